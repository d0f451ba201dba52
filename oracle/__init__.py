"""Oracle for the Sol-Attn single-pass sparse attention forward.

TEST INFRASTRUCTURE ONLY.  This package is a plain, slow, float64 CPU
restatement of the method, used to check the CUDA library.  Only the tests,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import it.  The library under ``video_diffusion_b200``
never imports it and shares no code with it.

Every function cites the passage it follows, as "<page>, <section / equation>".
The pages are:

* "Sol-Attn" visual paper explainer (mxino.github.io/illustrations/sol-attention):
  the only page that prints the formulas -- Eq. (4) the threshold, Eq. (5) the
  moments, Eq. (9) the denominator, Eq. (10) the numerator, Eq. (11) proxy reuse.
* "Sol-Attn: Accelerating Video Generation Inference via On-the-Fly Attention
  Sparsification" abstract (chatpaper / Hugging Face daily papers).
* The papers.ananclaw.com explainer (sections 3.1-3.3) and the bud-325 paper
  notes ("Method"), used only where the formula page is silent.

Pins: see ``tests/test_oracle_pins.py``.  Every function here is pinned by at
least one check that does not re-type its own formula; none is "parity unpinned"
except the generic-beta mixture as a whole, which is pinned only through the
special cases listed there (no page prints a worked numeric example).
"""

from .sol_attn import (  # noqa: F401
    BlockGeometry,
    block_geometry,
    pool_blocks,
    proxy_scores,
    row_moments,
    eq5_moments,
    diagonal_sigma,
    MOMENTS,
    threshold,
    select_blocks,
    route_head,
    attend_query_block,
    forward_head,
    forward,
    stats,
    dense_attention,
    NEAR_TIE,
)
