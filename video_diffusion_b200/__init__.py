"""B200-native Sol-Attn sparse attention forward (sm_100a CUDA kernels behind a C ABI).

The compiled library ``libsolattn.so`` sits next to this file.  The binding in
``video_diffusion_b200.api`` loads it on first use and raises if it is missing;
there is no CPU fallback.
"""

__all__ = ["api", "inputs"]
