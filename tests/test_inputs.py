"""Host checks of the seeded synthetic input generator."""

import torch

from video_diffusion_b200 import inputs as I


def test_filter_matrix_rows_sum_to_one_and_reflect():
    for n in (1, 3, 16, 45):
        F = I.gaussian_filter_matrix(n)
        torch.testing.assert_close(F.sum(1), torch.ones(n, dtype=torch.float64), rtol=0, atol=1e-12)
    # half-sample symmetric boundary: a constant field stays constant, and the
    # matrix is symmetric under flipping both axes
    F = I.gaussian_filter_matrix(21)
    torch.testing.assert_close(F, F.flip(0).flip(1))


def test_make_qkv_shapes_determinism_and_moments():
    Q, K, V = I.make_qkv((4, 16, 16), heads=2, d=64, seed=1000, dtype=torch.float32, text_tokens=8)
    assert Q.shape == (1, 2, 1032, 64)
    Q2, K2, V2 = I.make_qkv((4, 16, 16), heads=2, d=64, seed=1000, dtype=torch.float32, text_tokens=8)
    assert torch.equal(Q, Q2) and torch.equal(K, K2) and torch.equal(V, V2)
    # Q - K = 0.5 (N - N') has variance 0.5; Q and K share the smooth part
    diff = (Q - K)[0, 0, :1024]
    assert abs(diff.var().item() - 0.5) < 0.05
    assert abs(Q[0, 0, :1024].var().item() - 1.25) < 0.15
    corr = torch.corrcoef(torch.stack([Q[0, 0, :1024, 0], K[0, 0, :1024, 0]]))[0, 1]
    assert corr > 0.6  # smooth field shared by Q and K


def test_workload_table():
    wl = I.WORKLOADS["wan-720p"]
    assert wl.L == 75600 and wl.n_blocks == 591
    assert abs(wl.dense_flops() - 1.171e14) / 1.171e14 < 1e-3
    assert I.WORKLOADS["hunyuan-720p"].L == 119056
    assert I.WORKLOADS["wan-480p"].L == 32760
