"""Host-side logic of the benchmark (no GPU): FLOP counts of the workloads."""
import numpy as np
import pytest

import attn_inputs as ai
import bench


@pytest.mark.parametrize("L,causal,window", [(1, False, None), (37, True, (5, 0)),
                                             (200, False, (10, 3)), (64, False, (-1, 4)),
                                             (90, True, (1000, 0)), (50, False, (0, 0))])
def test_visible_pairs_brute_force(L, causal, window):
    i = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    vis = np.ones((L, L), dtype=bool)
    if window is not None:
        wl, wr = window
        if wl >= 0:
            vis &= j >= i - wl
        if wr >= 0:
            vis &= j <= i + wr
    if causal:
        vis &= j <= i
    if window is None:
        expected = L * L / 2.0 if causal else float(L * L)  # published L^2/2 convention
    else:
        expected = float(vis.sum())
    assert bench.visible_pairs(L, causal, window) == expected


def test_workload_flops():
    assert bench.workload_flops(ai.DENSE) == 4.0 * 4 * 16 * 2048 ** 2 * 128
    assert bench.workload_flops(ai.CAUSAL) == 4.0 * 2 * 16 * 8192 ** 2 * 128 / 2
    assert abs(bench.workload_flops(ai.VARLEN) - 5.643e12) / 5.643e12 < 1e-3
    # window 1024 back, causal: row i sees min(i, 1024) + 1 keys
    per_seq = sum(min(i, 1024) + 1 for i in range(8192))
    assert bench.workload_flops(ai.WINDOW) == 4.0 * 2 * 16 * 128 * per_seq
    assert bench.workload_flops(ai.CAUSAL_E4M3) == bench.workload_flops(ai.CAUSAL)


def test_e4m3_inputs_are_exact_and_in_range():
    import torch
    x = torch.randn(4096, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    x8, sc = ai.to_e4m3(x)
    assert x8.dtype == torch.float8_e4m3fn
    assert float(x8.float().abs().max()) <= 448.0
    assert sc == 2.0 ** round(np.log2(sc))  # a power of two
    # quantisation error is at most half an E4M3 step (relative 2^-4) above 2^-6
    xr = x.float() / sc
    big = xr.abs() >= 2.0 ** -6
    assert torch.all((x8.float() - xr).abs()[big] <= xr.abs()[big] * 2.0 ** -4 + 1e-12)


def test_source_hash_ignores_comments_and_launch_code():
    src = "a = 1; // note\n/* block\n comment */\nint f();\n\nint fwd_smem_bytes(int D) { return 0; }\n"
    assert bench._code_only(src) == "a = 1;\nint f();\nint fwd_smem_bytes(int D) { return 0; }"
    assert bench._device_part(src) == "a = 1; // note\n/* block\n comment */\nint f();\n"
    assert bench._code_only("x;  // a\n\n  y; /* b */\n") == "x;\n  y;"
