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


def test_reference_arm_prints_one_contract_line():
    """bench.py --impl reference times the oracle on the host and prints the
    contract's JSON line (here on the tiny workload, so it runs in seconds)."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    import time
    t0 = time.time()
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "2",
                        "--warmup", "3", "--workload", "B1-H1-N256-d64", "--ref-seconds", "0.5"],
                       capture_output=True, text=True, cwd=root, timeout=600)
    wall = time.time() - t0
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 3
    assert d["unit"] == "TFLOP/s" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["workload"] == "B1-H1-N256-d64"
    # the steps it reports are the steps it ran: they fit in the process's wall time
    assert d["steps"] * d["ms_per_step"] / 1e3 <= wall
    assert d["config"] == bench.bench_config(ai.TINY, 1)  # the same config as our arm's


def test_default_workload_is_the_largest_single_gpu_forward():
    """With no flags the bench measures the packed causal workload (the largest
    forward configuration, N up to 16384)."""
    import argparse
    import inspect
    src = inspect.getsource(bench.main)
    assert "default=ai.VARLEN.name" in src
    assert bench.workload_flops(ai.VARLEN) == max(bench.workload_flops(w) for w in ai.ALL.values()
                                                  if not w.e4m3)


def test_input_recipe_varlen_lengths():
    """The packed workload's lengths come from randint(512, 16385, 16) with seed 1."""
    assert ai.varlen_lengths() == [2910, 7918, 11825, 6298, 15585, 5661, 2365, 9874, 11314, 11831,
                                   4855, 1877, 14574, 2629, 15279, 1046]
    assert ai.VARLEN.total_tokens == 125841 and ai.VARLEN.N == 15585


def test_input_recipe_is_seeded_bf16():
    import torch
    a = ai.make_qkv(ai.TINY)
    b = ai.make_qkv(ai.TINY)
    assert all(torch.equal(x, y) for x, y in zip(a, b))
    assert all(x.dtype == torch.bfloat16 and tuple(x.shape) == (1, 256, 1, 64) for x in a)
    q4 = ai.make_qkv(ai.DENSE_X4)[0]
    q1 = ai.make_qkv(ai.DENSE)[0]
    assert torch.equal(q4.float(), q1.float() * 4)  # exact: a power-of-two multiple
