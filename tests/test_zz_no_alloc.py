"""The allocation-free forward entry point, attn_fwd_noalloc.

It serves callers that cannot call cudaMalloc (a framework that owns the whole
device memory pool, code that must not trigger an allocation's implicit
synchronisation, code running during stream capture): its scratch -- the kernel's
status word -- lives in a static device array inside the library.  Each test calls
it through the C ABI twice in a row and checks each result against the fp64 oracle
with the forward tolerance used everywhere else, and bitwise against the ordinary
entry point (both launch the same kernel with the same parameters).  This file is
collected last so a failure here cannot hide the other tests; it also passes when
run alone in a fresh process (the first call does the per-device set-up).
"""
import math
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import attn_inputs as ai
import oracle
from attn_check import compare_lse, compare_o

pytestmark = pytest.mark.gpu

DEV = "cuda"
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _ea():
    import exact_attention_103_b200 as ea
    return ea


def test_noalloc_dense_twice():
    ea = _ea()
    B, N, H, d = 2, 1100, 4, 128
    q, k, v = ai.make_custom(B, N, H, d, seed=31)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    o_fwd, l_fwd = ea.fwd(qd, kd, vd, causal=True)
    ea.get_device_status()
    o_ref, l_ref, _ = oracle.fwd(q.reshape(B * N, H, d), k.reshape(B * N, H, d),
                                 v.reshape(B * N, H, d), oracle.dense_cu(B, N), True,
                                 1 / math.sqrt(d))
    for call in range(2):
        o = torch.full_like(qd, float("nan"))
        lse = torch.full((B, H, N), float("nan"), dtype=torch.float32, device=DEV)
        ea.fwd_noalloc(qd, kd, vd, o, lse, causal=True, check=True)
        compare_o(o.cpu().reshape(B * N, H, d), o_ref, f"noalloc dense call {call}")
        compare_lse(lse.cpu(), oracle.lse_to_dense(l_ref, B, N), f"noalloc dense call {call}")
        assert torch.equal(o, o_fwd) and torch.equal(lse, l_fwd)


def test_noalloc_varlen_twice():
    ea = _ea()
    lengths = [300, 1, 700, 129]
    H, d = 2, 64
    q, k, v = ai.make_custom(0, 0, H, d, seed=32, lengths=lengths)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    cu_d = torch.from_numpy(cu).to(DEV)
    o_fwd, l_fwd = ea.fwd(qd, kd, vd, causal=False, cu_seqlens=cu_d, max_seqlen=max(lengths))
    ea.get_device_status()
    o_ref, l_ref, _ = oracle.fwd(q, k, v, cu, False, 1 / math.sqrt(d))
    for call in range(2):
        o = torch.full_like(qd, float("nan"))
        lse = torch.full((H, q.shape[0]), float("nan"), dtype=torch.float32, device=DEV)
        ea.fwd_noalloc(qd, kd, vd, o, lse, causal=False, cu_seqlens=cu_d,
                       max_seqlen=max(lengths), check=True)
        compare_o(o.cpu(), o_ref, f"noalloc varlen call {call}")
        compare_lse(lse.cpu(), l_ref, f"noalloc varlen call {call}")
        assert torch.equal(o, o_fwd) and torch.equal(lse, l_fwd)


def test_noalloc_reports_bad_cu_seqlens_then_recovers():
    """A cu_seqlens whose last entry is not total_tokens makes the kernel write
    nothing and record ATTN_ERR_INVALID_ARG in the static status word, which the
    call reads back (check=True); the next call clears the word and succeeds."""
    ea = _ea()
    lengths = [100, 100]
    H, d = 1, 64
    q, k, v = ai.make_custom(0, 0, H, d, seed=24, lengths=lengths)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    o = torch.full_like(qd, float("nan"))
    lse = torch.full((H, 200), float("nan"), dtype=torch.float32, device=DEV)
    bad = torch.tensor([0, 100, 150], dtype=torch.int32, device=DEV)  # cu[B] != 200
    with pytest.raises(ea.AttnError) as e:
        ea.fwd_noalloc(qd, kd, vd, o, lse, cu_seqlens=bad, max_seqlen=100, check=True)
    assert e.value.status == ea.ATTN_ERR_INVALID_ARG
    assert torch.isnan(o.float()).all(), "a rejected call wrote output"
    good = torch.tensor([0, 100, 200], dtype=torch.int32, device=DEV)
    ea.fwd_noalloc(qd, kd, vd, o, lse, cu_seqlens=good, max_seqlen=100, check=True)
    o_ref, l_ref, _ = oracle.fwd(q, k, v, np.array([0, 100, 200]), False, 1 / math.sqrt(d))
    compare_o(o.cpu(), o_ref, "noalloc after a rejected call")
    compare_lse(lse.cpu(), l_ref, "noalloc after a rejected call")


_FRESH = r"""
import sys, torch
sys.path.insert(0, sys.argv[1])
import attn_inputs as ai
import exact_attention_103_b200 as ea
q, k, v = (t.cuda() for t in ai.make_custom(1, 512, 2, 128, seed=5))
o = torch.empty_like(q)
lse = torch.empty((1, 2, 512), dtype=torch.float32, device="cuda")
ea.fwd_noalloc(q, k, v, o, lse, causal=True, check=True)   # set-up + kernel load
torch.cuda.synchronize()
free0 = torch.cuda.mem_get_info()[0]
for _ in range(3):
    ea.fwd_noalloc(q, k, v, o, lse, causal=True, check=True)
torch.cuda.synchronize()
free1 = torch.cuda.mem_get_info()[0]
print("FREE", free0, free1)
"""


def test_noalloc_in_fresh_process_takes_no_device_memory():
    """In a process of its own (the entry point's very first call there does the
    per-device set-up), further calls leave the device's free memory unchanged."""
    r = subprocess.run([sys.executable, "-c", _FRESH, ROOT], capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    line = [ln for ln in r.stdout.splitlines() if ln.startswith("FREE")][-1]
    free0, free1 = (int(x) for x in line.split()[1:])
    assert free0 == free1, f"free device memory changed: {free0} -> {free1}"
