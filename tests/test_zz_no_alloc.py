"""The allocation-free forward entry point, attn_fwd_noalloc.

It serves callers that cannot call cudaMalloc (a framework that owns the whole
device memory pool, code that must not trigger an allocation's implicit
synchronisation, code running during stream capture): its scratch -- the kernel's
status word -- lives in a static device array inside the library.  The test calls
it through the C ABI twice in a row and checks each result against the ordinary
entry point's output, with the forward tolerance used everywhere else.  This file
is collected last so a failure here cannot hide the other tests; it also passes
when run alone in a fresh process (the first call does the per-device set-up).
"""
import math

import numpy as np
import pytest
import torch

import attn_inputs as ai
from attn_check import compare_lse, compare_o

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _ea():
    import exact_attention_103_b200 as ea
    return ea


def test_noalloc_matches_fwd_dense_twice():
    ea = _ea()
    B, N, H, d = 2, 1100, 4, 128
    q, k, v = (t.to(DEV) for t in ai.make_custom(B, N, H, d, seed=31))
    o_ref, l_ref = ea.fwd(q, k, v, causal=True)
    ea.get_device_status()
    for _ in range(2):
        o = torch.full_like(q, float("nan"))
        lse = torch.full((B, H, N), float("nan"), dtype=torch.float32, device=DEV)
        ea.fwd_noalloc(q, k, v, o, lse, causal=True, check=True)
        compare_o(o.cpu(), o_ref.cpu(), "noalloc dense")
        compare_lse(lse.cpu(), l_ref.cpu(), "noalloc dense")


def test_noalloc_matches_fwd_varlen_twice():
    ea = _ea()
    lengths = [300, 1, 700, 129]
    H, d = 2, 64
    q, k, v = (t.to(DEV) for t in ai.make_custom(0, 0, H, d, seed=32, lengths=lengths))
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32, device=DEV)
    o_ref, l_ref = ea.fwd(q, k, v, causal=False, cu_seqlens=cu, max_seqlen=max(lengths))
    ea.get_device_status()
    for _ in range(2):
        o = torch.full_like(q, float("nan"))
        lse = torch.full((H, q.shape[0]), float("nan"), dtype=torch.float32, device=DEV)
        ea.fwd_noalloc(q, k, v, o, lse, causal=False, cu_seqlens=cu, max_seqlen=max(lengths),
                       check=True)
        compare_o(o.cpu(), o_ref.cpu(), "noalloc varlen")
        compare_lse(lse.cpu(), l_ref.cpu(), "noalloc varlen")
