"""GPU parity of the forward's mask hook (sliding window) and of the FMA-pipe
exponential, against the fp64 oracle, through the C ABI.

Window reading: key j is visible to query i iff i - left <= j <= i + right (an open
side is negative), on top of the causal rule.  Cases cover windows narrower than a
tile (rows whose first key tile is fully hidden), windows that straddle tile
boundaries, one-sided windows, windows wide enough to collapse to the causal or the
unmasked kernel, ragged sequence ends and packed varlen batches.
"""
import math

import numpy as np
import pytest
import torch

import attn_inputs as ai
import oracle
from attn_check import compare_lse, compare_o

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _ea():
    import exact_attention_103_b200 as ea
    return ea


def _dense(q, k, v, causal, scale, window=None, poly=0):
    ea = _ea()
    B, N, H, d = q.shape
    o, lse = ea.fwd(q.to(DEV), k.to(DEV), v.to(DEV), causal=causal, scale=scale, window=window,
                    exp_poly_per8=poly)
    ea.get_device_status()
    o_ref, l_ref, _ = oracle.fwd(q.reshape(B * N, H, d), k.reshape(B * N, H, d),
                                 v.reshape(B * N, H, d), oracle.dense_cu(B, N), causal, scale,
                                 window=window)
    return o.cpu(), lse.cpu(), o_ref.reshape(B, N, H, d), oracle.lse_to_dense(l_ref, B, N)


WINDOWS = [
    # B, N, H, d, causal, window, q_mult
    (1, 1024, 2, 128, True, (10, 0), 1.0),      # narrower than a tile: first tiles fully hidden
    (1, 1024, 2, 128, False, (5, 3), 4.0),
    (1, 700, 2, 128, True, (100, 0), 1.0),
    (2, 1000, 2, 128, False, (300, 50), 1.0),
    (1, 513, 2, 64, False, (0, 0), 1.0),        # each query sees only its own key
    (1, 900, 2, 128, False, (-1, 130), 1.0),    # right bound only
    (1, 900, 2, 64, False, (200, -1), 1.0),     # left bound only
    (1, 640, 2, 64, False, (127, 128), 1.0),    # bounds on tile edges
    (1, 2048, 2, 128, True, (1024, 0), 1.0),
    (1, 300, 1, 128, False, (299, 299), 1.0),   # collapses to the unmasked kernel
    (1, 300, 1, 128, True, (400, 7), 1.0),      # collapses to the causal kernel
    (3, 257, 2, 128, True, (64, 0), 4.0),       # 1-row tail
]


@pytest.mark.parametrize("B,N,H,d,causal,window,qm", WINDOWS)
def test_window_parity_dense(B, N, H, d, causal, window, qm):
    q, k, v = ai.make_custom(B, N, H, d, seed=7 * N + d + B)
    if qm != 1.0:
        q = (q.float() * qm).to(torch.bfloat16)
    scale = 1.0 / math.sqrt(d)
    o, lse, o_ref, l_ref = _dense(q, k, v, causal, scale, window)
    compare_o(o, o_ref, f"window {window} B{B} N{N} d{d} causal={causal}")
    compare_lse(lse, l_ref)


@pytest.mark.parametrize("lengths,d,causal,window", [
    ([5, 0, 300, 129, 700], 128, True, (200, 0)),
    ([5, 0, 300, 129, 700], 128, False, (64, 64)),
    ([1, 127, 128, 129, 256, 257, 1100], 64, True, (30, 0)),
])
def test_window_parity_varlen(lengths, d, causal, window):
    ea = _ea()
    H = 2
    q, k, v = ai.make_custom(0, 0, H, d, seed=sum(lengths) + 3, lengths=lengths)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    scale = 1.0 / math.sqrt(d)
    o, lse = ea.fwd(q.to(DEV), k.to(DEV), v.to(DEV), causal=causal, scale=scale,
                    cu_seqlens=torch.from_numpy(cu).to(DEV), max_seqlen=max(lengths),
                    window=window)
    ea.get_device_status()
    o_ref, l_ref, _ = oracle.fwd(q, k, v, cu, causal, scale, window=window)
    compare_o(o.cpu(), o_ref, f"varlen window {window}")
    compare_lse(lse.cpu(), l_ref)


def test_window_deterministic_and_canaries():
    ea = _ea()
    B, N, H, d = 1, 777, 3, 128
    q, k, v = (t.to(DEV) for t in ai.make_custom(B, N, H, d, seed=31))
    n_o, n_l, pad = B * N * H * d, B * H * N, 4096
    o_buf = torch.full((n_o + 2 * pad,), 7.0, dtype=torch.bfloat16, device=DEV)
    l_buf = torch.full((n_l + 2 * pad,), -3.0, dtype=torch.float32, device=DEV)
    o = o_buf[pad:pad + n_o].view(B, N, H, d)
    lse = l_buf[pad:pad + n_l].view(B, H, N)
    ea.fwd(q, k, v, causal=True, out=o, lse=lse, window=(90, 0))
    o2, l2 = ea.fwd(q, k, v, causal=True, window=(90, 0))
    ea.get_device_status()
    for buf, val in ((o_buf, 7.0), (l_buf, -3.0)):
        assert torch.all(buf[:pad] == val) and torch.all(buf[-pad:] == val)
    assert torch.equal(o, o2) and torch.equal(lse, l2)


# ------------------------------------------------ FMA-pipe exponential splits
POLY = [
    # B, N, H, d, causal, q_mult, window
    (2, 300, 3, 128, False, 1.0, None),
    (1, 768, 2, 128, True, 4.0, None),
    (1, 1000, 1, 64, False, 1.0, None),
    (1, 700, 2, 128, True, 1.0, (100, 0)),
]


@pytest.mark.parametrize("poly", [2, 8])
@pytest.mark.parametrize("B,N,H,d,causal,qm,window", POLY)
def test_exp_poly_parity(poly, B, N, H, d, causal, qm, window):
    """2 of 8 pairs (FA4-style partial offload) and 8 of 8 (every exponential on
    the polynomial) meet the same bar as the MUFU path."""
    q, k, v = ai.make_custom(B, N, H, d, seed=11 * N + poly)
    if qm != 1.0:
        q = (q.float() * qm).to(torch.bfloat16)
    scale = 1.0 / math.sqrt(d)
    o, lse, o_ref, l_ref = _dense(q, k, v, causal, scale, window, poly)
    compare_o(o, o_ref, f"poly {poly}/8 B{B} N{N} d{d} causal={causal} window={window}")
    compare_lse(lse, l_ref)


def test_exp_poly_varlen():
    ea = _ea()
    lengths = [1, 127, 128, 129, 256, 257, 700]
    H, d = 2, 128
    q, k, v = ai.make_custom(0, 0, H, d, seed=99, lengths=lengths)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    scale = 1.0 / math.sqrt(d)
    o, lse = ea.fwd(q.to(DEV), k.to(DEV), v.to(DEV), causal=True, scale=scale,
                    cu_seqlens=torch.from_numpy(cu).to(DEV), max_seqlen=max(lengths),
                    exp_poly_per8=8)
    ea.get_device_status()
    o_ref, l_ref, _ = oracle.fwd(q, k, v, cu, True, scale)
    compare_o(o.cpu(), o_ref, "varlen poly 8/8")
    compare_lse(lse.cpu(), l_ref)
