"""GPU parity of the CTA-pair forward (cta_pair: clusters of two CTAs running
tcgen05.mma.cta_group::2, each CTA holding half of every K/V tile) against the fp64
oracle, through the C ABI: dense, ragged, causal, varlen and windowed problems, and
the benchmark workloads at full size."""
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


PAIR_DENSE = [
    # B, N, H, causal, window
    (1, 512, 1, True, None),      # one item: two sub-tiles of 256 rows
    (1, 512, 1, False, None),
    (2, 700, 3, True, None),      # ragged: the second CTA's rows run past N
    (2, 700, 3, False, None),
    (1, 100, 2, False, None),     # every row in the leader's half
    (3, 257, 2, True, None),
    (1, 1100, 2, True, None),
    (1, 1024, 2, True, (100, 0)),
    (1, 900, 2, False, (50, 70)),
]


@pytest.mark.parametrize("B,N,H,causal,window", PAIR_DENSE)
def test_pair_parity_dense(B, N, H, causal, window):
    ea = _ea()
    d = 128
    q, k, v = ai.make_custom(B, N, H, d, seed=300 + N + H)
    o, lse = ea.fwd(q.to(DEV), k.to(DEV), v.to(DEV), causal=causal, window=window, cta_pair=True)
    ea.get_device_status()
    shp = (B * N, H, d)
    o_ref, l_ref, _ = oracle.fwd(q.reshape(shp), k.reshape(shp), v.reshape(shp), oracle.dense_cu(B, N),
                                 causal, 1 / math.sqrt(d), window=window)
    label = f"pair B{B} N{N} H{H} causal={causal} window={window}"
    compare_o(o.cpu().reshape(shp), o_ref, label)
    compare_lse(lse.cpu(), oracle.lse_to_dense(l_ref, B, N), label)


@pytest.mark.parametrize("causal", [False, True])
def test_pair_parity_varlen(causal):
    ea = _ea()
    lengths = [5, 0, 300, 129, 700, 1030, 512]
    H, d = 2, 128
    q, k, v = ai.make_custom(0, 0, H, d, seed=310, lengths=lengths)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    o, lse = ea.fwd(q.to(DEV), k.to(DEV), v.to(DEV), causal=causal,
                    cu_seqlens=torch.from_numpy(cu).to(DEV), max_seqlen=max(lengths), cta_pair=True)
    ea.get_device_status()
    o_ref, l_ref, _ = oracle.fwd(q, k, v, cu, causal, 1 / math.sqrt(d))
    compare_o(o.cpu(), o_ref, f"pair varlen causal={causal}")
    compare_lse(lse.cpu(), l_ref, f"pair varlen causal={causal}")


def test_pair_repeatable_and_close_to_single_cta():
    """Two pair launches are bitwise equal; pair and single-CTA outputs agree to
    within the rounding of the bf16 output."""
    ea = _ea()
    q, k, v = (t.to(DEV) for t in ai.make_custom(2, 1500, 4, 128, seed=311))
    a = ea.fwd(q, k, v, causal=True, cta_pair=True)
    b = ea.fwd(q, k, v, causal=True, cta_pair=True)
    c = ea.fwd(q, k, v, causal=True)
    ea.get_device_status()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    assert float((a[0].float() - c[0].float()).abs().max()) <= 1.6e-2
    assert float((a[1] - c[1]).abs().max()) <= 1e-5


@pytest.mark.parametrize("name", ["B2-H16-N8192-d128-causal", "varlen16-H16-d128-causal"])
def test_pair_full_workload(name):
    """The causal workloads at full size through the pair kernel: NaN-prefilled
    outputs all written; the causal N=8192 output compared whole, the packed one at
    a random row of every (sequence, head, 128-row block)."""
    ea = _ea()
    w = ai.ALL[name]
    q, k, v = ai.make_qkv(w)
    cu_t = torch.tensor(w.cu_seqlens(), dtype=torch.int32, device=DEV) if w.varlen else None
    o = torch.full(q.shape, float("nan"), dtype=torch.bfloat16, device=DEV)
    lse_shape = (w.H, w.total_tokens) if w.varlen else (w.B, w.H, w.N)
    lse = torch.full(lse_shape, float("nan"), dtype=torch.float32, device=DEV)
    ea.fwd(q.to(DEV), k.to(DEV), v.to(DEV), causal=True, cu_seqlens=cu_t,
           max_seqlen=w.N if w.varlen else None, out=o, lse=lse, cta_pair=True)
    ea.get_device_status()
    o = o.cpu().reshape(-1, w.H, w.d)
    lse = lse.cpu()
    if not w.varlen:
        lse = lse.permute(1, 0, 2).reshape(w.H, -1)
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    qp, kp, vp = (t.reshape(-1, w.H, w.d) for t in (q, k, v))
    cu = np.asarray(w.cu_seqlens())
    scale = 1.0 / math.sqrt(w.d)
    if not w.varlen:
        o_ref, l_ref, _ = oracle.fwd(qp, kp, vp, cu, True, scale)
        compare_o(o, o_ref, f"pair {name} (whole output)", raw_bar=True)
        compare_lse(lse, l_ref, f"pair {name}")
        return
    rng = np.random.default_rng(8)
    rows, heads = [], []
    for b, L in enumerate(w.seq_lengths()):
        for h in range(w.H):
            picks = {0, L - 1} | {int(rng.integers(t0, min(t0 + 128, L))) for t0 in range(0, L, 128)}
            rows += [cu[b] + i for i in sorted(picks)]
            heads += [h] * len(picks)
    rows, heads = np.asarray(rows), np.asarray(heads)
    o_ref, l_ref = oracle.fwd_rows(qp, kp, vp, cu, True, scale, rows, heads)
    compare_o(o[rows, heads], o_ref, f"pair {name} (every 128-row block)", raw_bar=True)
    compare_lse(lse[heads, rows], l_ref, f"pair {name}")
