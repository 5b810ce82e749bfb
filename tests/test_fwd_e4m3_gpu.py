"""GPU parity of the 8-bit forward (attn_fwd_e4m3) against the fp64 oracle run on
the dequantised inputs (x8 * scale), through the C ABI.  The tolerance reading is
in attn_check.compare_o_e4m3."""
import math

import numpy as np
import pytest
import torch

import attn_inputs as ai
import oracle
from attn_check import compare_lse, compare_o_e4m3

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _ea():
    import exact_attention_103_b200 as ea
    return ea


def test_selftest_umma_e4m3_tile():
    """kind::f8f6f4 building blocks on one tile: S = A B^T from shared memory,
    P = e4m3(S) packed four keys per TMEM column, O = P V with V MN-major."""
    ea = _ea()
    g = torch.Generator().manual_seed(8)
    a, b, v = (torch.randn(128, 128, generator=g).to(torch.float8_e4m3fn) for _ in range(3))
    s, o = ea.selftest_umma_e4m3(a.to(DEV), b.to(DEV), v.to(DEV))
    torch.cuda.synchronize()
    s_ref = a.double() @ b.double().T
    np.testing.assert_allclose(s.cpu().double().numpy(), s_ref.numpy(), rtol=0, atol=1e-3)
    p = s.cpu().to(torch.float8_e4m3fn).double()
    o_ref = p @ v.double()
    np.testing.assert_allclose(o.cpu().double().numpy(), o_ref.numpy(), rtol=1e-5, atol=1e-2)


def _quant(ts):
    out, sc = [], []
    for t in ts:
        t8, s = ai.to_e4m3(t)
        out.append(t8)
        sc.append(s)
    return out, tuple(sc)


def _deq(t8, s):
    return t8.double() * s


def _oracle(q8, k8, v8, sc, cu, causal, scale, window=None):
    """(O, LSE, A) of the dequantised inputs, packed [T,H,d] / [H,T]; A uses |V|."""
    q, k, v = (_deq(t, s) for t, s in zip((q8, k8, v8), sc))
    H, d = q.shape[-2], q.shape[-1]
    q, k, v = (t.reshape(-1, H, d) for t in (q, k, v))
    o, lse, _ = oracle.fwd(q, k, v, cu, causal, scale, window=window)
    a, _, _ = oracle.fwd(q, k, v.abs(), cu, causal, scale, window=window)
    return o, lse, a


CASES = [
    # B, N, H, causal, window
    (1, 256, 2, False, None),
    (1, 1, 1, True, None),
    (2, 300, 3, True, None),
    (1, 1000, 2, False, None),
    (3, 513, 2, True, None),
    (1, 700, 2, True, (100, 0)),
    (1, 640, 2, False, (127, 128)),
]


@pytest.mark.parametrize("B,N,H,causal,window", CASES)
def test_e4m3_parity_dense(B, N, H, causal, window):
    ea = _ea()
    d = 128
    (q8, k8, v8), sc = _quant(ai.make_custom(B, N, H, d, seed=13 * N + B))
    scale = 1.0 / math.sqrt(d)
    o, lse = ea.fwd(q8.to(DEV), k8.to(DEV), v8.to(DEV), causal=causal, scale=scale,
                    window=window, e4m3_scales=sc)
    ea.get_device_status()
    o_ref, l_ref, a_ref = _oracle(q8, k8, v8, sc, oracle.dense_cu(B, N), causal, scale, window)
    compare_o_e4m3(o.cpu().reshape(-1, H, d), o_ref, a_ref, f"e4m3 B{B} N{N} causal={causal}")
    compare_lse(lse.cpu(), oracle.lse_to_dense(l_ref, B, N))


def test_e4m3_peaked_rows():
    """Q x 4: sharply peaked rows, where most P~ are far below the row maximum."""
    ea = _ea()
    B, N, H, d = 1, 768, 2, 128
    q, k, v = ai.make_custom(B, N, H, d, seed=17)
    q = (q.float() * 4).to(torch.bfloat16)
    (q8, k8, v8), sc = _quant((q, k, v))
    scale = 1.0 / math.sqrt(d)
    for causal in (False, True):
        o, lse = ea.fwd(q8.to(DEV), k8.to(DEV), v8.to(DEV), causal=causal, scale=scale,
                        e4m3_scales=sc)
        ea.get_device_status()
        o_ref, l_ref, a_ref = _oracle(q8, k8, v8, sc, oracle.dense_cu(B, N), causal, scale)
        compare_o_e4m3(o.cpu().reshape(-1, H, d), o_ref, a_ref, f"e4m3 q x4 causal={causal}")
        compare_lse(lse.cpu(), oracle.lse_to_dense(l_ref, B, N))


def test_e4m3_parity_varlen():
    ea = _ea()
    lengths = [5, 0, 300, 129, 700]
    H, d = 2, 128
    (q8, k8, v8), sc = _quant(ai.make_custom(0, 0, H, d, seed=77, lengths=lengths))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    scale = 1.0 / math.sqrt(d)
    o, lse = ea.fwd(q8.to(DEV), k8.to(DEV), v8.to(DEV), causal=True, scale=scale,
                    cu_seqlens=torch.from_numpy(cu).to(DEV), max_seqlen=max(lengths),
                    e4m3_scales=sc)
    ea.get_device_status()
    o_ref, l_ref, a_ref = _oracle(q8, k8, v8, sc, cu, True, scale)
    compare_o_e4m3(o.cpu(), o_ref, a_ref, "e4m3 varlen")
    compare_lse(lse.cpu(), l_ref)


def test_e4m3_scales_are_applied():
    """The same 8-bit tensors with every scale doubled: S grows 4x (so a different
    softmax) and O carries V's factor 2 -- checked against the oracle."""
    ea = _ea()
    B, N, H, d = 1, 384, 2, 128
    (q8, k8, v8), sc = _quant(ai.make_custom(B, N, H, d, seed=5, std=0.5))
    sc2 = tuple(2 * s for s in sc)
    scale = 1.0 / math.sqrt(d)
    o, lse = ea.fwd(q8.to(DEV), k8.to(DEV), v8.to(DEV), scale=scale, e4m3_scales=sc2)
    ea.get_device_status()
    o_ref, l_ref, a_ref = _oracle(q8, k8, v8, sc2, oracle.dense_cu(B, N), False, scale)
    compare_o_e4m3(o.cpu().reshape(-1, H, d), o_ref, a_ref, "e4m3 doubled scales")
    compare_lse(lse.cpu(), oracle.lse_to_dense(l_ref, B, N))


def test_e4m3_deterministic():
    ea = _ea()
    (q8, k8, v8), sc = _quant(ai.make_custom(2, 1100, 4, 128, seed=21))
    q8, k8, v8 = q8.to(DEV), k8.to(DEV), v8.to(DEV)
    o1, l1 = ea.fwd(q8, k8, v8, causal=True, e4m3_scales=sc)
    o2, l2 = ea.fwd(q8, k8, v8, causal=True, e4m3_scales=sc)
    ea.get_device_status()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("name", ["B4-H16-N2048-d128-e4m3", "B2-H16-N8192-d128-causal-e4m3"])
def test_e4m3_full_workload_sampled(name):
    from test_fwd_gpu import _sample_rows
    ea = _ea()
    w = ai.ALL[name]
    q8, k8, v8, sc = ai.make_qkv_e4m3(w)
    scale = 1.0 / math.sqrt(w.d)
    o, lse = ea.fwd(q8.to(DEV), k8.to(DEV), v8.to(DEV), causal=w.causal, scale=scale,
                    e4m3_scales=sc)
    ea.get_device_status()
    o = o.cpu().reshape(-1, w.H, w.d)
    lse = lse.cpu().permute(1, 0, 2).reshape(w.H, -1)
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    rows, heads, cu = _sample_rows(w.seq_lengths(), w.H, 192, seed=len(name))
    q, k, v = (_deq(t, s).reshape(-1, w.H, w.d) for t, s in zip((q8, k8, v8), sc))
    o_ref, l_ref = oracle.fwd_rows(q, k, v, cu, w.causal, scale, rows, heads)
    a_ref, _ = oracle.fwd_rows(q, k, v.abs(), cu, w.causal, scale, rows, heads)
    compare_o_e4m3(o[rows, heads], o_ref, a_ref, name)
    compare_lse(lse[heads, rows], l_ref, name)


@pytest.mark.parametrize("causal", [False, True])
def test_e4m3_poly_split(causal):
    """2 of every 8 exponential pairs on the FMA-pipe polynomial, on the 8-bit path."""
    ea = _ea()
    B, N, H, d = 2, 600, 2, 128
    (q8, k8, v8), sc = _quant(ai.make_custom(B, N, H, d, seed=19))
    scale = 1.0 / math.sqrt(d)
    o, lse = ea.fwd(q8.to(DEV), k8.to(DEV), v8.to(DEV), causal=causal, scale=scale,
                    e4m3_scales=sc, exp_poly_per8=2)
    ea.get_device_status()
    o_ref, l_ref, a_ref = _oracle(q8, k8, v8, sc, oracle.dense_cu(B, N), causal, scale)
    compare_o_e4m3(o.cpu().reshape(-1, H, d), o_ref, a_ref, f"e4m3 poly 2/8 causal={causal}")
    compare_lse(lse.cpu(), oracle.lse_to_dense(l_ref, B, N))
