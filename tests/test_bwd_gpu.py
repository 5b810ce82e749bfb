"""GPU parity of the backward pass (dQ, dK, dV) against the fp64 oracle.

Tolerance: relative L2 error <= 2e-2 per gradient (the stated backward bar).
Inputs: seeded bf16 Q, K, V, dO; O and LSE from this library's forward.
"""
import math

import numpy as np
import pytest
import torch

import attn_inputs as ai
import oracle
from attn_check import log_parity, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"
REL_L2 = 2e-2


def _ea():
    import exact_attention_103_b200 as ea
    return ea


def _check(grads, refs, label):
    """||g - r|| <= 2e-2 ||r||, plus an absolute floor of 1e-5 per element in the
    norm for gradients that vanish exactly (one key: dS = dP - D = 0, so dQ = 0)."""
    for name, g, r in zip(("dq", "dk", "dv"), grads, refs):
        a, b = to_np(g), to_np(r)
        assert np.all(np.isfinite(a)), f"{label} {name}: non-finite"
        err = float(np.linalg.norm(a - b))
        bound = REL_L2 * float(np.linalg.norm(b)) + 1e-5 * math.sqrt(b.size)
        log_parity(f"{label} {name}", rel_l2=err / max(float(np.linalg.norm(b)), 1e-30))
        assert err <= bound, f"{label} {name}: |g-r| {err:.3e} > {bound:.3e} (|r| {np.linalg.norm(b):.3e})"


BWD_DENSE = [
    (1, 128, 1, 64, False),
    (1, 256, 2, 128, True),
    (2, 300, 3, 128, False),     # ragged last tile
    (2, 300, 3, 128, True),
    (1, 513, 2, 64, True),
    (1, 1, 1, 128, False),
    (1, 1100, 2, 128, True),     # nine tiles: the pipelined order wraps the ring several times
    (1, 1100, 2, 128, False),
    (1, 700, 2, 64, False),
]


@pytest.mark.parametrize("B,N,H,d,causal", BWD_DENSE)
def test_bwd_parity_dense(B, N, H, d, causal):
    ea = _ea()
    q, k, v, do = ai.make_custom(B, N, H, d, seed=100 + N + d, n=4)
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    o, lse = ea.fwd(qd, kd, vd, causal=causal)
    dq, dk, dv = ea.bwd(qd, kd, vd, o, lse, dod, causal=causal)
    ea.get_device_status()
    shp = (B * N, H, d)
    refs = oracle.bwd(q.reshape(shp), k.reshape(shp), v.reshape(shp), do.reshape(shp),
                      oracle.dense_cu(B, N), causal, 1 / math.sqrt(d))
    _check([g.cpu().reshape(shp) for g in (dq, dk, dv)], refs, f"B{B} N{N} H{H} d{d} c{causal}")


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_parity_varlen(causal):
    ea = _ea()
    lengths = [200, 1, 128, 333]
    H, d = 2, 128
    q, k, v, do = ai.make_custom(0, 0, H, d, seed=7, lengths=lengths, n=4)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    cu_d = torch.from_numpy(cu).to(DEV)
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    o, lse = ea.fwd(qd, kd, vd, causal=causal, cu_seqlens=cu_d, max_seqlen=max(lengths))
    grads = ea.bwd(qd, kd, vd, o, lse, dod, causal=causal, cu_seqlens=cu_d, max_seqlen=max(lengths))
    ea.get_device_status()
    refs = oracle.bwd(q, k, v, do, cu, causal, 1 / math.sqrt(d))
    _check([g.cpu() for g in grads], refs, f"varlen causal={causal}")


def test_bwd_bitwise_repeatable():
    ea = _ea()
    q, k, v, do = (t.to(DEV) for t in ai.make_custom(2, 640, 4, 128, seed=11, n=4))
    o, lse = ea.fwd(q, k, v, causal=True)
    a = ea.bwd(q, k, v, o, lse, do, causal=True, deterministic=True)
    b = ea.bwd(q, k, v, o, lse, do, causal=True, deterministic=True)
    c = ea.bwd(q, k, v, o, lse, do, causal=True, deterministic=False)
    ea.get_device_status()
    for x, y, z in zip(a, b, c):
        assert torch.equal(x, y) and torch.equal(x, z)


def test_bwd_full_workload():
    """The causal B2-H16-N8192-d128 backward at full size, as the benchmark runs it:
    run once normally and twice in deterministic mode, all three bitwise equal; dQ,
    dK and dV of four whole heads (both sequences, every row) against the oracle's
    textbook backward; every gradient finite."""
    ea = _ea()
    w = ai.BWD_CAUSAL
    q, k, v, do = ai.make_qkv(w, with_dout=True)
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    o, lse = ea.fwd(qd, kd, vd, causal=True)
    normal = ea.bwd(qd, kd, vd, o, lse, dod, causal=True, deterministic=False)
    det1 = ea.bwd(qd, kd, vd, o, lse, dod, causal=True, deterministic=True)
    det2 = ea.bwd(qd, kd, vd, o, lse, dod, causal=True, deterministic=True)
    ea.get_device_status()
    for name, a, b, c in zip(("dq", "dk", "dv"), normal, det1, det2):
        assert torch.equal(b, c), f"{name}: deterministic runs differ"
        assert torch.equal(a, b), f"{name}: normal and deterministic runs differ"
        assert torch.isfinite(a.float()).all(), f"{name}: non-finite"
    dq, dk, dv = (g.cpu() for g in normal)
    cu = oracle.dense_cu(w.B, w.N)
    for h in (0, 5, 10, 15):
        one = [t[:, :, h:h + 1].reshape(w.B * w.N, 1, w.d) for t in (q, k, v, do)]
        refs = oracle.bwd(*one, cu, True, 1 / math.sqrt(w.d))
        got = [g[:, :, h:h + 1].reshape(w.B * w.N, 1, w.d) for g in (dq, dk, dv)]
        _check(got, refs, f"full-size head {h}")


def test_bwd_peaked_rows():
    """Q x 4: sharply peaked probability rows (P close to one-hot)."""
    ea = _ea()
    B, N, H, d = 1, 640, 2, 128
    q, k, v, do = ai.make_custom(B, N, H, d, seed=12, n=4)
    q = (q.float() * 4).to(torch.bfloat16)
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    o, lse = ea.fwd(qd, kd, vd, causal=True)
    dq, dk, dv = ea.bwd(qd, kd, vd, o, lse, dod, causal=True)
    ea.get_device_status()
    shp = (B * N, H, d)
    refs = oracle.bwd(q.reshape(shp), k.reshape(shp), v.reshape(shp), do.reshape(shp),
                      oracle.dense_cu(B, N), True, 1 / math.sqrt(d))
    _check([g.cpu().reshape(shp) for g in (dq, dk, dv)], refs, "q x4")


def test_bwd_parity_varlen_d64():
    ea = _ea()
    lengths = [130, 7, 600, 256]
    H, d = 2, 64
    q, k, v, do = ai.make_custom(0, 0, H, d, seed=13, lengths=lengths, n=4)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    cu_d = torch.from_numpy(cu).to(DEV)
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    o, lse = ea.fwd(qd, kd, vd, causal=True, cu_seqlens=cu_d, max_seqlen=max(lengths))
    grads = ea.bwd(qd, kd, vd, o, lse, dod, causal=True, cu_seqlens=cu_d, max_seqlen=max(lengths))
    ea.get_device_status()
    refs = oracle.bwd(q, k, v, do, cu, True, 1 / math.sqrt(d))
    _check([g.cpu() for g in grads], refs, "varlen d64")


@pytest.mark.parametrize("B,N,H,d,causal,window", [
    (1, 700, 2, 128, True, (64, 0)),
    (1, 640, 2, 128, False, (100, 30)),
    (2, 300, 2, 64, False, (0, 0)),
    (1, 900, 2, 128, False, (-1, 130)),
    (1, 1100, 1, 128, True, (300, 0)),
])
def test_bwd_parity_window(B, N, H, d, causal, window):
    """The backward of the sliding-window forward (the mask hook) against the
    oracle's windowed textbook backward."""
    ea = _ea()
    q, k, v, do = ai.make_custom(B, N, H, d, seed=200 + N, n=4)
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    o, lse = ea.fwd(qd, kd, vd, causal=causal, window=window)
    dq, dk, dv = ea.bwd(qd, kd, vd, o, lse, dod, causal=causal, window=window)
    ea.get_device_status()
    shp = (B * N, H, d)
    refs = oracle.bwd(q.reshape(shp), k.reshape(shp), v.reshape(shp), do.reshape(shp),
                      oracle.dense_cu(B, N), causal, 1 / math.sqrt(d), window=window)
    _check([g.cpu().reshape(shp) for g in (dq, dk, dv)], refs, f"window {window} causal={causal}")


def test_bwd_parity_window_varlen():
    ea = _ea()
    lengths = [200, 1, 128, 333, 700]
    H, d = 2, 128
    window = (90, 0)
    q, k, v, do = ai.make_custom(0, 0, H, d, seed=201, lengths=lengths, n=4)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    cu_d = torch.from_numpy(cu).to(DEV)
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    o, lse = ea.fwd(qd, kd, vd, causal=True, cu_seqlens=cu_d, max_seqlen=max(lengths),
                    window=window)
    grads = ea.bwd(qd, kd, vd, o, lse, dod, causal=True, cu_seqlens=cu_d, max_seqlen=max(lengths),
                   window=window)
    ea.get_device_status()
    refs = oracle.bwd(q, k, v, do, cu, True, 1 / math.sqrt(d), window=window)
    _check([g.cpu() for g in grads], refs, "varlen window")


def test_bwd_varlen_checks_cu_seqlens_on_device():
    """The backward takes the packed token count from the caller (no read-back of
    cu_seqlens[B]) and checks cu_seqlens on the device: a last entry that is not
    the token count records ATTN_ERR_INVALID_ARG; a sequence that runs past the
    packed tensors is not processed (its gradients stay unwritten) and records the
    same; the next correct call succeeds."""
    ea = _ea()
    lengths = [100, 100]
    H, d = 1, 64
    q, k, v, do = ai.make_custom(0, 0, H, d, seed=25, lengths=lengths, n=4)
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    good = torch.tensor([0, 100, 200], dtype=torch.int32, device=DEV)
    o, lse = ea.fwd(qd, kd, vd, cu_seqlens=good, max_seqlen=100)
    ea.get_device_status()
    for bad in ([0, 100, 150], [0, 100, 260]):
        ea.bwd(qd, kd, vd, o, lse, dod, cu_seqlens=torch.tensor(bad, dtype=torch.int32, device=DEV),
               max_seqlen=100)
        with pytest.raises(ea.AttnError) as e:
            ea.get_device_status()
        assert e.value.status == ea.ATTN_ERR_INVALID_ARG, bad
    grads = ea.bwd(qd, kd, vd, o, lse, dod, cu_seqlens=good, max_seqlen=100)
    ea.get_device_status()
    refs = oracle.bwd(q, k, v, do, np.array([0, 100, 200]), False, 1 / math.sqrt(d))
    _check([g.cpu() for g in grads], refs, "varlen after rejected calls")
