"""GPU parity of the forward kernel against the fp64 oracle, through the C ABI.

Small and ragged shapes are compared element by element over the whole output;
the full benchmark workloads are compared on sampled rows (the oracle computes
those one by one) plus whole-output properties.
"""
import math

import numpy as np
import pytest
import torch

import attn_inputs as ai
import oracle
from attn_check import compare_lse, compare_o, to_np

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _lib():
    import exact_attention_103_b200 as ea
    return ea


def _dense_ref(q, k, v, causal, scale):
    B, N, H, d = q.shape
    o, lse, _ = oracle.fwd(q.reshape(B * N, H, d), k.reshape(B * N, H, d), v.reshape(B * N, H, d),
                           oracle.dense_cu(B, N), causal, scale)
    return o.reshape(B, N, H, d), oracle.lse_to_dense(lse, B, N)


def _run_dense(q, k, v, causal, scale, **kw):
    ea = _lib()
    o, lse = ea.fwd(q.to(DEV), k.to(DEV), v.to(DEV), causal=causal, scale=scale, **kw)
    ea.get_device_status()
    return o.cpu(), lse.cpu()


@pytest.mark.parametrize("d", [64, 128])
def test_selftest_umma_tile(d):
    """The kernel's tensor-core building blocks on one tile: S = A B^T (K-major
    smem operands), then bf16(S) V with P from TMEM and V MN-major."""
    ea = _lib()
    g = torch.Generator().manual_seed(d)
    a, b, v = (torch.randn(128, d, generator=g).to(torch.bfloat16) for _ in range(3))
    s, o = ea.selftest_umma(a.to(DEV), b.to(DEV), v.to(DEV))
    torch.cuda.synchronize()
    s_ref = a.double() @ b.double().T
    np.testing.assert_allclose(s.cpu().double().numpy(), s_ref.numpy(), rtol=0, atol=1e-3)
    p = s.cpu().to(torch.bfloat16).double()
    o_ref = p @ v.double()
    np.testing.assert_allclose(o.cpu().double().numpy(), o_ref.numpy(), rtol=1e-5, atol=1e-2)


SMALL = [
    # B, N, H, d, causal, q_mult
    (1, 256, 1, 64, False, 1.0),     # the tiny latency workload
    (1, 256, 1, 64, True, 1.0),
    (1, 1, 1, 128, False, 1.0),
    (1, 1, 1, 64, True, 1.0),
    (2, 300, 3, 128, False, 1.0),    # ragged last tile, two batches
    (2, 300, 3, 128, True, 1.0),
    (1, 129, 2, 64, True, 1.0),
    (3, 513, 2, 128, True, 1.0),     # several tile pairs plus a 1-row tail
    (1, 1000, 1, 64, False, 1.0),
    (2, 640, 2, 128, False, 4.0),    # Q x4: the running maximum moves often
    (1, 768, 2, 128, True, 4.0),
    (1, 100, 300, 64, False, 1.0),   # 300 one-sub-tile pairs: the split last wave holds empty
    (2, 100, 150, 128, False, 1.0),  # halves, and a CTA may claim more work after one
]


@pytest.mark.parametrize("B,N,H,d,causal,qm", SMALL)
def test_fwd_parity_dense(B, N, H, d, causal, qm):
    q, k, v = ai.make_custom(B, N, H, d, seed=B * 1000 + N + d)
    if qm != 1.0:
        q = (q.float() * qm).to(torch.bfloat16)
    scale = 1.0 / math.sqrt(d)
    o, lse = _run_dense(q, k, v, causal, scale)
    o_ref, lse_ref = _dense_ref(q, k, v, causal, scale)
    compare_o(o, o_ref, f"dense B{B} N{N} H{H} d{d} causal={causal} x{qm}")
    compare_lse(lse, lse_ref)


VARLEN = [
    ([5, 0, 300, 129], 128, True),
    ([5, 0, 300, 129], 128, False),
    ([1, 127, 128, 129, 256, 257, 700], 64, True),
    ([1, 127, 128, 129, 256, 257, 700], 128, False),
    ([1024, 3, 511], 128, True),
]


@pytest.mark.parametrize("lengths,d,causal", VARLEN)
def test_fwd_parity_varlen(lengths, d, causal):
    H = 2
    q, k, v = ai.make_custom(0, 0, H, d, seed=sum(lengths) + d, lengths=lengths)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    scale = 1.0 / math.sqrt(d)
    ea = _lib()
    o, lse = ea.fwd(q.to(DEV), k.to(DEV), v.to(DEV), causal=causal, scale=scale,
                    cu_seqlens=torch.from_numpy(cu).to(DEV), max_seqlen=max(lengths))
    ea.get_device_status()
    o_ref, lse_ref, _ = oracle.fwd(q, k, v, cu, causal, scale)
    compare_o(o.cpu(), o_ref, f"varlen {lengths} d{d} causal={causal}")
    compare_lse(lse.cpu(), lse_ref)


def test_plain_c_entry_point_varlen_reads_total():
    """attn_fwd (no options) reads cu_seqlens[B] itself; results equal attn_fwd_ex's."""
    ea = _lib()
    lengths = [200, 77, 390]
    H, d = 2, 128
    q, k, v = (t.to(DEV) for t in ai.make_custom(0, 0, H, d, seed=5, lengths=lengths))
    cu = torch.tensor([0, 200, 277, 667], dtype=torch.int32, device=DEV)
    o1, l1 = ea.fwd(q, k, v, causal=True, cu_seqlens=cu, max_seqlen=390)
    o2, l2 = torch.empty_like(q), torch.empty_like(l1)
    ea.fwd_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), o2.data_ptr(), l2.data_ptr(), 3, H, 390,
               d, True, 1 / math.sqrt(d), cu.data_ptr(), torch.cuda.current_stream().cuda_stream)
    ea.get_device_status()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_fwd_deterministic_bitwise():
    ea = _lib()
    q, k, v = (t.to(DEV) for t in ai.make_custom(2, 1100, 4, 128, seed=21))
    o1, l1 = ea.fwd(q, k, v, causal=True)
    o2, l2 = ea.fwd(q, k, v, causal=True)
    ea.get_device_status()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_fwd_writes_nothing_outside_outputs():
    """Guard regions around O and LSE keep their canary pattern."""
    ea = _lib()
    B, N, H, d = 1, 333, 3, 128
    q, k, v = (t.to(DEV) for t in ai.make_custom(B, N, H, d, seed=22))
    n_o, n_l, pad = B * N * H * d, B * H * N, 4096
    o_buf = torch.full((n_o + 2 * pad,), 7.0, dtype=torch.bfloat16, device=DEV)
    l_buf = torch.full((n_l + 2 * pad,), -3.0, dtype=torch.float32, device=DEV)
    o = o_buf[pad:pad + n_o].view(B, N, H, d)
    lse = l_buf[pad:pad + n_l].view(B, H, N)
    ea.fwd(q, k, v, causal=False, out=o, lse=lse)
    ea.get_device_status()
    for buf, val in ((o_buf, 7.0), (l_buf, -3.0)):
        assert torch.all(buf[:pad] == val) and torch.all(buf[-pad:] == val)
    o_ref, l_ref = _dense_ref(q.cpu(), k.cpu(), v.cpu(), False, 1 / math.sqrt(d))
    compare_o(o.cpu(), o_ref)
    compare_lse(lse.cpu(), l_ref)


def test_rescale_threshold_readings_agree():
    """tau = 0 (rescale whenever the maximum grows), 8 (default) and 64 (the
    largest allowed; rarely rescales) are all exact readings: same result within
    tolerance, and fewer rescales as tau grows."""
    ea = _lib()
    B, N, H, d = 1, 1024, 2, 128
    q, k, v = ai.make_custom(B, N, H, d, seed=23)
    q = (q.float() * 4).to(torch.bfloat16)
    o_ref, l_ref = _dense_ref(q, k, v, False, 1 / math.sqrt(d))
    outs = {}
    for tau in (0.0, 8.0, 64.0):
        stats = torch.zeros(2, dtype=torch.int64, device=DEV)
        o, lse = ea.fwd(q.to(DEV), k.to(DEV), v.to(DEV), rescale_threshold=tau, stats=stats)
        ea.get_device_status()
        compare_o(o.cpu(), o_ref, f"tau={tau}", raw_bar=False)  # Q x 4
        compare_lse(lse.cpu(), l_ref)
        outs[tau] = stats.cpu().tolist()
    # row-tiles after the first tile: every row of every 128-row sub-tile, 7 tiles each
    expected = B * H * (N // 128) * 128 * (N // 128 - 1)
    for tau, (resc, tiles) in outs.items():
        assert tiles == expected, (tau, tiles, expected)
    assert outs[0.0][0] >= outs[8.0][0] >= outs[64.0][0]


def test_invalid_cu_seqlens_recorded_on_device():
    """cu_seqlens that disagree with the packed token count make the kernel write
    nothing and record ATTN_ERR_INVALID_ARG in the device error word."""
    ea = _lib()
    q, k, v = (t.to(DEV) for t in ai.make_custom(0, 0, 1, 64, seed=24, lengths=[100, 100]))
    cu = torch.tensor([0, 100, 150], dtype=torch.int32, device=DEV)  # total 150 != 200
    ea.fwd(q, k, v, cu_seqlens=cu, max_seqlen=100)
    with pytest.raises(ea.AttnError) as e:
        ea.get_device_status()
    assert e.value.status == ea.ATTN_ERR_INVALID_ARG
    ea.get_device_status()  # cleared


# ----------------------------------------------------- full-size workloads
def _sample_rows(lengths, H, n, seed):
    """Sampled (token, head) rows: each sequence's first/last rows, rows around
    128-row tile boundaries, and random rows."""
    rng = np.random.default_rng(seed)
    cu = np.concatenate([[0], np.cumsum(lengths)])
    rows, heads = [], []
    for b, L in enumerate(lengths):
        picks = {0, L - 1, min(127, L - 1), min(128, L - 1), min(255, L - 1), min(256, L - 1),
                 (L - 1) // 2}
        picks |= set(rng.integers(0, L, size=max(1, n // len(lengths))).tolist())
        for i in sorted(picks):
            rows.append(cu[b] + i)
            heads.append(int(rng.integers(0, H)))
    return np.array(rows), np.array(heads), cu


def _run_workload(w, poly=0):
    """The workload through the C ABI into NaN-prefilled O and LSE (a row that the
    persistent schedule skipped stays NaN).  Returns CPU (o [T,H,d], lse [H,T])."""
    ea = _lib()
    q, k, v = ai.make_qkv(w)
    cu_t = None
    if w.varlen:
        cu_t = torch.tensor(w.cu_seqlens(), dtype=torch.int32, device=DEV)
    o = torch.full(q.shape, float("nan"), dtype=torch.bfloat16, device=DEV)
    lse_shape = (w.H, w.total_tokens) if w.varlen else (w.B, w.H, w.N)
    lse = torch.full(lse_shape, float("nan"), dtype=torch.float32, device=DEV)
    ea.fwd(q.to(DEV), k.to(DEV), v.to(DEV), causal=w.causal, scale=1.0 / math.sqrt(w.d),
           cu_seqlens=cu_t, max_seqlen=w.N if w.varlen else None, window=w.window,
           exp_poly_per8=poly, out=o, lse=lse)
    ea.get_device_status()
    o = o.cpu().reshape(-1, w.H, w.d)
    lse = lse.cpu()
    if not w.varlen:
        lse = lse.permute(1, 0, 2).reshape(w.H, -1)  # [B,H,N] -> [H, B*N]
    assert torch.isfinite(o.float()).all(), "an output row was not written"
    assert torch.isfinite(lse).all(), "an LSE entry was not written"
    return (q, k, v), o, lse


@pytest.mark.parametrize("name,poly", [("B1-H1-N256-d64", 0), ("B4-H16-N2048-d128", 0),
                                       ("B4-H16-N2048-d128", 2), ("B4-H16-N2048-d128-qx4", 0),
                                       ("B2-H16-N8192-d128-causal", 0),
                                       ("B2-H16-N8192-d128-causal-win1024", 0)])
def test_fwd_full_workload_whole_output(name, poly):
    """The benchmark workloads at full size, launched as the benchmark launches them,
    compared element by element over the WHOLE output against the oracle (a few
    seconds to half a minute of fp64 on the host cores each)."""
    w = ai.ALL[name]
    (q, k, v), o, lse = _run_workload(w, poly)
    qp, kp, vp = (t.reshape(-1, w.H, w.d) for t in (q, k, v))
    o_ref, l_ref, _ = oracle.fwd(qp, kp, vp, np.asarray(w.cu_seqlens()), w.causal,
                                 1.0 / math.sqrt(w.d), window=w.window)
    label = f"{name} poly={poly} (whole output)"
    compare_o(o, o_ref, label, raw_bar=w.q_mult == 1.0)
    compare_lse(lse, l_ref, label)


def test_fwd_varlen_workload_every_item():
    """The packed causal workload (16 sequences, 125 841 tokens): every output written
    (NaN-prefilled buffers), one random row of EVERY (sequence, head, 128-row
    sub-tile), each sequence's first 16 rows (they average the fewest keys, so |O|
    and the rounding error are largest there) and its last row compared with the
    oracle under the raw max-abs bar, and a second launch bitwise equal to the first."""
    w = ai.VARLEN
    (q, k, v), o, lse = _run_workload(w)
    rng = np.random.default_rng(7)
    cu = np.asarray(w.cu_seqlens())
    rows, heads = [], []
    for b, L in enumerate(w.seq_lengths()):
        for h in range(w.H):
            picks = set(range(min(16, L))) | {L - 1}
            for t0 in range(0, L, 128):
                picks.add(int(rng.integers(t0, min(t0 + 128, L))))
            rows += [cu[b] + i for i in sorted(picks)]
            heads += [h] * len(picks)
    rows, heads = np.asarray(rows), np.asarray(heads)
    o_ref, l_ref = oracle.fwd_rows(q, k, v, cu, True, 1.0 / math.sqrt(w.d), rows, heads)
    compare_o(o[rows, heads], o_ref, f"{w.name} ({rows.size} rows, every sub-tile)", raw_bar=True)
    compare_lse(lse[heads, rows], l_ref, w.name)
    _, o2, lse2 = _run_workload(w)
    assert torch.equal(o, o2) and torch.equal(lse, lse2), "repeat launch differs"


def test_wait_timeout_is_reported_and_the_context_stays_usable():
    """With the test-only fault option every CTA withholds its first query-tile
    copy, so the MMA warp's wait for it runs out (20 ms limit).  Each CTA records
    ATTN_ERR_TIMEOUT, the other roles see the CTA's abort flag, in-flight copies
    and MMAs drain, TMEM is freed, and the host reads the status; the next
    ordinary call still computes the right answer."""
    ea = _lib()
    B, N, H, d = 2, 1024, 4, 128
    q, k, v = ai.make_custom(B, N, H, d, seed=41)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    ea.fwd(qd, kd, vd, causal=True, timeout_ns=20_000_000, test_fault=1)
    with pytest.raises(ea.AttnError) as e:
        ea.get_device_status()
    assert e.value.status == ea.ATTN_ERR_TIMEOUT
    ea.get_device_status()  # cleared
    o, lse = ea.fwd(qd, kd, vd, causal=True)
    ea.get_device_status()
    o_ref, l_ref = _dense_ref(q, k, v, True, 1 / math.sqrt(d))
    compare_o(o.cpu(), o_ref, "after timeout")
    compare_lse(lse.cpu(), l_ref)


# ------------------------------------------------------------ size limits
@pytest.mark.parametrize("causal", [False, True])
def test_varlen_max_sequences(causal):
    """B = 1024 packed sequences (the varlen limit), lengths 0..9, compared in full."""
    ea = _lib()
    g = torch.Generator().manual_seed(71)
    lengths = [int(x) for x in torch.randint(0, 10, (1024,), generator=g)]
    H, d = 2, 64
    q, k, v = ai.make_custom(0, 0, H, d, seed=72, lengths=lengths)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    scale = 1.0 / math.sqrt(d)
    o, lse = ea.fwd(q.to(DEV), k.to(DEV), v.to(DEV), causal=causal, scale=scale,
                    cu_seqlens=torch.from_numpy(cu).to(DEV), max_seqlen=max(lengths))
    ea.get_device_status()
    o_ref, lse_ref, _ = oracle.fwd(q, k, v, cu, causal, scale)
    # Sequences of 0..9 tokens: output rows average at most 9 values, so |O| reaches 2
    # and beyond (the default rule then applies the half-ulp gate).
    compare_o(o.cpu(), o_ref, f"1024 sequences causal={causal}")
    compare_lse(lse.cpu(), lse_ref)


def test_varlen_max_length_sampled():
    """N = 131072 (the varlen limit): one sequence of that length plus a short one,
    causal, compared on sampled rows."""
    ea = _lib()
    lengths = [131072, 77]
    H, d = 1, 64
    q, k, v = ai.make_custom(0, 0, H, d, seed=73, lengths=lengths)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    scale = 1.0 / math.sqrt(d)
    o, lse = ea.fwd(q.to(DEV), k.to(DEV), v.to(DEV), causal=True, scale=scale,
                    cu_seqlens=torch.from_numpy(cu).to(DEV), max_seqlen=max(lengths))
    ea.get_device_status()
    o, lse = o.cpu(), lse.cpu()
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    rows, heads, cu64 = _sample_rows(lengths, H, 96, seed=74)
    rows = np.concatenate([rows, [131071, 131071 - 128, 131072, 131072 + 76]])
    heads = np.concatenate([heads, [0, 0, 0, 0]])
    o_ref, l_ref = oracle.fwd_rows(q, k, v, cu64, True, scale, rows, heads)
    compare_o(o[rows, heads], o_ref, "N=131072")
    compare_lse(lse[heads, rows], l_ref, "N=131072")


@pytest.mark.parametrize("varlen", [False, True])
def test_host_pipeline_matches_fwd(varlen):
    """Four calls through the overlapped host pipeline (two device buffer sets, so
    buffers are reused while neighbouring calls are in flight) give exactly the
    results of plain device calls."""
    ea = _lib()
    H, d = 2, 128
    lengths = [300, 5, 700] if varlen else None
    cu = None if lengths is None else torch.tensor(np.concatenate([[0], np.cumsum(lengths)]),
                                                   dtype=torch.int32)
    inputs = [ai.make_custom(2, 640, H, d, seed=80 + i, lengths=lengths) for i in range(4)]
    shape = inputs[0][0].shape
    pipe = ea.HostPipeline(shape, causal=True, cu_seqlens_host=None if cu is None else cu.pin_memory(),
                           max_seqlen=max(lengths) if varlen else None)
    outs = []
    for q, k, v in inputs:
        o_h = torch.empty(shape, dtype=torch.bfloat16, pin_memory=True)
        lse_shape = (H, shape[0]) if varlen else (shape[0], H, shape[1])
        l_h = torch.empty(lse_shape, dtype=torch.float32, pin_memory=True)
        pipe.submit(q.pin_memory(), k.pin_memory(), v.pin_memory(), o_h, l_h)
        outs.append((o_h, l_h))
    pipe.synchronize()
    ea.get_device_status()
    for (q, k, v), (o_h, l_h) in zip(inputs, outs):
        o, lse = ea.fwd(q.to(DEV), k.to(DEV), v.to(DEV), causal=True,
                        cu_seqlens=None if cu is None else cu.to(DEV),
                        max_seqlen=max(lengths) if varlen else None)
        ea.get_device_status()
        assert torch.equal(o.cpu(), o_h) and torch.equal(lse.cpu(), l_h)


def test_concurrent_streams_keep_their_own_work_counters():
    """Forward launches queued on four streams at once (the kernels may overlap on
    the GPU; each stream's launches use that stream's claim counters) give exactly
    the results of the same calls made one at a time."""
    ea = _lib()
    probs = [ai.make_custom(1, 700 + 130 * i, 3, 128, seed=90 + i) for i in range(4)]
    dev = [tuple(t.to(DEV) for t in p) for p in probs]
    serial = []
    for q, k, v in dev:
        serial.append(ea.fwd(q, k, v, causal=True))
    ea.get_device_status()
    streams = [torch.cuda.Stream() for _ in range(4)]
    torch.cuda.synchronize()
    outs = [[] for _ in range(4)]
    for rep in range(3):
        for i, (q, k, v) in enumerate(dev):
            with torch.cuda.stream(streams[i]):
                outs[i].append(ea.fwd(q, k, v, causal=True))
    torch.cuda.synchronize()
    ea.get_device_status()
    for i in range(4):
        for o, lse in outs[i]:
            assert torch.equal(o, serial[i][0]) and torch.equal(lse, serial[i][1])
