"""Pins for the fp64 oracle: what fixes it to something other than itself.

Each test checks the oracle against a closed form, a mathematical invariant, a
special case that reduces to a library routine (PyTorch's fp64 CPU
scaled_dot_product_attention / logsumexp / autograd), or finite differences.
A plausible mistake in the oracle -- a dropped scale, a wrong sign, a transposed
operand, an off-by-one causal mask, a missing max subtraction that overflows,
mixed-up heads or sequences -- fails at least one of them.
Definitions pinned: "FlashAttention 1-4 详解", section 原算法 (softmax(QK^T/sqrt(d))V),
Online Softmax 数学推导 (two-pass softmax and the online recurrences), and the
causal lower-triangle rule of section 其他优化.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from attn_inputs import make_custom


def _packed(t):
    """[B,N,H,d] or [T,H,d] tensor -> fp64 numpy [T,H,d]."""
    a = t.double().numpy()
    return a.reshape(-1, a.shape[-2], a.shape[-1])


def _sdpa_ref(q, k, v, causal, scale):
    """PyTorch fp64 CPU SDPA per sequence: q/k/v [B,N,H,d] fp64 -> O [B,N,H,d]."""
    qt, kt, vt = (x.double().permute(0, 2, 1, 3) for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=causal, scale=scale)
    return o.permute(0, 2, 1, 3).numpy()


# ---------------------------------------------------------------- closed forms

def test_two_key_closed_form():
    """One query, keys 0 and 1, values 0 and 1, scale 1: s = (0, x),
    O = e^x/(1+e^x) (the logistic function), LSE = ln(1+e^x).  With x = ln 3:
    O = 3/4 and LSE = ln 4 exactly."""
    x = math.log(3.0)
    q = np.array([[[x]], [[0.0]]])  # token 1 is a second query we ignore
    k = np.array([[[0.0]], [[1.0]]])
    v = np.array([[[0.0]], [[1.0]]])
    o, lse, _ = oracle.fwd(q, k, v, [0, 2], causal=False, scale=1.0)
    assert abs(o[0, 0, 0] - 0.75) < 1e-15
    assert abs(lse[0, 0] - math.log(4.0)) < 1e-15
    # query 1 has q = 0: uniform weights -> mean of values, LSE = ln 2.
    assert abs(o[1, 0, 0] - 0.5) < 1e-15
    assert abs(lse[0, 1] - math.log(2.0)) < 1e-15


def test_scale_is_applied_inside_softmax():
    """Same two keys, scale 1/2 and q = 2 ln 3: the scaled score is ln 3 again,
    so O = 3/4 -- a dropped or squared scale gives 9/10 or 0.63..."""
    x = 2.0 * math.log(3.0)
    q = np.array([[[x]], [[0.0]]])
    k = np.array([[[0.0]], [[1.0]]])
    v = np.array([[[0.0]], [[1.0]]])
    o, lse, _ = oracle.fwd(q, k, v, [0, 2], causal=False, scale=0.5)
    assert abs(o[0, 0, 0] - 0.75) < 1e-15
    assert abs(lse[0, 0] - math.log(4.0)) < 1e-15


def test_causal_three_token_closed_form():
    """Causal, d=1, q = k = 1, v = (1, 2, 4), scale ln 2: every visible score is ln 2,
    so row i averages v_0..v_i: O = (1, 1.5, 7/3); LSE_i = ln((i+1) * 2)."""
    q = np.ones((3, 1, 1))
    k = np.ones((3, 1, 1))
    v = np.array([1.0, 2.0, 4.0]).reshape(3, 1, 1)
    o, lse, _ = oracle.fwd(q, k, v, [0, 3], causal=True, scale=math.log(2.0))
    np.testing.assert_allclose(o[:, 0, 0], [1.0, 1.5, 7.0 / 3.0], rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse[0], [math.log(2 * (i + 1)) for i in range(3)], rtol=0, atol=1e-15)


# ------------------------------------------------------------------ invariants

@pytest.mark.parametrize("causal", [False, True])
def test_prob_rows_sum_to_one_and_mask(causal):
    q, k, _ = make_custom(1, 37, 2, 16, seed=3)
    cu = [0, 37]
    for h in range(2):
        P = oracle.probs(_packed(q), _packed(k), cu, causal, 0.25, 0, h)
        assert np.all(P >= 0)
        np.testing.assert_allclose(P.sum(axis=1), 1.0, rtol=0, atol=1e-12)
        if causal:
            assert np.all(np.triu(P, 1) == 0.0)
            assert P[0, 0] == 1.0
        else:
            assert np.all(P > 0)


@pytest.mark.parametrize("causal", [False, True])
def test_constant_v_returns_constant(causal):
    q, k, _ = make_custom(2, 50, 3, 8, seed=4)
    v = np.full((100, 3, 8), 0.0)
    v[:, :, :] = np.arange(8)[None, None, :] * 0.5 - 1.0
    o, _, _ = oracle.fwd(_packed(q), _packed(k), v, oracle.dense_cu(2, 50), causal, 0.3)
    np.testing.assert_allclose(o, v, rtol=0, atol=1e-12)


def test_causal_row0_returns_v0_exactly():
    q, k, v = make_custom(2, 40, 2, 32, seed=5)
    vp = _packed(v)
    o, lse, _ = oracle.fwd(_packed(q), _packed(k), vp, oracle.dense_cu(2, 40), True, 0.17)
    for b in range(2):
        assert np.array_equal(o[b * 40], vp[b * 40])
    # Row 0 sees one key: LSE = its scaled score.
    qp, kp = _packed(q), _packed(k)
    for h in range(2):
        s00 = 0.17 * float(np.dot(qp[0, h], kp[0, h]))
        assert abs(lse[h, 0] - s00) < 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_zero_q_returns_mean_of_visible_v(causal):
    _, k, v = make_custom(1, 33, 2, 16, seed=6)
    q = np.zeros((33, 2, 16))
    vp = _packed(v)
    o, lse, _ = oracle.fwd(q, _packed(k), vp, [0, 33], causal, 0.25)
    for i in range(33):
        n = i + 1 if causal else 33
        np.testing.assert_allclose(o[i], vp[:n].mean(axis=0), rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[:, i], math.log(n), rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_shift_invariance(causal):
    """Adding the same constant to every score of a row changes neither O nor the
    normalised weights; LSE moves by exactly that constant.  Realised by one extra
    dimension: q' = [q, 1], k' = [k, c], so s'_ij = s_ij + scale*c."""
    q, k, v = make_custom(1, 29, 2, 8, seed=7)
    qp, kp, vp = _packed(q), _packed(k), _packed(v)
    c = 3.0
    q2 = np.concatenate([qp, np.ones((29, 2, 1))], axis=2)
    k2 = np.concatenate([kp, np.full((29, 2, 1), c)], axis=2)
    v2 = np.concatenate([vp, np.zeros((29, 2, 1))], axis=2)
    o1, l1, _ = oracle.fwd(qp, kp, vp, [0, 29], causal, 0.5)
    o2, l2, _ = oracle.fwd(q2, k2, v2, [0, 29], causal, 0.5)
    np.testing.assert_allclose(o2[:, :, :8], o1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l2, l1 + 0.5 * c, rtol=0, atol=1e-12)


def test_large_scores_do_not_overflow():
    """Scores around 1e3 overflow exp() unless the row max is subtracted first."""
    q, k, v = make_custom(1, 16, 1, 8, seed=8)
    qp = _packed(q) * 200.0
    o, lse, _ = oracle.fwd(qp, _packed(k), _packed(v), [0, 16], False, 1.0)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    assert np.max(np.abs(lse)) > 700  # the scores really are that large


# ------------------------------------------------------- library special cases

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,N,H,d", [(1, 1, 1, 4), (2, 17, 3, 16), (1, 130, 2, 64)])
def test_matches_torch_sdpa_fp64(B, N, H, d, causal):
    q, k, v = make_custom(B, N, H, d, seed=11 + N)
    o, lse, _ = oracle.fwd(_packed(q), _packed(k), _packed(v), oracle.dense_cu(B, N), causal,
                           1.0 / math.sqrt(d))
    ref = _sdpa_ref(q, k, v, causal, None)  # PyTorch's default scale is 1/sqrt(d)
    np.testing.assert_allclose(o.reshape(B, N, H, d), ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_lse_matches_torch_logsumexp(causal):
    B, N, H, d = 2, 23, 2, 16
    scale = 0.3
    q, k, v = make_custom(B, N, H, d, seed=12)
    _, lse, _ = oracle.fwd(_packed(q), _packed(k), _packed(v), oracle.dense_cu(B, N), causal, scale)
    lse = oracle.lse_to_dense(lse, B, N)
    s = torch.einsum("bihc,bjhc->bhij", q.double(), k.double()) * scale
    if causal:
        s = s.masked_fill(torch.triu(torch.ones(N, N, dtype=torch.bool), 1), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_equals_per_sequence_sdpa(causal):
    lengths = [5, 1, 40, 17]
    H, d = 2, 16
    q, k, v = make_custom(0, 0, H, d, seed=13, lengths=lengths)
    cu = np.concatenate([[0], np.cumsum(lengths)])
    o, lse, _ = oracle.fwd(_packed(q), _packed(k), _packed(v), cu, causal, 0.25)
    for b, L in enumerate(lengths):
        sl = slice(cu[b], cu[b + 1])
        ref = _sdpa_ref(q[sl][None], k[sl][None], v[sl][None], causal, 0.25)[0]
        np.testing.assert_allclose(o[sl], ref, rtol=0, atol=1e-12)


def test_fwd_rows_equals_fwd():
    lengths = [70, 3, 129]
    q, k, v = make_custom(0, 0, 3, 32, seed=14, lengths=lengths)
    cu = np.concatenate([[0], np.cumsum(lengths)])
    o, lse, _ = oracle.fwd(_packed(q), _packed(k), _packed(v), cu, True, 0.2)
    rows = np.array([0, 69, 70, 72, 73, 150, 201])
    heads = np.array([0, 2, 1, 0, 2, 1, 0])
    o_r, l_r = oracle.fwd_rows(_packed(q), _packed(k), _packed(v), cu, True, 0.2, rows, heads)
    np.testing.assert_allclose(o_r, o[rows, heads], rtol=0, atol=1e-13)
    np.testing.assert_allclose(l_r, lse[heads, rows], rtol=0, atol=1e-13)


# ------------------------------------------------ online softmax == two-pass

@pytest.mark.parametrize("Br,Bc", [(1, 1), (16, 16), (128, 128), (7, 5), (64, 128)])
@pytest.mark.parametrize("tau", [0.0, 8.0 * math.log(2.0), 1e9])
@pytest.mark.parametrize("causal", [False, True])
def test_online_equals_two_pass(Br, Bc, tau, causal):
    lengths = [131, 45]
    q, k, v = make_custom(0, 0, 2, 16, seed=15, lengths=lengths, std=2.0)
    cu = np.concatenate([[0], np.cumsum(lengths)])
    args = (_packed(q), _packed(k), _packed(v), cu, causal, 0.4)
    o_ref, l_ref, _ = oracle.fwd(*args)
    o, l, n = oracle.online_fwd(*args, Br, Bc, tau)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l, l_ref, rtol=0, atol=1e-12)
    if tau >= 1e9 or Bc >= 131:
        assert n == 0


def test_rescale_count_falls_with_threshold():
    q, k, v = make_custom(1, 512, 2, 32, seed=16, std=2.0)
    args = (_packed(q), _packed(k), _packed(v), [0, 512], False, 0.5)
    counts = [oracle.online_fwd(*args, 128, 32, tau)[2] for tau in (0.0, 1.0, 4.0, 1e9)]
    assert counts[0] > 0 and counts[-1] == 0
    assert all(a >= b for a, b in zip(counts, counts[1:]))


# ------------------------------------------------------------------- backward

def _loss_grad_torch(q, k, v, dout, causal, scale):
    qt, kt, vt = (x.double().permute(0, 2, 1, 3).requires_grad_(True) for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=causal, scale=scale)
    (o * dout.double().permute(0, 2, 1, 3)).sum().backward()
    return [t.grad.permute(0, 2, 1, 3).numpy() for t in (qt, kt, vt)]


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_matches_torch_autograd_fp64(causal):
    B, N, H, d = 2, 19, 2, 8
    q, k, v, do = make_custom(B, N, H, d, seed=17, n=4)
    grads = oracle.bwd(_packed(q), _packed(k), _packed(v), _packed(do), oracle.dense_cu(B, N),
                       causal, 0.35)
    ref = _loss_grad_torch(q, k, v, do, causal, 0.35)
    for g, r in zip(grads, ref):
        np.testing.assert_allclose(g.reshape(B, N, H, d), r, rtol=0, atol=1e-11)


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_central_finite_differences(causal):
    """dL/dx for L = sum(dO * O), by central differences on a tiny problem."""
    lengths = [6, 4]
    H, d = 1, 3
    q, k, v, do = (t.double().numpy() for t in make_custom(0, 0, H, d, seed=18, lengths=lengths, n=4))
    cu = np.array([0, 6, 10])
    scale = 0.7
    grads = oracle.bwd(q, k, v, do, cu, causal, scale)

    def loss(qq, kk, vv):
        o, _, _ = oracle.fwd(qq, kk, vv, cu, causal, scale)
        return float(np.sum(o * do))

    eps = 1e-6
    for which, g in enumerate(grads):
        base = [q, k, v]
        num = np.zeros_like(g)
        for idx in np.ndindex(g.shape):
            plus = [a.copy() for a in base]
            minus = [a.copy() for a in base]
            plus[which][idx] += eps
            minus[which][idx] -= eps
            num[idx] = (loss(*plus) - loss(*minus)) / (2 * eps)
        np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-8)


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_key_shift_invariance(causal):
    """Adding one vector c to every key adds scale*<q_i,c> to each score of row i,
    which the softmax ignores; so sum_j dK_j = 0 for every (sequence, head)."""
    lengths = [33, 12]
    q, k, v, do = make_custom(0, 0, 2, 16, seed=19, lengths=lengths, n=4)
    cu = np.array([0, 33, 45])
    _, dk, _ = oracle.bwd(_packed(q), _packed(k), _packed(v), _packed(do), cu, causal, 0.25)
    for b in range(2):
        np.testing.assert_allclose(dk[cu[b]:cu[b + 1]].sum(axis=0), 0.0, rtol=0, atol=1e-11)


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_sampled_matches_torch_autograd(causal):
    """The per-position backward equals PyTorch fp64 autograd at the chosen rows."""
    lengths = [37, 70]
    H, d = 2, 16
    q, k, v, do = make_custom(0, 0, H, d, seed=20, lengths=lengths, n=4)
    cu = np.array([0, 37, 107])
    b, h = 1, 1
    sl = slice(37, 107)
    ref = _loss_grad_torch(q[sl][None], k[sl][None], v[sl][None], do[sl][None], causal, 0.3)
    rows = [0, 5, 69, 33]
    dq, dk, dv = oracle.bwd_sampled(_packed(q), _packed(k), _packed(v), _packed(do), cu, causal,
                                    0.3, b, h, rows, rows)
    np.testing.assert_allclose(dq, ref[0][0][rows, h], rtol=0, atol=1e-11)
    np.testing.assert_allclose(dk, ref[1][0][rows, h], rtol=0, atol=1e-11)
    np.testing.assert_allclose(dv, ref[2][0][rows, h], rtol=0, atol=1e-11)


# ------------------------------------------------------ sliding-window masks
# Reading of the mask hook: key j is visible to query i iff i - wl <= j <= i + wr
# (a negative bound is unbounded), on top of the causal rule when that is set.

def _window_bool_mask(N, wl, wr, causal):
    """The visibility rule written as a dense boolean matrix [i, j] (True = visible)."""
    i = torch.arange(N)[:, None]
    j = torch.arange(N)[None, :]
    vis = torch.ones(N, N, dtype=torch.bool)
    if wl >= 0:
        vis &= j >= i - wl
    if wr >= 0:
        vis &= j <= i + wr
    if causal:
        vis &= j <= i
    return vis


@pytest.mark.parametrize("wl,wr,causal", [(0, 0, False), (3, 0, True), (5, 2, False),
                                          (-1, 4, False), (7, -1, False), (16, 16, True),
                                          (200, 200, False)])
def test_window_matches_torch_sdpa_with_boolean_mask(wl, wr, causal):
    """Library special case: PyTorch fp64 SDPA given the visibility matrix as attn_mask."""
    B, N, H, d = 2, 37, 2, 16
    scale = 0.3
    q, k, v = make_custom(B, N, H, d, seed=21)
    o, lse, _ = oracle.fwd(_packed(q), _packed(k), _packed(v), oracle.dense_cu(B, N), causal,
                           scale, window=(wl, wr))
    mask = _window_bool_mask(N, wl, wr, causal)
    qt, kt, vt = (x.double().permute(0, 2, 1, 3) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale)
    np.testing.assert_allclose(o.reshape(B, N, H, d), ref.permute(0, 2, 1, 3).numpy(), rtol=0,
                               atol=1e-12)
    s = torch.einsum("bihc,bjhc->bhij", q.double(), k.double()) * scale
    ref_lse = torch.logsumexp(s.masked_fill(~mask, float("-inf")), dim=-1).numpy()
    np.testing.assert_allclose(oracle.lse_to_dense(lse, B, N), ref_lse, rtol=0, atol=1e-12)


def test_window_zero_returns_own_value_exactly():
    """wl = wr = 0: each query sees only its own key, so O_i = V_i exactly and
    LSE_i = scale * <q_i, k_i>."""
    q, k, v = make_custom(1, 19, 2, 8, seed=22)
    qp, kp, vp = _packed(q), _packed(k), _packed(v)
    o, lse, _ = oracle.fwd(qp, kp, vp, [0, 19], False, 0.7, window=(0, 0))
    np.testing.assert_array_equal(o, vp)
    np.testing.assert_allclose(lse, 0.7 * np.einsum("thc,thc->ht", qp, kp), rtol=0, atol=1e-12)


@pytest.mark.parametrize("wl,wr", [(2, 3), (0, 5), (4, 0), (-1, 1), (3, -1)])
def test_window_zero_q_returns_mean_of_window(wl, wr):
    """Q = 0 gives uniform weights: O_i is the mean of V over
    [max(0, i - wl), min(L - 1, i + wr)] and LSE_i = ln(count) -- an off-by-one at
    either edge of the window changes both."""
    L = 23
    _, k, v = make_custom(1, L, 1, 4, seed=23)
    vp = _packed(v)
    o, lse, _ = oracle.fwd(np.zeros((L, 1, 4)), _packed(k), vp, [0, L], False, 1.0,
                           window=(wl, wr))
    for i in range(L):
        lo = 0 if wl < 0 else max(0, i - wl)
        hi = L - 1 if wr < 0 else min(L - 1, i + wr)
        np.testing.assert_allclose(o[i, 0], vp[lo:hi + 1, 0].mean(axis=0), rtol=0, atol=1e-12)
        assert abs(lse[0, i] - math.log(hi - lo + 1)) < 1e-12


def test_window_two_key_closed_form():
    """Causal window of one key back: query i sees keys i-1 and i only.  With
    q_i = (x), k_{i-1} = (0), k_i = (1), v_{i-1} = 0, v_i = 1 and x = ln 3, the
    weight of key i is 3/4 (the two-key logistic closed form), whatever lies further back."""
    x = math.log(3.0)
    L = 6
    q = np.full((L, 1, 1), x)
    k = np.array([[[1.0 if t % 2 else 0.0]] for t in range(L)])
    v = k.copy()
    o, lse, _ = oracle.fwd(q, k, v, [0, L], True, 1.0, window=(1, 0))
    for i in range(1, L, 2):  # odd i: key i has k = 1, key i-1 has k = 0
        assert abs(o[i, 0, 0] - 0.75) < 1e-15
        assert abs(lse[0, i] - math.log(4.0)) < 1e-15


@pytest.mark.parametrize("wl,wr,causal", [(4, 1, False), (6, 0, True)])
def test_window_probs_zero_outside_and_rows_sum_to_one(wl, wr, causal):
    q, k, _ = make_custom(1, 31, 1, 8, seed=24)
    P = oracle.probs(_packed(q), _packed(k), [0, 31], causal, 0.5, 0, 0, window=(wl, wr))
    mask = _window_bool_mask(31, wl, wr, causal).numpy()
    assert np.all(P[~mask] == 0.0)
    assert np.all(P[mask] > 0.0)
    np.testing.assert_allclose(P.sum(axis=1), 1.0, rtol=0, atol=1e-14)


def test_window_rows_equal_full_and_wide_window_is_unmasked():
    """fwd_rows honours the window, and a window wider than the sequence masks nothing."""
    lengths = [50, 7, 90]
    q, k, v = make_custom(0, 0, 2, 16, seed=25, lengths=lengths)
    cu = np.concatenate([[0], np.cumsum(lengths)])
    qp, kp, vp = _packed(q), _packed(k), _packed(v)
    o, lse, _ = oracle.fwd(qp, kp, vp, cu, False, 0.25, window=(9, 4))
    rows = np.array([0, 5, 49, 50, 56, 57, 100, 146])
    heads = np.array([0, 1, 1, 0, 1, 0, 1, 0])
    o_r, l_r = oracle.fwd_rows(qp, kp, vp, cu, False, 0.25, rows, heads, window=(9, 4))
    np.testing.assert_allclose(o_r, o[rows, heads], rtol=0, atol=1e-13)
    np.testing.assert_allclose(l_r, lse[heads, rows], rtol=0, atol=1e-13)
    o_w, _, _ = oracle.fwd(qp, kp, vp, cu, True, 0.25, window=(1000, 1000))
    o_c, _, _ = oracle.fwd(qp, kp, vp, cu, True, 0.25)
    np.testing.assert_array_equal(o_w, o_c)


# ------------------------------------------------- windowed backward
@pytest.mark.parametrize("wl,wr,causal", [(3, 0, True), (5, 2, False), (0, 0, False), (-1, 3, False)])
def test_bwd_window_matches_torch_autograd_fp64(wl, wr, causal):
    """Library special case: PyTorch fp64 autograd through SDPA with the visibility
    matrix as a boolean mask."""
    B, N, H, d = 2, 21, 2, 8
    q, k, v, do = make_custom(B, N, H, d, seed=31, n=4)
    mask = _window_bool_mask(N, wl, wr, causal)
    qt, kt, vt = (x.double().permute(0, 2, 1, 3).requires_grad_(True) for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=0.4)
    (o * do.double().permute(0, 2, 1, 3)).sum().backward()
    refs = [t.grad.permute(0, 2, 1, 3).numpy().reshape(B * N, H, d) for t in (qt, kt, vt)]
    got = oracle.bwd(_packed(q), _packed(k), _packed(v), _packed(do), oracle.dense_cu(B, N),
                     causal, 0.4, window=(wl, wr))
    for g, r in zip(got, refs):
        np.testing.assert_allclose(g, r, rtol=0, atol=1e-11)


def test_bwd_window_central_finite_differences():
    """d/dx of L = sum(dO * O) by central differences for a few entries of q, k, v,
    with a causal one-key-back window on a packed pair of sequences."""
    lengths = [7, 5]
    H, d = 1, 4
    q, k, v, do = (_packed(t) for t in make_custom(0, 0, H, d, seed=32, lengths=lengths, n=4))
    cu = np.concatenate([[0], np.cumsum(lengths)])
    win = (1, 0)
    dq, dk, dv = oracle.bwd(q, k, v, do, cu, True, 0.7, window=win)

    def loss(q_, k_, v_):
        o, _, _ = oracle.fwd(q_, k_, v_, cu, True, 0.7, window=win)
        return float((o * do).sum())

    eps = 1e-6
    for arr, grad in ((q, dq), (k, dk), (v, dv)):
        for idx in [(0, 0, 0), (3, 0, 2), (6, 0, 1), (7, 0, 3), (11, 0, 0)]:
            plus, minus = arr.copy(), arr.copy()
            plus[idx] += eps
            minus[idx] -= eps
            args_p = [plus if a is arr else a for a in (q, k, v)]
            args_m = [minus if a is arr else a for a in (q, k, v)]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert abs(fd - grad[idx]) < 1e-6, (idx, fd, grad[idx])
