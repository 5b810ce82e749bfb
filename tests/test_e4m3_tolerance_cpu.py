"""The E4M3 tolerance reading, checked on the CPU: attention whose probabilities
are rounded to E4M3 before the PV product -- the one rounding the 8-bit path adds
-- stays inside the bar of attn_check.compare_o_e4m3 against the exact result.
As in the kernel, P~ = 2^(x - m_ref + shift) with the row sum l taken before
rounding; m_ref may sit up to tau below the row maximum (a stale reference) and
shift = floor(8 - tau) keeps P~ <= 256 inside the E4M3 range.  The rounding is
torch's float8_e4m3fn conversion; everything else is fp64."""
import math

import numpy as np
import pytest
import torch

from attn_check import compare_o_e4m3


def _o_with_e4m3_p(q, k, v, scale, causal, stale, tau):
    s = (q @ k.T) * scale * math.log2(math.e)
    if causal:
        s = np.where(np.tri(*s.shape, dtype=bool), s, -np.inf)
    m_ref = s.max(axis=1, keepdims=True) - stale
    shift = math.floor(8 - tau)
    p = np.exp2(s - m_ref + shift)
    assert p.max() <= 256.0
    l = p.sum(axis=1, keepdims=True)
    p8 = torch.from_numpy(p).to(torch.float8_e4m3fn).double().numpy()
    o = (p8 @ v) / l
    return torch.from_numpy(o).to(torch.bfloat16).double().numpy()  # O is stored as bf16


@pytest.mark.parametrize("tau", [2.0, 4.0, 6.0])
@pytest.mark.parametrize("N,causal,qm,stale", [(256, False, 1.0, 0.0), (512, True, 1.0, 0.0),
                                               (384, False, 4.0, 0.0), (384, True, 4.0, 1.0),
                                               (768, False, 6.0, 0.0), (1024, False, 1.0, 1.0)])
def test_e4m3_rounding_of_p_stays_inside_the_bar(N, causal, qm, stale, tau):
    """stale is a fraction of tau: the reference may lag the row maximum by up to tau."""
    g = torch.Generator().manual_seed(N)
    d = 128
    q, k, v = (torch.randn(N, d, generator=g, dtype=torch.float64).numpy() for _ in range(3))
    q = q * qm
    scale = 1 / math.sqrt(d)
    o8 = _o_with_e4m3_p(q, k, v, scale, causal, stale * tau, tau)
    s = (q @ k.T) * scale
    if causal:
        s = np.where(np.tri(N, dtype=bool), s, -np.inf)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    compare_o_e4m3(o8, p @ v, p @ np.abs(v), f"N{N} causal={causal} qx{qm} stale{stale} tau{tau}")


def test_without_the_factor_peaked_rows_break_the_bar():
    """tau = 8 leaves no room for the factor: peaked rows then lose mass to E4M3's
    subnormal range and the bound fails -- the reason for the factor."""
    g = torch.Generator().manual_seed(384)
    q, k, v = (torch.randn(384, 128, generator=g, dtype=torch.float64).numpy() for _ in range(3))
    q = q * 4.0
    scale = 1 / math.sqrt(128)
    o8 = _o_with_e4m3_p(q, k, v, scale, False, 0.0, 8.0)
    s = (q @ k.T) * scale
    p = np.exp(s - s.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    with pytest.raises(AssertionError):
        compare_o_e4m3(o8, p @ v, p @ np.abs(v))
