"""The forward kernel's FMA-pipe exponential on the GPU (attn_selftest_exp2): over
a dense grid of the range the kernel feeds it, the packed two-lane form equals the
scalar form bit for bit, equals the CPU float32 emulation of the same steps bit for
bit, and stays within the relative-error bound exp2_poly.h states against CUDA's
exp2f (whose own error, at most 2 ulp, is added to the bound)."""
import numpy as np
import pytest
import torch

from test_exp2_poly_cpu import _constants, _exp2_poly

pytestmark = pytest.mark.gpu


def test_exp2_poly_on_device_against_exp2f():
    import exact_attention_103_b200 as ea
    _, bound = _constants()
    x = np.concatenate([np.linspace(-124.0, 64.0, 4_000_001, dtype=np.float32),
                        np.array([-125.0, -126.0, -1000.0, -np.inf, 0.0, 1.0, -0.5, 0.5],
                                 dtype=np.float32)])
    xd = torch.from_numpy(x).cuda()
    y_poly, y_scalar, y_ref = (t.cpu().numpy() for t in ea.selftest_exp2(xd))
    torch.cuda.synchronize()
    assert np.array_equal(y_poly.view(np.uint32), y_scalar.view(np.uint32))
    assert np.array_equal(y_poly.view(np.uint32), _exp2_poly(x).view(np.uint32))
    ok = x >= -124.0
    rel = np.abs(y_poly[ok].astype(np.float64) / y_ref[ok].astype(np.float64) - 1.0)
    assert rel.max() <= bound * 1.01 + 2.5e-7, rel.max()
    assert np.all(np.isfinite(y_poly)) and np.all(y_poly > 0)
