"""Comparison helpers for GPU-vs-oracle parity tests (no attention arithmetic here).

Tolerances (forward): max-abs error of O <= 1e-2 plus half a bf16 ulp of the exact
value (the output is bf16, so rounding the exact result alone can cost half an
ulp: 1.6e-2 where |O| >= 4), relative L2 error of O <= 5e-3, LSE abs error <= 1e-3.
"""
from __future__ import annotations

import numpy as np
import torch

O_MAX_ABS = 1e-2
O_REL_L2 = 5e-3
LSE_ABS = 1e-3


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    """Half the bf16 spacing at |x| (8 significant bits)."""
    ax = np.abs(x)
    e = np.floor(np.log2(np.maximum(ax, 2.0 ** -126)))
    return 2.0 ** (e - 8)


def to_np(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().float().cpu().double().numpy()
    return np.asarray(t, dtype=np.float64)


def compare_o(o_gpu, o_ref, label: str = ""):
    """Asserts the forward-output bar; returns (raw max-abs, rel-L2)."""
    o, r = to_np(o_gpu), to_np(o_ref)
    assert o.shape == r.shape, (o.shape, r.shape)
    assert np.all(np.isfinite(o)), f"{label}: non-finite output"
    err = np.abs(o - r)
    bound = O_MAX_ABS + bf16_half_ulp(r)
    worst = np.argmax(err - bound)
    assert np.all(err <= bound), (
        f"{label}: |O-O_ref| = {err.flat[worst]:.3e} at {np.unravel_index(worst, err.shape)} "
        f"exceeds {bound.flat[worst]:.3e} (ref {r.flat[worst]:.4f}, got {o.flat[worst]:.4f})")
    rel = float(np.linalg.norm(o - r) / max(np.linalg.norm(r), 1e-30))
    assert rel <= O_REL_L2, f"{label}: rel-L2 {rel:.3e} > {O_REL_L2}"
    return float(err.max()), rel


def compare_lse(lse_gpu, lse_ref, label: str = ""):
    l, r = to_np(lse_gpu), to_np(lse_ref)
    assert l.shape == r.shape, (l.shape, r.shape)
    err = np.abs(l - r)
    assert np.all(err <= LSE_ABS), f"{label}: LSE error {err.max():.3e} > {LSE_ABS}"
    return float(err.max())
