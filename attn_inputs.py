"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds no attention arithmetic: it only draws random tensors and names
the workload shapes, so both the CUDA library's callers and the fp64 oracle can be
fed identical inputs.

Recipe: a CPU ``torch.Generator`` seeded per call; ``torch.randn`` in fp32, then a
cast to bf16 (so every value is exactly representable in both the bf16 kernel
inputs and the fp64 oracle).  Tensors are drawn in the order Q, K, V (then dO)
with shape ``[B, N, H, d]`` (dense) or ``[T, H, d]`` (packed variable length).
Variable-length batches draw their lengths uniformly from ``[lo, hi]`` with their
own generator (seed 1).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Tuple

import torch


@dataclass(frozen=True)
class Workload:
    """One attention forward problem: dense ``[B,N,H,d]`` or packed varlen."""
    name: str
    B: int
    H: int
    N: int              # dense sequence length, or the maximum length when varlen
    d: int
    causal: bool
    q_mult: float = 1.0  # exact power-of-two multiplier applied to the bf16 Q
    lengths: Optional[List[int]] = field(default=None)  # varlen sequence lengths
    # sliding window (left, right): key j visible to query i iff i-left <= j <= i+right
    window: Optional[Tuple[int, int]] = None
    e4m3: bool = False  # inputs quantised per tensor to E4M3 (see to_e4m3)

    @property
    def varlen(self) -> bool:
        return self.lengths is not None

    @property
    def total_tokens(self) -> int:
        return sum(self.lengths) if self.varlen else self.B * self.N

    def seq_lengths(self) -> List[int]:
        return list(self.lengths) if self.varlen else [self.N] * self.B

    def cu_seqlens(self) -> List[int]:
        cu = [0]
        for L in self.seq_lengths():
            cu.append(cu[-1] + L)
        return cu


def varlen_lengths(n: int = 16, lo: int = 512, hi: int = 16384, seed: int = 1) -> List[int]:
    """Sequence lengths uniform in [lo, hi] from their own seeded generator."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    return [int(x) for x in torch.randint(lo, hi + 1, (n,), generator=g)]


# The benchmark problems: tiny latency case, dense non-causal (and a variant with
# Q scaled by 4 so the running maximum moves often), long causal, packed causal
# varlen, the long causal problem under a 1024-key sliding window, the dense and
# long causal problems with E4M3 inputs, and the causal backward problem.
TINY = Workload("B1-H1-N256-d64", 1, 1, 256, 64, False)
DENSE = Workload("B4-H16-N2048-d128", 4, 16, 2048, 128, False)
DENSE_X4 = Workload("B4-H16-N2048-d128-qx4", 4, 16, 2048, 128, False, q_mult=4.0)
CAUSAL = Workload("B2-H16-N8192-d128-causal", 2, 16, 8192, 128, True)
_VL = varlen_lengths()
VARLEN = Workload("varlen16-H16-d128-causal", len(_VL), 16, max(_VL), 128, True, lengths=_VL)
WINDOW = Workload("B2-H16-N8192-d128-causal-win1024", 2, 16, 8192, 128, True, window=(1024, 0))
DENSE_E4M3 = Workload("B4-H16-N2048-d128-e4m3", 4, 16, 2048, 128, False, e4m3=True)
CAUSAL_E4M3 = Workload("B2-H16-N8192-d128-causal-e4m3", 2, 16, 8192, 128, True, e4m3=True)
BWD_CAUSAL = CAUSAL  # the backward problem uses the causal forward's shapes
BWD_NAME = CAUSAL.name + "-bwd"

ALL = {w.name: w for w in (TINY, DENSE, DENSE_X4, CAUSAL, VARLEN, WINDOW, DENSE_E4M3,
                           CAUSAL_E4M3)}


def make_qkv(w: Workload, seed: int = 0, with_dout: bool = False):
    """bf16 CPU tensors (q, k, v[, dout]) for workload ``w``.

    Dense: ``[B, N, H, d]``.  Varlen: ``[T, H, d]``.
    """
    g = torch.Generator(device="cpu").manual_seed(seed)
    shape = (w.total_tokens, w.H, w.d) if w.varlen else (w.B, w.N, w.H, w.d)
    out = []
    for _ in range(4 if with_dout else 3):
        out.append(torch.randn(shape, generator=g, dtype=torch.float32).to(torch.bfloat16))
    if w.q_mult != 1.0:
        out[0] = (out[0].float() * w.q_mult).to(torch.bfloat16)
    return tuple(out)


def to_e4m3(x: torch.Tensor):
    """Per-tensor 8-bit copy of a CPU tensor for the E4M3 entry point: returns
    (x8, scale) with x8 = e4m3(x / scale) (torch's float8_e4m3fn rounding) and
    scale the power of two that puts max|x| just below 448, so x8 * scale is the
    8-bit input the kernel sees (exactly representable in fp32 and fp64)."""
    import math
    amax = float(x.abs().max())
    scale = 2.0 ** math.ceil(math.log2(amax / 448.0)) if amax > 0 else 1.0
    return (x.float() / scale).to(torch.float8_e4m3fn), scale


def make_qkv_e4m3(w: Workload, seed: int = 0):
    """The bf16 draws of ``make_qkv`` quantised per tensor: (q8, k8, v8, scales)."""
    out, scales = [], []
    for t in make_qkv(w, seed):
        t8, sc = to_e4m3(t)
        out.append(t8)
        scales.append(sc)
    return out[0], out[1], out[2], tuple(scales)


def make_custom(B: int, N: int, H: int, d: int, seed: int = 0, lengths=None, n: int = 3,
                std: float = 1.0):
    """Generic seeded bf16 tensors for test shapes (dense when ``lengths`` is None)."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    shape = (sum(lengths), H, d) if lengths is not None else (B, N, H, d)
    return tuple((torch.randn(shape, generator=g, dtype=torch.float32) * std).to(torch.bfloat16)
                 for _ in range(n))
