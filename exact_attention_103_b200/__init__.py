"""Python binding of libattn: B200-native exact attention.

Argument marshalling only.  Every step of the computation runs in the CUDA
library ``libattn.so`` (built in-tree by ``build.py``); this module checks torch
tensors, allocates outputs with torch, and passes raw device pointers and the
current CUDA stream through the C ABI declared in ``include/attn.h``.  There is no
fallback: if the library is missing or the device is not an sm_100 GPU, calls
raise.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libattn.so")

ATTN_OK, ATTN_ERR_INVALID_ARG, ATTN_ERR_UNSUPPORTED = 0, 1, 2
ATTN_ERR_CUDA, ATTN_ERR_TIMEOUT, ATTN_ERR_WORKSPACE = 3, 4, 5

# Every symbol include/attn.h and include/attn_selftest.h declare.
EXPORTED_SYMBOLS = ("attn_fwd", "attn_fwd_ex", "attn_bwd", "attn_bwd_workspace_size",
                    "attn_get_device_status", "attn_status_string", "attn_last_error",
                    "attn_selftest_umma", "attn_fwd_noalloc", "attn_fwd_e4m3",
                    "attn_selftest_umma_e4m3", "attn_bwd_ex", "attn_selftest_exp2")


class AttnError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{status_string(status) if _lib else status}: {message}")
        self.status = status


class BwdOpts(ctypes.Structure):
    _fields_ = [("has_window", ctypes.c_int),
                ("window_left", ctypes.c_int),
                ("window_right", ctypes.c_int),
                ("timeout_ns", ctypes.c_uint64),
                ("total_tokens", ctypes.c_int64)]


class FwdOpts(ctypes.Structure):
    _fields_ = [("rescale_threshold", ctypes.c_float),
                ("stats", ctypes.c_void_p),
                ("timeout_ns", ctypes.c_uint64),
                ("total_tokens", ctypes.c_int64),
                ("test_fault", ctypes.c_int),
                ("has_window", ctypes.c_int),
                ("window_left", ctypes.c_int),
                ("window_right", ctypes.c_int),
                ("exp_poly_per8", ctypes.c_int),
                ("cta_pair", ctypes.c_int)]


_lib = None


def load_library(path: str = LIB_PATH):
    """Loads libattn.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libattn.so not found at {path}; build it with "
                           "`python -m exact_attention_103_b200.build`")
    lib = ctypes.CDLL(path)
    vp, ci, cf, cs = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.attn_fwd.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, vp, vp]
    lib.attn_fwd.restype = ci
    lib.attn_fwd_ex.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, vp,
                                ctypes.POINTER(FwdOpts), vp]
    lib.attn_fwd_ex.restype = ci
    lib.attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, vp, ci,
                             vp, cs, vp]
    lib.attn_bwd.restype = ci
    lib.attn_bwd_ex.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, vp, ci,
                                vp, cs, ctypes.POINTER(BwdOpts), vp]
    lib.attn_bwd_ex.restype = ci
    lib.attn_bwd_workspace_size.argtypes = [ci, ci, ci, ci, ci, ci]
    lib.attn_bwd_workspace_size.restype = cs
    lib.attn_get_device_status.argtypes = [vp]
    lib.attn_get_device_status.restype = ci
    lib.attn_status_string.argtypes = [ci]
    lib.attn_status_string.restype = ctypes.c_char_p
    lib.attn_last_error.argtypes = []
    lib.attn_last_error.restype = ctypes.c_char_p
    lib.attn_selftest_umma.argtypes = [vp, vp, vp, vp, vp, ci, vp]
    lib.attn_selftest_umma.restype = ci
    lib.attn_selftest_umma_e4m3.argtypes = [vp, vp, vp, vp, vp, vp]
    lib.attn_selftest_umma_e4m3.restype = ci
    lib.attn_fwd_e4m3.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, cf, cf, cf, vp,
                                  ctypes.POINTER(FwdOpts), vp]
    lib.attn_fwd_e4m3.restype = ci
    lib.attn_selftest_exp2.argtypes = [vp, vp, vp, vp, ci, vp]
    lib.attn_selftest_exp2.restype = ci
    lib.attn_fwd_noalloc.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, vp,
                                     ctypes.c_int64, ci, vp]
    lib.attn_fwd_noalloc.restype = ci
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load_library().attn_status_string(status).decode()


def last_error() -> str:
    return load_library().attn_last_error().decode()


def _check(status: int):
    if status != ATTN_OK:
        raise AttnError(status, last_error())


def _stream_ptr(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _need(t: torch.Tensor, name: str, dtype=torch.bfloat16):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
        scale: Optional[float] = None, cu_seqlens: Optional[torch.Tensor] = None,
        max_seqlen: Optional[int] = None, out: Optional[torch.Tensor] = None,
        lse: Optional[torch.Tensor] = None, rescale_threshold: Optional[float] = None,
        stats: Optional[torch.Tensor] = None, timeout_ns: int = 0,
        stream: Optional[torch.cuda.Stream] = None,
        test_fault: int = 0, window: Optional[Tuple[int, int]] = None,
        exp_poly_per8: int = 0,
        e4m3_scales: Optional[Tuple[float, float, float]] = None,
        cta_pair: bool = False
        ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Exact attention forward on the GPU.

    Dense: q, k, v are bf16 ``[B, N, H, d]``; returns O ``[B, N, H, d]`` and LSE
    ``[B, H, N]`` (fp32, natural log).  Varlen: q, k, v are packed ``[T, H, d]``,
    ``cu_seqlens`` is int32 ``[B+1]`` on the device and ``max_seqlen`` the longest
    sequence; LSE is ``[H, T]``.  ``scale`` defaults to ``1/sqrt(d)``.
    ``window = (left, right)`` keeps key j for query i only if
    ``i - left <= j <= i + right`` (negative = open side).  ``exp_poly_per8``
    (0, 2 or 8) moves that many of every 8 exponential pairs to the FMA pipe.
    ``e4m3_scales = (q_scale, k_scale, v_scale)`` selects the 8-bit entry point
    ``attn_fwd_e4m3``: q, k, v are then ``torch.float8_e4m3fn`` holding the real
    inputs divided by those per-tensor scales; O is still bf16.  ``cta_pair``
    runs the forward in clusters of two CTAs sharing each 512-row item
    (tcgen05.mma.cta_group::2; bf16, d = 128).
    """
    lib = load_library()
    in_dtype = torch.bfloat16 if e4m3_scales is None else torch.float8_e4m3fn
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, in_dtype)
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must have the same shape")
    d = q.shape[-1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    opts = FwdOpts(-1.0 if rescale_threshold is None else float(rescale_threshold),
                   None if stats is None else stats.data_ptr(), int(timeout_ns), 0, int(test_fault),
                   0 if window is None else 1, -1 if window is None else int(window[0]),
                   -1 if window is None else int(window[1]), int(exp_poly_per8),
                   int(bool(cta_pair)))
    if stats is not None:
        _need(stats, "stats", torch.int64)
    if cu_seqlens is None:
        if q.dim() != 4:
            raise ValueError("dense q must be [B, N, H, d]")
        B, N, H, _ = q.shape
        lse_shape = (B, H, N)
    else:
        if q.dim() != 3:
            raise ValueError("varlen q must be [T, H, d]")
        _need(cu_seqlens, "cu_seqlens", torch.int32)
        B = cu_seqlens.numel() - 1
        H = q.shape[1]
        if max_seqlen is None:
            raise ValueError("varlen needs max_seqlen")
        N = int(max_seqlen)
        lse_shape = (H, q.shape[0])
        opts.total_tokens = q.shape[0]
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    else:
        _need(out, "out")
        if out.shape != q.shape:
            raise ValueError("out has the wrong shape")
    if lse is None:
        lse = torch.empty(lse_shape, dtype=torch.float32, device=q.device)
    else:
        _need(lse, "lse", torch.float32)
        if tuple(lse.shape) != lse_shape:
            raise ValueError("lse has the wrong shape")
    if cu_seqlens is not None and q.shape[0] == 0:
        return out, lse
    cu_ptr = None if cu_seqlens is None else cu_seqlens.data_ptr()
    with torch.cuda.device(q.device):
        if e4m3_scales is None:
            st = lib.attn_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                 lse.data_ptr(), B, H, N, d, int(bool(causal)), float(scale),
                                 cu_ptr, ctypes.byref(opts), _stream_ptr(stream))
        else:
            qs, ks, vs = (float(x) for x in e4m3_scales)
            st = lib.attn_fwd_e4m3(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                   lse.data_ptr(), B, H, N, d, int(bool(causal)), float(scale),
                                   qs, ks, vs, cu_ptr, ctypes.byref(opts), _stream_ptr(stream))
    _check(st)
    return out, lse


def fwd_raw(q_ptr: int, k_ptr: int, v_ptr: int, o_ptr: int, lse_ptr: int, B: int, H: int, N: int,
            d: int, causal: bool, scale: float, cu_ptr: Optional[int] = None,
            stream_ptr: int = 0) -> None:
    """The plain C entry point ``attn_fwd`` on raw device pointers."""
    _check(load_library().attn_fwd(q_ptr, k_ptr, v_ptr, o_ptr, lse_ptr, B, H, N, d,
                                   int(bool(causal)), float(scale), cu_ptr, stream_ptr))


def fwd_from_host(q_host: torch.Tensor, k_host: torch.Tensor, v_host: torch.Tensor,
                  causal: bool = False, scale: Optional[float] = None,
                  cu_seqlens_host: Optional[torch.Tensor] = None,
                  max_seqlen: Optional[int] = None, device: str = "cuda",
                  stream: Optional[torch.cuda.Stream] = None,
                  out_host: Optional[torch.Tensor] = None,
                  lse_host: Optional[torch.Tensor] = None,
                  window: Optional[Tuple[int, int]] = None, exp_poly_per8: int = 0,
                  e4m3_scales: Optional[Tuple[float, float, float]] = None):
    """End-to-end call from host tensors: copies Q/K/V (and cu_seqlens) to the
    device, runs the forward, copies O and LSE back into host tensors (``out_host``
    / ``lse_host`` if given, ideally pinned; else new pinned tensors).  Returns
    (o_host, lse_host); they are complete once ``stream`` is synchronised."""
    s = stream if stream is not None else torch.cuda.current_stream()
    with torch.cuda.stream(s):
        q = q_host.to(device, non_blocking=True)
        k = k_host.to(device, non_blocking=True)
        v = v_host.to(device, non_blocking=True)
        cu = None if cu_seqlens_host is None else cu_seqlens_host.to(device, non_blocking=True)
        o, lse = fwd(q, k, v, causal=causal, scale=scale, cu_seqlens=cu, max_seqlen=max_seqlen,
                     stream=s, window=window, exp_poly_per8=exp_poly_per8,
                     e4m3_scales=e4m3_scales)
        o_h = out_host if out_host is not None else torch.empty(o.shape, dtype=o.dtype,
                                                                pin_memory=True)
        l_h = lse_host if lse_host is not None else torch.empty(lse.shape, dtype=lse.dtype,
                                                                pin_memory=True)
        o_h.copy_(o, non_blocking=True)
        l_h.copy_(lse, non_blocking=True)
    return o_h, l_h


class HostPipeline:
    """End-to-end forward from pinned host memory with the copies of neighbouring
    calls overlapped: call k's host-to-device copy runs while call k-1 computes and
    call k-2's results travel back, on three streams (copy in, compute, copy out)
    ordered by events.  ``depth`` device buffer sets rotate; every call still moves
    its own inputs to the device and its own O and LSE back.  Only plumbing lives
    here: the attention itself is ``fwd`` (the C ABI).

    ``shape``: the q/k/v shape of every call (dense ``[B,N,H,d]`` or packed
    ``[T,H,d]``); the other arguments are those of ``fwd``.
    """

    def __init__(self, shape, causal: bool = False, scale: Optional[float] = None,
                 cu_seqlens_host: Optional[torch.Tensor] = None, max_seqlen: Optional[int] = None,
                 device: str = "cuda", depth: int = 2,
                 window: Optional[Tuple[int, int]] = None, exp_poly_per8: int = 0,
                 e4m3_scales: Optional[Tuple[float, float, float]] = None):
        if depth < 1:
            raise ValueError("depth must be >= 1")
        self.dev = torch.device(device)
        self.kw = dict(causal=causal, scale=scale, max_seqlen=max_seqlen, window=window,
                       exp_poly_per8=exp_poly_per8, e4m3_scales=e4m3_scales)
        self.cu_host = cu_seqlens_host
        in_dtype = torch.bfloat16 if e4m3_scales is None else torch.float8_e4m3fn
        shape = tuple(shape)
        if cu_seqlens_host is None:
            B, N, H, _ = shape
            lse_shape = (B, H, N)
        else:
            lse_shape = (shape[1], shape[0])
        self.streams = [torch.cuda.Stream(self.dev) for _ in range(3)]
        self.slots = []
        for _ in range(depth):
            slot = {n: torch.empty(shape, dtype=in_dtype, device=self.dev) for n in ("q", "k", "v")}
            slot["o"] = torch.empty(shape, dtype=torch.bfloat16, device=self.dev)
            slot["lse"] = torch.empty(lse_shape, dtype=torch.float32, device=self.dev)
            slot["cu"] = (None if cu_seqlens_host is None else
                          torch.empty(cu_seqlens_host.shape, dtype=torch.int32, device=self.dev))
            for e in ("loaded", "computed", "drained"):
                slot[e] = torch.cuda.Event()
            self.slots.append(slot)
        self.calls = 0

    def submit(self, q_host: torch.Tensor, k_host: torch.Tensor, v_host: torch.Tensor,
               out_host: torch.Tensor, lse_host: torch.Tensor) -> torch.cuda.Event:
        """Queues one call; returns the event after which out_host / lse_host hold it."""
        h2d, comp, d2h = self.streams
        slot = self.slots[self.calls % len(self.slots)]
        self.calls += 1
        h2d.wait_event(slot["computed"])  # the slot's previous inputs have been read
        with torch.cuda.stream(h2d):
            for n, t in (("q", q_host), ("k", k_host), ("v", v_host)):
                slot[n].copy_(t, non_blocking=True)
            if slot["cu"] is not None:
                slot["cu"].copy_(self.cu_host, non_blocking=True)
            slot["loaded"].record(h2d)
        comp.wait_event(slot["loaded"])
        comp.wait_event(slot["drained"])  # the slot's previous outputs have left
        fwd(slot["q"], slot["k"], slot["v"], cu_seqlens=slot["cu"], out=slot["o"],
            lse=slot["lse"], stream=comp, **self.kw)
        slot["computed"].record(comp)
        d2h.wait_event(slot["computed"])
        with torch.cuda.stream(d2h):
            out_host.copy_(slot["o"], non_blocking=True)
            lse_host.copy_(slot["lse"], non_blocking=True)
            slot["drained"].record(d2h)
        return slot["drained"]

    def synchronize(self) -> None:
        for st in self.streams:
            st.synchronize()


def fwd_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
                lse: torch.Tensor, causal: bool = False, scale: Optional[float] = None,
                cu_seqlens: Optional[torch.Tensor] = None, max_seqlen: Optional[int] = None,
                total_tokens: Optional[int] = None, check: bool = True,
                stream: Optional[torch.cuda.Stream] = None) -> None:
    """The allocation-free forward ``attn_fwd_noalloc``: the caller supplies ``out``
    and ``lse`` (layouts as for ``fwd``); the library allocates no device memory.
    Varlen: ``total_tokens`` must equal ``cu_seqlens[B]`` (default: ``q.shape[0]``;
    pass it for a packed buffer longer than the batch).  With ``check`` the call
    synchronises the stream and raises on a kernel-recorded error; without it that
    status is not reported anywhere."""
    lib = load_library()
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out")):
        _need(t, n)
    _need(lse, "lse", torch.float32)
    d = q.shape[-1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if cu_seqlens is None:
        B, N, H, _ = q.shape
        total, cu_ptr = 0, None
    else:
        _need(cu_seqlens, "cu_seqlens", torch.int32)
        B, H, N = cu_seqlens.numel() - 1, q.shape[1], int(max_seqlen)
        total = q.shape[0] if total_tokens is None else int(total_tokens)
        cu_ptr = cu_seqlens.data_ptr()
    with torch.cuda.device(q.device):
        st = lib.attn_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                  lse.data_ptr(), B, H, N, d, int(bool(causal)), float(scale),
                                  cu_ptr, total, int(bool(check)), _stream_ptr(stream))
    _check(st)


def bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, lse: torch.Tensor,
        dout: torch.Tensor, causal: bool = False, scale: Optional[float] = None,
        cu_seqlens: Optional[torch.Tensor] = None, max_seqlen: Optional[int] = None,
        deterministic: bool = False, stream: Optional[torch.cuda.Stream] = None,
        window: Optional[Tuple[int, int]] = None):
    """Exact attention backward on the GPU: returns (dq, dk, dv), bf16, layout of q.

    ``o`` and ``lse`` are the forward's outputs (``window`` as given to ``fwd``).
    The workspace (the per-row <dO, O>) is allocated with torch.  Results are
    bitwise reproducible whether or not ``deterministic`` is set."""
    lib = load_library()
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout")):
        _need(t, n)
    _need(lse, "lse", torch.float32)
    d = q.shape[-1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if cu_seqlens is None:
        B, N, H, _ = q.shape
        total, cu_ptr = B * N, None
    else:
        _need(cu_seqlens, "cu_seqlens", torch.int32)
        B, H, N = cu_seqlens.numel() - 1, q.shape[1], int(max_seqlen)
        total, cu_ptr = q.shape[0], cu_seqlens.data_ptr()
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ws_bytes = lib.attn_bwd_workspace_size(B, H, N, d, total, int(bool(deterministic)))
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=q.device)
    with torch.cuda.device(q.device):
        opts = BwdOpts(0 if window is None else 1, -1 if window is None else int(window[0]),
                       -1 if window is None else int(window[1]), 0,
                       0 if cu_seqlens is None else int(total))
        st = lib.attn_bwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                             lse.data_ptr(), dout.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                             dv.data_ptr(), B, H, N, d, int(bool(causal)), float(scale), cu_ptr,
                             int(bool(deterministic)), ws.data_ptr(), ws.numel(),
                             ctypes.byref(opts), _stream_ptr(stream))
    _check(st)
    return dq, dk, dv


def get_device_status(stream: Optional[torch.cuda.Stream] = None) -> None:
    """Synchronises the stream; raises AttnError if a kernel recorded an error."""
    _check(load_library().attn_get_device_status(_stream_ptr(stream)))


def selftest_umma_e4m3(a: torch.Tensor, b: torch.Tensor, v: torch.Tensor):
    """The one-tile check of the 8-bit path: a, b, v are float8_e4m3fn [128, 128];
    returns (S = A B^T, O = e4m3(S) V), fp32."""
    for t, n in ((a, "a"), (b, "b"), (v, "v")):
        _need(t, n, torch.float8_e4m3fn)
        if tuple(t.shape) != (128, 128):
            raise ValueError(f"{n} must be [128, 128]")
    s_out = torch.empty((128, 128), dtype=torch.float32, device=a.device)
    o_out = torch.empty((128, 128), dtype=torch.float32, device=a.device)
    _check(load_library().attn_selftest_umma_e4m3(a.data_ptr(), b.data_ptr(), v.data_ptr(),
                                                  s_out.data_ptr(), o_out.data_ptr(),
                                                  _stream_ptr(None)))
    return s_out, o_out


def selftest_exp2(x: torch.Tensor):
    """The forward kernel's FMA-pipe exponential on a CUDA fp32 tensor x: returns
    (packed form, scalar form, exp2f), each like x."""
    _need(x, "x", torch.float32)
    outs = [torch.empty_like(x) for _ in range(3)]
    _check(load_library().attn_selftest_exp2(x.data_ptr(), outs[0].data_ptr(), outs[1].data_ptr(),
                                             outs[2].data_ptr(), x.numel(), _stream_ptr(None)))
    return tuple(outs)


def selftest_umma(a: torch.Tensor, b: torch.Tensor, v: torch.Tensor):
    """Runs the one-tile tensor-core check: returns (S = A B^T, O = bf16(S) V), fp32."""
    for t, n in ((a, "a"), (b, "b"), (v, "v")):
        _need(t, n)
    d = a.shape[1]
    s_out = torch.empty((128, 128), dtype=torch.float32, device=a.device)
    o_out = torch.empty((128, d), dtype=torch.float32, device=a.device)
    _check(load_library().attn_selftest_umma(a.data_ptr(), b.data_ptr(), v.data_ptr(),
                                             s_out.data_ptr(), o_out.data_ptr(), d,
                                             _stream_ptr(None)))
    return s_out, o_out
