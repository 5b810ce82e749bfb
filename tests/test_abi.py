"""The C ABI without a GPU: the library loads, exports every symbol the public
headers declare, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

import exact_attention_103_b200 as ea
from exact_attention_103_b200 import build as ea_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    ea_build.build()
    return ea.load_library()


def _declared_symbols():
    names = set()
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            names |= set(re.findall(r"ATTN_API\s+[^;(]*?\b(attn_\w+)\s*\(", text))
    return names


def test_every_declared_symbol_is_exported(lib):
    declared = _declared_symbols()
    assert {"attn_fwd", "attn_fwd_ex", "attn_bwd", "attn_get_device_status"} <= declared
    for name in declared:
        assert hasattr(lib, name), name
    assert declared == set(ea.EXPORTED_SYMBOLS)


def test_status_strings(lib):
    for code, name in enumerate(["ATTN_OK", "ATTN_ERR_INVALID_ARG", "ATTN_ERR_UNSUPPORTED",
                                 "ATTN_ERR_CUDA", "ATTN_ERR_TIMEOUT", "ATTN_ERR_WORKSPACE"]):
        assert ea.status_string(code) == name


FAKE = 0x10000  # 16-byte aligned, never dereferenced: validation returns first


def _fwd(lib, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, H=1, N=128, d=128, causal=0,
         scale=0.125, cu=None):
    return lib.attn_fwd(q, k, v, o, lse, B, H, N, d, causal, scale, cu, None)


def test_unsupported_head_dim(lib):
    assert _fwd(lib, d=96) == ea.ATTN_ERR_UNSUPPORTED
    assert "head dim" in ea.last_error()


@pytest.mark.parametrize("scale", [0.0, -1.0, float("inf"), float("nan")])
def test_bad_scale(lib, scale):
    assert _fwd(lib, scale=scale) == ea.ATTN_ERR_INVALID_ARG


def test_null_and_misaligned_pointers(lib):
    assert _fwd(lib, q=None) == ea.ATTN_ERR_INVALID_ARG
    assert _fwd(lib, o=None) == ea.ATTN_ERR_INVALID_ARG
    assert _fwd(lib, k=FAKE + 8) == ea.ATTN_ERR_INVALID_ARG
    assert _fwd(lib, lse=FAKE + 2) == ea.ATTN_ERR_INVALID_ARG


def test_negative_sizes(lib):
    assert _fwd(lib, B=-1) == ea.ATTN_ERR_INVALID_ARG
    assert _fwd(lib, H=0) == ea.ATTN_ERR_INVALID_ARG
    assert _fwd(lib, N=-5) == ea.ATTN_ERR_INVALID_ARG


def test_empty_problem_is_a_noop(lib):
    # Nothing is launched, so this succeeds without a device.
    assert _fwd(lib, B=0) == ea.ATTN_OK
    assert _fwd(lib, N=0, q=None) == ea.ATTN_OK


def test_varlen_limits(lib):
    assert _fwd(lib, B=1025, cu=FAKE) == ea.ATTN_ERR_UNSUPPORTED
    assert _fwd(lib, B=2, N=131073, cu=FAKE) == ea.ATTN_ERR_UNSUPPORTED
    assert _fwd(lib, B=2, cu=FAKE + 2) == ea.ATTN_ERR_INVALID_ARG


def test_bad_options(lib):
    for opts in (ea.FwdOpts(float("inf"), None, 0, 0, 0), ea.FwdOpts(65.0, None, 0, 0, 0),
                 ea.FwdOpts(-1.0, None, 0, 0, 2), ea.FwdOpts(-1.0, None, 0, 0, 0, 0, 0, 0, 3),
                 ea.FwdOpts(-1.0, None, 0, 0, 0, 0, 0, 0, -1)):
        st = lib.attn_fwd_ex(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 128, 0, 0.1, None,
                             ctypes.byref(opts), None)
        assert st == ea.ATTN_ERR_INVALID_ARG


def test_window_limit(lib):
    opts = ea.FwdOpts(-1.0, None, 0, 0, 0, 1, 64, 0, 0)
    st = lib.attn_fwd_ex(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 1 << 30, 64, 1, 0.1, None,
                         ctypes.byref(opts), None)
    assert st == ea.ATTN_ERR_UNSUPPORTED
    assert "window" in ea.last_error()


def test_backward_argument_checks(lib):
    def bwd(d=128, scale=0.1, B=1, dq=FAKE):
        return lib.attn_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, dq, FAKE, FAKE, B, 1, 128, d, 0,
                            scale, None, 0, None, 0, None)
    assert bwd(d=96) == ea.ATTN_ERR_UNSUPPORTED
    assert bwd(scale=0.0) == ea.ATTN_ERR_INVALID_ARG
    assert bwd(dq=None) == ea.ATTN_ERR_INVALID_ARG
    assert bwd(dq=FAKE + 4) == ea.ATTN_ERR_INVALID_ARG
    assert bwd(B=0) == ea.ATTN_OK


def test_backward_workspace_size(lib):
    # one fp32 per (token, head), rounded up to 256 bytes
    assert lib.attn_bwd_workspace_size(2, 16, 8192, 128, 2 * 8192, 0) == 2 * 8192 * 16 * 4
    assert lib.attn_bwd_workspace_size(1, 3, 5, 64, 5, 1) == 256
    assert lib.attn_bwd_workspace_size(0, 3, 5, 64, 0, 1) == 0


def test_e4m3_argument_checks(lib):
    def call(d=128, qs=1.0, opts=None, B=1):
        return lib.attn_fwd_e4m3(FAKE, FAKE, FAKE, FAKE, FAKE, B, 1, 128, d, 0, 0.1, qs, 1.0, 1.0,
                                 None, None if opts is None else ctypes.byref(opts), None)
    assert call(d=64) == ea.ATTN_ERR_UNSUPPORTED
    assert call(qs=0.0) == ea.ATTN_ERR_INVALID_ARG
    assert call(qs=float("nan")) == ea.ATTN_ERR_INVALID_ARG
    assert call(opts=ea.FwdOpts(-1.0, None, 0, 0, 0, 0, 0, 0, 8)) == ea.ATTN_ERR_UNSUPPORTED
    assert call(opts=ea.FwdOpts(9.0, None, 0, 0, 0, 0, 0, 0, 0)) == ea.ATTN_ERR_INVALID_ARG
    assert call(B=0) == ea.ATTN_OK


def test_backward_window_limit(lib):
    opts = ea.BwdOpts(1, 64, 0, 0)
    st = lib.attn_bwd_ex(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 1 << 30, 64,
                         1, 0.1, None, 0, None, 0, ctypes.byref(opts), None)
    assert st == ea.ATTN_ERR_UNSUPPORTED


def test_missing_library_fails_loudly():
    """No fallback: without the built library the binding raises (run in a fresh
    interpreter so the already-loaded library is not reused)."""
    import subprocess
    import sys
    code = ("import exact_attention_103_b200 as ea\n"
            "try:\n"
            "    ea.load_library('/nonexistent/libattn.so')\n"
            "except RuntimeError as e:\n"
            "    print('raised', 'not found' in str(e))\n")
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, cwd=ROOT,
                       timeout=300)
    assert r.stdout.strip() == "raised True", r.stdout + r.stderr


def test_cta_pair_limits(lib):
    """CTA pairs run bf16, d = 128, all-MUFU exponentials only."""
    for d, poly in ((64, 0), (128, 2)):
        opts = ea.FwdOpts(-1.0, None, 0, 0, 0, 0, 0, 0, poly, 1)
        st = lib.attn_fwd_ex(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, d, 0, 0.1, None,
                             ctypes.byref(opts), None)
        assert st == ea.ATTN_ERR_UNSUPPORTED, (d, poly)
        assert "cta_pair" in ea.last_error()
    opts = ea.FwdOpts(-1.0, None, 0, 0, 0, 0, 0, 0, 0, 1)
    st = lib.attn_fwd_e4m3(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 128, 0, 0.1, 1.0, 1.0, 1.0, None,
                           ctypes.byref(opts), None)
    assert st == ea.ATTN_ERR_UNSUPPORTED
