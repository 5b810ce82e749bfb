"""The pins are strong enough to catch plausible mistakes: each case plants one
mistake in a private copy of the oracle's C source (never in the oracle itself),
builds it, and checks that a pin from test_oracle_pins.py's families fails on it
while the real oracle passes the same check.  Each case runs in a fresh Python
process, so no mutant library shares a process (or a dlopen namespace) with the
real oracle or with another mutant."""
import importlib.util
import math
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
from attn_inputs import make_custom

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "attn_oracle.c")


def _mutant(tmp_path, old, new):
    text = open(SRC).read()
    assert text.count(old) == 1, old
    src = tmp_path / "attn_oracle_mutant.c"
    src.write_text(text.replace(old, new))
    spec = importlib.util.spec_from_file_location(f"oracle_mutant_{abs(hash(new))}",
                                                  os.path.join(ROOT, "oracle", "__init__.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod._SRC = str(src)
    mod._LIB_PATH = str(tmp_path / "liboracle_mutant.so")
    mod._lib = None
    return mod


def _packed(t):
    a = t.double().numpy()
    return a.reshape(-1, a.shape[-2], a.shape[-1])


def _sdpa_check(mod, causal):
    B, N, H, d = 2, 17, 3, 16
    q, k, v = make_custom(B, N, H, d, seed=11 + N)
    o, _, _ = mod.fwd(_packed(q), _packed(k), _packed(v), mod.dense_cu(B, N), causal, 1 / math.sqrt(d))
    qt, kt, vt = (x.double().permute(0, 2, 1, 3) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=causal)
    return np.allclose(o.reshape(B, N, H, d), ref.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-12)


def _lse_check(mod):
    B, N, H, d = 2, 23, 2, 16
    q, k, v = make_custom(B, N, H, d, seed=12)
    _, lse, _ = mod.fwd(_packed(q), _packed(k), _packed(v), mod.dense_cu(B, N), False, 0.3)
    s = torch.einsum("bihc,bjhc->bhij", q.double(), k.double()) * 0.3
    return np.allclose(mod.lse_to_dense(lse, B, N), torch.logsumexp(s, -1).numpy(), rtol=0, atol=1e-12)


def _overflow_check(mod):
    q, k, v = make_custom(1, 16, 1, 8, seed=8)
    o, lse, _ = mod.fwd(_packed(q) * 200.0, _packed(k), _packed(v), [0, 16], False, 1.0)
    return bool(np.all(np.isfinite(o)) and np.all(np.isfinite(lse)))


def _window_check(mod):
    L = 23
    _, k, v = make_custom(1, L, 1, 4, seed=23)
    vp = _packed(v)
    o, _, _ = mod.fwd(np.zeros((L, 1, 4)), _packed(k), vp, [0, L], False, 1.0, window=(2, 3))
    return all(np.allclose(o[i, 0], vp[max(0, i - 2):min(L, i + 4), 0].mean(axis=0), atol=1e-12)
               for i in range(L))


def _bwd_check(mod):
    B, N, H, d = 2, 19, 2, 8
    q, k, v, do = make_custom(B, N, H, d, seed=17, n=4)
    got = mod.bwd(_packed(q), _packed(k), _packed(v), _packed(do), mod.dense_cu(B, N), True, 0.35)
    qt, kt, vt = (x.double().permute(0, 2, 1, 3).requires_grad_(True) for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=0.35)
    (o * do.double().permute(0, 2, 1, 3)).sum().backward()
    refs = [t.grad.permute(0, 2, 1, 3).numpy().reshape(B * N, H, d) for t in (qt, kt, vt)]
    return all(np.allclose(g, r, rtol=0, atol=1e-10) for g, r in zip(got, refs))


def _online_check(mod):
    lengths = [131, 45]
    q, k, v = make_custom(0, 0, 2, 16, seed=9, lengths=lengths)
    q = (q.float() * 4).to(torch.bfloat16)
    cu = np.concatenate([[0], np.cumsum(lengths)])
    o2, l2, _ = mod.fwd(_packed(q), _packed(k), _packed(v), cu, False, 0.25)
    o1, l1, _ = mod.online_fwd(_packed(q), _packed(k), _packed(v), cu, False, 0.25, 16, 16, 0.0)
    return np.allclose(o1, o2, rtol=0, atol=1e-12) and np.allclose(l1, l2, rtol=0, atol=1e-12)


MUTATIONS = [
    ("dropped scale", "    srow[j - lo] = scale * acc;", "    srow[j - lo] = acc;",
     lambda m: _sdpa_check(m, False)),
    ("causal off by one", "  if (causal && i + 1 < b) b = i + 1;", "  if (causal && i < b) b = i > 0 ? i : 1;",
     lambda m: _sdpa_check(m, True)),
    ("no max subtraction", "srow[j] = exp(srow[j] - m); l += srow[j];", "srow[j] = exp(srow[j]); l += srow[j];",
     _overflow_check),
    ("LSE without the max", "  *lse_out = m + log(l);", "  *lse_out = log(l);", _lse_check),
    ("window edge off by one", "  if (wl >= 0 && i - wl > a) a = i - wl;",
     "  if (wl >= 0 && i - wl + 1 > a) a = i - wl + 1;", _window_check),
    ("backward sign", "const double ds = prow[j] * (dp - Di);", "const double ds = prow[j] * (Di - dp);",
     _bwd_check),
    ("rescale factor inverted", "const double alpha = exp(m[r] - rowmax);",
     "const double alpha = exp(rowmax - m[r]);", _online_check),
]


def _run_case(index, tmp_dir):
    """Child-process body: print whether the real oracle and the mutant pass the check."""
    import pathlib
    name, old, new, check = MUTATIONS[index]
    real = check(oracle)
    with np.errstate(all="ignore"):
        mutant = check(_mutant(pathlib.Path(tmp_dir), old, new))
    print(f"RESULT real={int(real)} mutant={int(mutant)}")


@pytest.mark.parametrize("index", range(len(MUTATIONS)), ids=[m[0] for m in MUTATIONS])
def test_pin_catches_planted_mistake(tmp_path, index):
    name = MUTATIONS[index][0]
    code = ("import sys; sys.path[:0] = [sys.argv[1], sys.argv[2]]; "
            "import test_oracle_mutations as t; t._run_case(int(sys.argv[3]), sys.argv[4])")
    run = subprocess.run([sys.executable, "-c", code, ROOT, os.path.join(ROOT, "tests"),
                          str(index), str(tmp_path)], capture_output=True, text=True, timeout=300)
    out = [ln for ln in run.stdout.splitlines() if ln.startswith("RESULT ")]
    assert run.returncode == 0 and out, f"{name}: child failed\n{run.stdout}\n{run.stderr}"
    assert out[-1].split()[1] == "real=1", f"the real oracle fails the {name} check"
    assert out[-1].split()[2] == "mutant=0", f"{name} went unnoticed"
