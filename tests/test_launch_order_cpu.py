"""The backward's overlapped launch keeps stream order (CPU, reads the kernel source).

The dQ kernel is launched as a programmatic dependent of the dK/dV kernel, so its
CTAs may run while dK/dV's last wave does.  For the work the stream runs next to
see dK, dV written, every way out of the dQ kernel passes a wait on that grid,
and the dK/dV kernel signals its dependents; both are checked here."""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "exact_attention_103_b200", "csrc", "attn_bwd_sm100.cu")
WAIT = 'asm volatile("griddepcontrol.wait;" ::: "memory");'


def _kernel_body(src: str, name: str) -> str:
    i = src.index(name + "(")
    j = src.index("{", src.index(")", i))
    depth = 0
    for k in range(j, len(src)):
        if src[k] == "{":
            depth += 1
        elif src[k] == "}":
            depth -= 1
            if depth == 0:
                return src[j:k + 1]
    raise AssertionError("unbalanced braces in " + name)


def test_every_exit_of_the_dq_kernel_waits_for_the_dkdv_grid():
    src = open(SRC).read()
    body = _kernel_body(src, "bwd_dq_kernel")
    lines = [l.strip() for l in body.split("\n") if l.strip()]
    bare = [i for i, l in enumerate(lines) if l == "return;"]
    assert bare, "the early exit is expected"
    for i in bare:
        assert lines[i - 1] == WAIT, lines[i - 1]
    assert lines[-1] == "}" and lines[-2] == WAIT, lines[-3:]


def test_dkdv_signals_dependents_and_dq_is_launched_as_one():
    src = open(SRC).read()
    dkdv = _kernel_body(src, "bwd_dkdv_kernel")
    first = [l.strip() for l in dkdv.split("\n") if l.strip() and not l.strip().startswith("//")]
    assert 'asm volatile("griddepcontrol.launch_dependents;" ::: "memory");' in first[:4], first[:4]
    assert re.search(r"cudaLaunchAttributeProgrammaticStreamSerialization", src)
    assert re.search(r"programmaticStreamSerializationAllowed\s*=\s*1", src)
