"""The forward kernel's setmaxnreg split adds up (CPU, reads the kernel source).

The kernel launches kThreads threads; three warps share each SM sub-partition, so
every thread starts with the budget ptxas gives at that launch size.  Warpgroup 2
lowers its budget and warpgroups 0 and 1 raise theirs; an increase that asks for
more registers than the decrease released would wait forever, so the arithmetic
is checked here, before anything runs on a GPU."""
import math
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "exact_attention_103_b200", "csrc", "attn_fwd_sm100.cu")

REGS_PER_SM = 65536
SUB_PARTITIONS = 4
ALLOC_GRANULE = 8  # registers per thread are allocated in multiples of 8


def _source():
    with open(SRC) as f:
        return f.read()


def _launch_budget(threads: int) -> int:
    warps = threads // 32
    warps_per_sub = math.ceil(warps / SUB_PARTITIONS)
    per_thread = REGS_PER_SM // SUB_PARTITIONS // (warps_per_sub * 32)
    return per_thread // ALLOC_GRANULE * ALLOC_GRANULE


def test_setmaxnreg_split_fits_the_launch_budget():
    src = _source()
    threads = int(re.search(r"constexpr int kThreads = (\d+);", src).group(1))
    dec = [int(x) for x in re.findall(r"setmaxnreg\.dec\.sync\.aligned\.u32 (\d+);", src)]
    inc = [int(x) for x in re.findall(r"setmaxnreg\.inc\.sync\.aligned\.u32 (\d+);", src)]
    assert len(dec) == 1 and len(inc) == 1, (dec, inc)
    dec, inc = dec[0], inc[0]
    assert threads == 384, "warpgroup 2 must be complete (4 warps) for setmaxnreg"
    launch = _launch_budget(threads)
    assert launch == 168
    for v in (dec, inc):
        assert v % ALLOC_GRANULE == 0 and 24 <= v <= 256
    assert dec < launch < inc
    released = 4 * 32 * (launch - dec)   # warpgroup 2: producer, MMA issuer, two idle warps
    taken = 8 * 32 * (inc - launch)      # warpgroups 0 and 1: the softmax warps
    assert taken <= released, (taken, released)
    # each sub-partition holds one warp of each warpgroup after the change
    assert (2 * inc + dec) * 32 <= REGS_PER_SM // SUB_PARTITIONS
    assert threads * launch <= REGS_PER_SM


def test_each_warpgroup_changes_its_budget_once_at_its_branch_head():
    """The increase is the first statement of the softmax branch and the decrease the
    first statement of warpgroup 2's branch, one instruction each, so every warp of
    a warpgroup executes the same setmaxnreg."""
    lines = [l.strip() for l in _source().split("\n")]
    i_inc = next(i for i, l in enumerate(lines) if "setmaxnreg.inc" in l)
    i_dec = next(i for i, l in enumerate(lines) if "setmaxnreg.dec" in l)
    assert lines[i_inc - 1] == "if (warp < 8) {", lines[i_inc - 1]
    assert lines[i_dec - 1] == "} else {", lines[i_dec - 1]
    assert lines[i_dec + 1] == "if (warp == 8) {", lines[i_dec + 1]
