"""No TMA or bulk load in the CUDA sources uses cluster multicast (CPU, reads the sources).

Every copy loads this GPU's own tiles into the CTA that issued it; multicast is
used only by tcgen05.commit (barrier arrivals), never by a data copy."""
import glob
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "exact_attention_103_b200", "csrc")


def test_bulk_copies_never_multicast():
    files = sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                   + glob.glob(os.path.join(CSRC, "*.h")))
    assert files
    bulk_lines = 0
    for path in files:
        for n, line in enumerate(open(path), 1):
            code = line.split("//")[0]
            if "cp.async.bulk" in code:
                bulk_lines += 1
                assert "multicast" not in code, f"{os.path.basename(path)}:{n}: {line.strip()}"
            if "multicast" in code:
                assert "tcgen05.commit" in code, f"{os.path.basename(path)}:{n}: {line.strip()}"
    assert bulk_lines > 0  # the scan saw the copy instructions
