"""Static checks on the CUDA sources (CPU): rules the kernels must keep on any number of GPUs.

- No TMA or bulk load with cluster multicast: every load in this library reads this GPU's own
  memory, and the multi-GPU benchmark path must never meet such a load.
- Every mbarrier wait goes through the bounded helpers (a deadline, then an error bit).
"""
import os
import re

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "mxfp8_block_scaled_07_b200",
                    "csrc")


def sources():
    for name in sorted(os.listdir(CSRC)):
        if name.endswith((".cu", ".cuh")):
            with open(os.path.join(CSRC, name)) as f:
                yield name, f.read()


def test_no_multicast_loads():
    for name, text in sources():
        for line in text.splitlines():
            if "cp.async.bulk" in line and "multicast" in line:
                raise AssertionError(f"{name}: multicast bulk/TMA load: {line.strip()}")


def test_mbarrier_waits_are_bounded():
    for name, text in sources():
        # The only raw try_wait is inside the bounded helpers of ptx.cuh.
        raw = [m.start() for m in re.finditer(r"mbarrier\.try_wait", text)]
        if name == "ptx.cuh":
            assert len(raw) == 1
        else:
            assert not raw, f"{name}: raw mbarrier wait"
        assert "mbarrier.test_wait" not in text
