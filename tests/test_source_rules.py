"""Source-level rules of the CUDA library, checked on the host.

* No kernel traps or asserts on the device: faults are reported through the
  status word, and a trapped kernel would take its context down.
* No TMA or bulk load with cluster multicast: every load of the library may
  run in multi-GPU jobs (one process per GPU), where such loads are not used.
* No batched memory-copy entry points of the runtime or driver.
* Every spin on an mbarrier is bounded: the waits go through the helpers that
  carry an iteration or time limit.
"""
import glob
import os
import re

CSRC = os.path.join(os.path.dirname(__file__), "..", "int4_quantized_flashattention_b200", "csrc")


def _sources():
    files = sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                   + glob.glob(os.path.join(CSRC, "*.h")))
    assert files
    return {os.path.basename(f): open(f).read() for f in files}


def _code(text):
    """The text without // and /* */ comments."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.sub(r"//[^\n]*", "", text)


def test_no_device_trap_or_assert():
    for name, text in _sources().items():
        code = _code(text)
        assert "__trap" not in code and "trap;" not in code, name
        assert not re.search(r"(?<!static_)\bassert\s*\(", code), name


def test_no_multicast_loads():
    for name, text in _sources().items():
        assert ".multicast::cluster" not in _code(text), name


def test_no_batched_copies():
    for name, text in _sources().items():
        assert not re.search("[Mm]emcpy(3D)?" + "Batch" + "Async", text), name


def test_mbarrier_spins_are_bounded():
    """Every loop around mbar_try_wait / mbar_test_wait has a bound in its
    condition (an iteration counter) or sits in the time-limited helper."""
    for name, text in _sources().items():
        code = _code(text)
        for m in re.finditer(r"while\s*\(([^;{]*mbar_(?:try|test)_wait[^;{]*)\)", code):
            cond = m.group(1)
            assert "kSpinLimit" in cond or "Limit" in cond, (name, cond)
