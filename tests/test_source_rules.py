"""Source-level rules of the CUDA library, checked on the host.

* No kernel traps or asserts on the device: faults are reported through the
  status word, and a trapped kernel would take its context down.
* No TMA or bulk load with cluster multicast: every load of the library may
  run in multi-GPU jobs (one process per GPU), where such loads are not used.
  (The pair attention's tcgen05.commit multicast is a completion signal, not a
  load, and is the one multicast form allowed.)
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
    """The only cluster-multicast form in the library is the tcgen05.commit
    completion signal of the CTA-pair attention (an mbarrier arrive in both
    CTAs); no TMA or bulk copy names multicast."""
    for name, text in _sources().items():
        for line in _code(text).splitlines():
            if ".multicast::cluster" in line:
                assert "tcgen05.commit" in line and "cp.async" not in line, (name, line.strip())
        assert not re.search(r"cp\.async\.bulk[^;]*multicast", _code(text)), name


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


_COLLECTIVE = re.compile(r"__(?:shfl(?:_xor|_up|_down)?|any|all|ballot)_sync\s*\(")


def _blank_calls(code):
    """The code with the argument lists of every full-mask warp collective
    replaced by a placeholder, so that only the context of each call is left."""
    out = []
    i = 0
    for m in _COLLECTIVE.finditer(code):
        if m.start() < i:
            continue
        out.append(code[i:m.start()])
        depth = 0
        j = m.end() - 1
        while True:
            depth += code[j] == "("
            depth -= code[j] == ")"
            j += 1
            if depth == 0:
                break
        out.append("WARP_COLLECTIVE")
        i = j
    out.append(code[i:])
    return "".join(out)


def _statements(code):
    return re.split(r"[;{}]", code)


def test_warp_collectives_are_not_conditional_operands():
    """A full-mask shuffle or vote must be reached by every lane of the warp.
    Written as an operand of ?:, && or ||, it is skipped by the lanes whose
    condition short-circuits, and the lanes that reach it wait for them for
    ever (the hang of the quantise kernel whose 'mq == 0 ? 0 : shfl' skipped
    the shuffle on lanes of zero rows and of tokens past N).  Collectives are
    evaluated into a value first and combined afterwards."""
    for name, text in _sources().items():
        for st in _statements(_blank_calls(_code(text))):
            if "WARP_COLLECTIVE" not in st:
                continue
            assert "?" not in st and "&&" not in st and "||" not in st, (name, st.strip())


_TMEM_COLLECTIVE = re.compile(r"\btmem_(?:ld|st)_h\d*\s*(?:<[^>]*>)?\s*\(")


def _blank_tmem_calls(code):
    """The code with every warp-collective tensor-memory load / store helper
    call (tcgen05.ld / tcgen05.st .sync.aligned) replaced by the placeholder."""
    return _TMEM_COLLECTIVE.sub("WARP_COLLECTIVE(", code)


def test_warp_collectives_are_not_under_per_lane_branches():
    """No full-mask collective -- shuffle, vote, or tensor-memory load/store
    (tcgen05.ld / st are .sync.aligned: every lane of the warp must execute
    them) -- sits inside an if/else whose condition depends on the lane or on a
    per-row flag or value (validity, the dumped tile, a row's rescale factor).
    Such branches guard only the per-lane work; the collective runs for the
    whole warp, with a warp vote deciding whether it runs at all."""
    per_lane = re.compile(r"\b(lane|threadIdx|row_ok|valid|nvalid|in_range|dump_tile|sc|grow|change|near_bound|write)\b")
    for name, text in _sources().items():
        code = _blank_calls(_blank_tmem_calls(_code(text)))
        for m in re.finditer("WARP_COLLECTIVE", code):
            # walk outwards through the enclosing braces and check each opener
            depth = 0
            i = m.start()
            while i > 0:
                i -= 1
                c = code[i]
                if c == "}":
                    depth += 1
                elif c == "{":
                    if depth == 0:
                        head = code[max(0, i - 300):i]
                        head = head[max(head.rfind(";"), head.rfind("}"), head.rfind("{")) + 1:]
                        if re.match(r"\s*(?:else\s+)?if\s*\(", head):
                            assert not per_lane.search(head), (name, head.strip())
                    else:
                        depth -= 1


def test_collective_rule_flags_the_conditional_shuffle():
    """The checker itself: the statement that hung the quantise kernel is
    flagged, and its corrected form (shuffle first, select after) is not."""
    bad = "const float iq = mq == 0.0f ? 0.0f : __shfl_sync(0xFFFFFFFFu, rcp7, lane & ~1);"
    good = ("const float sh = __shfl_sync(0xFFFFFFFFu, rcp7, lane & ~1);\n"
            "const float iq = mq == 0.0f ? 0.0f : sh;")
    flagged = lambda src: any("WARP_COLLECTIVE" in st and ("?" in st or "&&" in st or "||" in st)  # noqa: E731
                              for st in _statements(_blank_calls(src)))
    assert flagged(bad)
    assert not flagged(good)
    assert flagged("if (reset || __any_sync(0xFFFFFFFFu, change)) {")


def test_collective_rule_flags_tensor_memory_access_under_a_row_condition():
    """The checker flags a tensor-memory load guarded by a per-row value (the
    rescale of one row's output accumulator), and accepts the warp-voted form."""
    bad = ("if (sc != 1.0f) {\n  uint32_t f[32];\n  tmem_ld_h<32, kHD>(tF + c, f);\n}\n")
    good = ("const bool any_rescale = __any_sync(0xFFFFFFFFu, sc != 1.0f);\n"
            "if (any_rescale) {\n  uint32_t f[32];\n  tmem_ld_h<32, kHD>(tF + c, f);\n}\n")
    per_lane = re.compile(r"\b(lane|threadIdx|row_ok|valid|nvalid|in_range|dump_tile|sc|grow|change|near_bound|write)\b")

    def flagged(src):
        code = _blank_calls(_blank_tmem_calls(src))
        for m in re.finditer("WARP_COLLECTIVE", code):
            head = code[:m.start()]
            i = head.rfind("{")
            opener = head[:i]
            opener = opener[max(opener.rfind(";"), opener.rfind("}"), opener.rfind("{")) + 1:]
            if re.match(r"\s*(?:else\s+)?if\s*\(", opener) and per_lane.search(opener):
                return True
        return False
    assert flagged(bad)
    assert not flagged(good)
