"""C-ABI library: it loads, exports every entry point include/ra.h declares, and
its host-side validation rejects bad arguments before any launch (no GPU)."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ra.h")


def _no_gpu():
    """Checks that pass validation and reach a launch use fake pointers: they
    run only where no GPU is visible (the launch then fails with RA_ERR_CUDA)."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("reaches a launch with fake pointers; host-only check")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ra_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def ra():
    import __graft_entry__
    __graft_entry__.build()
    import int4_quantized_flashattention_b200 as ra
    ra.lib()
    return ra


def test_header_declares_the_entry_points():
    names = _declared()
    for n in ("ra_rope_rotate_quant", "ra_attn_int4", "ra_attn_bf16_fallback", "ra_test_int4_codes",
              "ra_rope_bf16", "ra_workspace_bytes", "ra_sync_status", "ra_status_string",
              "ra_attn_int4_opts", "ra_test_int4_codes_opts", "ra_attn_int4_qfused",
              "ra_rope_rotate_quant_s8", "ra_attn_int4_s8"):
        assert n in names


def test_library_exports_every_declared_symbol(ra):
    L = ra.lib()
    missing = [n for n in _declared() if not hasattr(L, n)]
    assert not missing, missing


def test_status_strings(ra):
    for s in range(5):
        assert ra.status_string(s)
    assert ra.status_string(0) == "ok"


def _wan(ra, **kw):
    args = dict(B=1, H=40, D=128, seg=(44, 42, 42), grid=(21, 30, 52), rot=ra.ROT_INTERLEAVED,
                block_q=128, block_k=64)
    args.update(kw)
    return ra.Problem.make(**args)


def test_workspace_bytes(ra):
    p = _wan(ra)
    ws = ra.workspace_bytes(p)
    # tables + fp64 channel sums + fp32 maxima per chunk of 256 tokens + reciprocals
    nchunk = -(-p.N // 256)
    assert ws >= 40 * nchunk * 128 * 12
    assert ws < 64 << 20
    bad = _wan(ra, D=96, seg=(32, 32, 32))
    assert ra.workspace_bytes(bad) == 0


@pytest.mark.parametrize("field,value", [
    ("D", 96), ("N", 0), ("block_k", 48), ("block_q", 100), ("rot", 4), ("theta", -1.0), ("B", 0),
])
def test_invalid_problem_rejected(ra, field, value):
    p = _wan(ra)
    setattr(p, field, value)
    fake = C.c_void_p(0x10000)
    rc = ra.lib().ra_attn_int4(C.byref(p), *([fake] * 7), None, None)
    assert rc == 1


def test_bad_segments_rejected(ra):
    for seg in ((43, 43, 42), (44, 42, 40), (0, 64, 64)):
        p = _wan(ra, seg=seg)
        fake = C.c_void_p(0x10000)
        assert ra.lib().ra_attn_int4(C.byref(p), *([fake] * 7), None, None) == 1


def test_misaligned_or_null_pointer_rejected(ra):
    p = _wan(ra)
    good = C.c_void_p(0x10000)
    bad = C.c_void_p(0x10004)
    L = ra.lib()
    for i in range(7):
        args = [good] * 7
        args[i] = bad
        assert L.ra_attn_int4(C.byref(p), *args, None, None) == 1
        args[i] = None
        assert L.ra_attn_int4(C.byref(p), *args, None, None) == 1
    assert L.ra_attn_int4(C.byref(p), *([good] * 7), bad, None) == 1  # lse misaligned


def test_workspace_too_small_rejected(ra):
    p = _wan(ra)
    good = C.c_void_p(0x10000)
    need = ra.workspace_bytes(p)
    rc = ra.lib().ra_rope_rotate_quant(C.byref(p), 1, *([good] * 13), C.c_size_t(need - 16), None)
    assert rc == 1
    rc = ra.lib().ra_rope_rotate_quant(C.byref(p), 7, *([good] * 13), C.c_size_t(need), None)
    assert rc == 1   # unknown input dtype


def test_block_k_128_is_dispatched(ra):
    """block_k = 128 (the CTA-pair kernel) passes validation and is not
    refused as unsupported, in every mode; without a GPU the launch itself
    then fails with RA_ERR_CUDA."""
    _no_gpu()
    p = _wan(ra, block_k=128)
    good = C.c_void_p(0x10000)
    L = ra.lib()
    assert L.ra_attn_int4(C.byref(p), *([good] * 7), None, None) not in (1, 2)
    for pm, lm in ((1, 0), (2, 0), (0, 1), (1, 1), (2, 1)):
        opts = ra.AttnOpts(pm, lm)
        assert L.ra_attn_int4_opts(C.byref(p), C.byref(opts), *([good] * 7), None, None) not in (1, 2)


def test_ablation_options_are_validated_before_any_launch(ra):
    """Out-of-range switches are invalid; switches other than the defaults are
    implemented for block_k = 64 and 128 only."""
    good = C.c_void_p(0x10000)
    L = ra.lib()
    p = _wan(ra)
    for pm, lm in ((3, 0), (-1, 0), (0, 2)):
        opts = ra.AttnOpts(pm, lm)
        assert L.ra_attn_int4_opts(C.byref(p), C.byref(opts), *([good] * 7), None, None) == 1
        assert L.ra_test_int4_codes_opts(C.byref(p), C.byref(opts), *([good] * 6), 0, 0, 0,
                                         None, None, None, good, None, None) == 1
    p32 = _wan(ra, block_k=32)
    for pm, lm in ((1, 0), (2, 0), (0, 1)):
        opts = ra.AttnOpts(pm, lm)
        assert L.ra_attn_int4_opts(C.byref(p32), C.byref(opts), *([good] * 7), None, None) == 2


def test_test_entry_rejects_bad_tile(ra):
    p = _wan(ra)
    good = C.c_void_p(0x10000)
    L = ra.lib()
    ntiles = -(-p.N // 128)
    for b, h, t in ((1, 0, 0), (0, 40, 0), (0, 0, ntiles), (-1, 0, 0)):
        rc = L.ra_test_int4_codes(C.byref(p), *([good] * 6), b, h, t, None, None, None, good, None, None)
        assert rc == 1


def test_qfused_entry_validates_before_any_launch(ra):
    """ra_attn_int4_qfused: invalid problems, bad pointers or a short workspace
    are RA_ERR_INVALID_ARG, block sizes other than 64 RA_ERR_UNSUPPORTED, all
    before any launch (no GPU needed)."""
    L = ra.lib()
    good, bad = C.c_void_p(0x10000), C.c_void_p(0x10004)
    p = _wan(ra)
    need = ra.workspace_bytes(p)

    def call(pp, dt=1, ptrs=None, ws=need, lse=None):
        ptrs = ptrs or [good] * 6
        return L.ra_attn_int4_qfused(C.byref(pp), dt, *ptrs[:6], good, C.c_size_t(ws), good, lse, None)
    assert call(p, dt=7) == 1
    for i in range(6):
        ptrs = [good] * 6
        ptrs[i] = bad
        assert call(p, ptrs=ptrs) == 1
        ptrs[i] = None
        assert call(p, ptrs=ptrs) == 1
    assert call(p, ws=need - 16) == 1
    assert call(p, lse=bad) == 1
    q = _wan(ra)
    q.D = 96
    assert call(q) == 1
    assert call(_wan(ra, block_k=32)) == 2
    assert call(_wan(ra, block_k=128)) == 2


def test_kv_only_prologue_needs_all_three_q_pointers_null(ra):
    """ra_rope_rotate_quant accepts q, q4 and sq all NULL (K and V only); a
    partial set is RA_ERR_INVALID_ARG.  The full-NULL call passes validation
    (without a GPU it then fails at the launch with RA_ERR_CUDA)."""
    _no_gpu()
    L = ra.lib()
    good = C.c_void_p(0x10000)
    p = _wan(ra)
    need = C.c_size_t(ra.workspace_bytes(p))
    base = [good] * 13
    for drop in ((0,), (4,), (5,), (0, 4), (0, 5), (4, 5)):
        args = list(base)
        for i in drop:
            args[i] = None
        assert L.ra_rope_rotate_quant(C.byref(p), 1, *args, need, None) == 1, drop
    args = list(base)
    for i in (0, 4, 5):
        args[i] = None
    assert L.ra_rope_rotate_quant(C.byref(p), 1, *args, need, None) not in (1, 2)


def test_s8_entries_validate_before_any_launch(ra):
    """ra_attn_int4_s8 / ra_rope_rotate_quant_s8: bad arguments are
    RA_ERR_INVALID_ARG and block sizes other than 64 RA_ERR_UNSUPPORTED before
    any launch (no GPU needed)."""
    L = ra.lib()
    good, bad = C.c_void_p(0x10000), C.c_void_p(0x10004)
    p = _wan(ra)
    for i in range(7):
        args = [good] * 7
        args[i] = bad
        assert L.ra_attn_int4_s8(C.byref(p), *args, None, None) == 1
        args[i] = None
        assert L.ra_attn_int4_s8(C.byref(p), *args, None, None) == 1
    assert L.ra_attn_int4_s8(C.byref(p), *([good] * 7), bad, None) == 1
    assert L.ra_attn_int4_s8(C.byref(_wan(ra, block_k=32)), *([good] * 7), None, None) == 2
    assert L.ra_attn_int4_s8(C.byref(_wan(ra, block_k=128)), *([good] * 7), None, None) == 2
    need = ra.workspace_bytes(p)
    assert L.ra_rope_rotate_quant_s8(C.byref(p), 1, *([good] * 13), C.c_size_t(need - 16), None) == 1
    assert L.ra_rope_rotate_quant_s8(C.byref(p), 7, *([good] * 13), C.c_size_t(need), None) == 1
