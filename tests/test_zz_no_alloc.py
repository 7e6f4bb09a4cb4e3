"""The allocation-free prologue entry point, ra_rope_rotate_quant_noalloc.

It serves callers that may not allocate device memory when they run the
prologue (an engine plugin's execute step, a service with a fixed memory
budget): its scratch lives in a fixed array inside the library.  This file is
collected last so that, if it fails, a run that stops at the first failure has
already run every other test.  It passes alone in a fresh process too.
"""
import ctypes as C

import numpy as np
import pytest

from synth import inputs as si
from tests import gpu_util as gu


@pytest.fixture(scope="module")
def ra():
    import __graft_entry__
    __graft_entry__.build()
    import int4_quantized_flashattention_b200 as ra
    return ra


def _c_entry(ra):
    fn = ra.lib().ra_rope_rotate_quant_noalloc
    fn.restype = C.c_int
    fn.argtypes = [C.POINTER(ra.Problem), C.c_int] + [C.c_void_p] * 13
    return fn


def test_oversized_problem_is_rejected_without_launch(ra):
    """A problem needing more scratch than the fixed array holds returns
    RA_ERR_UNSUPPORTED before anything is launched (no GPU needed)."""
    p = ra.Problem.make(1, 128, 128, (44, 42, 42), (33, 45, 80), block_k=64)
    assert ra.workspace_bytes(p) > (32 << 20)
    fake = C.c_void_p(0x10000)
    assert _c_entry(ra)(C.byref(p), 1, *([fake] * 12), None) == 2


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_on_two_calls(ra):
    import torch
    dev = gu.device()
    wl = si.WORKLOADS["small"].with_(H=3, grid=(2, 10, 10))  # N = 200: ragged blocks
    x = si.make_inputs(wl)
    p = gu.problem_for(ra, wl)
    q, k, v, pos = gu.to_device(x, wl, dev)
    ref = {n: t.clone() for n, t in ra.rope_rotate_quant(p, q, k, v, pos).items()}
    assert ra.sync_status() == 0
    fn = _c_entry(ra)
    free_after = []
    for call in range(2):
        out = {n: torch.full_like(t, 0x5A if t.dtype == torch.uint8 else 7) for n, t in ref.items()}
        ptr = lambda t: C.c_void_p(t.data_ptr())  # noqa: E731
        rc = fn(C.byref(p), 1, ptr(q), ptr(k), ptr(v), ptr(pos),
                ptr(out["q4"]), ptr(out["sq"]), ptr(out["k4"]), ptr(out["sk"]), ptr(out["k_mean"]),
                ptr(out["v4"]), ptr(out["sv"]), ptr(out["v_colsum"]),
                C.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert rc == 0, call
        assert ra.sync_status() == 0
        torch.cuda.synchronize()
        free_after.append(torch.cuda.mem_get_info()[0])
        for n in ref:
            a, b = out[n].cpu().numpy(), ref[n].cpu().numpy()
            if n in ("q4", "k4", "v4"):
                import oracle
                frac, mx = gu.code_agreement(a, b, oracle)
                assert frac >= 0.9999 and mx <= 1, (call, n)
            elif n == "v_colsum":
                assert np.array_equal(a, b), (call, n)
            else:
                assert np.allclose(a, b, rtol=1e-6, atol=0), (call, n)
    # The point of the entry: once the first call has looked up the array (and
    # the kernels are loaded), a call takes no device memory.
    assert free_after[1] == free_after[0], free_after


def test_noalloc_source_calls_no_allocator():
    """The allocation-free entry's source names no device allocator or free
    (host check, no GPU needed)."""
    import os
    import re
    path = os.path.join(os.path.dirname(__file__), "..", "int4_quantized_flashattention_b200", "csrc", "ra_noalloc.cu")
    code = re.sub(r"//[^\n]*", "", open(path).read())
    for name in ("cudaMalloc", "cudaFree", "cuMemAlloc", "cuMemFree", "cudaMallocAsync", "cudaMallocManaged"):
        assert name not in code, name
