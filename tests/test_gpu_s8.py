"""The byte code layout (ra_rope_rotate_quant_s8 / ra_attn_int4_s8): one code
per byte, natural channel order (Q and K as FP8 E4M3 values equal to the
code, V as the int8 value 16 x code), loaded by TMA straight into the MMA
operand tiles; Q K^T runs in FP8 with an fp32 accumulator.  The codes must be
the packed prologue's codes bit for bit, every other prologue output
identical, and the attention's out and lse identical to ra_attn_int4 on the
packed codes (which also shows the FP8 Q K^T is exact); the packed path is
checked against the oracle in test_gpu_int4.py.
"""
import numpy as np
import pytest

from synth import inputs as si
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ra():
    import __graft_entry__
    __graft_entry__.build()
    import int4_quantized_flashattention_b200 as ra
    return ra


def _unpack16(packed):
    import oracle
    return (oracle.unpack_codes(packed).astype(np.int16) * 16).astype(np.int8)


def _e4m3(c):
    """FP8 E4M3 byte of each integer code in [-7, 7] (sign, 4 exponent bits
    with bias 7, 3 mantissa bits), written out from the format's definition."""
    c = np.asarray(c, np.int64)
    a = np.abs(c)
    e = np.floor(np.log2(np.maximum(a, 1))).astype(np.int64)
    m = ((a / np.exp2(e) - 1.0) * 8).astype(np.int64)
    byte = np.where(a == 0, 0, ((e + 7) << 3) | m) | np.where(c < 0, 0x80, 0)
    return byte.astype(np.uint8)


def test_e4m3_table():
    assert list(_e4m3(np.arange(-7, 8))) == [0xCE, 0xCC, 0xCA, 0xC8, 0xC4, 0xC0, 0xB8, 0x00,
                                             0x38, 0x40, 0x44, 0x48, 0x4A, 0x4C, 0x4E]


def _run(ra, wl):
    import torch
    dev = gu.device()
    x = si.make_inputs(wl)
    p = gu.problem_for(ra, wl)
    q, k, v, pos = gu.to_device(x, wl, dev)
    packed = ra.rope_rotate_quant(p, q, k, v, pos)
    lse_ref = torch.empty(wl.B, wl.H, wl.N, dtype=torch.float32, device=dev)
    out_ref = ra.attn_int4(p, packed, lse=lse_ref)
    assert ra.sync_status() == 0
    s8 = ra.rope_rotate_quant_s8(p, q, k, v, pos)
    assert ra.sync_status() == 0
    import oracle
    for a, b in (("q8", "q4"), ("k8", "k4")):
        got = s8[a].cpu().numpy().reshape(-1, wl.D)
        ref = _e4m3(oracle.unpack_codes(packed[b].cpu().numpy().reshape(-1, wl.D // 2)))
        assert np.array_equal(got, ref), a
    got = s8["v8"].cpu().numpy().reshape(-1, wl.D)
    assert np.array_equal(got, _unpack16(packed["v4"].cpu().numpy().reshape(-1, wl.D // 2)))
    for name in ("sq", "sk", "k_mean", "sv", "v_colsum"):
        assert torch.equal(s8[name], packed[name]), name
    # K and V only (q = None): the same K and V outputs, nothing for Q
    kv = ra.rope_rotate_quant_s8(p, None, k, v, pos)
    assert ra.sync_status() == 0
    assert set(kv) == {"k8", "sk", "k_mean", "v8", "sv", "v_colsum"}
    for name, t in kv.items():
        assert torch.equal(t, s8[name]), name
    out = torch.full_like(out_ref, float("nan"))
    lse = torch.full_like(lse_ref, float("nan"))
    ra.attn_int4_s8(p, s8, out=out, lse=lse)
    assert ra.sync_status() == 0
    assert torch.equal(out.view(torch.int16), out_ref.view(torch.int16))
    assert torch.equal(lse.view(torch.int32), lse_ref.view(torch.int32))


@pytest.mark.parametrize("D,seg,rot,grid", [
    (128, (44, 42, 42), 1, (3, 10, 10)),   # N = 300: ragged query tile and key block
    (128, (16, 56, 56), 2, (2, 5, 9)),     # N = 90: one partial block
    (64, (24, 20, 20), 1, (5, 9, 11)),     # D = 64, N = 495
    (64, (24, 20, 20), 0, (1, 1, 7)),      # N = 7
    (128, (44, 42, 42), 3, (1, 1, 1)),     # N = 1
])
def test_s8_equals_packed(ra, D, seg, rot, grid):
    wl = si.WORKLOADS["small"].with_(H=2, D=D, seg=seg, grid=grid, rot=rot, block_k=64)
    _run(ra, wl)


def test_s8_at_the_wan_shape(ra):
    _run(ra, si.WORKLOADS["wan"])


def test_s8_sharp(ra):
    _run(ra, si.WORKLOADS["small"].with_(H=2, sharp=True))
