"""GPU parity of the bf16 fallback (plain 3D RoPE to bf16, then bf16
FlashAttention) against the CPU oracle: the oracle's RoPE without rotation and
unquantised fp64 softmax attention (papernotes page, key design 3: the
fallback is ordinary bf16 attention on the RoPE'd inputs).

Acceptance:
  * RoPE'd q and k: the kernel rounds its fp32 RoPE to bf16, the oracle its own
    (fp32 arithmetic in the same order) to bf16; identical on >= 99.9 % of
    elements and within one bf16 unit elsewhere.
  * Attention output against fp64 attention on the same bf16 inputs: relative
    L2 <= 5e-3.  Budget: P is rounded to bf16 before P.V (relative error
    <= 2^-9 per weight, averaging over the keys) and the output is rounded to
    bf16 (RMS relative error 2^-9/sqrt(3) ~ 1.1e-3).
  * lse within 2e-3 of the fp64 log-sum-exp (ex2.approx and fp32 sums).
"""
import math

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


def _bf16_ulps(a, b):
    """|a - b| in units of the bf16 spacing of max(|a|, |b|)."""
    m = np.maximum(np.abs(a), np.abs(b))
    ulp = np.where(m > 0, 2.0 ** (np.floor(np.log2(np.where(m > 0, m, 1.0))) - 7), 2.0 ** -133)
    return np.abs(a - b) / ulp


def _run(ra, orc, wl, heads=None):
    import torch
    dev = gu.device()
    x = si.make_inputs(wl)
    p = gu.problem_for(ra, wl)
    q, k, v, pos = gu.to_device(x, wl, dev)
    qr, kr = ra.rope_bf16(p, q, k, pos)
    vb = v.to(torch.bfloat16) if v.dtype != torch.bfloat16 else v
    lse = torch.empty(wl.B, wl.H, wl.N, dtype=torch.float32, device=dev)
    out = ra.attn_bf16_fallback(p, qr, kr, vb, lse=lse)
    assert ra.sync_status() == 0
    po = orc.problem(wl)
    po.rot = 0
    qr_h, kr_h = qr.float().cpu().numpy(), kr.float().cpu().numpy()
    v_h = vb.float().cpu().numpy()
    out_h, lse_h = out.float().cpu().numpy(), lse.cpu().numpy()
    num = den = 0.0
    for h in (range(wl.H) if heads is None else heads):
        for name, src, got in (("q", x["q"], qr_h), ("k", x["k"], kr_h)):
            ref = gu.bf16_round(orc.rope_rotate(po, src[0, h], x["pos"]))
            u = _bf16_ulps(got[0, h], ref)
            assert u.max() <= 1.0, (name, h, u.max())
            assert np.mean(u == 0) >= 0.999, (name, h)
        q64, k64, v64 = (a[0, h].astype(np.float64) for a in (qr_h, kr_h, v_h))
        ref = orc.reference_attention_fp64(q64, k64, v64)
        s = q64 @ k64.T / math.sqrt(wl.D)
        m = s.max(axis=1)
        ref_lse = m + np.log(np.exp(s - m[:, None]).sum(axis=1))
        assert np.max(np.abs(lse_h[0, h] - ref_lse)) <= 2e-3, h
        num += float(np.sum((out_h[0, h] - ref) ** 2))
        den += float(np.sum(ref ** 2))
    assert math.sqrt(num / den) <= 5e-3, math.sqrt(num / den)


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_bf16_fallback_small_workloads(ra, orc, name):
    _run(ra, orc, si.WORKLOADS[name])


@pytest.mark.parametrize("D,seg,bk,grid", [
    (128, (44, 42, 42), 64, (2, 10, 10)),    # N = 200: ragged key block and query tile
    (128, (44, 42, 42), 32, (3, 7, 13)),     # N = 273
    (128, (16, 56, 56), 16, (2, 5, 9)),      # N = 90
    (64, (24, 20, 20), 64, (5, 9, 11)),      # N = 495, D = 64
    (128, (44, 42, 42), 64, (1, 1, 1)),      # N = 1
])
def test_bf16_fallback_shapes(ra, orc, D, seg, bk, grid):
    wl = si.WORKLOADS["small"].with_(name=f"bf16_{D}_{bk}", D=D, seg=seg, block_k=bk, grid=grid, H=2)
    _run(ra, orc, wl)


def test_bf16_fallback_long_sequence(ra, orc):
    """4096 keys (64 blocks): many running-maximum changes and folds."""
    wl = si.WORKLOADS["sweep4096"].with_(H=2)
    _run(ra, orc, wl, heads=(0, 1))


def test_bf16_fallback_wan_sampled(ra, orc):
    """The bf16 fallback at the size bench.py times it (wan: H = 40, N = 32760):
    RoPE of three whole heads, attention on sampled query rows (first, middle
    and ragged last tiles of three heads) against fp64 attention over all keys."""
    import torch
    wl = si.WORKLOADS["wan"]
    dev = gu.device()
    x = si.make_inputs(wl)
    p = gu.problem_for(ra, wl)
    q, k, v, pos = gu.to_device(x, wl, dev)
    qr, kr = ra.rope_bf16(p, q, k, pos)
    lse = torch.empty(wl.B, wl.H, wl.N, dtype=torch.float32, device=dev)
    out = ra.attn_bf16_fallback(p, qr, kr, v, lse=lse)
    assert ra.sync_status() == 0
    po = orc.problem(wl)
    po.rot = 0
    num = den = 0.0
    for h in (0, 19, 39):
        qr_h, kr_h = qr[0, h].float().cpu().numpy(), kr[0, h].float().cpu().numpy()
        for name, src, got in (("q", x["q"], qr_h), ("k", x["k"], kr_h)):
            ref = gu.bf16_round(orc.rope_rotate(po, src[0, h], x["pos"]))
            u = _bf16_ulps(got, ref)
            assert u.max() <= 1.0, (name, h, u.max())
            assert np.mean(u == 0) >= 0.999, (name, h)
        v64 = v[0, h].float().cpu().numpy().astype(np.float64)
        k64 = kr_h.astype(np.float64)
        rows = np.concatenate([np.arange(0, 128), np.arange(16384, 16512), np.arange(wl.N - 120, wl.N)])
        q64 = qr_h[rows].astype(np.float64)
        ref = orc.reference_attention_fp64(q64, k64, v64)
        s = q64 @ k64.T / math.sqrt(wl.D)
        m = s.max(axis=1)
        ref_lse = m + np.log(np.exp(s - m[:, None]).sum(axis=1))
        got = out[0, h].float().cpu().numpy()[rows]
        assert np.max(np.abs(lse[0, h].cpu().numpy()[rows] - ref_lse)) <= 2e-3, h
        num += float(np.sum((got - ref) ** 2))
        den += float(np.sum(ref ** 2))
    assert math.sqrt(num / den) <= 5e-3, math.sqrt(num / den)
