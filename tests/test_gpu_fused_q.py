"""The fused-Q attention (ra_attn_int4_qfused): the attention kernel's
widening warps apply the prologue's RoPE, rotation and per-token INT4 to the
raw Q (papernotes page, highlights: the rotation rides on the elementwise RoPE
pass).  Its codes and scales must be the prologue's bit for bit, so the
output and lse must equal ra_attn_int4 on the full prologue's codes exactly;
that path is itself checked against the oracle in test_gpu_int4.py, and the
oracle is compared here once more at relative L2 1e-3.  The K/V-only prologue
(q, q4, sq NULL) must give the full prologue's K and V outputs bit for bit.
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


def _run(ra, wl, with_oracle=False):
    import torch
    dev = gu.device()
    x = si.make_inputs(wl)
    p = gu.problem_for(ra, wl)
    q, k, v, pos = gu.to_device(x, wl, dev)
    full = ra.rope_rotate_quant(p, q, k, v, pos)
    lse_ref = torch.empty(wl.B, wl.H, wl.N, dtype=torch.float32, device=dev)
    out_ref = ra.attn_int4(p, full, lse=lse_ref)
    assert ra.sync_status() == 0
    kv = ra.rope_rotate_quant(p, None, k, v, pos)
    assert ra.sync_status() == 0
    assert set(kv) == {"k4", "sk", "k_mean", "v4", "sv", "v_colsum"}
    for name, t in kv.items():
        assert torch.equal(t, full[name]), name
    # poison the output first: every element must be written
    out = torch.full_like(out_ref, float("nan"))
    lse = torch.full_like(lse_ref, float("nan"))
    ra.attn_int4_qfused(p, q, pos, kv, out=out, lse=lse)
    assert ra.sync_status() == 0
    assert torch.equal(out.view(torch.int16), out_ref.view(torch.int16))
    assert torch.equal(lse.view(torch.int32), lse_ref.view(torch.int32))
    if with_oracle:
        import oracle
        orc_p = oracle.problem(wl)
        h = 0
        ref = oracle.prologue_head(orc_p, x["q"][0, h], x["k"][0, h], x["v"][0, h], x["pos"])
        o = oracle.attention_int4_rows(orc_p, ref, 0, wl.N)["out"]
        got = out[0, h].float().cpu().numpy()
        assert gu.rel_l2(got, gu.bf16_round(o)) <= 1e-3


@pytest.mark.parametrize("rot", [0, 1, 2, 3])
@pytest.mark.parametrize("D,seg", [(128, (44, 42, 42)), (64, (24, 20, 20))])
def test_fused_q_equals_unfused(ra, rot, D, seg):
    # N = 300: two items' worth of 128-row tiles with a ragged last tile and a
    # ragged last key block; two heads.
    wl = si.WORKLOADS["small"].with_(H=2, D=D, seg=seg, grid=(3, 10, 10), rot=rot, block_k=64)
    _run(ra, wl, with_oracle=(rot == 2 and D == 128))


def test_fused_q_fp32_inputs(ra):
    wl = si.WORKLOADS["tiny"].with_(grid=(2, 8, 9), block_q=128, block_k=64)   # fp32, D = 64, N = 144
    _run(ra, wl, with_oracle=True)


def test_fused_q_at_the_wan_shape(ra):
    # The full Wan shape (N = 32760, 40 heads): every item of the grid runs.
    _run(ra, si.WORKLOADS["wan"])


def test_fused_q_sharp(ra):
    wl = si.WORKLOADS["small"].with_(H=2, grid=(4, 8, 8), sharp=True)
    _run(ra, wl, with_oracle=True)
