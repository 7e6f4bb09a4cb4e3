"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
on seeded inputs and the oracle on the same inputs."""
from __future__ import annotations

import numpy as np
import pytest

from synth import inputs as si


def device():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU test selected but no CUDA device is visible")
    return torch.device("cuda:0")


def problem_for(ra, wl):
    return ra.Problem.make(wl.B, wl.H, wl.D, wl.seg, wl.grid, theta=wl.theta, rot=wl.rot,
                           block_q=wl.block_q, block_k=wl.block_k)


def to_device(x, wl, dev):
    import torch
    if wl.dtype == "bf16":
        t = lambda n: torch.from_numpy(x[n + "_bits"]).view(torch.bfloat16).to(dev)  # noqa: E731
    else:
        t = lambda n: torch.from_numpy(x[n]).to(dev)  # noqa: E731
    return t("q"), t("k"), t("v"), torch.from_numpy(x["pos"]).to(dev)


def gpu_forward(ra, wl, x, dev, with_lse=False, p_mode=0, l_mode=0):
    import torch
    p = problem_for(ra, wl)
    q, k, v, pos = to_device(x, wl, dev)
    codes = ra.rope_rotate_quant(p, q, k, v, pos)
    lse = torch.empty(wl.B, wl.H, wl.N, dtype=torch.float32, device=dev) if with_lse else None
    out = ra.attn_int4(p, codes, lse=lse, p_mode=p_mode, l_mode=l_mode)
    assert ra.sync_status() == 0
    host = {k2: t.cpu().numpy() for k2, t in codes.items()}
    host["out"] = out.float().cpu().numpy()
    if with_lse:
        host["lse"] = lse.cpu().numpy()
    return p, codes, host


def bf16_round(a):
    return si.bf16_bits_to_f32(si.f32_to_bf16_bits(np.asarray(a, np.float32)))


def rel_l2(got, ref):
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))


def code_agreement(a4, b4, orc):
    """(fraction equal, max |difference|) of two packed code arrays."""
    a = orc.unpack_codes(a4).astype(np.int16)
    b = orc.unpack_codes(b4).astype(np.int16)
    return float((a == b).mean()), int(np.abs(a - b).max()) if a.size else 0


def head_codes(host, bh):
    """The GPU prologue outputs of one head in the oracle's per-head layout."""
    b, h = bh
    return {k: host[k][b, h] for k in ("q4", "sq", "k4", "sk", "v4", "sv", "v_colsum")} | {
        "colsum": host["v_colsum"][b, h]}
