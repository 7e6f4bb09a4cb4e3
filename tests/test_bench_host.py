"""Host-side logic of bench.py that needs no GPU: the algorithmic byte count of
the prologue, the workload description, and the rule that the committed DRAM
traffic is reported only for the kernel sources it was measured on."""
import hashlib
import os

import pytest

import bench
from synth import inputs as si


def test_prologue_bytes_by_hand():
    """Wan with 128-key blocks: reads Q once, K and V twice (bf16, 5 x 335,462,400
    bytes); writes three packed code tensors (3 x 83,865,600), two per-token
    scale tensors (2 x 5,241,600), three per-channel vectors (3 x 20,480) and
    the colsums (4 x 40 x 256 x 128): 1,944,696,320 bytes."""
    wl = si.WORKLOADS["wan"].with_(block_k=128)
    assert bench.prologue_bytes(wl) == 1_944_696_320
    # 64-key blocks double the colsum rows (512 per head)
    assert bench.prologue_bytes(si.WORKLOADS["wan"]) == 1_944_696_320 + 4 * 40 * 256 * 128


@pytest.mark.parametrize("rot,name", [(0, "none"), (1, "interleaved"), (2, "half"), (3, "full")])
def test_config_names_every_rotation_mode(rot, name):
    c = bench._config(si.WORKLOADS["small"].with_(rot=rot))
    assert c["rot"] == name and name in c["workload"]
    assert c["N"] == 256 and c["block_k"] == 64


def _fake_tree(tmp_path, sources, recorded_sources):
    csrc = tmp_path / "int4_quantized_flashattention_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name, text in sources.items():
        (csrc / name).write_bytes(text)
    h = hashlib.sha256()
    for name in ("ra_attn_int4.cu", "ra_common.cuh"):
        h.update(recorded_sources[name])
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "launches_wan.md").write_text(
        f"traffic_bytes_per_launch: 12345\nkernel_sources_sha256: {h.hexdigest()}\n")


def test_traffic_is_reported_only_for_the_measured_sources(tmp_path, monkeypatch):
    src = {"ra_attn_int4.cu": b"kernel v1", "ra_common.cuh": b"helpers"}
    _fake_tree(tmp_path, src, src)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench._attn_traffic() == 12345
    (tmp_path / "int4_quantized_flashattention_b200" / "csrc" / "ra_attn_int4.cu").write_bytes(b"kernel v2")
    assert bench._attn_traffic() is None



def test_launch_count_per_step_by_rotation_mode():
    """The interleaved rotation builds two RoPE tables (the fused one and the
    plain one of the channel reduce), the other modes one: reduce, finalize,
    quantise and the attention make the rest."""
    assert bench.kernels_per_step(1) == 6
    for rot in (0, 2, 3):
        assert bench.kernels_per_step(rot) == 5


def test_reference_arm_marks_its_time_as_extrapolated():
    """--impl reference on a small workload: the line carries the sample's own
    time beside the extrapolated step time, and the e2e object the contract
    asks for (no host-device copies)."""
    import argparse
    args = argparse.Namespace(workload="tiny", block_k=None, steps=1, warmup=3, ref_seconds=1.0)
    r = bench.run_reference(args)
    assert r["impl"] == "reference" and r["extrapolated"] is True
    assert r["sample_ms_per_step"] > 0 and r["ms_per_step"] > 0
    assert r["cpu_baseline"]["kind"] == "oracle" and r["cpu_baseline"]["cores"] >= 1
    assert r["e2e"]["h2d_bytes_per_step"] == 0 and r["e2e"]["d2h_bytes_per_step"] == 0
    assert r["e2e"]["value"] == r["value"]
