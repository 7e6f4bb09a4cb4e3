"""Accuracy of the INT4 method itself, measured with the oracle (test
infrastructure; no GPU).

For sampled heads of the Wan-like and HunyuanVideo-like workloads, the oracle's
INT4 attention output is compared (cosine and relative L2, over a fixed sample
of query rows spread across the sequence, each against all keys) with
unquantised fp64 softmax attention on the RoPE'd inputs, for every rotation
mode (none, interleaved 2x2, half, full D x D Hadamard) and the P-code /
denominator modes of the attention (range-rectified codes against the running
maximum with the code-sum denominator -- the method -- and the alternatives it
is compared with: the fp32 denominator, codes against each block's own maximum,
symmetric codes).  Inputs follow the seeded recipe of synth/inputs.py, with and
without the per-row RMS normalisation of Q and K.

  python -m oracle.method_accuracy [--rows 512] [--heads 0,19]

prints one markdown table row per (workload, recipe, rotation, mode).
"""
from __future__ import annotations

import argparse
import os
import sys

import numpy as np

if __package__ in (None, ""):
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import oracle  # noqa: E402
from synth import inputs as si  # noqa: E402

ROTATIONS = (("none", 0), ("interleaved", 1), ("half", 2), ("full", 3))
MODES = (("range, code-sum l", 0, 0), ("range, fp32 l", 0, 1), ("block-local max", 1, 0), ("symmetric P", 2, 0))


def sample_rows(n: int, count: int) -> np.ndarray:
    """count query rows in 128-row groups spread evenly over [0, n)."""
    groups = max(1, count // 128)
    starts = np.linspace(0, max(0, n - 128), groups).astype(int) // 128 * 128
    return np.unique(np.concatenate([np.arange(s, min(s + 128, n)) for s in starts]))


def head_accuracy(wl, x, head: int, rows: np.ndarray):
    """{(rotation, mode name): (cosine, relative L2)} for one head."""
    res = {}
    q, k, v, pos = x["q"][0, head], x["k"][0, head], x["v"][0, head], x["pos"]
    p0 = oracle.problem(wl.with_(rot=0))
    qr, kr = oracle.rope_rotate(p0, q, pos), oracle.rope_rotate(p0, k, pos)
    ref = oracle.reference_attention_fp64(qr[rows], kr, v)
    for rname, rot in ROTATIONS:
        for mname, pm, lm in MODES:
            p = oracle.problem(wl.with_(rot=rot), p_mode=pm, l_mode=lm)
            h = oracle.prologue_head(p, q, k, v, pos)
            # rows are whole 128-row groups (sample_rows), in order
            out = np.concatenate([oracle.attention_int4_rows(p, h, int(r0), min(int(r0) + 128, wl.N))["out"]
                                  for r0 in np.unique(rows // 128 * 128)])
            assert out.shape == ref.shape
            a, b = out.ravel(), ref.ravel()
            cos = float(a @ b / np.linalg.norm(a) / np.linalg.norm(b))
            rel = float(np.linalg.norm(a - b) / np.linalg.norm(b))
            res[(rname, mname)] = (cos, rel)
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--rows", type=int, default=512)
    ap.add_argument("--heads", default="0,19")
    ap.add_argument("--workloads", default="wan,hunyuan")
    args = ap.parse_args()
    heads = tuple(int(h) for h in args.heads.split(","))
    print("| workload | inputs | rotation | P codes / denominator | cosine | rel. L2 |")
    print("|---|---|---|---|---|---|")
    for name in args.workloads.split(","):
        for recipe, norm in (("RMS-normalised", True), ("literal recipe", False)):
            wl = si.WORKLOADS[name].with_(rms_norm=norm)
            x = si.make_inputs(wl, heads=heads)
            rows = sample_rows(wl.N, args.rows)
            acc = {}
            for hi, _ in enumerate(heads):
                for key, (c, r) in head_accuracy(wl, {k2: (v2[:, hi:hi + 1] if v2.ndim == 4 else v2)
                                                     for k2, v2 in x.items()}, 0, rows).items():
                    acc.setdefault(key, []).append((c, r))
            for (rname, mname), vals in acc.items():
                c = float(np.mean([v[0] for v in vals]))
                r = float(np.mean([v[1] for v in vals]))
                print(f"| {name} | {recipe} | {rname} | {mname} | {c:.4f} | {r:.4f} |", flush=True)


if __name__ == "__main__":
    main()
