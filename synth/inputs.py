"""Seeded synthetic inputs for the RotateAttention attention workloads.

This module is shared by the CPU oracle's tests and by the CUDA path's tests and
benchmark.  It draws random tensors with the shapes and outlier structure of
video-DiT attention and contains none of the method's arithmetic: no RoPE, no
rotation, no smoothing, no quantisation, no attention.

Workloads (all B=1; positions enumerate a frames x height x width grid):

  tiny     H=1,  grid 2x4x4    (N=32),     D=64,  segments 24/20/20, interleaved, fp32
  small    H=2,  grid 4x8x8    (N=256),    D=128, segments 44/42/42, half,        bf16
  wan      H=40, grid 21x30x52 (N=32760),  D=128, segments 44/42/42, interleaved, bf16
  hunyuan  H=24, grid 33x45x80 (N=118800), D=128, segments 16/56/56, half,        bf16
  sweep-N  H=40, D=128, 44/42/42, N in {4096, 8192, 16384, 32760, 65536},
           interleaved (sweepN) and half rotation (sweepN_half); sweepN_sharp
           is the interleaved sweep with the sharp-P variant

Outlier recipe (the pages report that after 3D RoPE the Q/K outliers sit inside
each frame/height/width segment, mostly in its first half, and are shared by Q
and K -- RotateAttention, papernotes page, "key design 1"):

  * Q, K ~ N(0, 1) per element.
  * A seeded subset of channels, drawn from the first half of every segment, is
    multiplied by a per-channel factor; the same channels and factors are used
    for Q and K of a head.  tiny: 50% of each first half, factor 20.  others:
    25% of all channels (taken from the first halves), factor ~ U(10, 30).
  * K gets a per-channel offset ~ U(-3, 3) (the channel bias that motivates K
    smoothing).
  * Every Q and K row is then divided by its root-mean-square over the D
    channels (the q/k RMS normalisation video DiTs apply before RoPE).  Without
    it the recipe's logits q.k/sqrt(D) have a standard deviation near 200 and
    every softmax row is already one-hot; with it the deviation is about 2, and
    the sharp variant below (x8) is the near-one-hot case.
  * V ~ N(0, 1); for bf16 workloads 5% of channels are multiplied by 8.  The
    wan / hunyuan / sweep workloads then right-multiply V by the normalised
    128-point Sylvester Hadamard matrix: the offline V transform the pages
    absorb into W_v and W_o ("key design 3"), applied here to the synthetic V.
  * sharp=True multiplies Q by 8 (near one-hot softmax rows).
  * rms_norm=False skips the normalisation (the recipe as literally stated,
    used only to measure what the normalisation changes in the accuracy).

bf16 tensors are produced from fp32 by round-to-nearest-even and returned as
uint16 bit patterns so that both sides read exactly the same values.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Tuple

import numpy as np

ROT_INTERLEAVED = 1
ROT_HALF = 2


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    grid: Tuple[int, int, int]
    D: int
    seg: Tuple[int, int, int]
    rot: int
    block_q: int
    block_k: int
    dtype: str          # "f32" or "bf16"
    seed: int
    theta: float = 10000.0
    v_hadamard: bool = False
    sharp: bool = False
    rms_norm: bool = True      # False: the literal recipe, without the per-row RMS normalisation

    @property
    def N(self) -> int:
        return self.grid[0] * self.grid[1] * self.grid[2]

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    def attn_ops(self) -> float:
        """Algorithmic integer ops of one attention call: 4 * N^2 * D * H * B."""
        return 4.0 * self.N * self.N * self.D * self.H * self.B


SWEEP_GRIDS = {
    4096: (1, 64, 64),
    8192: (2, 64, 64),
    16384: (4, 64, 64),
    32760: (21, 30, 52),
    65536: (16, 64, 64),
}


def _sweep(n: int, i: int, rot: int) -> Workload:
    return Workload(f"sweep{n}", 1, 40, SWEEP_GRIDS[n], 128, (44, 42, 42), rot,
                    128, 64, "bf16", 10 + i, v_hadamard=True)


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", 1, 1, (2, 4, 4), 64, (24, 20, 20), ROT_INTERLEAVED,
                     16, 16, "f32", 0),
    "small": Workload("small", 1, 2, (4, 8, 8), 128, (44, 42, 42), ROT_HALF,
                      128, 64, "bf16", 1),
    "wan": Workload("wan", 1, 40, (21, 30, 52), 128, (44, 42, 42), ROT_INTERLEAVED,
                    128, 64, "bf16", 2, v_hadamard=True),
    "hunyuan": Workload("hunyuan", 1, 24, (33, 45, 80), 128, (16, 56, 56), ROT_HALF,
                        128, 64, "bf16", 3, v_hadamard=True),
}
for _i, _n in enumerate(sorted(SWEEP_GRIDS)):
    WORKLOADS[f"sweep{_n}"] = _sweep(_n, _i, ROT_INTERLEAVED)
    # the sweep in the other rotation mode (same tensors, same seed)
    WORKLOADS[f"sweep{_n}_half"] = _sweep(_n, _i, ROT_HALF).with_(name=f"sweep{_n}_half")
    # the sharp-P variant (Q x8: near one-hot softmax rows), interleaved rotation
    WORKLOADS[f"sweep{_n}_sharp"] = _sweep(_n, _i, ROT_INTERLEAVED).with_(name=f"sweep{_n}_sharp", sharp=True)


def positions(grid: Tuple[int, int, int]) -> np.ndarray:
    """[N, 3] int32 (frame, row, col) with token n = (f * Gh + y) * Gw + x."""
    gf, gh, gw = grid
    f, y, x = np.meshgrid(np.arange(gf), np.arange(gh), np.arange(gw), indexing="ij")
    return np.stack([f.ravel(), y.ravel(), x.ravel()], axis=1).astype(np.int32)


def sylvester_hadamard(n: int) -> np.ndarray:
    """Normalised Sylvester Hadamard matrix H_n (n a power of two), float64."""
    h = np.ones((1, 1))
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h / np.sqrt(n)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _outlier_channels(rng: np.random.Generator, wl: Workload) -> np.ndarray:
    """Channel indices drawn from the first half of each RoPE segment."""
    chans = []
    off = 0
    for dj in wl.seg:
        half = np.arange(off, off + dj // 2)
        if wl.name == "tiny":
            k = len(half) // 2                       # 50% of the first half
        else:
            k = int(round(0.25 * dj))                # 25% of the segment's channels
            k = min(k, len(half))
        chans.append(rng.choice(half, size=k, replace=False))
        off += dj
    return np.sort(np.concatenate(chans))


def make_inputs(wl: Workload, heads: Tuple[int, ...] | None = None) -> Dict[str, np.ndarray]:
    """Draw Q, K, V [B, H, N, D] and positions [N, 3] for a workload.

    heads restricts generation to a subset of heads (others are not drawn); each
    head has its own generator stream seeded by (seed, b, h), so a head's data
    does not depend on which other heads were requested.

    Returns float32 arrays under 'q','k','v' (the exact values both sides use)
    and, for bf16 workloads, the uint16 bit patterns under 'q_bits' etc.
    """
    B, H, N, D = wl.B, wl.H, wl.N, wl.D
    hs = tuple(range(H)) if heads is None else tuple(heads)
    out = {name: np.empty((B, len(hs), N, D), dtype=np.float32) for name in ("q", "k", "v")}
    hmat = sylvester_hadamard(D).astype(np.float32) if wl.v_hadamard else None
    for b in range(B):
        for hi, h in enumerate(hs):
            rng = np.random.default_rng([wl.seed, b, h])
            q = rng.standard_normal((N, D), dtype=np.float32)
            k = rng.standard_normal((N, D), dtype=np.float32)
            v = rng.standard_normal((N, D), dtype=np.float32)
            ch = _outlier_channels(rng, wl)
            if wl.name == "tiny":
                fac = np.full(len(ch), 20.0, dtype=np.float32)
            else:
                fac = rng.uniform(10.0, 30.0, size=len(ch)).astype(np.float32)
            q[:, ch] *= fac
            k[:, ch] *= fac
            k += rng.uniform(-3.0, 3.0, size=D).astype(np.float32)
            if wl.rms_norm:
                q /= np.sqrt(np.mean(q * q, axis=1, keepdims=True, dtype=np.float32))
                k /= np.sqrt(np.mean(k * k, axis=1, keepdims=True, dtype=np.float32))
            if wl.dtype == "bf16":
                vch = rng.choice(D, size=max(1, int(round(0.05 * D))), replace=False)
                v[:, vch] *= 8.0
            if hmat is not None:
                v = v @ hmat
            if wl.sharp:
                q *= 8.0
            out["q"][b, hi], out["k"][b, hi], out["v"][b, hi] = q, k, v
    if wl.dtype == "bf16":
        for name in ("q", "k", "v"):
            bits = f32_to_bf16_bits(out[name])
            out[name + "_bits"] = bits
            out[name] = bf16_bits_to_f32(bits)
    out["pos"] = positions(wl.grid)
    return out
