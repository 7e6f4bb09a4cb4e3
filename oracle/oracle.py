"""numpy front end of the C oracle (test infrastructure; see ra_oracle.c).

Every function here marshals numpy arrays into the C routines; the arithmetic
lives in ra_oracle.c.  Arrays of one head are [N, D]; packed code arrays are
[N, D/2] uint8 (element 2t in the low nibble, 4-bit two's complement).
"""
from __future__ import annotations

import ctypes as C
import math
from typing import Dict, Optional

import numpy as np

from . import build_oracle

_lib = None


class OrcProblem(C.Structure):
    _fields_ = [("B", C.c_int), ("H", C.c_int), ("N", C.c_int), ("D", C.c_int),
                ("seg", C.c_int * 3), ("grid", C.c_int * 3), ("theta", C.c_double),
                ("rot", C.c_int), ("block_q", C.c_int), ("block_k", C.c_int),
                ("p_mode", C.c_int), ("l_mode", C.c_int)]


# Ablation switches of the attention (reading R11 in ra_oracle.c).
P_RANGE, P_LOCAL, P_SYMMETRIC = 0, 1, 2
L_CODES, L_FP32 = 0, 1


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build_oracle.build())
        P = C.POINTER
        vp = C.c_void_p
        _lib.orc_table_len.argtypes = [P(OrcProblem)]
        _lib.orc_rope_tables.argtypes = [P(OrcProblem), vp, vp]
        _lib.orc_rope_rotate.argtypes = [P(OrcProblem), vp, vp, vp, C.c_int]
        _lib.orc_prologue_head.argtypes = [P(OrcProblem)] + [vp] * 14
        _lib.orc_p_code.argtypes = [C.c_float, C.c_float]
        _lib.orc_p_code_sym.argtypes = [C.c_float, C.c_float]
        _lib.orc_attention_int4_rows.argtypes = [P(OrcProblem)] + [vp] * 7 + [C.c_int, C.c_int] + [vp] * 5
        _lib.orc_attention_int4_rows_given_codes.argtypes = [P(OrcProblem)] + [vp] * 8 + [C.c_int, C.c_int, vp, vp]
        _lib.orc_attention_exact_blocked_rows.argtypes = [P(OrcProblem), vp, vp, vp, C.c_int, C.c_int, vp, vp]
        _lib.orc_rotation_matrix.argtypes = [P(OrcProblem), vp]
        _lib.orc_rope_matrix.argtypes = [P(OrcProblem), vp, vp]
        _lib.orc_num_threads.argtypes = []
    return _lib


def problem(wl=None, *, N=None, D=None, seg=None, grid=None, theta=10000.0, rot=1,
            block_q=128, block_k=64, B=1, H=1, p_mode=P_RANGE, l_mode=L_CODES) -> OrcProblem:
    """Build the C problem struct from a synth.inputs.Workload or keywords."""
    if wl is not None:
        B, H, D, seg, grid = wl.B, wl.H, wl.D, wl.seg, wl.grid
        theta, rot, block_q, block_k = wl.theta, wl.rot, wl.block_q, wl.block_k
        N = wl.N
    if N is None:
        N = grid[0] * grid[1] * grid[2]
    p = OrcProblem()
    p.B, p.H, p.N, p.D = B, H, N, D
    p.seg[:] = list(seg)
    p.grid[:] = list(grid)
    p.theta, p.rot, p.block_q, p.block_k = float(theta), int(rot), int(block_q), int(block_k)
    p.p_mode, p.l_mode = int(p_mode), int(l_mode)
    return p


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what}: invalid arguments")


def num_threads() -> int:
    return int(lib().orc_num_threads())


def rope_tables(p: OrcProblem):
    n = lib().orc_table_len(C.byref(p))
    a = np.empty(n, np.float32)
    b = np.empty(n, np.float32)
    _check(lib().orc_rope_tables(C.byref(p), _ptr(a), _ptr(b)), "rope_tables")
    return a, b


def rope_rotate(p: OrcProblem, x: np.ndarray, pos: np.ndarray, swap_order: bool = False) -> np.ndarray:
    """RoPE + rotation of one head's rows x [N, D] (fp32), per the oracle's rules."""
    if x.shape != (p.N, p.D) or len(pos) != p.N:
        raise ValueError(f"rope_rotate: x {x.shape} / pos {len(pos)} do not match N={p.N}, D={p.D}")
    x = np.ascontiguousarray(x, np.float32)
    pos = np.ascontiguousarray(pos, np.int32)
    out = np.empty_like(x)
    _check(lib().orc_rope_rotate(C.byref(p), _ptr(x), _ptr(pos), _ptr(out), int(swap_order)),
           "rope_rotate")
    return out


def prologue_head(p: OrcProblem, q: np.ndarray, k: np.ndarray, v: np.ndarray, pos: np.ndarray,
                  want_rot: bool = False) -> Dict[str, np.ndarray]:
    """Prologue of one head: returns q4, sq, k4, sk, kmean, v4, sv, colsum (+ q_rot, k_rot)."""
    N, D = p.N, p.D
    q = np.ascontiguousarray(q, np.float32)
    k = np.ascontiguousarray(k, np.float32)
    v = np.ascontiguousarray(v, np.float32)
    pos = np.ascontiguousarray(pos, np.int32)
    nb = (N + p.block_k - 1) // p.block_k
    r = {
        "q4": np.empty((N, D // 2), np.uint8), "sq": np.empty(N, np.float32),
        "k4": np.empty((N, D // 2), np.uint8), "sk": np.empty(N, np.float32),
        "kmean": np.empty(D, np.float32), "v4": np.empty((N, D // 2), np.uint8),
        "sv": np.empty(D, np.float32), "colsum": np.empty((nb, D), np.int32),
    }
    if want_rot:
        r["q_rot"] = np.empty((N, D), np.float32)
        r["k_rot"] = np.empty((N, D), np.float32)
    rc = lib().orc_prologue_head(C.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(pos),
                                 _ptr(r["q4"]), _ptr(r["sq"]), _ptr(r["k4"]), _ptr(r["sk"]),
                                 _ptr(r["kmean"]), _ptr(r["v4"]), _ptr(r["sv"]), _ptr(r["colsum"]),
                                 _ptr(r.get("q_rot")), _ptr(r.get("k_rot")))
    _check(rc, "prologue_head")
    return r


def p_code(S: float, m: float) -> int:
    return int(lib().orc_p_code(C.c_float(S), C.c_float(m)))


def p_code_sym(S: float, m: float) -> int:
    return int(lib().orc_p_code_sym(C.c_float(S), C.c_float(m)))


def attention_int4_rows(p: OrcProblem, h: Dict[str, np.ndarray], row0: int, row1: int,
                        dumps: bool = False) -> Dict[str, np.ndarray]:
    """INT4 attention of rows [row0, row1) of one head from its prologue outputs h."""
    N, D = p.N, p.D
    R = row1 - row0
    nb = (N + p.block_k - 1) // p.block_k
    out = np.empty((R, D), np.float64)
    lse = np.empty(R, np.float64)
    r = {"out": out, "lse": lse}
    if dumps:
        r["s_int"] = np.empty((R, N), np.int32)
        r["codes"] = np.empty((R, N), np.int8)
        r["acc"] = np.empty((R, nb, D), np.int32)
    args = [np.ascontiguousarray(h[k]) for k in ("q4", "sq", "k4", "sk", "v4", "sv", "colsum")]
    rc = lib().orc_attention_int4_rows(C.byref(p), *[_ptr(a) for a in args], int(row0), int(row1),
                                       _ptr(out), _ptr(lse), _ptr(r.get("s_int")),
                                       _ptr(r.get("codes")), _ptr(r.get("acc")))
    _check(rc, "attention_int4_rows")
    return r


def attention_int4_rows_given_codes(p: OrcProblem, h: Dict[str, np.ndarray], codes: np.ndarray,
                                    row0: int, row1: int) -> Dict[str, np.ndarray]:
    """INT4 attention of rows [row0, row1) with the P codes given ([rows, N] int8)."""
    R = row1 - row0
    out = np.empty((R, p.D), np.float64)
    lse = np.empty(R, np.float64)
    codes = np.ascontiguousarray(codes, np.int8)
    assert codes.shape == (R, p.N)
    args = [np.ascontiguousarray(h[k]) for k in ("q4", "sq", "k4", "sk", "v4", "sv", "colsum")]
    rc = lib().orc_attention_int4_rows_given_codes(C.byref(p), *[_ptr(a) for a in args], _ptr(codes),
                                                   int(row0), int(row1), _ptr(out), _ptr(lse))
    _check(rc, "attention_int4_rows_given_codes")
    return {"out": out, "lse": lse}


def attention_exact_blocked_rows(p: OrcProblem, q: np.ndarray, k: np.ndarray, v: np.ndarray,
                                 row0: int = 0, row1: Optional[int] = None):
    """The same blocked online-softmax recurrence on unquantised fp64 inputs."""
    row1 = p.N if row1 is None else row1
    q = np.ascontiguousarray(q, np.float64)
    k = np.ascontiguousarray(k, np.float64)
    v = np.ascontiguousarray(v, np.float64)
    out = np.empty((row1 - row0, p.D), np.float64)
    lse = np.empty(row1 - row0, np.float64)
    _check(lib().orc_attention_exact_blocked_rows(C.byref(p), _ptr(q), _ptr(k), _ptr(v),
                                                  int(row0), int(row1), _ptr(out), _ptr(lse)),
           "attention_exact_blocked_rows")
    return out, lse


def rotation_matrix(p: OrcProblem) -> np.ndarray:
    R = np.empty((p.D, p.D), np.float64)
    _check(lib().orc_rotation_matrix(C.byref(p), _ptr(R)), "rotation_matrix")
    return R


def rope_matrix(p: OrcProblem, pos3) -> np.ndarray:
    M = np.empty((p.D, p.D), np.float64)
    pos3 = np.ascontiguousarray(pos3, np.int32)
    _check(lib().orc_rope_matrix(C.byref(p), _ptr(pos3), _ptr(M)), "rope_matrix")
    return M


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    """[..., D/2] uint8 -> [..., D] int8 (low nibble = even element, two's complement)."""
    lo = (packed & 0xF).astype(np.int8)
    hi = (packed >> 4).astype(np.int8)
    lo = np.where(lo >= 8, lo - 16, lo).astype(np.int8)
    hi = np.where(hi >= 8, hi - 16, hi).astype(np.int8)
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), np.int8)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


def reference_attention_fp64(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """Unquantised softmax(q k^T / sqrt(D)) v of one head in fp64 (the accuracy reference)."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    s = q @ k.T / math.sqrt(q.shape[1])
    s -= s.max(axis=1, keepdims=True)
    p = np.exp(s)
    return (p @ v) / p.sum(axis=1, keepdims=True)
