"""RotateAttention INT4 attention forward for NVIDIA B200 (sm_100a).

Thin ctypes binding over the C-ABI library libra.so (see include/ra.h): every
function below only checks and marshals torch tensors (device memory and the
current CUDA stream) and calls the entry point of the same name.  All the work
runs in the library's CUDA kernels; there is no other implementation, and the
module raises if the library is missing.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Dict, Optional, Sequence

import torch

__all__ = [
    "ROT_NONE", "ROT_INTERLEAVED", "ROT_HALF", "ROT_FULL", "RaError", "Problem", "lib", "workspace_bytes",
    "rope_rotate_quant", "attn_int4", "test_int4_codes", "rope_bf16", "attn_bf16_fallback",
    "attn_int4_qfused", "rope_rotate_quant_s8", "attn_int4_s8", "sync_status", "library_path", "AttnOpts", "P_RANGE", "P_LOCAL_MAX", "P_SYMMETRIC", "L_CODES", "L_FP32",
]

ROT_NONE, ROT_INTERLEAVED, ROT_HALF, ROT_FULL = 0, 1, 2, 3
DT_F32, DT_BF16 = 0, 1
P_RANGE, P_LOCAL_MAX, P_SYMMETRIC = 0, 1, 2   # ra_attn_opts.p_mode
L_CODES, L_FP32 = 0, 1                        # ra_attn_opts.l_mode

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libra.so")
_lib = None


class RaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn}: {status_string(status)} (status {status})")
        self.status = status


class Problem(C.Structure):
    """ra_problem: B, H, N, D, seg[3], grid[3], theta, rot, block_q, block_k."""
    _fields_ = [("B", C.c_int), ("H", C.c_int), ("N", C.c_int), ("D", C.c_int),
                ("seg", C.c_int * 3), ("grid", C.c_int * 3), ("theta", C.c_float),
                ("rot", C.c_int), ("block_q", C.c_int), ("block_k", C.c_int)]

    @classmethod
    def make(cls, B: int, H: int, D: int, seg: Sequence[int], grid: Sequence[int], *, N: Optional[int] = None,
             theta: float = 10000.0, rot: int = ROT_INTERLEAVED, block_q: int = 128, block_k: int = 64) -> "Problem":
        p = cls()
        p.B, p.H, p.D = B, H, D
        p.N = int(grid[0] * grid[1] * grid[2]) if N is None else int(N)
        p.seg[:] = list(seg)
        p.grid[:] = list(grid)
        p.theta, p.rot, p.block_q, p.block_k = float(theta), int(rot), int(block_q), int(block_k)
        return p


class AttnOpts(C.Structure):
    """ra_attn_opts: the ablation switches of the INT4 attention."""
    _fields_ = [("p_mode", C.c_int), ("l_mode", C.c_int)]


def _opts(p_mode: int, l_mode: int):
    return None if (p_mode, l_mode) == (P_RANGE, L_CODES) else C.byref(AttnOpts(int(p_mode), int(l_mode)))


def lib():
    """Loads libra.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(library_path):
            raise RuntimeError(f"{library_path} is missing: build it with __graft_entry__.build()")
        L = C.CDLL(library_path)
        P, vp, sz = C.POINTER(Problem), C.c_void_p, C.c_size_t
        L.ra_status_string.restype = C.c_char_p
        L.ra_status_string.argtypes = [C.c_int]
        L.ra_workspace_bytes.restype = sz
        L.ra_workspace_bytes.argtypes = [P]
        L.ra_rope_rotate_quant.argtypes = [P, C.c_int] + [vp] * 13 + [sz, vp]
        L.ra_attn_int4.argtypes = [P] + [vp] * 9
        L.ra_test_int4_codes.argtypes = [P] + [vp] * 6 + [C.c_int] * 3 + [vp] * 6
        L.ra_attn_int4_opts.argtypes = [P, vp] + [vp] * 9
        L.ra_test_int4_codes_opts.argtypes = [P, vp] + [vp] * 6 + [C.c_int] * 3 + [vp] * 6
        L.ra_rope_bf16.argtypes = [P, C.c_int] + [vp] * 6 + [sz, vp]
        L.ra_attn_bf16_fallback.argtypes = [P] + [vp] * 6
        L.ra_attn_int4_qfused.argtypes = [P, C.c_int] + [vp] * 7 + [sz] + [vp] * 3
        L.ra_rope_rotate_quant_s8.argtypes = [P, C.c_int] + [vp] * 13 + [sz, vp]
        L.ra_attn_int4_s8.argtypes = [P] + [vp] * 9
        L.ra_sync_status.argtypes = [vp]
        for name in ("ra_rope_rotate_quant", "ra_attn_int4", "ra_test_int4_codes", "ra_rope_bf16",
                     "ra_attn_bf16_fallback", "ra_sync_status", "ra_attn_int4_opts", "ra_test_int4_codes_opts",
                     "ra_attn_int4_qfused", "ra_rope_rotate_quant_s8", "ra_attn_int4_s8"):
            getattr(L, name).restype = C.c_int
        _lib = L
    return _lib


def status_string(s: int) -> str:
    return lib().ra_status_string(int(s)).decode()


def _check(fn: str, rc: int):
    if rc != 0:
        raise RaError(fn, rc)


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: Optional[torch.Tensor], dtype=None, shape=None, name="tensor"):
    if t is None:
        return None
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return C.c_void_p(t.data_ptr())


def _in_dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return DT_BF16
    if t.dtype == torch.float32:
        return DT_F32
    raise ValueError("inputs must be bfloat16 or float32")


def workspace_bytes(p: Problem) -> int:
    return int(lib().ra_workspace_bytes(C.byref(p)))


def _nblocks(p: Problem) -> int:
    return (p.N + p.block_k - 1) // p.block_k


def rope_rotate_quant(p: Problem, q: Optional[torch.Tensor], k: torch.Tensor, v: torch.Tensor, pos: torch.Tensor,
                      out: Optional[Dict[str, torch.Tensor]] = None, workspace: Optional[torch.Tensor] = None,
                      stream=None) -> Dict[str, torch.Tensor]:
    """ra_rope_rotate_quant: returns q4, sq, k4, sk, k_mean, v4, sv, v_colsum.
    q = None runs K and V only (for attn_int4_qfused); q4 and sq are then absent."""
    B, H, N, D = p.B, p.H, p.N, p.D
    dev = k.device
    if out is None:
        out = {} if q is None else {
            "q4": torch.empty(B, H, N, D // 2, dtype=torch.uint8, device=dev),
            "sq": torch.empty(B, H, N, dtype=torch.float32, device=dev)}
        out.update({
            "k4": torch.empty(B, H, N, D // 2, dtype=torch.uint8, device=dev),
            "sk": torch.empty(B, H, N, dtype=torch.float32, device=dev),
            "k_mean": torch.empty(B, H, D, dtype=torch.float32, device=dev),
            "v4": torch.empty(B, H, N, D // 2, dtype=torch.uint8, device=dev),
            "sv": torch.empty(B, H, D, dtype=torch.float32, device=dev),
            "v_colsum": torch.empty(B, H, _nblocks(p), D, dtype=torch.int32, device=dev),
        })
    if workspace is None:
        workspace = torch.empty(max(workspace_bytes(p), 16), dtype=torch.uint8, device=dev)
    dt = _in_dtype(k)
    shp = (B, H, N, D)
    rc = lib().ra_rope_rotate_quant(
        C.byref(p), dt, _ptr(q, k.dtype, shp, "q"), _ptr(k, k.dtype, shp, "k"), _ptr(v, k.dtype, shp, "v"),
        _ptr(pos, torch.int32, (N, 3), "pos"),
        _ptr(out.get("q4") if q is not None else None, torch.uint8, (B, H, N, D // 2)),
        _ptr(out.get("sq") if q is not None else None, torch.float32, (B, H, N)),
        _ptr(out["k4"], torch.uint8, (B, H, N, D // 2)), _ptr(out["sk"], torch.float32, (B, H, N)),
        _ptr(out["k_mean"], torch.float32, (B, H, D)), _ptr(out["v4"], torch.uint8, (B, H, N, D // 2)),
        _ptr(out["sv"], torch.float32, (B, H, D)), _ptr(out["v_colsum"], torch.int32, (B, H, _nblocks(p), D)),
        _ptr(workspace, torch.uint8), C.c_size_t(workspace.numel()), C.c_void_p(_stream(stream)))
    _check("ra_rope_rotate_quant", rc)
    return out


def attn_int4(p: Problem, codes: Dict[str, torch.Tensor], out: Optional[torch.Tensor] = None,
              lse: Optional[torch.Tensor] = None, stream=None, p_mode: int = P_RANGE,
              l_mode: int = L_CODES) -> torch.Tensor:
    """ra_attn_int4 (ra_attn_int4_opts for the ablation switches) on the
    prologue's outputs; returns out [B, H, N, D] bf16."""
    B, H, N, D = p.B, p.H, p.N, p.D
    if out is None:
        out = torch.empty(B, H, N, D, dtype=torch.bfloat16, device=codes["q4"].device)
    rc = lib().ra_attn_int4_opts(
        C.byref(p), _opts(p_mode, l_mode), _ptr(codes["q4"], torch.uint8, (B, H, N, D // 2)), _ptr(codes["sq"], torch.float32, (B, H, N)),
        _ptr(codes["k4"], torch.uint8, (B, H, N, D // 2)), _ptr(codes["sk"], torch.float32, (B, H, N)),
        _ptr(codes["v4"], torch.uint8, (B, H, N, D // 2)), _ptr(codes["sv"], torch.float32, (B, H, D)),
        _ptr(out, torch.bfloat16, (B, H, N, D), "out"), _ptr(lse, torch.float32, (B, H, N), "lse"),
        C.c_void_p(_stream(stream)))
    _check("ra_attn_int4_opts", rc)
    return out


def rope_rotate_quant_s8(p: Problem, q: Optional[torch.Tensor], k: torch.Tensor, v: torch.Tensor,
                         pos: torch.Tensor, out: Optional[Dict[str, torch.Tensor]] = None,
                         workspace: Optional[torch.Tensor] = None, stream=None) -> Dict[str, torch.Tensor]:
    """ra_rope_rotate_quant_s8: returns q8, sq, k8, sk, k_mean, v8, sv, v_colsum with
    the codes one per byte [B, H, N, D]: q8, k8 FP8 E4M3 bytes (uint8 tensors),
    v8 int8 16 x code (q = None: K and V only)."""
    B, H, N, D = p.B, p.H, p.N, p.D
    dev = k.device
    if out is None:
        out = {} if q is None else {
            "q8": torch.empty(B, H, N, D, dtype=torch.uint8, device=dev),
            "sq": torch.empty(B, H, N, dtype=torch.float32, device=dev)}
        out.update({
            "k8": torch.empty(B, H, N, D, dtype=torch.uint8, device=dev),
            "sk": torch.empty(B, H, N, dtype=torch.float32, device=dev),
            "k_mean": torch.empty(B, H, D, dtype=torch.float32, device=dev),
            "v8": torch.empty(B, H, N, D, dtype=torch.int8, device=dev),
            "sv": torch.empty(B, H, D, dtype=torch.float32, device=dev),
            "v_colsum": torch.empty(B, H, _nblocks(p), D, dtype=torch.int32, device=dev),
        })
    if workspace is None:
        workspace = torch.empty(max(workspace_bytes(p), 16), dtype=torch.uint8, device=dev)
    shp = (B, H, N, D)
    rc = lib().ra_rope_rotate_quant_s8(
        C.byref(p), _in_dtype(k), _ptr(q, k.dtype, shp, "q"), _ptr(k, k.dtype, shp, "k"), _ptr(v, k.dtype, shp, "v"),
        _ptr(pos, torch.int32, (N, 3), "pos"),
        _ptr(out.get("q8") if q is not None else None, torch.uint8, shp),
        _ptr(out.get("sq") if q is not None else None, torch.float32, (B, H, N)),
        _ptr(out["k8"], torch.uint8, shp), _ptr(out["sk"], torch.float32, (B, H, N)),
        _ptr(out["k_mean"], torch.float32, (B, H, D)), _ptr(out["v8"], torch.int8, shp),
        _ptr(out["sv"], torch.float32, (B, H, D)), _ptr(out["v_colsum"], torch.int32, (B, H, _nblocks(p), D)),
        _ptr(workspace, torch.uint8), C.c_size_t(workspace.numel()), C.c_void_p(_stream(stream)))
    _check("ra_rope_rotate_quant_s8", rc)
    return out


def attn_int4_s8(p: Problem, codes: Dict[str, torch.Tensor], out: Optional[torch.Tensor] = None,
                 lse: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """ra_attn_int4_s8 on rope_rotate_quant_s8's outputs; returns out [B, H, N, D] bf16."""
    B, H, N, D = p.B, p.H, p.N, p.D
    shp = (B, H, N, D)
    if out is None:
        out = torch.empty(shp, dtype=torch.bfloat16, device=codes["q8"].device)
    rc = lib().ra_attn_int4_s8(
        C.byref(p), _ptr(codes["q8"], torch.uint8, shp), _ptr(codes["sq"], torch.float32, (B, H, N)),
        _ptr(codes["k8"], torch.uint8, shp), _ptr(codes["sk"], torch.float32, (B, H, N)),
        _ptr(codes["v8"], torch.int8, shp), _ptr(codes["sv"], torch.float32, (B, H, D)),
        _ptr(out, torch.bfloat16, shp, "out"), _ptr(lse, torch.float32, (B, H, N), "lse"),
        C.c_void_p(_stream(stream)))
    _check("ra_attn_int4_s8", rc)
    return out


def attn_int4_qfused(p: Problem, q: torch.Tensor, pos: torch.Tensor, codes: Dict[str, torch.Tensor],
                     out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                     workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """ra_attn_int4_qfused: INT4 attention that quantises the raw Q itself;
    codes holds k4, sk, v4, sv (rope_rotate_quant with q = None).  Returns out."""
    B, H, N, D = p.B, p.H, p.N, p.D
    dev = q.device
    if out is None:
        out = torch.empty(B, H, N, D, dtype=torch.bfloat16, device=dev)
    if workspace is None:
        workspace = torch.empty(max(workspace_bytes(p), 16), dtype=torch.uint8, device=dev)
    rc = lib().ra_attn_int4_qfused(
        C.byref(p), _in_dtype(q), _ptr(q, q.dtype, (B, H, N, D), "q"), _ptr(pos, torch.int32, (N, 3), "pos"),
        _ptr(codes["k4"], torch.uint8, (B, H, N, D // 2)), _ptr(codes["sk"], torch.float32, (B, H, N)),
        _ptr(codes["v4"], torch.uint8, (B, H, N, D // 2)), _ptr(codes["sv"], torch.float32, (B, H, D)),
        _ptr(workspace, torch.uint8), C.c_size_t(workspace.numel()),
        _ptr(out, torch.bfloat16, (B, H, N, D), "out"), _ptr(lse, torch.float32, (B, H, N), "lse"),
        C.c_void_p(_stream(stream)))
    _check("ra_attn_int4_qfused", rc)
    return out


def test_int4_codes(p: Problem, codes: Dict[str, torch.Tensor], b: int, h: int, q_tile: int, stream=None,
                    p_mode: int = P_RANGE, l_mode: int = L_CODES):
    """ra_test_int4_codes(_opts): returns (out, lse, s_dump, p_dump, acc_dump) for tile q_tile of head (b, h)."""
    B, H, N, D = p.B, p.H, p.N, p.D
    dev = codes["q4"].device
    out = torch.empty(B, H, N, D, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(B, H, N, dtype=torch.float32, device=dev)
    s = torch.zeros(128, N, dtype=torch.int32, device=dev)
    pc = torch.zeros(128, N, dtype=torch.int8, device=dev)
    acc = torch.zeros(128, _nblocks(p), D, dtype=torch.int32, device=dev)
    rc = lib().ra_test_int4_codes_opts(
        C.byref(p), _opts(p_mode, l_mode), _ptr(codes["q4"], torch.uint8), _ptr(codes["sq"], torch.float32),
        _ptr(codes["k4"], torch.uint8), _ptr(codes["sk"], torch.float32),
        _ptr(codes["v4"], torch.uint8), _ptr(codes["sv"], torch.float32),
        int(b), int(h), int(q_tile), _ptr(s), _ptr(pc), _ptr(acc), _ptr(out), _ptr(lse),
        C.c_void_p(_stream(stream)))
    _check("ra_test_int4_codes_opts", rc)
    return out, lse, s, pc, acc


def rope_bf16(p: Problem, q: torch.Tensor, k: torch.Tensor, pos: torch.Tensor,
              workspace: Optional[torch.Tensor] = None, stream=None):
    """ra_rope_bf16: 3D RoPE (no rotation) of q and k to bf16."""
    B, H, N, D = p.B, p.H, p.N, p.D
    qo = torch.empty(B, H, N, D, dtype=torch.bfloat16, device=q.device)
    ko = torch.empty_like(qo)
    if workspace is None:
        workspace = torch.empty(max(workspace_bytes(p), 16), dtype=torch.uint8, device=q.device)
    shp = (B, H, N, D)
    rc = lib().ra_rope_bf16(C.byref(p), _in_dtype(q), _ptr(q, q.dtype, shp, "q"), _ptr(k, q.dtype, shp, "k"),
                            _ptr(pos, torch.int32, (N, 3), "pos"), _ptr(qo), _ptr(ko),
                            _ptr(workspace, torch.uint8), C.c_size_t(workspace.numel()),
                            C.c_void_p(_stream(stream)))
    _check("ra_rope_bf16", rc)
    return qo, ko


def attn_bf16_fallback(p: Problem, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                       out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None, stream=None):
    """ra_attn_bf16_fallback: softmax(q k^T / sqrt(D)) v, bf16 in / out."""
    B, H, N, D = p.B, p.H, p.N, p.D
    shp = (B, H, N, D)
    if out is None:
        out = torch.empty(shp, dtype=torch.bfloat16, device=q.device)
    rc = lib().ra_attn_bf16_fallback(C.byref(p), _ptr(q, torch.bfloat16, shp, "q"), _ptr(k, torch.bfloat16, shp, "k"),
                                     _ptr(v, torch.bfloat16, shp, "v"), _ptr(out, torch.bfloat16, shp, "out"),
                                     _ptr(lse, torch.float32, (B, H, N), "lse"), C.c_void_p(_stream(stream)))
    _check("ra_attn_bf16_fallback", rc)
    return out


def sync_status(stream=None) -> int:
    """ra_sync_status: synchronises the stream and returns (and clears) the device status."""
    return int(lib().ra_sync_status(C.c_void_p(_stream(stream))))


def rope_rotate_quant_noalloc(p: Problem, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, pos: torch.Tensor,
                              out: Dict[str, torch.Tensor], stream=None) -> Dict[str, torch.Tensor]:
    """ra_rope_rotate_quant_noalloc: the prologue without a workspace argument.

    For callers that cannot allocate device memory while they run (the library
    keeps a fixed scratch array of RA_STATIC_SCRATCH_BYTES per GPU instead).  The
    caller supplies every output tensor in `out` (keys as rope_rotate_quant
    returns).  The first call on a device should precede any stream capture, and
    calls that may overlap on the GPU share, and race on, the one scratch array.
    """
    L = lib()
    fn = L.ra_rope_rotate_quant_noalloc
    fn.restype = C.c_int
    fn.argtypes = [C.POINTER(Problem), C.c_int] + [C.c_void_p] * 13
    B, H, N, D = p.B, p.H, p.N, p.D
    shp = (B, H, N, D)
    rc = fn(C.byref(p), _in_dtype(q), _ptr(q, q.dtype, shp, "q"), _ptr(k, q.dtype, shp, "k"),
            _ptr(v, q.dtype, shp, "v"), _ptr(pos, torch.int32, (N, 3), "pos"),
            _ptr(out["q4"], torch.uint8, (B, H, N, D // 2)), _ptr(out["sq"], torch.float32, (B, H, N)),
            _ptr(out["k4"], torch.uint8, (B, H, N, D // 2)), _ptr(out["sk"], torch.float32, (B, H, N)),
            _ptr(out["k_mean"], torch.float32, (B, H, D)), _ptr(out["v4"], torch.uint8, (B, H, N, D // 2)),
            _ptr(out["sv"], torch.float32, (B, H, D)), _ptr(out["v_colsum"], torch.int32, (B, H, _nblocks(p), D)),
            C.c_void_p(_stream(stream)))
    _check("ra_rope_rotate_quant_noalloc", rc)
    return out
