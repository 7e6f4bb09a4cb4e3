// Per-token RoPE, RoPE-aware rotation and symmetric INT4 quantisation of
// eight channels of a token row, shared by the prologue and by the attention
// kernel's fused-Q path (which must reproduce the prologue's Q codes bit for
// bit).  RotateAttention (arXiv 2607.02584), papernotes page "key design 1"
// (3D RoPE, the rotation M' = R M) and gecl notes "Key Insight" (per-token
// INT4).
//
// Every value that decides a code is computed in fp32 with explicit
// round-to-nearest (or explicitly fused) operations in a fixed order, so the
// results do not depend on the compiler's contraction setting.
//
// Thread layout: a thread works on the 8 consecutive channels [c0, c0 + 8) of
// a token; the D/8 threads of a token form a contiguous group of lanes.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "ra_internal.h"

namespace ra {

struct SegInfo {
  int off[3];     // first channel of each segment
  int dj[3];      // channels of each segment
  int toff[3];    // first table entry of each segment
  int grid[3];
  int D;
  float hscale;   // fp32 rounding of 1/sqrt(D), the full rotation's scale
};

__device__ __forceinline__ void load8(const void* base, size_t elem_off, int dtype, float* x) {
  if (dtype == 1) {
    const uint4 u = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(base) + elem_off);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  } else {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + elem_off);
    const float4 a = p[0], b = p[1];
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
}

__device__ __forceinline__ int seg_of(const SegInfo& s, int d) {
  return d < s.off[1] ? 0 : (d < s.off[2] ? 1 : 2);
}

// Eight channels of one token as loaded from memory: one 16-byte word for bf16,
// two for fp32.  Loads use the read-only path.
template <bool kBf16>
struct Raw8 {
  uint4 u[kBf16 ? 1 : 2];
};

template <bool kBf16>
__device__ __forceinline__ void load_raw8(const void* base, size_t elem_off, Raw8<kBf16>& r) {
  if constexpr (kBf16) {
    r.u[0] = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(base) + elem_off));
  } else {
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const float*>(base) + elem_off);
    r.u[0] = __ldg(p);
    r.u[1] = __ldg(p + 1);
  }
}

template <bool kBf16>
__device__ __forceinline__ void unpack8(const Raw8<kBf16>& r, float* x) {
  if constexpr (kBf16) {
    const uint32_t w[4] = {r.u[0].x, r.u[0].y, r.u[0].z, r.u[0].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  } else {
    x[0] = __uint_as_float(r.u[0].x); x[1] = __uint_as_float(r.u[0].y);
    x[2] = __uint_as_float(r.u[0].z); x[3] = __uint_as_float(r.u[0].w);
    x[4] = __uint_as_float(r.u[1].x); x[5] = __uint_as_float(r.u[1].y);
    x[6] = __uint_as_float(r.u[1].z); x[7] = __uint_as_float(r.u[1].w);
  }
}

// Per-thread constants of the RoPE table lookup: the segment and the pair of
// each of the thread's 4 channel pairs, computed once.
struct RopePlan {
  int seg[4], off[4], stride[4];
  // Half rotation: output channels c0 + 2p and c0 + 2p + 1 (one segment)
  // take the sum and the difference of channels u and w = u + Dj/2 of the
  // RoPE'd row: hp[p] = 4u | 4w << 16 (byte offsets into the row).
  uint32_t hp[4];
  __device__ __forceinline__ void init(const SegInfo& s, int c0) {
#pragma unroll
    for (int pr = 0; pr < 4; ++pr) {
      const int d = c0 + 2 * pr;
      const int j = seg_of(s, d);
      seg[pr] = j;
      off[pr] = s.toff[j] + ((d - s.off[j]) >> 1);
      stride[pr] = s.dj[j] >> 1;
    }
#pragma unroll
    for (int pr = 0; pr < 4; ++pr) {
      const int d = c0 + 2 * pr;  // segments start at even channels: d, d + 1 share one
      const int j = seg_of(s, d);
      const uint32_t u = static_cast<uint32_t>(s.off[j] + ((d - s.off[j]) >> 1));
      hp[pr] = (4u * u) | ((4u * (u + (s.dj[j] >> 1))) << 16);
    }
  }
};

// Table coefficients (a, b) of the thread's 4 channel pairs for a token at grid
// position gp (one position per segment; out-of-grid positions are reported
// in *status and clamped so every table access stays in bounds).
__device__ __forceinline__ void rope_coef8p(const SegInfo& s, const RopePlan& rp, const float2* tab,
                                            const int* gp, float2* cf, uint32_t* status) {
  int g[3];
#pragma unroll
  for (int j = 0; j < 3; ++j) {
    g[j] = gp[j];
    if (g[j] < 0 || g[j] >= s.grid[j]) {
      atomicOr(status, kStatusBadPosition);
      g[j] = g[j] < 0 ? 0 : s.grid[j] - 1;
    }
  }
#pragma unroll
  for (int pr = 0; pr < 4; ++pr) {
    const int gj = rp.seg[pr] == 0 ? g[0] : (rp.seg[pr] == 1 ? g[1] : g[2]);
    const int idx = rp.off[pr] + gj * rp.stride[pr];
    cf[pr] = __ldg(tab + idx);
  }
}

// Full rotation: the token row times H_D / sqrt(D) (Sylvester Hadamard), as
// butterflies (a, b) -> (a + b, a - b) on channels d apart, d = 1, 2, ..., D/2
// in that order, then one fp32 scaling.  The thread holds channels
// [c0, c0 + 8): distances 1, 2, 4 are in its registers, distances 8 ... D/2
// pair it with the lanes 1 ... D/16 apart in its token's lane group.
__device__ __forceinline__ void hadamard8(const SegInfo& s, int c0, float* x) {
#pragma unroll
  for (int d = 1; d < 8; d <<= 1)
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (!(i & d)) {
        const float a = x[i], b = x[i + d];
        x[i] = __fadd_rn(a, b);
        x[i + d] = __fsub_rn(a, b);
      }
  const int g = c0 >> 3;  // this thread's place among the token's D/8 lanes
  for (int m = 1; m < (s.D >> 3); m <<= 1) {
    const bool upper = (g & m) != 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float o = __shfl_xor_sync(0xFFFFFFFFu, x[i], m);
      x[i] = upper ? __fsub_rn(o, x[i]) : __fadd_rn(x[i], o);
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) x[i] = __fmul_rn(x[i], s.hscale);
}

// The same arithmetic as rope_rotate8, from coefficients already loaded (rot
// 3: the full Hadamard rotation after the RoPE pairs).  Every output is
// fl(fl(x0 a) +- fl(x1 b)) with scalar round-to-nearest operations (packed
// f32x2 products measured no faster here).  The half rotation stores the
// RoPE'd row (two 16-byte stores per thread) and reads each output pair's two
// inputs u, w = u + Dj/2 back at the byte offsets in rp.hp.
__device__ __forceinline__ void rope_apply8(const SegInfo& s, const RopePlan& rp, int rot, const float2* cf,
                                            int c0, float* x, float* row) {
#pragma unroll
  for (int pr = 0; pr < 4; ++pr) {
    const float a = cf[pr].x, b = cf[pr].y;
    const float x0 = x[2 * pr], x1 = x[2 * pr + 1];
    if (rot == 1) {
      x[2 * pr] = __fadd_rn(__fmul_rn(x0, a), __fmul_rn(x1, b));
      x[2 * pr + 1] = __fsub_rn(__fmul_rn(x0, b), __fmul_rn(x1, a));
    } else {
      x[2 * pr] = __fsub_rn(__fmul_rn(x0, a), __fmul_rn(x1, b));
      x[2 * pr + 1] = __fadd_rn(__fmul_rn(x0, b), __fmul_rn(x1, a));
    }
  }
  if (rot == 2) {
    const float r2 = 0.70710678118654752440f;  // fp32 rounding of 1/sqrt(2)
    float4* const r4 = reinterpret_cast<float4*>(row + c0);
    r4[0] = make_float4(x[0], x[1], x[2], x[3]);
    r4[1] = make_float4(x[4], x[5], x[6], x[7]);
    __syncwarp();
    const char* const rb = reinterpret_cast<const char*>(row);
#pragma unroll
    for (int pr = 0; pr < 4; ++pr) {
      const uint32_t h = rp.hp[pr];
      const float u = *reinterpret_cast<const float*>(rb + (h & 0xFFFFu));
      const float w = *reinterpret_cast<const float*>(rb + (h >> 16));
      x[2 * pr] = __fmul_rn(__fadd_rn(u, w), r2);
      x[2 * pr + 1] = __fmul_rn(__fsub_rn(u, w), r2);
    }
    __syncwarp();
  }
  if (rot == 3) hadamard8(s, c0, x);
}


// For two elements: the bits of 1.5 * 2^23 + 8 + rint(x * inv), i.e.
// 0x4B400000 + (code + 8) with code + 8 in [1, 15].  One f32x2 fused
// multiply-add: the product x * inv is exact inside the FMA and the single
// rounding to the integer grid of [2^23, 2^24) (ties to even; the offset is
// even) is the rint of the exact product.
//   * No clamp is needed: inv = fl(7/amax) with |x| <= amax (the token's or
//     channel's own maximum), so |x * inv| <= 7 (1 + 2^-23) < 7.5 and rint
//     already lies in [-7, 7]; amax = 0 gives inv = 0 and code 0.
//   * The exact product is the decision on purpose: an f32x2 multiply and an
//     f32x2 add in sequence are fused by the compiler even when written with
//     explicit round-to-nearest (measured: the codes of exact fp32 ties
//     x * inv = k + 1/2 followed the unrounded product), so a two-rounding
//     decision would need scalar operations at twice the instruction count.
constexpr uint32_t kQBits = 0x4B400000u;       // bits of 1.5 * 2^23
constexpr float kQMagic8 = 12582920.0f;        // 1.5 * 2^23 + 8
__device__ __forceinline__ void quant4_bits2(float x0, float x1, float inv0, float inv1, uint32_t* b) {
  const float2 t = __ffma2_rn(make_float2(x0, x1), make_float2(inv0, inv1), make_float2(kQMagic8, kQMagic8));
  b[0] = __float_as_uint(t.x);
  b[1] = __float_as_uint(t.y);
}

// Packs the nibbles of eight quant4_bits2 results, element 2t in the low
// nibble: sum_i 16^i b_i (integer multiply-adds) minus the known sum of the
// 0x4B400000 parts leaves the nibbles code + 8 (at most 15: no carries);
// XOR with 8 in every nibble turns code + 8 into the two's complement code.
constexpr uint32_t kQBitsRep = kQBits * 0x11111111u;   // sum_i 16^i 0x4B400000 mod 2^32
__device__ __forceinline__ uint32_t pack8_bits(const uint32_t* b) {
  uint32_t acc = b[7];
#pragma unroll
  for (int i = 6; i >= 0; --i) acc = acc * 16u + b[i];
  return (acc - kQBitsRep) ^ 0x88888888u;
}

// The byte code layout (V): one code per byte, held in the byte's high nibble
// (the s8 value 16 x code, the low nibble zero), channels in natural order.  For
// four quant4_bits2 results b[0..3] (channels c..c+3) the little-endian word
// of their bytes: sum_i 256^i b_i minus the known offsets leaves the bytes
// code + 8 (at most 15: no carries), shifted into the high nibble; XOR 0x80
// turns (code + 8) * 16 into the s8 value 16 x code.
constexpr uint32_t kQBitsRep4 = kQBits * 0x01010101u;   // sum_i 256^i 0x4B400000 mod 2^32
__device__ __forceinline__ uint32_t pack4_s8_bits(const uint32_t* b) {
  uint32_t acc = b[3];
  acc = acc * 256u + b[2];
  acc = acc * 256u + b[1];
  acc = acc * 256u + b[0];
  return ((acc - kQBitsRep4) << 4) ^ 0x80808080u;
}

// FP8 E4M3 bytes of four codes (channels c..c+3, little-endian) from their
// quant4_bits2 results: the code as a float is the bits' value minus
// 1.5 * 2^23 + 8 (exact), and every integer in [-7, 7] is exact in E4M3.
__device__ __forceinline__ uint32_t pack4_e4m3_bits(const uint32_t* b) {
  float c[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) c[i] = __fsub_rn(__uint_as_float(b[i]), kQMagic8);
  uint16_t lo, hi;
  // the first source goes to the upper byte of each pair
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(c[1]), "f"(c[0]));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(c[3]), "f"(c[2]));
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

// Max over the D/8 threads of a token (a contiguous lane group of size lpt).
__device__ __forceinline__ float group_max(float v, int lpt) {
  for (int o = lpt >> 1; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

// Segment offsets, table offsets and grid of a problem (host).
SegInfo seg_info(const ra_problem& p);

}  // namespace ra
