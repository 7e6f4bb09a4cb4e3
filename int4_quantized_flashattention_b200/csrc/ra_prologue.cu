// Fused prologue of the RotateAttention INT4 forward (memory-bound):
//   3D RoPE + RoPE-aware rotation of Q and K, K smoothing, per-token INT4 of Q
//   and K, per-channel INT4 of V and per-block V column sums; plus the plain
//   RoPE to bf16 that feeds the bf16 fallback.  Rotation modes: interleaved
//   (H2 fused into the RoPE table), half (pairs i, i + Dj/2), full (the row
//   times a D x D Hadamard matrix), none.
// Method: RotateAttention (arXiv 2607.02584), papernotes page "overall
// framework" and "key design 1"; gecl notes "Key Insight" (per-token INT4).
//
// Every value that decides a code is computed in fp32 with explicit
// round-to-nearest intrinsics in a fixed order (no contraction), so codes
// match an fp32 reference of the same definition bit for bit.
//
// Layout: token rows are staged in shared memory by bulk copies; a thread
// works on 8 consecutive channels of a token (D/8 threads per token, 16-byte
// shared-memory reads).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "ra_common.cuh"
#include "ra_internal.h"
#include "ra_rope.cuh"

namespace ra {
namespace {

__device__ uint32_t g_prologue_status = 0;

constexpr int kThreads = 256;
constexpr int kChunk = 256;  // tokens per CTA; a multiple of every block_k

// Reads the token's grid position; a position outside the grid is reported and
// clamped so every table access stays in bounds.
__device__ __forceinline__ int grid_pos(const SegInfo& s, const int32_t* pos, int n, int j) {
  int g = pos[3 * n + j];
  if (g < 0 || g >= s.grid[j]) {
    atomicOr(&g_prologue_status, kStatusBadPosition);
    g = g < 0 ? 0 : s.grid[j] - 1;
  }
  return g;
}

// RoPE (+ rotation) of this thread's 8 channels [c0, c0+8) of token n.
//   rot 1 (interleaved, fused table): y0 = x0 a + x1 b, y1 = x0 b - x1 a
//   rot 0 / 2: y0 = x0 c - x1 s, y1 = x0 s + x1 c; rot 2 then pairs i, i + Dj/2
//   through the per-warp row buffer `row` (D floats for this token).
__device__ __forceinline__ void rope_rotate8(const SegInfo& s, const float2* tab,
                                             const int32_t* pos, int n, int rot, int c0, float* x,
                                             float* row) {
#pragma unroll
  for (int pr = 0; pr < 4; ++pr) {
    const int d = c0 + 2 * pr;
    const int j = seg_of(s, d);
    const int k = (d - s.off[j]) >> 1;
    const int g = grid_pos(s, pos, n, j);
    const int idx = s.toff[j] + g * (s.dj[j] >> 1) + k;
    const float2 ab = __ldg(tab + idx);
    const float a = ab.x, b = ab.y;
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
#pragma unroll
    for (int i = 0; i < 8; ++i) row[c0 + i] = x[i];
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int d = c0 + i;
      const int j = seg_of(s, d);
      const int h = s.dj[j] >> 1;
      const int t = (d - s.off[j]) >> 1;
      const float u = row[s.off[j] + t], w = row[s.off[j] + t + h];
      x[i] = (d - s.off[j]) & 1 ? __fmul_rn(__fsub_rn(u, w), r2) : __fmul_rn(__fadd_rn(u, w), r2);
    }
    __syncwarp();
  }
}


struct PrologueArgs {
  SegInfo s;
  int N, D, rot, dtype, block_k, nchunk;
  int bk_log2;  // block_k = 2^bk_log2
  const void *q, *k, *v;
  const int32_t* pos;
  const float2* tab;   // RoPE table entries (a, b) of the rotation mode
  const float2* tab0;  // plain RoPE table (cos, sin): the reduce pass
  double* ksum;     // [BH, nchunk, D]
  float* vmax;      // [BH, nchunk, D]
  float* vinv;      // [BH, D]
  uint8_t *q4, *k4, *v4;   // packed codes [BH, N, D/2], or bytes [BH, N, D] when s8 (Q, K: E4M3 codes; V: 16 x code)
  float *sq, *sk, *k_mean, *sv;
  int32_t* colsum;
  int s8;                  // code layout: 0 packed nibbles, 1 one code per byte
};

// Table entry e -> (segment j, position g, pair k); angle g * theta^(-2k/Dj) in
// fp64, entries rounded once to fp32.  rot 1 stores the fused H2 block.
__global__ void rope_table_kernel(SegInfo s, int total, double theta, int rot, float2* tab) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= total) return;
  const int j = e < s.toff[1] ? 0 : (e < s.toff[2] ? 1 : 2);
  const int npair = s.dj[j] >> 1;
  const int g = (e - s.toff[j]) / npair, k = (e - s.toff[j]) % npair;
  const double freq = pow(theta, -2.0 * static_cast<double>(k) / static_cast<double>(s.dj[j]));
  const double phi = static_cast<double>(g) * freq;
  const double c = cos(phi), sn = sin(phi);
  float a, b;
  if (rot == 1) {
    a = static_cast<float>((c + sn) / sqrt(2.0));
    b = static_cast<float>((c - sn) / sqrt(2.0));
  } else {
    a = static_cast<float>(c);
    b = static_cast<float>(sn);
  }
  tab[e] = make_float2(a, b);
}

// Rows of kSub tokens of the input tensors are staged in shared memory by bulk
// asynchronous copies, kStg sub-chunks ahead of the threads that use them, so
// each SM keeps tens of kilobytes of loads in flight.  Thread 0 issues the
// copies; every stage has one mbarrier that completes on the copied bytes.
constexpr int kSub = 32;   // tokens per stage
// Two stages per pass: more stages in flight (4 or 6 for the reduce pass, 3
// for the quantise pass at two CTAs per SM) measured no faster.
constexpr int kStgR = 2;   // stages of the channel-reduce pass (K, V)
constexpr int kStgQ = 2;   // stages of the quantise pass (Q, K, V)

template <bool kBf16, int NT, int kStg>
struct StageIO {
  static constexpr int kEl = kBf16 ? 2 : 4;
  // Issues the copies of sub-chunk sc (tokens n0 + sc*kSub ...) of NT tensors
  // into stage sc % kStg; a sub-chunk past N only completes the barrier.
  static __device__ __forceinline__ void issue(const void* const* src, size_t head, int D, int N, int n0, int sc,
                                               uint8_t* stg, uint64_t* full) {
    const int s = sc % kStg;
    const int t0 = n0 + sc * kSub;
    const int cnt = min(kSub, N - t0);
    if (cnt <= 0) {
      mbar_arrive(full + s);
      return;
    }
    const uint32_t tb = kSub * D * kEl, bytes = static_cast<uint32_t>(cnt) * D * kEl;
    mbar_arrive_expect_tx(full + s, NT * bytes);
    for (int i = 0; i < NT; ++i)
      bulk_g2s(stg + (s * NT + i) * tb, static_cast<const uint8_t*>(src[i]) + (head + static_cast<size_t>(t0) * D) * kEl,
               bytes, full + s);
  }
  // This thread's 8 channels of token ti of tensor i in stage s.
  static __device__ __forceinline__ void read(const uint8_t* stg, int D, int s, int i, int ti, int c0, Raw8<kBf16>& r) {
    const uint8_t* p = stg + ((s * NT + i) * kSub + ti) * D * kEl + c0 * kEl;
    r.u[0] = *reinterpret_cast<const uint4*>(p);
    if constexpr (!kBf16) r.u[1] = *reinterpret_cast<const uint4*>(p + 16);
  }
  static constexpr int stage_bytes(int D) { return NT * kSub * D * kEl; }
};

// Waits (bounded) for stage s's copies; returns false in every thread of the
// CTA if any thread gave up.
__device__ __forceinline__ bool stage_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  const int r = mbar_wait_ex(bar, parity, abort, 64u);
  return !__syncthreads_or(r <= 0);
}

// Pass 1: per chunk of tokens, fp64 channel sums of the RoPE'd K (before the
// rotation, which is linear and the same for every token: the finalize pass
// applies it to the mean) and channel maxima of |V|.
template <bool kBf16, int kD>
__global__ void __launch_bounds__(kThreads, 3) prologue_reduce_kernel(PrologueArgs a) {
  using IO = StageIO<kBf16, 2, kStgR>;
  constexpr int kRot = 0;
  __shared__ __align__(16) float rows[1][4][128];   // (unused by the plain RoPE)
  __shared__ uint64_t full[kStgR];
  __shared__ int abort_flag;
  extern __shared__ __align__(128) uint8_t stg[];
  const int bh = blockIdx.y, chunk = blockIdx.x;
  const int lpt = kD >> 3, tpw = 32 / lpt;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tok_in_warp = lane / lpt, c0 = (lane % lpt) * 8;
  float* const row = rows[0][0];
  const int step = (kThreads / 32) * tpw;
  const int n0 = chunk * kChunk;
  const size_t head = static_cast<size_t>(bh) * a.N * kD;
  const void* src[2] = {a.k, a.v};
  RopePlan rp;
  rp.init(a.s, c0);
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStgR; ++s) mbar_init(full + s, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0)
    for (int sc = 0; sc < kStgR; ++sc) IO::issue(src, head, kD, a.N, n0, sc, stg, full);
  double ks[8];
  float vm[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) { ks[i] = 0.0; vm[i] = 0.0f; }
  bool ok = true;
  for (int sc = 0; sc < kChunk / kSub && ok; ++sc) {
    const int s = sc % kStgR;
    if (!(ok = stage_wait(full + s, (sc / kStgR) & 1, &abort_flag))) break;
    // Two tokens per thread in flight (latency of the position and table loads).
#pragma unroll 2
    for (int ti = warp * tpw + tok_in_warp; ti - tok_in_warp < kSub; ti += step) {
      const int n = n0 + sc * kSub + ti;
      const bool valid = n < a.N;
      float x[8], y[8];
      float2 cf[4];
      int gp[3] = {0, 0, 0};
      if (valid) {
        Raw8<kBf16> rk, rv;
        IO::read(stg, kD, s, 0, ti, c0, rk);
        IO::read(stg, kD, s, 1, ti, c0, rv);
        unpack8<kBf16>(rk, x);
        unpack8<kBf16>(rv, y);
#pragma unroll
        for (int j = 0; j < 3; ++j) gp[j] = __ldg(a.pos + 3 * n + j);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) { x[i] = 0.0f; y[i] = 0.0f; }
      }
      rope_coef8p(a.s, rp, a.tab0, gp, cf, &g_prologue_status);
      rope_apply8(a.s, rp, kRot, cf, c0, x, row);
      if (valid) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          ks[i] += static_cast<double>(x[i]);
          vm[i] = fmaxf(vm[i], fabsf(y[i]));
        }
      }
    }
    __syncthreads();  // stage s consumed
    if (threadIdx.x == 0 && sc + kStgR < kChunk / kSub) IO::issue(src, head, kD, a.N, n0, sc + kStgR, stg, full);
  }
  if (!ok) {
    if (threadIdx.x == 0) atomicOr(&g_prologue_status, kStatusTimeout);
    return;
  }
  // Per-thread partials to shared memory (reusing the stage buffers), folded
  // in thread order per channel.
  double* red_s = reinterpret_cast<double*>(stg);
  float* red_m = reinterpret_cast<float*>(stg + kThreads * 8 * sizeof(double));
#pragma unroll
  for (int i = 0; i < 8; ++i) { red_s[threadIdx.x * 8 + i] = ks[i]; red_m[threadIdx.x * 8 + i] = vm[i]; }
  __syncthreads();
  for (int d = threadIdx.x; d < kD; d += kThreads) {
    const int c = d >> 3, i = d & 7;
    double sum = 0.0;
    float mx = 0.0f;
    for (int t = c; t < kThreads; t += lpt) {
      sum += red_s[t * 8 + i];
      mx = fmaxf(mx, red_m[t * 8 + i]);
    }
    const size_t o = (static_cast<size_t>(bh) * a.nchunk + chunk) * kD + d;
    a.ksum[o] = sum;
    a.vmax[o] = mx;
  }
}

// Per head and channel: K mean (fp64 sum over chunks in order; the rotation
// applied to the mean in fp64; rounded once), V scale amax/7 and reciprocal
// 7/amax.  One CTA of 128 threads per head; threads d >= D only take part in
// the barrier.
__global__ void prologue_finalize_kernel(PrologueArgs a) {
  __shared__ double m[128];
  const int bh = blockIdx.x, d = threadIdx.x;
  const bool active = d < a.D;
  if (active) {
    double sum = 0.0;
    float mx = 0.0f;
    const size_t o0 = static_cast<size_t>(bh) * a.nchunk * a.D + d;
    int c = 0;
    // Eight chunks' loads in flight at a time; the sum keeps the chunk order.
    for (; c + 8 <= a.nchunk; c += 8) {
      double s8[8];
      float m8[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        s8[u] = a.ksum[o0 + static_cast<size_t>(c + u) * a.D];
        m8[u] = a.vmax[o0 + static_cast<size_t>(c + u) * a.D];
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        sum += s8[u];
        mx = fmaxf(mx, m8[u]);
      }
    }
    for (; c < a.nchunk; ++c) {
      sum += a.ksum[o0 + static_cast<size_t>(c) * a.D];
      mx = fmaxf(mx, a.vmax[o0 + static_cast<size_t>(c) * a.D]);
    }
    a.sv[bh * a.D + d] = __fdiv_rn(mx, 7.0f);
    a.vinv[bh * a.D + d] = mx == 0.0f ? 0.0f : __fdiv_rn(7.0f, mx);
    m[d] = sum / static_cast<double>(a.N);   // mean of the RoPE'd K (before the rotation)
  }
  __syncthreads();
  if (!active) return;
  const double r2 = 0.70710678118654752440;   // 1/sqrt(2) in fp64
  double mu;
  if (a.rot == 1) {
    const int e = d & ~1;
    mu = (d & 1) ? (m[e] - m[e + 1]) * r2 : (m[e] + m[e + 1]) * r2;
  } else if (a.rot == 2) {
    const int j = seg_of(a.s, d);
    const int o = a.s.off[j], h = a.s.dj[j] >> 1, i = (d - o) >> 1;
    mu = ((d - o) & 1) ? (m[o + i] - m[o + i + h]) * r2 : (m[o + i] + m[o + i + h]) * r2;
  } else if (a.rot == 3) {
    double acc = 0.0;
    for (int e = 0; e < a.D; ++e) acc += (__popc(e & d) & 1) ? -m[e] : m[e];
    mu = acc * (1.0 / sqrt(static_cast<double>(a.D)));
  } else {
    mu = m[d];
  }
  a.k_mean[bh * a.D + d] = static_cast<float>(mu);
}

// Pass 2: quantise.  Q, K: rotate (K also smoothed), per-token scale and codes.
// V: per-channel codes, column sums per key block.  Q and K of a token share
// the RoPE coefficients; column sums are kept per thread while a warp stays in
// one key block, then combined across the warp's tokens and added to shared
// memory.  kQ = false leaves Q out (the attention kernel's fused-Q path
// quantises Q itself): only K and V are staged and written.
template <bool kBf16, int kRot, int kD, bool kQ, bool kS8>
__global__ void __launch_bounds__(kThreads, 3) prologue_quant_kernel(PrologueArgs a) {
  constexpr int kNT = kQ ? 3 : 2;          // staged tensors
  constexpr int iK = kQ ? 1 : 0, iV = iK + 1;
  using IO = StageIO<kBf16, kNT, kStgQ>;
  // Row buffer of the half rotation's exchange (one token row per warp slot).
  __shared__ __align__(16) float rows[kRot == 2 ? kThreads / 32 : 1][4][128];
  __shared__ int csum[kChunk / 16][128];
  __shared__ uint64_t full[kStgQ];
  __shared__ int abort_flag;
  extern __shared__ __align__(128) uint8_t stg[];
  const int bh = blockIdx.y, chunk = blockIdx.x;
  const int lpt = kD >> 3, tpw = 32 / lpt;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tok_in_warp = lane / lpt, c0 = (lane % lpt) * 8;
  float* const row = rows[kRot == 2 ? warp : 0][kRot == 2 ? tok_in_warp : 0];
  const int step = (kThreads / 32) * tpw;
  const int nblk = kChunk / a.block_k;
  const int n0 = chunk * kChunk;
  const size_t head = static_cast<size_t>(bh) * a.N * kD;
  const size_t head4 = static_cast<size_t>(bh) * a.N * (kD / 2);
  const void* src[3] = {kQ ? a.q : a.k, kQ ? a.k : a.v, a.v};
  RopePlan rp;
  rp.init(a.s, c0);
  for (int i = threadIdx.x; i < nblk * kD; i += kThreads) csum[i / kD][i % kD] = 0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStgQ; ++s) mbar_init(full + s, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  float kmean[8], vinv[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    kmean[i] = a.k_mean[bh * kD + c0 + i];
    vinv[i] = a.vinv[bh * kD + c0 + i];
  }
  __syncthreads();
  if (threadIdx.x == 0)
    for (int sc = 0; sc < kStgQ; ++sc) IO::issue(src, head, kD, a.N, n0, sc, stg, full);
  int cacc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  int cblk = (warp * tpw) >> a.bk_log2;  // key block of this warp's first tokens
  // Adds this warp's per-thread column sums of block cblk to shared memory:
  // lanes holding the same channels (lpt apart) are combined first.
  auto flush = [&]() {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      for (int o = lpt; o < 32; o <<= 1) cacc[i] += __shfl_xor_sync(0xFFFFFFFFu, cacc[i], o);
    if (tok_in_warp == 0) {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (cacc[i] != 0) atomicAdd(&csum[cblk][c0 + i], cacc[i]);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) cacc[i] = 0;
  };
  bool ok = true;
  for (int sc = 0; sc < kChunk / kSub && ok; ++sc) {
    const int s = sc % kStgQ;
    if (!(ok = stage_wait(full + s, (sc / kStgQ) & 1, &abort_flag))) break;
    // Two tokens per thread in flight: independent work to hide the latency
    // of the position and table loads and of the shuffles.
#pragma unroll 2
    for (int ti = warp * tpw + tok_in_warp; ti - tok_in_warp < kSub; ti += step) {
      const int n = n0 + sc * kSub + ti;
      const bool valid = n < a.N;
      const int blk = (sc * kSub + ti - tok_in_warp) >> a.bk_log2;  // the same for the warp's tokens
      if (blk != cblk) {
        flush();
        cblk = blk;
      }
      float xq[8] = {}, xk[8], xv[8];
      float2 cf[4];
      int gp[3] = {0, 0, 0};
      if (valid) {
        Raw8<kBf16> rq, rk, rv;
        if constexpr (kQ) {
          IO::read(stg, kD, s, 0, ti, c0, rq);
          unpack8<kBf16>(rq, xq);
        }
        IO::read(stg, kD, s, iK, ti, c0, rk);
        IO::read(stg, kD, s, iV, ti, c0, rv);
        unpack8<kBf16>(rk, xk);
        unpack8<kBf16>(rv, xv);
#pragma unroll
        for (int j = 0; j < 3; ++j) gp[j] = __ldg(a.pos + 3 * n + j);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) { xq[i] = 0.0f; xk[i] = 0.0f; xv[i] = 0.0f; }
      }
      rope_coef8p(a.s, rp, a.tab, gp, cf, &g_prologue_status);
      if constexpr (kQ) rope_apply8(a.s, rp, kRot, cf, c0, xq, row);
      rope_apply8(a.s, rp, kRot, cf, c0, xk, row);
      float mq = 0.0f, mk = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        xk[i] = __fsub_rn(xk[i], kmean[i]);
        mq = fmaxf(mq, fabsf(xq[i]));
        mk = fmaxf(mk, fabsf(xk[i]));
      }
      if constexpr (kQ) mq = group_max(mq, lpt);
      mk = group_max(mk, lpt);
      const float iq = mq == 0.0f ? 0.0f : __fdiv_rn(7.0f, mq);
      const float ik = mk == 0.0f ? 0.0f : __fdiv_rn(7.0f, mk);
      uint32_t bq[8], bk[8], bv[8];
#pragma unroll
      for (int i = 0; i < 8; i += 2) {
        if constexpr (kQ) quant4_bits2(xq[i], xq[i + 1], iq, iq, bq + i);
        quant4_bits2(xk[i], xk[i + 1], ik, ik, bk + i);
        quant4_bits2(xv[i], xv[i + 1], vinv[i], vinv[i + 1], bv + i);
      }
      if (valid) {
        const size_t o4 = head4 + static_cast<size_t>(n) * (kD / 2) + (c0 >> 1);
        if constexpr (kS8) {
          const size_t o8 = head + static_cast<size_t>(n) * kD + c0;
          if constexpr (kQ) *reinterpret_cast<uint2*>(a.q4 + o8) = make_uint2(pack4_e4m3_bits(bq), pack4_e4m3_bits(bq + 4));
          *reinterpret_cast<uint2*>(a.k4 + o8) = make_uint2(pack4_e4m3_bits(bk), pack4_e4m3_bits(bk + 4));
          *reinterpret_cast<uint2*>(a.v4 + o8) = make_uint2(pack4_s8_bits(bv), pack4_s8_bits(bv + 4));
        } else {
          if constexpr (kQ) *reinterpret_cast<uint32_t*>(a.q4 + o4) = pack8_bits(bq);
          *reinterpret_cast<uint32_t*>(a.k4 + o4) = pack8_bits(bk);
          *reinterpret_cast<uint32_t*>(a.v4 + o4) = pack8_bits(bv);
        }
        if (c0 == 0) {
          if constexpr (kQ) a.sq[static_cast<size_t>(bh) * a.N + n] = __fdiv_rn(mq, 7.0f);
          a.sk[static_cast<size_t>(bh) * a.N + n] = __fdiv_rn(mk, 7.0f);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) cacc[i] += static_cast<int>(bv[i] - (kQBits + 8u));
      }
    }
    __syncthreads();  // stage s consumed
    if (threadIdx.x == 0 && sc + kStgQ < kChunk / kSub) IO::issue(src, head, kD, a.N, n0, sc + kStgQ, stg, full);
  }
  if (!ok) {
    if (threadIdx.x == 0) atomicOr(&g_prologue_status, kStatusTimeout);
    return;
  }
  flush();
  __syncthreads();
  const int nb_total = (a.N + a.block_k - 1) / a.block_k;
  for (int i = threadIdx.x; i < nblk * kD; i += kThreads) {
    const int bl = i / kD, d = i % kD;
    const int gb = chunk * nblk + bl;
    if (gb < nb_total) a.colsum[(static_cast<size_t>(bh) * nb_total + gb) * kD + d] = csum[bl][d];
  }
}

// RoPE only (rotation off) to bf16, round to nearest even.
__global__ void __launch_bounds__(kThreads) rope_bf16_kernel(PrologueArgs a, __nv_bfloat16* qo,
                                                             __nv_bfloat16* ko) {
  __shared__ float rows[kThreads / 32][4][128];
  const int bh = blockIdx.y, chunk = blockIdx.x;
  const int lpt = a.D >> 3, tpw = 32 / lpt;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tok_in_warp = lane / lpt, c0 = (lane % lpt) * 8;
  const int n0 = chunk * kChunk;
  const size_t head = static_cast<size_t>(bh) * a.N * a.D;
  for (int base = n0; base < n0 + kChunk; base += (kThreads / 32) * tpw) {
    const int n = base + warp * tpw + tok_in_warp;
    if (n >= a.N) continue;
    float x[8];
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      load8(which ? a.k : a.q, head + static_cast<size_t>(n) * a.D + c0, a.dtype, x);
      rope_rotate8(a.s, a.tab, a.pos, n, 0, c0, x, rows[warp][tok_in_warp]);
      uint32_t w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 h2 = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
        w[i] = *reinterpret_cast<const uint32_t*>(&h2);
      }
      __nv_bfloat16* dst = (which ? ko : qo) + head + static_cast<size_t>(n) * a.D + c0;
      *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

}  // namespace

SegInfo seg_info(const ra_problem& p) {
  SegInfo s;
  int o = 0, t = 0;
  for (int j = 0; j < 3; ++j) {
    s.off[j] = o;
    s.dj[j] = p.seg[j];
    s.toff[j] = t;
    s.grid[j] = p.grid[j];
    o += p.seg[j];
    t += p.grid[j] * (p.seg[j] / 2);
  }
  s.D = p.D;
  s.hscale = static_cast<float>(1.0 / sqrt(static_cast<double>(p.D)));
  return s;
}

size_t rope_table_len(const ra_problem& p) {
  size_t t = 0;
  for (int j = 0; j < 3; ++j) t += static_cast<size_t>(p.grid[j]) * (p.seg[j] / 2);
  return t;
}

int prologue_nchunk(const ra_problem& p) { return (p.N + kChunk - 1) / kChunk; }

static size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

WorkspaceLayout workspace_layout(const ra_problem& p) {
  WorkspaceLayout w;
  const size_t bh = static_cast<size_t>(p.B) * p.H, T = rope_table_len(p), nc = prologue_nchunk(p);
  size_t o = 0;
  w.tab = o; o = align256(o + T * sizeof(float2));
  w.tab0 = o; o = align256(o + T * sizeof(float2));
  w.ksum = o;  o = align256(o + bh * nc * p.D * sizeof(double));
  w.vmax = o;  o = align256(o + bh * nc * p.D * sizeof(float));
  w.vinv = o;  o = align256(o + bh * p.D * sizeof(float));
  w.total = o;
  return w;
}

template <typename K>
static cudaError_t set_smem(K kern, int bytes) {
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

static cudaError_t launch_tables(const ra_problem& p, int rot, float2* tab, cudaStream_t st) {
  const SegInfo s = seg_info(p);
  const int T = static_cast<int>(rope_table_len(p));
  rope_table_kernel<<<(T + 255) / 256, 256, 0, st>>>(s, T, static_cast<double>(p.theta), rot, tab);
  return cudaGetLastError();
}

// The quantise pass, with or without Q, in one code layout.
template <bool kBf16, int kRot, int kD, bool kS8>
static cudaError_t launch_quant(const PrologueArgs& a, dim3 grid, int quant_bytes, cudaStream_t st) {
  cudaError_t e;
  if (a.q) {
    if ((e = set_smem(prologue_quant_kernel<kBf16, kRot, kD, true, kS8>, quant_bytes)) != cudaSuccess) return e;
    prologue_quant_kernel<kBf16, kRot, kD, true, kS8><<<grid, kThreads, quant_bytes, st>>>(a);
  } else {
    const int kv_bytes = quant_bytes / 3 * 2;
    if ((e = set_smem(prologue_quant_kernel<kBf16, kRot, kD, false, kS8>, kv_bytes)) != cudaSuccess) return e;
    prologue_quant_kernel<kBf16, kRot, kD, false, kS8><<<grid, kThreads, kv_bytes, st>>>(a);
  }
  return cudaGetLastError();
}

// The three passes (channel reduce, finalize, quantise) for one input type and
// rotation mode and head dimension.
template <bool kBf16, int kRot, int kD>
static cudaError_t launch_passes3(const PrologueArgs& a, dim3 grid, int red_bytes, int quant_bytes,
                                  cudaStream_t st) {
  cudaError_t e;
  if ((e = set_smem(prologue_reduce_kernel<kBf16, kD>, red_bytes)) != cudaSuccess) return e;
  prologue_reduce_kernel<kBf16, kD><<<grid, kThreads, red_bytes, st>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  prologue_finalize_kernel<<<grid.y, 128, 0, st>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (a.s8) return launch_quant<kBf16, kRot, kD, true>(a, grid, quant_bytes, st);
  return launch_quant<kBf16, kRot, kD, false>(a, grid, quant_bytes, st);
}

template <bool kBf16, int kRot>
static cudaError_t launch_passes(const PrologueArgs& a, dim3 grid, int red_bytes, int quant_bytes,
                                 cudaStream_t st) {
  return a.D == 128 ? launch_passes3<kBf16, kRot, 128>(a, grid, red_bytes, quant_bytes, st)
                    : launch_passes3<kBf16, kRot, 64>(a, grid, red_bytes, quant_bytes, st);
}

cudaError_t launch_prologue(const ra_problem& p, int dtype, const void* q, const void* k, const void* v,
                            const int32_t* pos, uint8_t* q4, float* sq, uint8_t* k4, float* sk,
                            float* k_mean, uint8_t* v4, float* sv, int32_t* colsum, void* ws,
                            cudaStream_t st, bool s8) {
  const WorkspaceLayout w = workspace_layout(p);
  char* base = static_cast<char*>(ws);
  PrologueArgs a;
  a.s = seg_info(p);
  a.N = p.N; a.D = p.D; a.rot = p.rot; a.dtype = dtype; a.block_k = p.block_k;
  a.bk_log2 = __builtin_ctz(static_cast<unsigned>(p.block_k));
  a.nchunk = prologue_nchunk(p);
  a.q = q; a.k = k; a.v = v; a.pos = pos;
  a.tab = reinterpret_cast<const float2*>(base + w.tab);
  a.tab0 = reinterpret_cast<const float2*>(base + (p.rot == 1 ? w.tab0 : w.tab));
  a.ksum = reinterpret_cast<double*>(base + w.ksum);
  a.vmax = reinterpret_cast<float*>(base + w.vmax);
  a.vinv = reinterpret_cast<float*>(base + w.vinv);
  a.q4 = q4; a.k4 = k4; a.v4 = v4; a.sq = sq; a.sk = sk; a.k_mean = k_mean; a.sv = sv;
  a.colsum = colsum;
  a.s8 = s8 ? 1 : 0;
  cudaError_t e = launch_tables(p, p.rot, reinterpret_cast<float2*>(base + w.tab), st);
  if (e != cudaSuccess) return e;
  if (p.rot == 1) {  // the fused table differs from the plain one
    e = launch_tables(p, 0, reinterpret_cast<float2*>(base + w.tab0), st);
    if (e != cudaSuccess) return e;
  }
  const dim3 grid(a.nchunk, p.B * p.H);
  // Dynamic shared memory: the staged sub-chunks (the reduce pass reuses it
  // for its per-thread partial sums, 12 bytes x 8 channels x threads).
  const int el = dtype == 1 ? 2 : 4;
  const int red_bytes = kStgR * 2 * kSub * p.D * el > kThreads * 8 * 12 ? kStgR * 2 * kSub * p.D * el : kThreads * 8 * 12;
  const int quant_bytes = kStgQ * 3 * kSub * p.D * el;
  switch (dtype * 4 + p.rot) {
#define RA_PRO(DT, ROT)                                                                              \
  case DT * 4 + ROT:                                                                                 \
    e = launch_passes<DT == 1, ROT>(a, grid, red_bytes, quant_bytes, st);                            \
    break;
    RA_PRO(0, 0) RA_PRO(0, 1) RA_PRO(0, 2) RA_PRO(0, 3)
    RA_PRO(1, 0) RA_PRO(1, 1) RA_PRO(1, 2) RA_PRO(1, 3)
#undef RA_PRO
    default:
      return cudaErrorInvalidValue;
  }
  return e;
}

cudaError_t launch_rope_table(const ra_problem& p, void* ws, const float2** tab, cudaStream_t st) {
  const WorkspaceLayout w = workspace_layout(p);
  float2* t = reinterpret_cast<float2*>(static_cast<char*>(ws) + w.tab);
  *tab = t;
  return launch_tables(p, p.rot, t, st);
}

cudaError_t launch_rope_bf16(const ra_problem& p, int dtype, const void* q, const void* k,
                             const int32_t* pos, void* qo, void* ko, void* ws, cudaStream_t st) {
  const WorkspaceLayout w = workspace_layout(p);
  char* base = static_cast<char*>(ws);
  PrologueArgs a{};
  a.s = seg_info(p);
  a.N = p.N; a.D = p.D; a.rot = 0; a.dtype = dtype; a.block_k = p.block_k;
  a.bk_log2 = __builtin_ctz(static_cast<unsigned>(p.block_k));
  a.nchunk = prologue_nchunk(p);
  a.q = q; a.k = k; a.pos = pos;
  a.tab = reinterpret_cast<const float2*>(base + w.tab);
  cudaError_t e = launch_tables(p, 0, reinterpret_cast<float2*>(base + w.tab), st);
  if (e != cudaSuccess) return e;
  rope_bf16_kernel<<<dim3(a.nchunk, p.B * p.H), kThreads, 0, st>>>(a, static_cast<__nv_bfloat16*>(qo),
                                                                   static_cast<__nv_bfloat16*>(ko));
  return cudaGetLastError();
}

cudaError_t read_prologue_status(uint32_t* out) {
  uint32_t zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(out, g_prologue_status, sizeof(uint32_t));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_prologue_status, &zero, sizeof(uint32_t));
}

}  // namespace ra
