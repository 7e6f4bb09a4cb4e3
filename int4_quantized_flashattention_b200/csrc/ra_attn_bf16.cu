// bf16 FlashAttention forward on sm_100a: the selective-precision fallback of
// RotateAttention (papernotes page, key design 3): softmax(q k^T / sqrt(D)) v
// on bf16 RoPE'd q, k and v, fp32 accumulation, bf16 output.
//
// B200 design (the INT4 kernel's pipeline without the widening step):
//   * TMA loads bf16 Q, K and V tiles straight into 128B-swizzled shared
//     memory, 64 channels (128 bytes) per box.
//   * QK^T: tcgen05.mma kind::f16 (bf16 in, fp32 out), A = Q (smem, K-major),
//     B = K (smem, K-major), D = S in TMEM, M = 128, N = block_k; two S
//     buffers per query tile.
//   * Softmax: two threads per query row (.16x32bx2 TMEM accesses), exp2 of the
//     scaled scores against the running row maximum, P = bf16(p) stored into
//     TMEM over the S columns it came from; the row sum uses the fp32 p.
//   * P.V: tcgen05.mma kind::f16 with A = P from TMEM and B = V (smem,
//     MN-major), D = an fp32 accumulator in TMEM that keeps accumulating across
//     key blocks; when a row maximum grows the output gains (w_old - w_new)
//     times the accumulator (the weighted segment sums telescope), so the
//     accumulator is only reset at the end of a query tile.
//   * Persistent CTAs, two 128-row query tiles per CTA sharing each K/V tile.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "ra_common.cuh"
#include "ra_internal.h"

namespace ra {
namespace {

__device__ uint32_t g_bf16_status = 0;

constexpr int kThreads = 768;  // 24 warps: see the role map in the kernel
constexpr int kRows = 128;     // query rows per tile = MMA M
constexpr int kTiles = 2;      // query tiles per CTA

template <int D, int BN>
struct CfgB {
  static constexpr int kHalves = D / 64;               // 64-channel (128-byte) boxes per row
  static constexpr int kKS = 2, kVS = 2;               // K and V stages
  static constexpr int kQBytes = kRows * D * 2;        // one bf16 Q tile
  static constexpr int kKBytes = BN * D * 2;
  static constexpr int kVBytes = BN * D * 2;
  static constexpr int kQHalf = kRows * 128;           // one 64-channel box of Q
  static constexpr int kKHalf = BN * 128;
  static constexpr int oQ = 0;
  static constexpr int oK = oQ + kTiles * kQBytes;
  static constexpr int oV = oK + kKS * kKBytes;
  static constexpr int kFRow = D / 4 + 4;              // floats of F per thread in smem (padded)
  static constexpr int oF = oV + kVS * kVBytes;
  static constexpr int oBar = oF + kTiles * 2 * kRows * kFRow * 4;
  static constexpr int kNumBars = 2 + 2 * kKS + 2 * kVS + 4 + 4 + 4 + 2;
  static constexpr int oMisc = oBar + kNumBars * 8;
  static constexpr int kSmem = oMisc + 16 + 1024;
  static constexpr uint32_t kIdescQK = instr_desc(kCfmtF32, 1, 1, 0, 0, kRows, BN);
  static constexpr uint32_t kIdescPV = instr_desc(kCfmtF32, 1, 1, 0, 1, kRows, D);
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(BN == 16 || BN == 32 || BN == 64, "block_k");
  static_assert(kSmem <= 232448, "shared memory");
};

struct BarsB {
  uint64_t* q_full; uint64_t* q_free;
  uint64_t* k_full; uint64_t* k_empty;
  uint64_t* v_full; uint64_t* v_empty;
  uint64_t* s_full;   // [tile][buf]
  uint64_t* p_full;   // [tile][buf]
  uint64_t* pv_done;  // [tile][buf]
  uint64_t* drain;    // [issuer]
};

struct AttnBf16Params {
  int N, BH, nblocks, npairs, nitems;
  float scale;        // 1/sqrt(D)
  __nv_bfloat16* out;
  float* lse;
};

__device__ __forceinline__ void set_status_b(uint32_t bits) { atomicOr(&g_bf16_status, bits); }

__device__ __forceinline__ bool wait_b(uint64_t* bar, uint32_t parity, volatile int* abort, uint32_t backoff_ns = 16) {
  return mbar_wait_ex(bar, parity, abort, backoff_ns) > 0;
}

__device__ __forceinline__ float max3b(float a, float b, float c) { return fmaxf(a, fmaxf(b, c)); }

template <int n>
__device__ __forceinline__ float tree_max_b(const float* x) {
  if constexpr (n == 1) return x[0];
  else if constexpr (n == 2) return fmaxf(x[0], x[1]);
  else if constexpr (n == 3) return max3b(x[0], x[1], x[2]);
  else return max3b(tree_max_b<n / 3>(x), tree_max_b<n / 3>(x + n / 3), tree_max_b<n - 2 * (n / 3)>(x + 2 * (n / 3)));
}

template <int D, int BN>
__global__ void __launch_bounds__(kThreads, 1)
attn_bf16_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const AttnBf16Params prm) {
  using C = CfgB<D, BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::oBar);
  BarsB B;
  {
    uint64_t* b = bar;
    B.q_full = b++; B.q_free = b++;
    B.k_full = b; b += C::kKS; B.k_empty = b; b += C::kKS;
    B.v_full = b; b += C::kVS; B.v_empty = b; b += C::kVS;
    B.s_full = b; b += 4; B.p_full = b; b += 4; B.pv_done = b; b += 4; B.drain = b; b += 2;
  }
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::oMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::oMisc + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(B.q_full, 1); mbar_init(B.q_free, 2);
    for (int s = 0; s < C::kKS; ++s) { mbar_init(B.k_full + s, 1); mbar_init(B.k_empty + s, 2); }
    for (int s = 0; s < C::kVS; ++s) { mbar_init(B.v_full + s, 1); mbar_init(B.v_empty + s, 2); }
    for (int s = 0; s < 4; ++s) { mbar_init(B.s_full + s, 1); mbar_init(B.p_full + s, 8); mbar_init(B.pv_done + s, 1); }
    mbar_init(B.drain, 1);
    mbar_init(B.drain + 1, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_q); prefetch_tmap(&tm_k); prefetch_tmap(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;
  const int nb = prm.nblocks;
  // Roles: warp 0 TMA producer, warps 1 and 2 MMA issuers of query tiles 0 and
  // 1 (warp 1 owns TMEM), warps 3-7 idle, warps 8-15 and 16-23 softmax of query
  // tiles 0 and 1 (two threads per row, 16 rows per warp).
  if (warp < 8) {
    if (warp < 4) asm volatile("setmaxnreg.dec.sync.aligned.u32 56;");
    else asm volatile("setmaxnreg.dec.sync.aligned.u32 40;");
    if (warp == 0 && lane == 0) {
      // ------------------------------------------------------------ TMA producer
      uint32_t g = 0, li = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < prm.nitems && ok; item += gridDim.x, ++li) {
        const int bh = item / prm.npairs, pair = item % prm.npairs;
        if (!(ok = wait_b(B.q_free, (li & 1) ^ 1, abort_flag, 256u))) break;
        mbar_arrive_expect_tx(B.q_full, kTiles * C::kQBytes);
        for (int tt = 0; tt < kTiles; ++tt)
          for (int h = 0; h < C::kHalves; ++h)
            tma_load_3d(smem + C::oQ + tt * C::kQBytes + h * C::kQHalf, &tm_q, B.q_full, h * 64,
                        pair * 2 * kRows + tt * kRows, bh);
        for (int t = 0; t < nb && ok; ++t, ++g) {
          const int ks = g % C::kKS, vs = g % C::kVS;
          if (!(ok = wait_b(B.k_empty + ks, ((g / C::kKS) & 1) ^ 1, abort_flag, 256u))) break;
          mbar_arrive_expect_tx(B.k_full + ks, C::kKBytes);
          for (int h = 0; h < C::kHalves; ++h)
            tma_load_3d(smem + C::oK + ks * C::kKBytes + h * C::kKHalf, &tm_k, B.k_full + ks, h * 64, t * BN, bh);
          if (!(ok = wait_b(B.v_empty + vs, ((g / C::kVS) & 1) ^ 1, abort_flag, 256u))) break;
          mbar_arrive_expect_tx(B.v_full + vs, C::kVBytes);
          for (int h = 0; h < C::kHalves; ++h)
            tma_load_3d(smem + C::oV + vs * C::kVBytes + h * C::kKHalf, &tm_v, B.v_full + vs, h * 64, t * BN, bh);
        }
      }
      // Wait (bounded) for the copies of the last stages to land.
      for (uint32_t k = (g > (uint32_t)C::kKS ? g - C::kKS : 0); k < g; ++k) {
        uint32_t it = 0;
        while (!mbar_try_wait(B.k_full + (k % C::kKS), (k / C::kKS) & 1) && ++it < kSpinLimit) {}
        it = 0;
        while (!mbar_try_wait(B.v_full + (k % C::kVS), (k / C::kVS) & 1) && ++it < kSpinLimit) {}
      }
      if (!ok) set_status_b(kStatusTimeout);
    } else if ((warp == 1 || warp == 2) && lane == 0) {
      // ------------------------------------------------------------ MMA issuers
      // Per tile: P.V(g), then QK(g+2) into the S buffer whose P P.V(g) has
      // just read (after P.V(g) has completed: MMAs into different
      // accumulators are not ordered).
      const int tt = warp - 1;
      const uint32_t sQ = smem_u32(smem + C::oQ) + tt * C::kQBytes;
      const uint32_t sK = smem_u32(smem + C::oK);
      const uint32_t sV = smem_u32(smem + C::oV);
      const uint32_t tS0 = tbase + tt * 256;
      const uint32_t tA = tS0 + 128;
      uint32_t li = 0, g0 = 0;
      bool ok = true;
      auto issue_qk = [&](uint32_t gq, bool last_of_item) -> bool {
        const uint32_t buf = gq & 1;
        if (gq >= 2) {
          if (!wait_b(B.pv_done + tt * 2 + buf, ((gq - 2) >> 1) & 1, abort_flag, 32u)) return false;
        }
        const int ks = gq % C::kKS;
        if (!wait_b(B.k_full + ks, (gq / C::kKS) & 1, abort_flag, 32u)) return false;
        tc_fence_after();
        const uint32_t tS = tS0 + buf * 64;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk & 3) * 32;  // 16 channels = 32 bytes per K step
          const uint64_t adesc = smem_desc(sQ + (kk >> 2) * C::kQHalf + off, 16, 1024, kSwizzle128B);
          const uint64_t bdesc = smem_desc(sK + ks * C::kKBytes + (kk >> 2) * C::kKHalf + off, 16, 1024, kSwizzle128B);
          mma_f16_ss(tS, adesc, bdesc, C::kIdescQK, kk > 0 ? 1u : 0u);
        }
        mma_commit(B.s_full + tt * 2 + buf);
        mma_commit(B.k_empty + ks);
        if (last_of_item) mma_commit(B.q_free);
        return true;
      };
      for (int item = blockIdx.x; item < prm.nitems && ok; item += gridDim.x, ++li, g0 += nb) {
        if (!(ok = wait_b(B.q_full, li & 1, abort_flag, 32u))) break;
        tc_fence_after();
        for (int t = 0; t < 2 && t < nb && ok; ++t) ok = issue_qk(g0 + t, t == nb - 1);
        for (int t = 0; t < nb && ok; ++t) {
          const uint32_t gg = g0 + t;
          const int vs = gg % C::kVS;
          const uint32_t buf = gg & 1;
          if (!(ok = wait_b(B.v_full + vs, (gg / C::kVS) & 1, abort_flag, 32u))) break;
          if (!(ok = wait_b(B.p_full + tt * 2 + buf, (gg >> 1) & 1, abort_flag, 32u))) break;
          tc_fence_after();
          const uint32_t tP = tS0 + buf * 64;
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            // V: [BN keys x D] bf16, MN-major; 64-channel boxes C::kKHalf apart,
            // 8-key groups 1024 bytes apart.
            const uint64_t bdesc = smem_desc(sV + vs * C::kVBytes + kk * 16 * 128, C::kKHalf, 1024, kSwizzle128B);
            mma_f16_ts(tA, tP + kk * 8, bdesc, C::kIdescPV, 1);
          }
          mma_commit(B.pv_done + tt * 2 + buf);
          mma_commit(B.v_empty + vs);
          if (t + 2 < nb) ok = issue_qk(gg + 2, t + 2 == nb - 1);
        }
      }
      mma_commit(B.drain + tt);
      uint32_t it = 0;
      while (!mbar_try_wait(B.drain + tt, 0) && ++it < kSpinLimit) {}
      if (!ok) set_status_b(kStatusTimeout);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 96;");
    // -------------------------------------------------------------- softmax
    // Two threads per query row: lane l < 16 takes the first half of every key
    // block and of the output columns of its row, lane l + 16 the second halves.
    constexpr int kHK = BN / 2;          // keys of a block per thread
    constexpr int kHD = D / 2;           // output columns per thread
    constexpr int kFr = kHD / 2;         // of which in registers (the rest in shared memory)
    const int sw = warp - 8;
    const int tt = sw >> 3;
    const int sub = (sw >> 2) & 1;
    const int quad = warp & 3;
    const int hh = lane >> 4;
    const int r = quad * 32 + sub * 16 + (lane & 15);
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32 + sub * 16) << 16;
    const uint32_t tA = tbase + tt * 256 + 128 + lane_off;
    float4* Fs = reinterpret_cast<float4*>(smem + C::oF) + ((tt * 2 + hh) * kRows + r) * (C::kFRow / 4);
    const float kLog2e = 1.4426950408889634f;
    const float ci = prm.scale;                 // 1/sqrt(D)
    const float cpi = __fmul_rn(ci, kLog2e);
    const float2 cpi2 = make_float2(cpi, cpi);
    uint32_t g = 0;
    bool ok = true;
    float2 F2[kFr / 2];
    // F += coef * (fp32 accumulator A); with reset, A is then set to zero.
    auto fold = [&](float coef, bool reset) {
      const float2 w2 = make_float2(coef, coef);
#pragma unroll
      for (int c = 0; c < kHD; c += 32) {
        uint32_t a[32];
        tmem_ld_h<32, kHD>(tA + c, a);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int col = c + 4 * q;
          const float2 lo = make_float2(__uint_as_float(a[4 * q]), __uint_as_float(a[4 * q + 1]));
          const float2 hi = make_float2(__uint_as_float(a[4 * q + 2]), __uint_as_float(a[4 * q + 3]));
          if (col < kFr) {
            F2[col / 2] = __ffma2_rn(w2, lo, F2[col / 2]);
            F2[col / 2 + 1] = __ffma2_rn(w2, hi, F2[col / 2 + 1]);
          } else {
            const float4 f = Fs[(col - kFr) / 4];
            const float2 nl = __ffma2_rn(w2, lo, make_float2(f.x, f.y));
            const float2 nh = __ffma2_rn(w2, hi, make_float2(f.z, f.w));
            Fs[(col - kFr) / 4] = make_float4(nl.x, nl.y, nh.x, nh.y);
          }
        }
        if (reset) {
          uint32_t z[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) z[i] = 0u;
          tmem_st_h<32, kHD>(tA + c, z);
        }
      }
    };
    {
      uint32_t z[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) z[i] = 0u;
#pragma unroll
      for (int c = 0; c < kHD; c += 32) tmem_st_h<32, kHD>(tA + c, z);
    }
    for (int item = blockIdx.x; item < prm.nitems && ok; item += gridDim.x) {
      const int bh = item / prm.npairs, pair = item % prm.npairs;
      const int row = (pair * 2 + tt) * kRows + r;
      const bool row_ok = row < prm.N;
#pragma unroll
      for (int i = 0; i < kFr / 2; ++i) F2[i] = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int q = 0; q < (kHD - kFr) / 4; ++q) Fs[q] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      float m_run = -INFINITY, m_ref = 0.0f, w = 1.0f, Lf = 0.0f, Lrun = 0.0f;
      for (int t = 0; t < nb; ++t, ++g) {
        const uint32_t buf = g & 1;
        const uint32_t tS = tbase + tt * 256 + buf * 64 + lane_off;
        if (!(ok = wait_b(B.s_full + tt * 2 + buf, (g >> 1) & 1, abort_flag))) break;
        __syncwarp();
        tc_fence_after();
        const int nvalid = min(BN, prm.N - t * BN);
        uint32_t raw[kHK];
        tmem_ld_h<kHK, kHK>(tS, raw);
        float* sv = reinterpret_cast<float*>(raw);
        if (nvalid < BN) {  // last, ragged block: keys past N do not take part
#pragma unroll
          for (int j = 0; j < kHK; ++j)
            if (hh * kHK + j >= nvalid) sv[j] = -INFINITY;
        }
        float vmax = tree_max_b<kHK>(sv);
        vmax = fmaxf(vmax, __shfl_xor_sync(0xFFFFFFFFu, vmax, 16));
        const float m_blk = __fmul_rn(vmax, ci);
        const float m_new = fmaxf(m_run, m_blk);
        const bool grow = m_new > m_run;
        const float Mp = __fmul_rn(m_new, kLog2e);
        const float2 nMp2 = make_float2(-Mp, -Mp);
        // p = exp2(s cpi - m log2 e); P = bf16(p), two keys per word.
        uint32_t words[kHK / 2];
        float2 psum2 = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int q = 0; q < kHK / 2; ++q) {
          const float2 x = __ffma2_rn(make_float2(sv[2 * q], sv[2 * q + 1]), cpi2, nMp2);
          const float2 pe = make_float2(ex2_approx(x.x), ex2_approx(x.y));
          psum2 = __fadd2_rn(psum2, pe);
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(pe.x, pe.y);
          words[q] = *reinterpret_cast<const uint32_t*>(&b2);
        }
        float psum = psum2.x + psum2.y;
        psum += __shfl_xor_sync(0xFFFFFFFFu, psum, 16);
        tmem_st_h<kHK / 2, kHK / 2>(tS, words);
        // Weight of the coming segment; a rescale moves the reference max.
        float w_new = w, sc = 1.0f;
        if (t == 0) {
          m_ref = m_new;
          w_new = 1.0f;
        } else if (grow) {
          const float xx = __fmul_rn(m_new - m_ref, kLog2e);
          if (xx > 64.0f) {
            sc = ex2_approx(-xx);
            m_ref = m_new;
            w_new = 1.0f;
          } else {
            w_new = ex2_approx(xx);
          }
        }
        if (__any_sync(0xFFFFFFFFu, (t > 0) && grow)) {
          if (!(ok = wait_b(B.pv_done + tt * 2 + ((g - 1) & 1), ((g - 1) >> 1) & 1, abort_flag))) break;
          __syncwarp();
          tc_fence_after();
          if (sc != 1.0f) {
            const float2 sc2 = make_float2(sc, sc);
#pragma unroll
            for (int i = 0; i < kFr / 2; ++i) F2[i] = __fmul2_rn(F2[i], sc2);
            for (int q = 0; q < (kHD - kFr) / 4; ++q) {
              const float4 f = Fs[q];
              Fs[q] = make_float4(f.x * sc, f.y * sc, f.z * sc, f.w * sc);
            }
            Lf *= sc;
            w *= sc;
          }
          fold(w - w_new, false);
          Lf = fmaf(w, Lrun, Lf);
          Lrun = 0.0f;
        }
        w = w_new;
        Lrun += psum;
        m_run = m_new;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(B.p_full + tt * 2 + buf);
      }
      if (!ok) break;
      if (!(ok = wait_b(B.pv_done + tt * 2 + ((g - 1) & 1), ((g - 1) >> 1) & 1, abort_flag))) break;
      __syncwarp();
      tc_fence_after();
      fold(w, true);
      Lf = fmaf(w, Lrun, Lf);
      if (row_ok) {
        const float inv = 1.0f / Lf;
        const float* Fsf = reinterpret_cast<const float*>(Fs);
        __nv_bfloat16* orow = prm.out + (static_cast<size_t>(bh) * prm.N + row) * D + hh * kHD;
#pragma unroll
        for (int c = 0; c < kHD; c += 8) {
          uint32_t pk[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int i0 = c + 2 * u;
            const float f0 = i0 < kFr ? F2[i0 >> 1].x : Fsf[i0 - kFr];
            const float f1 = i0 < kFr ? F2[i0 >> 1].y : Fsf[i0 + 1 - kFr];
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(f0 * inv, f1 * inv);
            pk[u] = *reinterpret_cast<const uint32_t*>(&h2);
          }
          *reinterpret_cast<uint4*>(orow + c) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
        if (prm.lse && hh == 0) prm.lse[static_cast<size_t>(bh) * prm.N + row] = m_ref + logf(Lf);
      }
    }
    if (!ok) set_status_b(kStatusTimeout);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, 512);
}
// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 get_encoder_b() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 3D map over bf16 [BH, N, D]; box = 64 channels (128 bytes) x rows, 128-byte
// swizzle, zero fill past N.
bool make_bf16_map(CUtensorMap* m, const void* base, int BH, int N, int D, int rows) {
  auto enc = get_encoder_b();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(N) * D * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(rows), 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, int BN>
cudaError_t launch_cfg_b(const ra_problem& p, const void* q, const void* k, const void* v,
                         const AttnBf16Params& prm, cudaStream_t st) {
  using C = CfgB<D, BN>;
  CUtensorMap mq, mk, mv;
  const int BH = p.B * p.H;
  if (!make_bf16_map(&mq, q, BH, p.N, D, kRows) || !make_bf16_map(&mk, k, BH, p.N, D, BN) ||
      !make_bf16_map(&mv, v, BH, p.N, D, BN))
    return cudaErrorInvalidValue;
  auto kern = attn_bf16_kernel<D, BN>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  int dev = 0, nsm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const int grid = prm.nitems < nsm ? prm.nitems : nsm;
  kern<<<grid, kThreads, C::kSmem, st>>>(mq, mk, mv, prm);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_bf16(const ra_problem& p, const void* q, const void* k, const void* v, void* out,
                             float* lse, cudaStream_t st, int* unsupported) {
  AttnBf16Params prm{};
  prm.N = p.N;
  prm.BH = p.B * p.H;
  prm.nblocks = (p.N + p.block_k - 1) / p.block_k;
  prm.npairs = (p.N + 2 * kRows - 1) / (2 * kRows);
  prm.nitems = prm.BH * prm.npairs;
  prm.scale = static_cast<float>(1.0 / sqrt(static_cast<double>(p.D)));
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.lse = lse;
  *unsupported = 0;
#define RA_CASE(DD, BB) \
  if (p.D == DD && p.block_k == BB) return launch_cfg_b<DD, BB>(p, q, k, v, prm, st);
  RA_CASE(128, 64)
  RA_CASE(128, 32)
  RA_CASE(128, 16)
  RA_CASE(64, 64)
  RA_CASE(64, 32)
  RA_CASE(64, 16)
#undef RA_CASE
  *unsupported = 1;
  return cudaSuccess;
}

cudaError_t read_attn_bf16_status(uint32_t* out) {
  uint32_t zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(out, g_bf16_status, sizeof(uint32_t));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_bf16_status, &zero, sizeof(uint32_t));
}

}  // namespace ra
