// INT4 attention forward of RotateAttention on sm_100a for key blocks of 128:
// a CTA pair (a cluster of two, tcgen05 cta_group::2) computes one 256-row
// query tile.
//
// Method (papernotes page, flowchart D-F and key design 2), as in the
// single-CTA kernel for smaller blocks:
//   S_ij = (S_int_ij * s_k[j]) * (s_q[i] / sqrt(D)),  S_int = sum_d q4 k4 (exact)
//   online softmax over key blocks of 128 keys with the running row max m
//   P codes c_ij = clamp(rint(15 exp(S_ij - m)), 0, 15) - 8
//   acc_t = sum_j (c_ij + 8) v4_jd  (= sum_j c_ij v4_jd + 8 colsum_t)
//   O = sum_t alpha-chain (s_v/15) acc_t / sum_t alpha-chain sum_j (c_ij+8)/15
//   plus the ablation modes (block-local maximum, symmetric codes, fp32
//   denominator) selected by MODE.
//
// B200 design:
//   * One pair MMA covers M = 256 query rows: CTA r of the pair holds rows
//     128r..128r+127 of the tile (its half of A and of every accumulator) and
//     half of every B operand: keys 64r..64r+63 of each K block for Q K^T
//     (N = 128 keys) and channels rD/2..rD/2+D/2-1 of each V block for P.V
//     (N = D).  Each CTA therefore widens only half of every K and V block,
//     and both S and P.V cover 128 keys per step.
//   * Packed nibbles are widened to s8 as 16 x code (as in the single-CTA
//     kernel), which scales S_int by 256 and acc by 16, both exact.
//   * Tensor memory per CTA (512 columns, allocated for the pair): two S
//     buffers of 128 columns (Q K^T of block g+1 runs while the softmax works
//     on block g; the P codes of a block overwrite the first 32 columns of its
//     S buffer), the s32 P.V accumulator A (D columns, kept across blocks and
//     holding the bits of 1.5 * 2^23 before P.V accumulates onto it, so an
//     integer x reads back as the float 1.5 * 2^23 + x) and the fp32 output
//     accumulator F (D columns).  The only cross-warp dependency per block is
//     P.V(g) -> Q K^T(g+2), which has a whole softmax step of slack.
//   * Warp roles per CTA (16 warps): 0 TMA producer, 1 MMA issuer (even CTA)
//     and tensor-memory owner, 2-3 idle, 4-7 widening, 8-15 softmax (two
//     threads per query row, 64 keys and D/2 accumulator columns each).
//   * Cross-CTA signalling: the widening and softmax warps of both CTAs arrive
//     on the even CTA's barriers (mapa + release at cluster scope); the MMA
//     completions arrive on both CTAs' barriers (tcgen05.commit multicast).
//     Every wait is bounded in time; a timeout raises the abort flag of both
//     CTAs and the device status word.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "ra_common.cuh"
#include "ra_internal.h"

namespace ra {
namespace {

__device__ uint32_t g_pair_status = 0;
// First timed-out wait: (site << 24) | (block counter & 0xFFFF) << 8 | (cluster rank << 7) | (cluster & 0x7F).
__device__ uint32_t g_pair_diag = 0;

constexpr int kThreadsP = 512;   // 16 warps
constexpr int kBK = 128;         // keys per block
constexpr int kRowsP = 128;      // query rows per CTA (M = 256 per pair)
constexpr uint32_t kMagicP = 0x4B400000u;  // bits of 1.5 * 2^23
constexpr float kMagicPF = 12582912.0f;

constexpr int align1k(int x) { return (x + 1023) / 1024 * 1024; }

template <int D, bool DUMP>
struct PairCfg {
  static constexpr int kStages = 4;                       // K/V/scale/packed pipeline depth
  static constexpr int kQw = kRowsP * D;                  // widened Q half (K-major, D bytes per row)
  static constexpr int kQPk = kRowsP * D / 2;             // packed Q half
  static constexpr int kKRows = kBK / 2;                  // keys of a block held by one CTA
  static constexpr int kKw = kKRows * D;                  // widened K half (K-major)
  static constexpr int kVRow = D / 2;                     // widened bytes per key of the V half (MN-major)
  static constexpr int kVw = kBK * kVRow;                 // widened V half
  static constexpr int kKPk = kKRows * D / 2;             // packed K half
  static constexpr int kVPk = kBK * D / 4;                // packed V half
  static constexpr int oQ = 0;
  static constexpr int oQPk = oQ + kQw;
  static constexpr int oKw = align1k(oQPk + kQPk);
  static constexpr int oVw = oKw + kStages * align1k(kKw);
  static constexpr int oPk = oVw + kStages * align1k(kVw);
  static constexpr int oKsc = oPk + kStages * (kKPk + kVPk);
  // DUMP variant: every softmax thread's accumulator columns at the previous
  // read-back (to dump each block's own P.V result without changing the fold
  // schedule of the kernel).
  static constexpr int oPrev = oKsc + kStages * kBK * 4;
  static constexpr int kPrevBytes = DUMP ? 256 * (D / 2) * 4 : 0;
  static constexpr int oBar = oPrev + kPrevBytes;
  static constexpr int kNumBars = 16 + 8 * kStages;
  static constexpr int oMisc = oBar + kNumBars * 8;
  static constexpr int kSmem = oMisc + 16 + 1024;        // + alignment slack
  static constexpr int kKwStride = align1k(kKw);
  static constexpr int kVwStride = align1k(kVw);
  static constexpr uint32_t kSwzQK = D == 128 ? kSwizzle128B : kSwizzle64B;
  static constexpr uint32_t kSwzV = D == 128 ? kSwizzle64B : kSwizzle32B;
  static constexpr uint32_t kIdescQK = instr_desc(kCfmtS32, 1, 1, 0, 0, 2 * kRowsP, kBK);
  static constexpr uint32_t kIdescPV = instr_desc(kCfmtS32, 0, 1, 0, 1, 2 * kRowsP, D);
  // tensor memory columns
  static constexpr uint32_t tS = 0, tA = 256, tF = 384;   // S buffer b at tS + 128 b
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(kSmem <= 227 * 1024, "shared memory");
};

struct PairBars {
  // local to each CTA
  uint64_t* qpk_full; uint64_t* qpk_empty; uint64_t* q_free;
  uint64_t* pk_full; uint64_t* pk_empty;     // [stage]
  uint64_t* kw_empty; uint64_t* vw_empty;    // [stage], MMA commits (multicast)
  uint64_t* ksc_full; uint64_t* ksc_empty;   // [stage]
  uint64_t* s_full;                          // [S buffer], MMA commits (multicast): Q K^T done
  uint64_t* pv_done;                         // [S buffer], MMA commits (multicast): P.V done
  // arrived on by both CTAs; used in the even CTA only
  uint64_t* kw_full; uint64_t* vw_full;      // [stage]
  uint64_t* q_full;
  uint64_t* p_full;                          // [S buffer]: P codes stored by every softmax warp
  uint64_t* drain;
};

struct PairParams {
  int N, BH, nblocks, ntiles, nitems;
  float inv_sqrt_d;
  const float* sq;
  const float* sk;
  const float* sv;
  __nv_bfloat16* out;
  float* lse;
  int dump_bh, dump_tile;   // tile in units of 128 rows
  int32_t* dump_s;
  int8_t* dump_p;
  int32_t* dump_acc;
};

__device__ __forceinline__ void widen_chunk_p(const uint8_t* src, uint8_t* dst_lo, uint8_t* dst_hi) {
  const uint4 w = *reinterpret_cast<const uint4*>(src);
  uint4 lo, hi;
  lo.x = (w.x << 4) & 0xF0F0F0F0u; hi.x = w.x & 0xF0F0F0F0u;
  lo.y = (w.y << 4) & 0xF0F0F0F0u; hi.y = w.y & 0xF0F0F0F0u;
  lo.z = (w.z << 4) & 0xF0F0F0F0u; hi.z = w.z & 0xF0F0F0F0u;
  lo.w = (w.w << 4) & 0xF0F0F0F0u; hi.w = w.w & 0xF0F0F0F0u;
  *reinterpret_cast<uint4*>(dst_lo) = lo;
  *reinterpret_cast<uint4*>(dst_hi) = hi;
}

// Widening of ROWS rows of PK packed bytes each into a swizzled tile with
// rows of 2 * PK bytes, by 128 threads; offsets computed once.  Packed chunk
// pc (16 bytes, 32 codes) of a row becomes widened chunks 2pc (low nibbles:
// even elements) and 2pc + 1 (high nibbles: odd elements).
template <int ROWS, int PK>
struct WidenPlanP {
  static constexpr int kPc = PK / 16;
  static constexpr int kChunks = ROWS * kPc;
  static constexpr int kIter = (kChunks + 127) / 128;
  static_assert(kChunks % 128 == 0, "whole iterations");
  uint32_t src[kIter], lo[kIter], hi[kIter];
  __device__ __forceinline__ void init(int tid) {
#pragma unroll
    for (int k = 0; k < kIter; ++k) {
      const int idx = tid + 128 * k;
      const int r = idx / kPc, pc = idx % kPc;
      src[k] = static_cast<uint32_t>(r * PK + pc * 16);
      lo[k] = swz_offset3(r, 2 * pc, 2 * PK);
      hi[k] = swz_offset3(r, 2 * pc + 1, 2 * PK);
    }
  }
  __device__ __forceinline__ void run(const uint8_t* pk, uint8_t* wide) const {
#pragma unroll
    for (int k = 0; k < kIter; ++k) widen_chunk_p(pk + src[k], wide + lo[k], wide + hi[k]);
  }
};

// As WidenPlanP, by 64 threads.
template <int ROWS, int PK>
struct WidenPlanP64 {
  static constexpr int kPc = PK / 16;
  static constexpr int kChunks = ROWS * kPc;
  static constexpr int kIter = kChunks / 64;
  static_assert(kChunks % 64 == 0, "whole iterations");
  uint32_t src[kIter], lo[kIter], hi[kIter];
  __device__ __forceinline__ void init(int tid) {
#pragma unroll
    for (int k = 0; k < kIter; ++k) {
      const int idx = tid + 64 * k;
      const int r = idx / kPc, pc = idx % kPc;
      src[k] = static_cast<uint32_t>(r * PK + pc * 16);
      lo[k] = swz_offset3(r, 2 * pc, 2 * PK);
      hi[k] = swz_offset3(r, 2 * pc + 1, 2 * PK);
    }
  }
  __device__ __forceinline__ void run(const uint8_t* pk, uint8_t* wide) const {
#pragma unroll
    for (int k = 0; k < kIter; ++k) widen_chunk_p(pk + src[k], wide + lo[k], wide + hi[k]);
  }
};

// Widening of ROWS rows (once per item) by 64 threads, offsets computed on the fly.
template <int ROWS, int PK>
__device__ __forceinline__ void widen_rows(const uint8_t* pk, uint8_t* wide, int tid) {
  constexpr int kPc = PK / 16;
#pragma unroll 4
  for (int idx = tid; idx < ROWS * kPc; idx += 64) {
    const int r = idx / kPc, pc = idx % kPc;
    widen_chunk_p(pk + r * PK + pc * 16, wide + swz_offset3(r, 2 * pc, 2 * PK), wide + swz_offset3(r, 2 * pc + 1, 2 * PK));
  }
}

// Widened position n (0..D-1) of a row -> channel (32-position groups: 16
// even channels, then 16 odd ones).
__host__ __device__ constexpr int wide_to_dim_p(int n) {
  return (n & ~31) + 8 * ((n & 15) >> 2) + 2 * (n & 3) + ((n >> 4) & 1);
}

__device__ __forceinline__ float max3p(float a, float b, float c) { return fmaxf(a, fmaxf(b, c)); }
template <int n>
__device__ __forceinline__ float tree_max_p(const float* x) {
  if constexpr (n == 1) return x[0];
  else if constexpr (n == 2) return fmaxf(x[0], x[1]);
  else if constexpr (n == 3) return max3p(x[0], x[1], x[2]);
  else return max3p(tree_max_p<n / 3>(x), tree_max_p<n / 3>(x + n / 3), tree_max_p<n - 2 * (n / 3)>(x + 2 * (n / 3)));
}

struct Abort {
  volatile int* local;
  uint32_t peer;  // shared::cluster address of the peer CTA's flag
  __device__ __forceinline__ void raise() const {
    *local = 1;
    st_cluster_u32(peer, 1u);
  }
};

__device__ __forceinline__ void note_timeout_p(uint32_t site, uint32_t g, uint32_t rank) {
  atomicCAS(&g_pair_diag, 0u, (site << 24) | ((g & 0xFFFFu) << 8) | (rank << 7) | (cluster_id_x() & 0x7Fu));
  atomicOr(&g_pair_status, kStatusTimeout);
}

// Bounded wait; on a timeout both CTAs' abort flags are raised.  Waits on
// barriers completed by the pair's MMA commits or by this CTA's own threads
// acquire at CTA scope; the MMA issuer's waits on the operands widened by
// both CTAs (generic stores made visible to the tensor core's async proxy)
// acquire at cluster scope.
__device__ __forceinline__ bool pwait(uint64_t* bar, uint32_t parity, const Abort& ab, uint32_t site, uint32_t g,
                                      uint32_t rank, uint32_t backoff_ns = 32, bool cluster_scope = false) {
  const int r = cluster_scope ? mbar_wait_cluster(bar, parity, ab.local, backoff_ns)
                              : mbar_wait_ex(bar, parity, ab.local, backoff_ns);
  if (r < 0) {
    ab.raise();
    note_timeout_p(site, g, rank);
  }
  return r > 0;
}

// As pwait, for all 32 lanes of a warp together: the lanes test the barrier
// and decide as one (warp votes), so the warp stays converged through the wait
// and the warp-collective tensor-memory accesses after it.
__device__ __forceinline__ bool pwait_warp(uint64_t* bar, uint32_t parity, const Abort& ab, uint32_t site, uint32_t g,
                                           uint32_t rank, uint32_t backoff_ns = 32) {
  const bool first = mbar_test_wait(bar, parity);
  if (__all_sync(0xFFFFFFFFu, first)) return true;
  const uint64_t t0 = global_ns();
  uint32_t sleep = 16;
  for (uint32_t n = 1;; ++n) {
    __nanosleep(sleep);
    const bool done = mbar_test_wait(bar, parity);
    if (__all_sync(0xFFFFFFFFu, done)) return true;
    sleep = min(sleep * 2, backoff_ns);
    if ((n & 31u) == 0) {
      const bool aborted = *ab.local != 0;
      const bool late = global_ns() - t0 > kWaitLimitNs;
      const bool any_aborted = __any_sync(0xFFFFFFFFu, aborted);
      const bool any_late = __any_sync(0xFFFFFFFFu, late);
      if (any_late && !any_aborted) {
        if ((threadIdx.x & 31) == 0) {
          ab.raise();
          note_timeout_p(site, g, rank);
        }
      }
      if (any_aborted || any_late) return false;
    }
  }
}

// MODE bits 0-1: P codes (0 range-rectified, 1 block-local maximum, 2
// symmetric); bit 2: fp32 denominator.
template <int D, bool DUMP, int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreadsP, 1)
attn_int4_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const PairParams prm) {
  using C = PairCfg<D, DUMP>;
  extern __shared__ uint8_t smem_raw[];
  // Same 1024-aligned layout in both CTAs (the pair MMA reads both at the same offsets).
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::oBar);
  constexpr int S = C::kStages;
  PairBars B;
  {
    uint64_t* b = bar;
    B.qpk_full = b++; B.qpk_empty = b++; B.q_free = b++; B.q_full = b++; B.drain = b++;
    B.s_full = b; b += 2; B.pv_done = b; b += 2; B.p_full = b; b += 2;
    B.pk_full = b; b += S; B.pk_empty = b; b += S;
    B.kw_empty = b; b += S; B.vw_empty = b; b += S;
    B.ksc_full = b; b += S; B.ksc_empty = b; b += S;
    B.kw_full = b; b += S; B.vw_full = b; b += S;
  }
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::oMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::oMisc + 4);
  const uint32_t rank = cluster_ctarank();
  const Abort ab{abort_flag, map_shared_rank(smem_u32(smem + C::oMisc + 4), rank ^ 1u)};
  // shared::cluster address of a barrier in the even CTA
  auto lead = [&](uint64_t* b) { return map_shared_rank(smem_u32(b), 0u); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(B.qpk_full, 1); mbar_init(B.qpk_empty, 2); mbar_init(B.q_free, 1);
    mbar_init(B.q_full, 4); mbar_init(B.drain, 1);
    for (int i = 0; i < 2; ++i) { mbar_init(B.s_full + i, 1); mbar_init(B.pv_done + i, 1); mbar_init(B.p_full + i, 16); }
    for (int s = 0; s < S; ++s) {
      mbar_init(B.pk_full + s, 1); mbar_init(B.pk_empty + s, 4);
      mbar_init(B.kw_empty + s, 1); mbar_init(B.vw_empty + s, 1);
      mbar_init(B.ksc_full + s, 2); mbar_init(B.ksc_empty + s, 8);
      mbar_init(B.kw_full + s, 4); mbar_init(B.vw_full + s, 4);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, 512);
    tmem_relinquish_pair();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_q); prefetch_tmap(&tm_k); prefetch_tmap(&tm_v);
  }
  // Both CTAs' barriers are initialised before any remote arrival.
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;

  const int nb = prm.nblocks;
  const uint32_t cl = cluster_id_x(), ncl = cluster_count_x();
  if (warp < 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 64;");
    if (warp == 0) {
      // ------------------------------------------------------------ TMA producer (each CTA)
      if (lane == 0) {
        uint32_t g = 0, li = 0;
        bool ok = true;
        for (int item = cl; item < prm.nitems && ok; item += ncl, ++li) {
          const int bh = item / prm.ntiles, tile = item % prm.ntiles;
          if (!(ok = pwait(B.qpk_empty, (li & 1) ^ 1, ab, 1u, li, rank, 256u))) break;
          mbar_arrive_expect_tx(B.qpk_full, C::kQPk);
          tma_load_3d(smem + C::oQPk, &tm_q, B.qpk_full, 0, tile * 2 * kRowsP + rank * kRowsP, bh);
          for (int t = 0; t < nb; ++t, ++g) {
            const int s = g % S;
            if (!(ok = pwait(B.pk_empty + s, ((g / S) & 1) ^ 1, ab, 2u, g, rank, 256u))) break;
            mbar_arrive_expect_tx(B.pk_full + s, C::kKPk + C::kVPk);
            uint8_t* dst = smem + C::oPk + s * (C::kKPk + C::kVPk);
            tma_load_3d(dst, &tm_k, B.pk_full + s, 0, t * kBK + rank * C::kKRows, bh);
            tma_load_3d(dst + C::kKPk, &tm_v, B.pk_full + s, rank * (D / 4), t * kBK, bh);
          }
        }
        // Wait (bounded) for the copies of the last stages to land.
        for (uint32_t k = (g > static_cast<uint32_t>(S) ? g - S : 0); k < g; ++k) {
          uint32_t it = 0;
          while (!mbar_try_wait(B.pk_full + (k % S), (k / S) & 1) && ++it < kSpinLimit) {}
        }
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer (even CTA)
      if (rank == 0 && lane == 0) {
        const uint32_t sQ = smem_u32(smem + C::oQ);
        const uint32_t sKw = smem_u32(smem + C::oKw);
        const uint32_t sVw = smem_u32(smem + C::oVw);
        // Event loop over this cluster's blocks (numbered across its items):
        // QK(g) into S buffer g & 1 once K(g) is widened in both CTAs, Q for
        // the first block of an item, and P.V(g - 2) (which reads the P codes
        // in that buffer) has completed; P.V(g) once the P codes of block g
        // are in place and V(g) is widened.  Whichever is ready is issued, so
        // a late K tile never holds up a P.V.
        const uint32_t my_items = prm.nitems > static_cast<int>(cl) ? (prm.nitems - cl + ncl - 1) / ncl : 0u;
        const uint32_t total = my_items * static_cast<uint32_t>(nb);
        uint32_t qk = 0, pv = 0;
        uint32_t sleep = 16, idle = 0;
        uint64_t t_idle = 0;
        bool ok = true;
        while (pv < total) {
          bool progressed = false;
          if (qk < total && qk < pv + 2) {
            const uint32_t li = qk / nb, t = qk % nb;
            const int ks = qk % S;
            const uint32_t sb = qk & 1;
            if ((t != 0 || mbar_test_wait_cluster(B.q_full, li & 1)) &&
                (qk < 2 || mbar_test_wait(B.pv_done + sb, ((qk - 2) >> 1) & 1)) &&
                mbar_test_wait_cluster(B.kw_full + ks, (qk / S) & 1)) {
              tc_fence_after();
#pragma unroll
              for (int kk = 0; kk < D / 32; ++kk) {
                const uint64_t adesc = smem_desc(sQ + kk * 32, 16, 8 * D, C::kSwzQK);
                const uint64_t bdesc = smem_desc(sKw + ks * C::kKwStride + kk * 32, 16, 8 * D, C::kSwzQK);
                mma_i8_ss_pair(tbase + C::tS + sb * 128, adesc, bdesc, C::kIdescQK, kk > 0 ? 1u : 0u);
              }
              mma_commit_pair(B.s_full + sb);
              mma_commit_pair(B.kw_empty + ks);
              if (t == static_cast<uint32_t>(nb) - 1) mma_commit_pair(B.q_free);
              ++qk;
              progressed = true;
            }
          }
          if (pv < qk) {
            const int vs = pv % S;
            const uint32_t pb = pv & 1;
            if (mbar_test_wait_cluster(B.vw_full + vs, (pv / S) & 1) && mbar_test_wait(B.p_full + pb, (pv >> 1) & 1)) {
              tc_fence_after();
#pragma unroll
              for (int kk = 0; kk < kBK / 32; ++kk) {
                const uint64_t bdesc = smem_desc(sVw + vs * C::kVwStride + kk * 32 * C::kVRow, C::kVw,
                                                 8 * C::kVRow, C::kSwzV);
                mma_i8_ts_pair(tbase + C::tA, tbase + C::tS + pb * 128 + kk * 8, bdesc, C::kIdescPV, 1u);
              }
              mma_commit_pair(B.pv_done + pb);
              mma_commit_pair(B.vw_empty + vs);
              ++pv;
              progressed = true;
            }
          }
          if (progressed) {
            sleep = 16;
            idle = 0;
            continue;
          }
          // Nothing ready: back off; a wait that lasts past the bound aborts.
          if (idle == 0) t_idle = global_ns();
          __nanosleep(sleep);
          sleep = min(sleep * 2, 64u);
          if ((++idle & 31u) == 0) {
            if (*abort_flag) { ok = false; break; }
            if (global_ns() - t_idle > kWaitLimitNs) {
              ab.raise();
              note_timeout_p(3u, pv, rank);
              ok = false;
              break;
            }
          }
        }
        (void)ok;
        // Every MMA issued by this thread completes before tensor memory is released.
        mma_commit_pair(B.drain);
        uint32_t it = 0;
        while (!mbar_try_wait(B.drain, 0) && ++it < kSpinLimit) {}
      }
    } else if (warp >= 4) {
      // ------------------------------------------------------------ widening (each CTA)
      // Warps 4-5 widen Q (once per item) and the K half of every block and
      // stage the block's key scales; warps 6-7 widen the V half.  The two
      // groups run independently, each up to kStages blocks ahead.
      const int wt = (threadIdx.x - 128) & 63;  // thread within its group
      const bool kgroup = warp < 6;
      uint32_t g = 0, li = 0;
      bool ok = true;
      if (kgroup) {
        WidenPlanP64<C::kKRows, D / 2> planK;
        planK.init(wt);
        const uint32_t q_full_l = lead(B.q_full);
        for (int item = cl; item < prm.nitems && ok; item += ncl, ++li) {
          const int bh = item / prm.ntiles;
          const float* skh = prm.sk + static_cast<size_t>(bh) * prm.N;
          // Scales of keys wt and wt + 64 of a block, loaded one block ahead.
          auto load_sc = [&](int t, int j) -> float {
            const int key = t * kBK + j;
            return key < prm.N ? __ldg(skh + key) * (1.0f / 256.0f) : __int_as_float(0x7FC00000);
          };
          float sc0 = load_sc(0, wt), sc1 = load_sc(0, wt + 64);
          if (!(ok = pwait_warp(B.qpk_full, li & 1, ab, 8u, li, rank, 256u))) break;
          if (!(ok = pwait_warp(B.q_free, (li & 1) ^ 1, ab, 9u, li, rank, 256u))) break;
          widen_rows<kRowsP, D / 2>(smem + C::oQPk, smem + C::oQ, wt);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) { mbar_arrive(B.qpk_empty); mbar_arrive_cluster(q_full_l); }
          for (int t = 0; t < nb; ++t, ++g) {
            const int s = g % S;
            const uint32_t ph = ((g / S) & 1) ^ 1;
            if (!(ok = pwait_warp(B.pk_full + s, (g / S) & 1, ab, 10u, g, rank, 128u))) break;
            const uint8_t* pk = smem + C::oPk + s * (C::kKPk + C::kVPk);
            if (!(ok = pwait_warp(B.kw_empty + s, ph, ab, 11u, g, rank, 256u))) break;
            planK.run(pk, smem + C::oKw + s * C::kKwStride);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) { mbar_arrive_cluster(lead(B.kw_full + s)); mbar_arrive(B.pk_empty + s); }
            // The next block's scales, requested after the cluster-scope
            // release above (which would otherwise wait for these loads).
            const float nx0 = t + 1 < nb ? load_sc(t + 1, wt) : 0.0f;
            const float nx1 = t + 1 < nb ? load_sc(t + 1, wt + 64) : 0.0f;
            // Per-key scales of the whole block (both CTAs' softmax rows use
            // all 128 keys).  Keys past N get a NaN scale: their score is NaN,
            // which the maximum ignores, and their code bytes are masked.
            if (!(ok = pwait_warp(B.ksc_empty + s, ph, ab, 12u, g, rank, 256u))) break;
            float* ksc = reinterpret_cast<float*>(smem + C::oKsc) + s * kBK;
            ksc[wt] = sc0;
            ksc[wt + 64] = sc1;
            __syncwarp();
            if (lane == 0) mbar_arrive(B.ksc_full + s);
            sc0 = nx0;
            sc1 = nx1;
          }
        }
      } else {
        WidenPlanP64<kBK, D / 4> planV;
        planV.init(wt);
        for (int item = cl; item < prm.nitems && ok; item += ncl, ++li) {
          for (int t = 0; t < nb; ++t, ++g) {
            const int s = g % S;
            const uint32_t ph = ((g / S) & 1) ^ 1;
            if (!(ok = pwait_warp(B.pk_full + s, (g / S) & 1, ab, 10u, g, rank, 128u))) break;
            const uint8_t* pk = smem + C::oPk + s * (C::kKPk + C::kVPk);
            if (!(ok = pwait_warp(B.vw_empty + s, ph, ab, 13u, g, rank, 256u))) break;
            planV.run(pk + C::kKPk, smem + C::oVw + s * C::kVwStride);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) { mbar_arrive_cluster(lead(B.vw_full + s)); mbar_arrive(B.pk_empty + s); }
          }
        }
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 192;");
    // -------------------------------------------------------------- softmax (each CTA)
    // Two threads per query row: lane l < 16 takes keys 0-63 of every block
    // and accumulator columns 0..D/2-1 of its row, lane l + 16 keys 64-127 and
    // columns D/2..D-1 (.16x32bx2 tensor-memory accesses).
    constexpr int kHK = kBK / 2;         // keys of a block per thread
    constexpr int kHD = D / 2;           // accumulator columns per thread
    const int sw = warp - 8;             // softmax warp 0..7
    const int quad = warp & 3;           // tensor-memory lane quadrant of this warp
    const int sub = sw >> 2;             // half of the quadrant
    const int hh = lane >> 4;            // half of the keys / columns
    const int r = quad * 32 + sub * 16 + (lane & 15);  // row within this CTA's 128
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32 + sub * 16) << 16;
    const uint32_t tA = tbase + C::tA + lane_off;
    const uint32_t tF = tbase + C::tF + lane_off;
    int32_t* prev = DUMP ? reinterpret_cast<int32_t*>(smem + C::oPrev) + (sw * 32 + lane) * kHD : nullptr;
    const float kLog2e = 1.4426950408889634f;
    const float2 kNegMagic2 = make_float2(-kMagicPF, -kMagicPF);
    // Byte-lane magics: fp32 values in [2^23, 2^24) with a zero low byte whose
    // bits K0..K3 satisfy K0 + K1 2^8 + K2 2^16 + K3 2^24 = 0 mod 2^32, so
    // t0 + t1 2^8 + t2 2^16 + t3 2^24 of the rounded sums is the packed word.
    const float2 kMagLo = make_float2(8388608.0f, 11862016.0f);   // bits 0x4B000000, 0x4B350000
    const float2 kMagHi = make_float2(8421376.0f, kMagicPF);      // bits 0x4B008000, 0x4B400000
    constexpr int kPMode = MODE & 3;
    constexpr bool kLf = (MODE & 4) != 0;
    constexpr float kLevels = kPMode == 2 ? 7.0f : 15.0f;
    constexpr int kZero = kPMode == 2 ? 0 : 8;
    const float2 kLv2 = make_float2(kLevels, kLevels);
    const uint32_t p_full_l[2] = {lead(B.p_full), lead(B.p_full + 1)};
    uint32_t g = 0;
    bool ok = true;

    // F += coef * (A - magic) over this thread's columns; with reset, A is set
    // back to the magic (integer zero).  Without reset, A keeps accumulating
    // across a change of the row maximum: with segments s_k of P.V results
    // between changes, A_k = s_1 + ... + s_k and segment weights w_k,
    // sum_k w_k s_k = sum_k (w_k - w_(k+1)) A_k + w_last A_last, so each change
    // adds (w_old - w_new) A to F and the last fold adds w_last A.
    // Stores are not waited for here: the wait before the next arrive (or
    // before the next load of these columns) covers them.
    auto fold = [&](float coef, bool reset) __attribute__((always_inline)) {
      const float2 w2 = make_float2(coef, coef);
      uint32_t a[kHD], f[kHD];
      // every column of this thread in one round trip (D = 64: one pair of loads)
      if constexpr (kHD == 64) {
        tmem_ld_h32_quad<kHD>(tA, tF, tA + 32, tF + 32, a, f, a + 32, f + 32);
      } else {
        tmem_ld_h32_pair<kHD>(tA, tF, a, f);
      }
#pragma unroll
      for (int q = 0; q < kHD; q += 2) {
        const float2 x = __fadd2_rn(make_float2(__uint_as_float(a[q]), __uint_as_float(a[q + 1])), kNegMagic2);
        const float2 y = __ffma2_rn(w2, x, make_float2(__uint_as_float(f[q]), __uint_as_float(f[q + 1])));
        f[q] = __float_as_uint(y.x);
        f[q + 1] = __float_as_uint(y.y);
      }
#pragma unroll
      for (int c = 0; c < kHD; c += 32) {
        tmem_st_h32_nw<kHD>(tF + c, f + c);
        if (reset) tmem_fill_h32_nw<kHD>(tA + c, kMagicP);
      }
    };
    // DUMP: the accumulator of the block whose P.V completed last, as the
    // difference to the previous read-back (A itself keeps accumulating).  The
    // whole warp reads tensor memory; only rows of the dumped tile write.
    auto dump_acc = [&](int blk, int row_in_tile, bool was_reset, bool write) {
#pragma unroll 1
      for (int c = 0; c < kHD; c += 32) {
        uint32_t a[32];
        tmem_ld_h<32, kHD>(tA + c, a);
        if (write) {
#pragma unroll 1
          for (int i = 0; i < 32; ++i) {
            const int cur = static_cast<int>(a[i]) - static_cast<int>(kMagicP);
            const int before = was_reset ? 0 : prev[c + i];
            prm.dump_acc[(static_cast<size_t>(row_in_tile) * nb + blk) * D + wide_to_dim_p(hh * kHD + c + i)] =
                (cur - before) / 16;
            prev[c + i] = cur;
          }
        }
      }
    };
    // Reads S of block gs (after its Q K^T) from S buffer gs & 1; both halves
    // of the warp read 64 keys.
    auto take_s = [&](uint32_t gs, uint32_t* raw) __attribute__((always_inline)) -> bool {
      if (!pwait_warp(B.s_full + (gs & 1), (gs >> 1) & 1, ab, 14u, gs, rank, 16u)) return false;
      if (!pwait_warp(B.ksc_full + gs % S, (gs / S) & 1, ab, 15u, gs, rank, 16u)) return false;
      tc_fence_after();
      tmem_ld_h64<kHK>(tbase + C::tS + (gs & 1) * 128 + lane_off, raw);
      return true;
    };
    // v = S_int * s_k (256 S_int is exact in fp32 and s_k/256 a power-of-two
    // scaling, so v is S_int * s_k rounded once) and the row maximum of the
    // block over both halves.  Keys past N have a NaN scale, which the
    // maximum ignores.
    auto scale_max = [&](uint32_t gs, const uint32_t* raw, float2* v) __attribute__((always_inline)) -> float {
      const float4* ksc = reinterpret_cast<const float4*>(smem + C::oKsc) + (gs % S) * (kBK / 4) + hh * (kHK / 4);
#pragma unroll
      for (int j = 0; j < kHK; j += 4) {
        const float4 sc = ksc[j / 4];
        const float2 a = make_float2(static_cast<float>(static_cast<int>(raw[j])), static_cast<float>(static_cast<int>(raw[j + 1])));
        const float2 b = make_float2(static_cast<float>(static_cast<int>(raw[j + 2])), static_cast<float>(static_cast<int>(raw[j + 3])));
        v[j / 2] = __fmul2_rn(a, make_float2(sc.x, sc.y));
        v[j / 2 + 1] = __fmul2_rn(b, make_float2(sc.z, sc.w));
      }
      const float vm = tree_max_p<kHK>(reinterpret_cast<const float*>(v));
      return fmaxf(vm, __shfl_xor_sync(0xFFFFFFFFu, vm, 16));  // the row's other half
    };
    // A starts at the magic (integer zero).
#pragma unroll
    for (int c = 0; c < kHD; c += 32) tmem_fill_h<32, kHD>(tA + c, kMagicP);

    for (int item = cl; item < prm.nitems && ok; item += ncl) {
      const int bh = item / prm.ntiles, tile = item % prm.ntiles;
      const int row = tile * 2 * kRowsP + static_cast<int>(rank) * kRowsP + r;
      const bool row_ok = row < prm.N;
      const float ci = row_ok ? __fmul_rn(prm.sq[static_cast<size_t>(bh) * prm.N + row], prm.inv_sqrt_d) : 0.0f;
      const float cpi = __fmul_rn(ci, kLog2e);
      const float2 cpi2 = make_float2(cpi, cpi);
      const bool dump_tile = DUMP && bh == prm.dump_bh && tile * 2 + static_cast<int>(rank) == prm.dump_tile && row_ok;
#pragma unroll
      for (int c = 0; c < kHD; c += 32) tmem_fill_h32_nw<kHD>(tF + c, 0u);   // F = 0 (waited for before any load of F)
      bool dump_reset = true;   // DUMP: A was reset since the last read-back
      float m_run = -INFINITY, m_ref = 0.0f, w = 1.0f, Lf = 0.0f;
      int Lrun = 0;          // code sum of the row since the last fold (denominator)
      float Lrun_e = 0.0f;   // fp32 sum of exp(S - m) since the last fold (fp32 denominator)
      int Labs = 0;          // code sum of the row since the last reset of A (magnitude bound)
      const uint32_t g0 = g;

      auto dump_s = [&](int t, const uint32_t* raw) __attribute__((always_inline)) {
        if (dump_tile && prm.dump_s) {
          const int nv = min(kBK, prm.N - t * kBK);
          for (int j = 0; j < kHK; ++j)
            if (hh * kHK + j < nv)
              prm.dump_s[static_cast<size_t>(r) * prm.N + t * kBK + hh * kHK + j] = static_cast<int32_t>(raw[j]) / 256;
        }
      };
      // Step for block t: read and release S, scale, maximum, codes, fold.
      auto step = [&](int t) {
        const uint32_t gg = g0 + t;
        float2 v[kHK / 2];
        float vmax;
        {
          uint32_t raw[kHK];
          if (!(ok = take_s(gg, raw))) return;
          if (DUMP) dump_s(t, raw);
          vmax = scale_max(gg, raw, v);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(B.ksc_empty + gg % S);
        const int nvalid = min(kBK, prm.N - t * kBK);
        const float m_blk = __fmul_rn(vmax, ci);
        const float m_new = fmaxf(m_run, m_blk);
        const bool grow = m_new > m_run;
        const float Mp = __fmul_rn(kPMode == 1 ? m_blk : m_new, kLog2e);  // the max the codes use
        const float2 nMp2 = make_float2(-Mp, -Mp);
        // P code c + 8 = rint(15 exp2(y)): adding 15 e to a magic in [2^23, 2^24)
        // with a zero low byte rounds it to an integer in the low byte of the bits.
        uint32_t words[kHK / 4];
        float2 esum = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int q = 0; q < kHK / 4; ++q) {
          const float2 x01 = __ffma2_rn(v[2 * q], cpi2, nMp2);
          const float2 x23 = __ffma2_rn(v[2 * q + 1], cpi2, nMp2);
          float2 e01 = make_float2(ex2_approx(x01.x), ex2_approx(x01.y));
          float2 e23 = make_float2(ex2_approx(x23.x), ex2_approx(x23.y));
          const float2 t01 = __ffma2_rn(kLv2, e01, kMagLo);
          const float2 t23 = __ffma2_rn(kLv2, e23, kMagHi);
          if constexpr (kLf) {
            if (nvalid < kBK) {  // keys past N (NaN scores) do not count
              const int j = hh * kHK + 4 * q;
              e01 = make_float2(j < nvalid ? e01.x : 0.0f, j + 1 < nvalid ? e01.y : 0.0f);
              e23 = make_float2(j + 2 < nvalid ? e23.x : 0.0f, j + 3 < nvalid ? e23.y : 0.0f);
            }
            esum = __fadd2_rn(esum, __fadd2_rn(e01, e23));
          }
          // Integer multiply-adds pack the four low bytes; keys past N give
          // NaN bits, which form a suffix of the word and only carry into
          // higher (also masked) bytes.
          const uint32_t lo = __float_as_uint(t01.y) * 256u + __float_as_uint(t01.x);
          const uint32_t hi = __float_as_uint(t23.y) * 256u + __float_as_uint(t23.x);
          words[q] = hi * 65536u + lo;
        }
        if (nvalid < kBK) {  // last, ragged block: codes of keys past N are 0
#pragma unroll
          for (int q = 0; q < kHK / 4; ++q) {
            const int lim = nvalid - hh * kHK - 4 * q;
            words[q] &= lim >= 4 ? 0xFFFFFFFFu : (lim <= 0 ? 0u : (0xFFFFFFFFu >> (8 * (4 - lim))));
          }
        }
        // P codes of block t over the first 32 columns of its S buffer: word q
        // of half hh (keys 64 hh + 4q .. +3) is column 16 hh + q.
        tmem_st_h16_nw<kHK / 4>(tbase + C::tS + (gg & 1) * 128 + lane_off, words);
        // Sum of the row's codes (+8 each): bytes are at most 15, so plain
        // word additions of 16 words cannot carry between bytes.
        uint32_t ws4[4] = {0u, 0u, 0u, 0u};   // four independent chains
#pragma unroll
        for (int q = 0; q < kHK / 4; ++q) ws4[q & 3] += words[q];
        const uint32_t wsum = (ws4[0] + ws4[1]) + (ws4[2] + ws4[3]);
        int lq = static_cast<int>(__dp4a(wsum, 0x01010101u, 0u));
        lq += __shfl_xor_sync(0xFFFFFFFFu, lq, 16);
        float le = 0.0f;
        if constexpr (kLf) {
          le = esum.x + esum.y;
          le += __shfl_xor_sync(0xFFFFFFFFu, le, 16);
        }
        if (DUMP && dump_tile && prm.dump_p) {
          for (int j = 0; j < kHK; ++j)
            if (hh * kHK + j < nvalid)
              prm.dump_p[static_cast<size_t>(r) * prm.N + t * kBK + hh * kHK + j] =
                  static_cast<int8_t>(((words[j >> 2] >> (8 * (j & 3))) & 0xFF) - kZero);
        }
        // Weight of the coming segment; a rescale moves the reference max.
        float w_new = w, sc = 1.0f;
        if (t == 0) {
          m_ref = m_new;
          w_new = 1.0f;
        } else if (grow) {
          const float x = __fmul_rn(m_new - m_ref, kLog2e);
          if (x > 64.0f) {
            sc = ex2_approx(-x);
            m_ref = m_new;
            w_new = 1.0f;
          } else {
            w_new = ex2_approx(x);
          }
        }
        if constexpr (kPMode == 1) w_new = t == 0 ? 1.0f : ex2_approx(__fmul_rn(m_blk - m_ref, kLog2e));
        const bool change = grow || (kPMode == 1 && w_new != w);
        // Fold when a row's maximum grows (its earlier codes used the old
        // maximum); reset A when its magnitude bound nears the exact range of
        // the read-back (|A| < 2^22).  Every vote is taken by every lane.
        const bool near_bound = (Labs + 15 * kBK) * 112 >= (1 << 22) - 4096;
        const bool reset = __any_sync(0xFFFFFFFFu, (t > 0) && near_bound);
        const bool any_change = __any_sync(0xFFFFFFFFu, (t > 0) && change);
        // Tensor-memory accesses are warp-collective: a rescale of one row's F
        // is done by the whole warp (sc = 1 for the other rows).
        const bool any_rescale = __any_sync(0xFFFFFFFFu, sc != 1.0f);
        bool dump_now = false;
        if constexpr (DUMP) {
          const bool any_dump = __any_sync(0xFFFFFFFFu, dump_tile);
          dump_now = any_dump && t > 0;
        }
        if (reset || any_change || dump_now) {
          // A holds the P.V results up to block t - 1.
          if (!(ok = pwait_warp(B.pv_done + ((gg - 1) & 1), ((gg - 1) >> 1) & 1, ab, 16u, gg, rank, 16u))) return;
          tc_fence_after();
          if (DUMP && dump_now) {
            dump_acc(t - 1, r, dump_reset, dump_tile);
            dump_reset = false;
          }
        }
        if (reset || any_change) {
          if (any_rescale) {  // new reference maximum of some row: rescale F and the denominator
            tmem_wait_st();
#pragma unroll
            for (int c = 0; c < kHD; c += 32) {
              uint32_t f[32];
              tmem_ld_h<32, kHD>(tF + c, f);
#pragma unroll
              for (int i = 0; i < 32; ++i) f[i] = __float_as_uint(__uint_as_float(f[i]) * sc);
              tmem_st_h32_nw<kHD>(tF + c, f);
            }
            tmem_wait_st();
            Lf *= sc;
            w *= sc;
          }
          fold(reset ? w : w - w_new, reset);
          Lf = fmaf(w, kLf ? Lrun_e : static_cast<float>(Lrun), Lf);
          Lrun = 0;
          Lrun_e = 0.0f;
          if (reset) {
            Labs = 0;
            dump_reset = true;
          }
        }
        w = w_new;
        Labs += lq;
        Lrun += lq;
        Lrun_e += le;
        m_run = m_new;
        tmem_wait_st();   // the P codes (and any fold's stores) are in tensor memory
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(p_full_l[gg & 1]);
      };

      for (int t = 0; t < nb && ok; ++t) step(t);
      g = g0 + nb;
      if (!ok) break;
      // Last block: fold the accumulator into F (and reset it), normalise, store.
      if (!(ok = pwait_warp(B.pv_done + ((g - 1) & 1), ((g - 1) >> 1) & 1, ab, 17u, g, rank, 16u))) break;
      tc_fence_after();
      if constexpr (DUMP) {
        const bool any_dump = __any_sync(0xFFFFFFFFu, dump_tile);
        if (any_dump) dump_acc(nb - 1, r, dump_reset, dump_tile);
      }
      Lf = fmaf(w, kLf ? Lrun_e : static_cast<float>(Lrun), Lf);
      const float inv = 1.0f / (kLf ? 16.0f * kLevels * Lf : 16.0f * Lf);
      const float* sv = prm.sv + static_cast<size_t>(bh) * D;
      __nv_bfloat16* orow = prm.out + (static_cast<size_t>(bh) * prm.N + (row_ok ? row : 0)) * D;
      const float2 w2 = make_float2(w, w);
#pragma unroll
      for (int c = 0; c < kHD; c += 32) {
        uint32_t a[32], f[32];
        tmem_ld_h32_pair<kHD>(tA + c, tF + c, a, f);
        float fo[32];
#pragma unroll
        for (int q = 0; q < 32; q += 2) {
          const float2 x = __fadd2_rn(make_float2(__uint_as_float(a[q]), __uint_as_float(a[q + 1])), kNegMagic2);
          const float2 y = __ffma2_rn(w2, x, make_float2(__uint_as_float(f[q]), __uint_as_float(f[q + 1])));
          fo[q] = y.x;
          fo[q + 1] = y.y;
        }
        tmem_fill_h32_nw<kHD>(tA + c, kMagicP);
        if (row_ok) {
          // Widened positions hh * D/2 + c + (4a + b) and + 16 hold channels
          // d = hh * D/2 + c + 8a + 2b and d + 1.
          const int c0 = hh * kHD + c;
          uint32_t pk[16];
#pragma unroll
          for (int a4 = 0; a4 < 4; ++a4)
#pragma unroll
            for (int b4 = 0; b4 < 4; ++b4) {
              const int d = c0 + 8 * a4 + 2 * b4;
              const __nv_bfloat162 h2 = __floats2bfloat162_rn(fo[4 * a4 + b4] * __ldg(sv + d) * inv,
                                                              fo[16 + 4 * a4 + b4] * __ldg(sv + d + 1) * inv);
              pk[4 * a4 + b4] = *reinterpret_cast<const uint32_t*>(&h2);
            }
          uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
          for (int u = 0; u < 4; ++u) dst[u] = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
        }
      }
      if (row_ok && prm.lse && hh == 0)
        prm.lse[static_cast<size_t>(bh) * prm.N + row] = m_ref + logf(kLf ? Lf : Lf * (1.0f / kLevels));
    }
  }
  // Both CTAs finish every access to each other's shared and tensor memory
  // (remote arrivals, pair MMAs) before either frees its tensor memory or exits.
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tbase, 512);
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 get_encoder_p() {
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

// 3D map over packed codes [BH, N, D/2] bytes; box = box_x bytes x rows; zero fill past N.
bool make_code_map_p(CUtensorMap* m, const void* base, int BH, int N, int D, int box_x, int rows) {
  auto enc = get_encoder_p();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D / 2), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D / 2), static_cast<cuuint64_t>(N) * (D / 2)};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box_x), static_cast<cuuint32_t>(rows), 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, bool DUMP, int MODE>
cudaError_t launch_pair_cfg(const ra_problem& p, const uint8_t* q4, const uint8_t* k4, const uint8_t* v4,
                            const PairParams& prm, cudaStream_t st) {
  using C = PairCfg<D, DUMP>;
  CUtensorMap mq, mk, mv;
  const int BH = p.B * p.H;
  if (!make_code_map_p(&mq, q4, BH, p.N, D, D / 2, kRowsP) ||
      !make_code_map_p(&mk, k4, BH, p.N, D, D / 2, C::kKRows) ||
      !make_code_map_p(&mv, v4, BH, p.N, D, D / 4, kBK))
    return cudaErrorInvalidValue;
  auto kern = attn_int4_pair_kernel<D, DUMP, MODE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  static int max_clusters = 0;
  if (max_clusters == 0) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2);
    cfg.blockDim = dim3(kThreadsP);
    cfg.dynamicSmemBytes = C::kSmem;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) {
      cudaGetLastError();
      int dev = 0, nsm = 0;
      cudaGetDevice(&dev);
      cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
      n = nsm / 2;
    }
    max_clusters = n;
  }
  const int clusters = prm.nitems < max_clusters ? prm.nitems : max_clusters;
  kern<<<2 * clusters, kThreadsP, C::kSmem, st>>>(mq, mk, mv, prm);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_int4_pair(const ra_problem& p, const uint8_t* q4, const float* sq, const uint8_t* k4,
                                  const float* sk, const uint8_t* v4, const float* sv, void* out, float* lse,
                                  const AttnDump* dump, int mode, cudaStream_t st, int* unsupported) {
  PairParams prm{};
  prm.N = p.N;
  prm.BH = p.B * p.H;
  prm.nblocks = (p.N + kBK - 1) / kBK;
  prm.ntiles = (p.N + 2 * kRowsP - 1) / (2 * kRowsP);
  prm.nitems = prm.BH * prm.ntiles;
  prm.inv_sqrt_d = static_cast<float>(1.0 / sqrt(static_cast<double>(p.D)));
  prm.sq = sq; prm.sk = sk; prm.sv = sv;
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.lse = lse;
  prm.dump_bh = -1;
  prm.dump_tile = -1;
  const bool dmp = dump != nullptr;
  if (dmp) {
    prm.dump_bh = dump->bh; prm.dump_tile = dump->q_tile;
    prm.dump_s = dump->s; prm.dump_p = dump->p; prm.dump_acc = dump->acc;
  }
  *unsupported = 0;
  if (p.block_k != kBK) {
    *unsupported = 1;
    return cudaSuccess;
  }
#define RA_PCASE(DD, MM)                                                                    \
  if (p.D == DD && mode == MM)                                                              \
    return dmp ? launch_pair_cfg<DD, true, MM>(p, q4, k4, v4, prm, st)                      \
               : launch_pair_cfg<DD, false, MM>(p, q4, k4, v4, prm, st);
  RA_PCASE(128, 0)
  RA_PCASE(64, 0)
  RA_PCASE(128, 1)
  RA_PCASE(128, 2)
  RA_PCASE(128, 4)
  RA_PCASE(128, 5)
  RA_PCASE(128, 6)
  RA_PCASE(64, 1)
  RA_PCASE(64, 2)
  RA_PCASE(64, 4)
  RA_PCASE(64, 5)
  RA_PCASE(64, 6)
#undef RA_PCASE
  *unsupported = 1;
  return cudaSuccess;
}

cudaError_t read_attn_pair_status(uint32_t* out) {
  uint32_t zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(out, g_pair_status, sizeof(uint32_t));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_pair_status, &zero, sizeof(uint32_t));
}

cudaError_t read_attn_pair_diag(uint32_t* out) {
  uint32_t zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(out, g_pair_diag, sizeof(uint32_t));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_pair_diag, &zero, sizeof(uint32_t));
}

}  // namespace ra
