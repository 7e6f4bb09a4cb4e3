// INT4 attention forward of RotateAttention on sm_100a (tcgen05 kind::i8).
//
// Method (papernotes page, flowchart D-F and key design 2):
//   S_ij = (S_int_ij * s_k[j]) * (s_q[i] / sqrt(D)),  S_int = sum_d q4 k4 (exact)
//   online softmax over key blocks of block_k keys with the running row max m
//   P codes c_ij = clamp(rint(15 exp(S_ij - m)), 0, 15) - 8
//   acc_t = sum_j (c_ij + 8) v4_jd  (= sum_j c_ij v4_jd + 8 colsum_t: the
//           zero-point correction folded into the integer accumulator)
//   O = sum_t alpha-chain (s_v/15) acc_t / sum_t alpha-chain sum_j (c_ij+8)/15
//   Ablation modes (the alternatives key design 2 is compared with): codes
//   against each block's own maximum, weighted exp(m_block - m) (LOCAL);
//   SageAttention-style codes rint(7 exp(S - m)) in [0, 7], no zero point
//   (SYMMETRIC); the denominator as the fp32 sum of exp(S - m) (FP32 l).
//
// B200 design:
//   * No 4-bit integer MMA exists on sm_100a; packed nibbles are widened to s8
//     in shared memory (as 16 x code: the high nibble in place, the low nibble
//     shifted up), which scales S_int by 256 and acc by 16, both exact powers
//     of two folded into the fp32 scales.  The widened K dimension of Q and K
//     follows the same channel permutation, which leaves S_int unchanged.
//   * QK^T: tcgen05.mma kind::i8, A = Q (smem), B = K (smem), D = S (s32, TMEM).
//   * P codes are produced as unsigned bytes c + 8 in [0, 15] and stored into
//     TMEM over the S columns they came from; P.V is a TMEM-A kind::i8 MMA
//     (A u8, B s8, V MN-major), so the accumulator is sum_j (c_ij + 8) v_jd.
//   * The s32 P.V accumulator stays in TMEM across key blocks and is folded
//     into the fp32 output (registers) only when the running maximum of a row
//     of the warp grows, or when its magnitude bound requires it.  The
//     accumulator is pre-loaded with the bits of 1.5 * 2^23 so that it reads
//     back as a float with one subtraction.
//   * Two 128-row query tiles per CTA share every K/V tile; warp roles:
//     TMA producer, two MMA issuers, four widening warps and 16 softmax warps
//     (two threads per query row, each with half of the keys of a block and
//     half of the output columns).  Persistent CTAs, one per SM.
//   * Variants (MODE bits): the ablation switches; fused Q (warp 3 produces
//     each item's packed Q from the raw Q); the byte code layout (Q, K as FP8
//     E4M3 codes and V as 16 x code, TMA'd straight into the operand tiles, an
//     FP8 Q K^T with an exact fp32 S, no widening).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "ra_common.cuh"
#include "ra_internal.h"
#include "ra_rope.cuh"

namespace ra {
namespace {

__device__ uint32_t g_attn_status = 0;
// First timed-out wait: (site << 24) | (block counter & 0xFFFF) << 8 | (cta & 0xFF).
__device__ uint32_t g_attn_diag = 0;

constexpr int kThreads = 768;   // 24 warps: see the role map in the kernel
constexpr int kRows = 128;          // query rows per tile = MMA M
constexpr int kTiles = 2;           // query tiles per CTA
constexpr uint32_t kMagic = 0x4B400000u;  // bits of 1.5 * 2^23
constexpr float kMagicF = 12582912.0f;

template <int D, int BN>
struct Cfg {
  static constexpr int kPackRow = D / 2;                // packed bytes per row
  static constexpr int kKeysPV = BN < 32 ? 32 : BN;     // P.V MMA K extent
  static constexpr int kPS = 4, kKS = 4, kVS = 4;       // pipeline stages
  static constexpr int kQBytes = kRows * D;             // one widened Q tile
  static constexpr int kQPkBytes = kRows * kPackRow;
  static constexpr int kKwBytes = BN * D;
  static constexpr int kVwBytes = kKeysPV * D;
  static constexpr int kPkHalf = BN * kPackRow;         // packed K (or V) of one block
  // shared-memory map (bytes from a 1024-aligned base)
  static constexpr int oQ = 0;
  static constexpr int oQPk = oQ + kTiles * kQBytes;
  static constexpr int oKw = oQPk + kTiles * kQPkBytes;
  static constexpr int oVw = oKw + kKS * ((kKwBytes + 1023) / 1024) * 1024;
  static constexpr int oPk = oVw + kVS * ((kVwBytes + 1023) / 1024) * 1024;
  static constexpr int oKsc = oPk + kPS * 2 * kPkHalf;
  // Half of every softmax thread's fp32 output accumulator columns live in
  // shared memory (the other half in registers); padded against bank conflicts.
  static constexpr int kFRow = D / 4 + 4;                 // floats per thread (padded)
  static constexpr int oF = oKsc + kKS * BN * 4;
  static constexpr int oBar = oF + kTiles * 2 * kRows * kFRow * 4;
  static constexpr int kNumBars = 4 + 2 * kPS + 2 * kKS + 2 * kVS + 4 + 4 + 4 + 2 + 4;
  static constexpr int oMisc = oBar + kNumBars * 8;
  // Fused-Q path: the Q warp's half-rotation row exchange (32 / (D/8) token
  // rows of D floats = 1 KB) and a ring of two items' per-row Q scales.
  static constexpr int oQx = oMisc + 64;
  static constexpr int oSq = oQx + 1024;
  static constexpr int kSmem = oSq + 2 * kTiles * kRows * 4 + 1024;   // + alignment slack
  static constexpr int kKwStride = ((kKwBytes + 1023) / 1024) * 1024;
  static constexpr int kVwStride = ((kVwBytes + 1023) / 1024) * 1024;
  static constexpr uint32_t kSwz = D == 128 ? kSwizzle128B : kSwizzle64B;
  static constexpr uint32_t kIdescQK = instr_desc(kCfmtS32, 1, 1, 0, 0, kRows, BN);
  // byte layout: Q and K hold FP8 E4M3 codes, S accumulates in fp32 (exact:
  // |S_int| <= 49 D < 2^13)
  static constexpr uint32_t kIdescQKf8 = instr_desc(kCfmtF32, 0, 0, 0, 0, kRows, BN);
  static constexpr uint32_t kIdescPV = instr_desc(kCfmtS32, 0, 1, 0, 1, kRows, D);
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(BN == 16 || BN == 32 || BN == 64, "block_k");
};

struct Bars {
  uint64_t* qpk_full; uint64_t* qpk_empty; uint64_t* q_full; uint64_t* q_free;
  uint64_t* pk_full; uint64_t* pk_empty;
  uint64_t* kw_full; uint64_t* kw_empty;
  uint64_t* vw_full; uint64_t* vw_empty;
  uint64_t* s_full;   // [tile][buf]
  uint64_t* p_full;   // [tile][buf]
  uint64_t* pv_done;  // [tile][buf]: P.V of the blocks whose P sits in S buffer buf
  uint64_t* drain;    // [issuer]
  uint64_t* sq_full;  // [slot] fused Q: an item's per-row Q scales are in shared memory
  uint64_t* sq_empty; // [slot] fused Q: every softmax warp has read them
};

struct AttnParams {
  int N, BH, nblocks, npairs, nitems;
  float inv_sqrt_d;
  const float* sq;
  const float* sk;
  const float* sv;
  __nv_bfloat16* out;
  float* lse;
  // dump variant
  int dump_bh, dump_tile;
  int32_t* dump_s;
  int8_t* dump_p;
  int32_t* dump_acc;
  // fused-Q variant: raw Q [BH, N, D] (bf16 or fp32), positions, RoPE table
  const void* qraw;
  int qdtype, rot;
  const int32_t* pos;
  const float2* tab;
  SegInfo seg;
};

// Widens one 16-byte chunk of packed codes (32 channels) into two 16-byte
// chunks of s8 holding 16 x code: low nibbles first, then high nibbles.
__device__ __forceinline__ void widen_chunk(const uint8_t* src, uint8_t* dst_lo, uint8_t* dst_hi) {
  const uint4 w = *reinterpret_cast<const uint4*>(src);
  uint4 lo, hi;
  lo.x = (w.x << 4) & 0xF0F0F0F0u; hi.x = w.x & 0xF0F0F0F0u;
  lo.y = (w.y << 4) & 0xF0F0F0F0u; hi.y = w.y & 0xF0F0F0F0u;
  lo.z = (w.z << 4) & 0xF0F0F0F0u; hi.z = w.z & 0xF0F0F0F0u;
  lo.w = (w.w << 4) & 0xF0F0F0F0u; hi.w = w.w & 0xF0F0F0F0u;
  *reinterpret_cast<uint4*>(dst_lo) = lo;
  *reinterpret_cast<uint4*>(dst_hi) = hi;
}

// Widens `rows` packed rows (D/2 bytes each, linear) into a swizzled tile of
// D-byte rows; threads [tid0, tid0 + nthr) share the work.
template <int D>
__device__ __forceinline__ void widen_tile(const uint8_t* pk, uint8_t* wide, int rows, int tid, int nthr) {
  constexpr int kPc = D / 32;  // packed 16-byte chunks per row
  for (int idx = tid; idx < rows * kPc; idx += nthr) {
    const int r = idx / kPc, pc = idx % kPc;
    widen_chunk(pk + r * (D / 2) + pc * 16, wide + swz_offset(r, 2 * pc, D), wide + swz_offset(r, 2 * pc + 1, D));
  }
}

// Per-thread chunk offsets of widen_tile for a fixed tile height, computed
// once: every K/V block has the same layout, so the widening warps only load,
// widen and store in their loop.
template <int D, int ROWS>
struct WidenPlan {
  static constexpr int kChunks = ROWS * (D / 32);
  static constexpr int kIter = (kChunks + 127) / 128;
  uint32_t src[kIter], lo[kIter], hi[kIter];
  __device__ __forceinline__ void init(int tid) {
#pragma unroll
    for (int k = 0; k < kIter; ++k) {
      const int idx = tid + 128 * k;
      const int r = idx / (D / 32), pc = idx % (D / 32);
      src[k] = idx < kChunks ? static_cast<uint32_t>(r * (D / 2) + pc * 16) : ~0u;
      lo[k] = swz_offset(r, 2 * pc, D);
      hi[k] = swz_offset(r, 2 * pc + 1, D);
    }
  }
  __device__ __forceinline__ void run(const uint8_t* pk, uint8_t* wide) const {
#pragma unroll
    for (int k = 0; k < kIter; ++k)
      if (kChunks % 128 == 0 || src[k] != ~0u) widen_chunk(pk + src[k], wide + lo[k], wide + hi[k]);
  }
};

// Widened position n (0..D-1) of a row -> channel.
__host__ __device__ constexpr int wide_to_dim(int n) {
  return (n & ~31) + 8 * ((n & 15) >> 2) + 2 * (n & 3) + ((n >> 4) & 1);
}

__device__ __forceinline__ float max3(float a, float b, float c) { return fmaxf(a, fmaxf(b, c)); }

// Maximum of n values as a tree of 3-way maxima (short dependency chains).
template <int n>
__device__ __forceinline__ float tree_max(const float* x) {
  if constexpr (n == 1) return x[0];
  else if constexpr (n == 2) return fmaxf(x[0], x[1]);
  else if constexpr (n == 3) return max3(x[0], x[1], x[2]);
  else return max3(tree_max<n / 3>(x), tree_max<n / 3>(x + n / 3), tree_max<n - 2 * (n / 3)>(x + 2 * (n / 3)));
}

__device__ __forceinline__ void set_status(uint32_t bits) { atomicOr(&g_attn_status, bits); }

// Fused Q of one item (query tiles 2 pair and 2 pair + 1 of head bh), by one
// warp: the prologue's per-token arithmetic (RoPE, rotation, amax, 7/amax, one
// f32x2 FMA per code pair and the nibble packing, shared through ra_rope.cuh,
// so the codes and scales are bit-identical to ra_rope_rotate_quant's),
// written as packed rows into the packed-Q staging tiles (the layout the TMA
// would load) and the per-row scales amax/7 into sqs[tile * 128 + row].  D/8
// lanes per row, two rows per lane in flight; rows past N get codes 0 and
// scale 0.  Every lane runs every pass (the shuffles and the half rotation's
// warp synchronisation are unconditional).
template <int D>
__device__ __forceinline__ void fused_q_pack(const AttnParams& prm, uint8_t* qpk, float* rows, float* sqs, int bh,
                                             int pair, int lane) {
  constexpr int lpt = D / 8;        // lanes per row
  constexpr int rpp = 32 / lpt;     // rows per pass
  const int tok = lane / lpt, c0 = (lane % lpt) * 8;
  float* const row = rows + tok * D;   // this row's exchange slot
  RopePlan rp;
  rp.init(prm.seg, c0);
  const size_t head = static_cast<size_t>(bh) * prm.N * D;
#pragma unroll 2
  for (int base = 0; base < kTiles * kRows; base += rpp) {
    const int rr = base + tok;
    const int tt = rr / kRows, r = rr % kRows;
    const int n = (pair * kTiles + tt) * kRows + r;
    const bool valid = n < prm.N;
    float x[8];
    int gp[3] = {0, 0, 0};
    if (valid) {
      load8(prm.qraw, head + static_cast<size_t>(n) * D + c0, prm.qdtype, x);
#pragma unroll
      for (int j = 0; j < 3; ++j) gp[j] = __ldg(prm.pos + 3 * n + j);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) x[i] = 0.0f;
    }
    float2 cf[4];
    rope_coef8p(prm.seg, rp, prm.tab, gp, cf, &g_attn_status);
    rope_apply8(prm.seg, rp, prm.rot, cf, c0, x, row);
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(x[i]));
    m = group_max(m, lpt);
    const float inv = m == 0.0f ? 0.0f : __fdiv_rn(7.0f, m);
    uint32_t b[8];
#pragma unroll
    for (int i = 0; i < 8; i += 2) quant4_bits2(x[i], x[i + 1], inv, inv, b + i);
    *reinterpret_cast<uint32_t*>(qpk + tt * (kRows * D / 2) + r * (D / 2) + (c0 >> 1)) = pack8_bits(b);
    if (c0 == 0) sqs[rr] = valid ? __fdiv_rn(m, 7.0f) : 0.0f;
  }
}

// Records the first wait that gave up (site id, block counter, CTA) for diagnosis.
__device__ __forceinline__ void note_timeout(uint32_t site, uint32_t g) {
  atomicCAS(&g_attn_diag, 0u, (site << 24) | ((g & 0xFFFFu) << 8) | (blockIdx.x & 0xFFu));
}

__device__ __forceinline__ bool wait_at(uint64_t* bar, uint32_t parity, volatile int* abort, uint32_t site,
                                        uint32_t g, uint32_t backoff_ns = 16) {
  const int r = mbar_wait_ex(bar, parity, abort, backoff_ns);
  if (r < 0) note_timeout(site, g);
  return r > 0;
}

// MODE bits 0-1: P codes (0 range-rectified, 1 block-local maximum, 2
// symmetric); bit 2: fp32 denominator; bit 3: fused Q (warp 3 computes Q's
// packed codes and scales from the raw Q in place of the TMA load of q4);
// bit 4: byte code layout (one code per byte, natural channel order; Q and K
// as FP8 E4M3 codes, V as 16 x code in s8): the TMA loads Q, K and V straight
// into the MMA operand tiles, Q K^T runs as kind::f8f6f4 with an fp32 S (no
// integer conversion in the softmax), and warps 4-7 only stage the per-key
// scales.
template <int D, int BN, bool DUMP, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
attn_int4_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const AttnParams prm) {
  using C = Cfg<D, BN>;
  constexpr bool kFQ = (MODE & 8) != 0;
  constexpr bool kS8 = (MODE & 16) != 0;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base; pointer arithmetic on the shared array keeps the
  // shared address space visible to the compiler (LDS/STS, not generic LD/ST).
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::oBar);
  Bars B;
  {
    uint64_t* b = bar;
    B.qpk_full = b++; B.qpk_empty = b++; B.q_full = b++; B.q_free = b++;
    B.pk_full = b; b += C::kPS; B.pk_empty = b; b += C::kPS;
    B.kw_full = b; b += C::kKS; B.kw_empty = b; b += C::kKS;
    B.vw_full = b; b += C::kVS; B.vw_empty = b; b += C::kVS;
    B.s_full = b; b += 4; B.p_full = b; b += 4; B.pv_done = b; b += 4; B.drain = b; b += 2;
    B.sq_full = b; b += 2; B.sq_empty = b; b += 2;
  }
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::oMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::oMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    // s8 layout: the TMA fills Q, K and V tiles (one expect-tx arrival each);
    // a K stage also waits for the four scale warps.
    mbar_init(B.qpk_full, 1); mbar_init(B.qpk_empty, 4); mbar_init(B.q_full, kS8 ? 1 : 4); mbar_init(B.q_free, 2);
    for (int s = 0; s < C::kPS; ++s) { mbar_init(B.pk_full + s, 1); mbar_init(B.pk_empty + s, 4); }
    for (int s = 0; s < C::kKS; ++s) { mbar_init(B.kw_full + s, kS8 ? 1 + 4 : 4); mbar_init(B.kw_empty + s, 2 + 16); }
    for (int s = 0; s < C::kVS; ++s) { mbar_init(B.vw_full + s, kS8 ? 1 : 4); mbar_init(B.vw_empty + s, 2); }
    for (int s = 0; s < 4; ++s) { mbar_init(B.s_full + s, 1); mbar_init(B.p_full + s, 8); mbar_init(B.pv_done + s, 1); }
    mbar_init(B.drain, 1);
    mbar_init(B.drain + 1, 1);
    for (int s = 0; s < 2; ++s) { mbar_init(B.sq_full + s, 1); mbar_init(B.sq_empty + s, 16); }
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
  // Roles: warp 0 TMA producer, warp 1 MMA issuer of tile 0 and TMEM owner,
  // warp 2 MMA issuer of tile 1, warp 3 idle, warps 4-7 widen codes (one per
  // SM sub-partition), warps 8-15 and 16-23 softmax of query tiles 0 and 1
  // (two threads per row, 16 rows per warp).
  if (warp < 8) {
    if (warp < 4) asm volatile("setmaxnreg.dec.sync.aligned.u32 56;");
    else asm volatile("setmaxnreg.dec.sync.aligned.u32 40;");
    if (warp == 0) {
      // ------------------------------------------------------------ TMA producer
      if (kS8 && lane == 0) {
        // s8 layout: K and V of each block into their operand stages, and the
        // item's Q tiles after its first block (once the previous item's QK
        // products have been issued).
        uint32_t g = 0, li = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < prm.nitems && ok; item += gridDim.x, ++li) {
          const int bh = item / prm.npairs, pair = item % prm.npairs;
          for (int t = 0; t < nb; ++t, ++g) {
            const int ks = g % C::kKS, vs = g % C::kVS;
            if (!(ok = wait_at(B.kw_empty + ks, ((g / C::kKS) & 1) ^ 1, abort_flag, 14u, g, 256u))) break;
            mbar_arrive_expect_tx(B.kw_full + ks, C::kKwBytes);
            tma_load_3d(smem + C::oKw + ks * C::kKwStride, &tm_k, B.kw_full + ks, 0, t * BN, bh);
            if (!(ok = wait_at(B.vw_empty + vs, ((g / C::kVS) & 1) ^ 1, abort_flag, 16u, g, 256u))) break;
            mbar_arrive_expect_tx(B.vw_full + vs, C::kVwBytes);
            tma_load_3d(smem + C::oVw + vs * C::kVwStride, &tm_v, B.vw_full + vs, 0, t * BN, bh);
            if (t == 0) {
              if (!(ok = wait_at(B.q_free, (li & 1) ^ 1, abort_flag, 1u, li, 256u))) break;
              mbar_arrive_expect_tx(B.q_full, kTiles * C::kQBytes);
              for (int tt = 0; tt < kTiles; ++tt)
                tma_load_3d(smem + C::oQ + tt * C::kQBytes, &tm_q, B.q_full, 0, pair * 2 * kRows + tt * kRows, bh);
            }
          }
        }
        // Wait (bounded) for the copies of the last stages to land.
        for (uint32_t k = (g > (uint32_t)C::kKS ? g - C::kKS : 0); k < g; ++k) {
          uint32_t it = 0;
          while (!mbar_try_wait(B.vw_full + (k % C::kVS), (k / C::kVS) & 1) && ++it < kSpinLimit) {}
        }
        if (!ok) set_status(kStatusTimeout);
      } else if (!kS8 && lane == 0) {
        uint32_t g = 0, li = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < prm.nitems && ok; item += gridDim.x, ++li) {
          const int bh = item / prm.npairs, pair = item % prm.npairs;
          if constexpr (!kFQ) {
            ok = wait_at(B.qpk_empty, (li & 1) ^ 1, abort_flag, 1u, li, 256u);
            if (!ok) break;
            mbar_arrive_expect_tx(B.qpk_full, kTiles * C::kQPkBytes);
            for (int tt = 0; tt < kTiles; ++tt)
              tma_load_3d(smem + C::oQPk + tt * C::kQPkBytes, &tm_q, B.qpk_full, 0, pair * 2 * kRows + tt * kRows, bh);
          }
          for (int t = 0; t < nb; ++t, ++g) {
            const int s = g % C::kPS;
            ok = wait_at(B.pk_empty + s, ((g / C::kPS) & 1) ^ 1, abort_flag, 14u, g, 256u);
            if (!ok) break;
            mbar_arrive_expect_tx(B.pk_full + s, 2 * C::kPkHalf);
            uint8_t* dst = smem + C::oPk + s * 2 * C::kPkHalf;
            tma_load_3d(dst, &tm_k, B.pk_full + s, 0, t * BN, bh);
            tma_load_3d(dst + C::kPkHalf, &tm_v, B.pk_full + s, 0, t * BN, bh);
          }
        }
        // Wait (bounded) for the copies of the last stages to land.
        for (uint32_t k = (g > (uint32_t)C::kPS ? g - C::kPS : 0); k < g; ++k) {
          uint64_t* fb = B.pk_full + (k % C::kPS);
          uint32_t it = 0;
          while (!mbar_try_wait(fb, (k / C::kPS) & 1) && ++it < kSpinLimit) {}
        }
        if (!ok) set_status(kStatusTimeout);
      }
    } else if (warp == 1 || warp == 2) {
      // ------------------------------------------------------------ MMA issuers
      // One issuing thread per query tile, so each tile's pipeline advances at
      // its own pace (within the shared K/V stage window).  Per tile: P.V(g),
      // then QK(g+2) into the S buffer whose P codes P.V(g) has just read.
      if (lane == 0) {
        const int tt = warp - 1;
        const uint32_t sQ = smem_u32(smem + C::oQ) + tt * C::kQBytes;
        const uint32_t sKw = smem_u32(smem + C::oKw);
        const uint32_t sVw = smem_u32(smem + C::oVw);
        const uint32_t tS0 = tbase + tt * 256;
        const uint32_t tA = tS0 + 128;
        uint32_t li = 0, g0 = 0;
        bool ok = true;
        // QK(gq) into S buffer gq & 1; before that, P.V(gq - 2) (which reads the
        // P codes stored in that buffer) must have completed.  pv_done has one
        // barrier per S buffer, so P.V(gq - 4), the previous completion on it,
        // is done and the awaited phase is the barrier's current one.
        auto issue_qk = [&](uint32_t gq, bool last_of_item) -> bool {
          const uint32_t buf = gq & 1;
          if (gq >= 2) {
            if (!wait_at(B.pv_done + tt * 2 + buf, ((gq - 2) >> 1) & 1, abort_flag, 6u, gq, 32u)) return false;
          }
          const int ks = gq % C::kKS;
          if (!wait_at(B.kw_full + ks, (gq / C::kKS) & 1, abort_flag, 5u, gq, 32u)) return false;
          tc_fence_after();
          const uint32_t tS = tS0 + buf * 64;
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk) {
            const uint64_t adesc = smem_desc(sQ + kk * 32, 16, 8 * D, C::kSwz);
            const uint64_t bdesc = smem_desc(sKw + ks * C::kKwStride + kk * 32, 16, 8 * D, C::kSwz);
            if constexpr (kS8) mma_f8_ss(tS, adesc, bdesc, C::kIdescQKf8, kk > 0 ? 1u : 0u);
            else mma_i8_ss(tS, adesc, bdesc, C::kIdescQK, kk > 0 ? 1u : 0u);
          }
          mma_commit(B.s_full + tt * 2 + buf);
          mma_commit(B.kw_empty + ks);
          if (last_of_item) mma_commit(B.q_free);
          return true;
        };
        for (int item = blockIdx.x; item < prm.nitems && ok; item += gridDim.x, ++li, g0 += nb) {
          if (!(ok = wait_at(B.q_full, li & 1, abort_flag, 4u, li, 32u))) break;
          tc_fence_after();
          for (int t = 0; t < 2 && t < nb && ok; ++t) ok = issue_qk(g0 + t, t == nb - 1);
          for (int t = 0; t < nb && ok; ++t) {
            const uint32_t gg = g0 + t;
            const int vs = gg % C::kVS;
            const uint32_t buf = gg & 1;
            if (!(ok = wait_at(B.vw_full + vs, (gg / C::kVS) & 1, abort_flag, 2u, gg, 32u))) break;
            if (!(ok = wait_at(B.p_full + tt * 2 + buf, (gg >> 1) & 1, abort_flag, 3u, gg, 32u))) break;
            tc_fence_after();
            const uint32_t tP = tS0 + buf * 64;
#pragma unroll
            for (int kk = 0; kk < C::kKeysPV / 32; ++kk) {
              const uint64_t bdesc = smem_desc(sVw + vs * C::kVwStride + kk * 32 * D, 8 * D * (C::kKeysPV / 8),
                                               8 * D, C::kSwz);
              mma_i8_ts(tA, tP + kk * 8, bdesc, C::kIdescPV, 1);
            }
            mma_commit(B.pv_done + tt * 2 + buf);
            mma_commit(B.vw_empty + vs);
            if (t + 2 < nb) ok = issue_qk(gg + 2, t + 2 == nb - 1);
          }
        }
        // Drain: every MMA issued by this thread has completed before TMEM is released.
        mma_commit(B.drain + tt);
        uint32_t it = 0;
        while (!mbar_try_wait(B.drain + tt, 0) && ++it < kSpinLimit) {}
        if (!ok) set_status(kStatusTimeout);
      }
    } else if (warp == 3) {
      // ------------------------------------------------------------ fused-Q warp
      // Produces each item's packed Q (in place of the TMA load) and its
      // per-row scales, as soon as the widening warps have consumed the
      // previous item's packed Q: a whole item of slack.
      if constexpr (kFQ) {
        uint32_t li = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < prm.nitems && ok; item += gridDim.x, ++li) {
          const uint32_t slot = li & 1;
          if (!(ok = wait_at(B.qpk_empty, (li & 1) ^ 1, abort_flag, 22u, li, 256u))) break;
          if (!(ok = wait_at(B.sq_empty + slot, ((li >> 1) & 1) ^ 1, abort_flag, 20u, li, 256u))) break;
          fused_q_pack<D>(prm, smem + C::oQPk, reinterpret_cast<float*>(smem + C::oQx),
                          reinterpret_cast<float*>(smem + C::oSq) + slot * kTiles * kRows, item / prm.npairs,
                          item % prm.npairs, lane);
          __syncwarp();
          if (lane == 0) { mbar_arrive(B.qpk_full); mbar_arrive(B.sq_full + slot); }
        }
        if (!ok) set_status(kStatusTimeout);
      }
    } else if (warp >= 4 && kS8) {
      // ------------------------------------------------------------ scale warps (s8 layout)
      // The TMA fills the operand tiles; these warps only stage each block's
      // per-key scales (the K stage's barrier waits for them too).
      const int wt = threadIdx.x - 128;  // 0..127
      uint32_t g = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < prm.nitems && ok; item += gridDim.x) {
        const int bh = item / prm.npairs;
        for (int t = 0; t < nb; ++t, ++g) {
          const int ks = g % C::kKS;
          if (!(ok = wait_at(B.kw_empty + ks, ((g / C::kKS) & 1) ^ 1, abort_flag, 15u, g, 256u))) break;
          if (wt < BN) {
            const int j = t * BN + wt;
            float* ksc = reinterpret_cast<float*>(smem + C::oKsc) + ks * BN;
            ksc[wt] = j < prm.N ? prm.sk[static_cast<size_t>(bh) * prm.N + j] : __int_as_float(0x7FC00000);
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(B.kw_full + ks);
        }
      }
      if (!ok) set_status(kStatusTimeout);
    } else if (warp >= 4) {
      // ------------------------------------------------------------ widening warps
      const int wt = threadIdx.x - 128;  // 0..127
      WidenPlan<D, BN> plan;
      plan.init(wt);
      uint32_t g = 0, li = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < prm.nitems && ok; item += gridDim.x, ++li) {
        const int bh = item / prm.npairs;
        // The packed Q of the item (TMA, or the fused-Q warp) is widened once
        // the previous item's QK products have been issued (q_free).
        if (!(ok = wait_at(B.qpk_full, li & 1, abort_flag, 7u, li, 256u))) break;
        if (!(ok = wait_at(B.q_free, (li & 1) ^ 1, abort_flag, 8u, li, 256u))) break;
        for (int tt = 0; tt < kTiles; ++tt)
          widen_tile<D>(smem + C::oQPk + tt * C::kQPkBytes, smem + C::oQ + tt * C::kQBytes, kRows, wt, 128);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) { mbar_arrive(B.qpk_empty); mbar_arrive(B.q_full); }
        for (int t = 0; t < nb; ++t, ++g) {
          const int s = g % C::kPS, ks = g % C::kKS, vs = g % C::kVS;
          if (!(ok = wait_at(B.pk_full + s, (g / C::kPS) & 1, abort_flag, 9u, g, 128u))) break;
          if (!(ok = wait_at(B.kw_empty + ks, ((g / C::kKS) & 1) ^ 1, abort_flag, 15u, g, 256u))) break;
          const uint8_t* pk = smem + C::oPk + s * 2 * C::kPkHalf;
          plan.run(pk, smem + C::oKw + ks * C::kKwStride);
          if (wt < BN) {
            const int j = t * BN + wt;
            float* ksc = reinterpret_cast<float*>(smem + C::oKsc) + ks * BN;
            // Keys past N get a NaN scale: their score is NaN, which the
            // maximum ignores, and their code bytes are masked in the softmax.
            ksc[wt] = j < prm.N ? prm.sk[static_cast<size_t>(bh) * prm.N + j] * (1.0f / 256.0f)
                                : __int_as_float(0x7FC00000);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(B.kw_full + ks);
          if (!(ok = wait_at(B.vw_empty + vs, ((g / C::kVS) & 1) ^ 1, abort_flag, 16u, g, 256u))) break;
          plan.run(pk + C::kPkHalf, smem + C::oVw + vs * C::kVwStride);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) { mbar_arrive(B.vw_full + vs); mbar_arrive(B.pk_empty + s); }
        }
      }
      if (!ok) set_status(kStatusTimeout);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 96;");
    // -------------------------------------------------------------- softmax
    // Two threads per query row.  A softmax warp covers 16 rows of its TMEM lane
    // quadrant; lane l < 16 takes the first half of every key block and of the
    // accumulator columns of its row, lane l + 16 the second halves of the same
    // row (.16x32bx2 TMEM accesses).
    constexpr int kHK = BN / 2;          // keys of a block per thread
    constexpr int kHD = D / 2;           // accumulator columns per thread
    constexpr int kFr = kHD / 2;         // of which in registers (the rest in shared memory)
    const int sw = warp - 8;             // softmax warp 0..15
    const int tt = sw >> 3;              // query tile
    const int sub = (sw >> 2) & 1;       // half of the lane quadrant
    const int quad = warp & 3;           // TMEM lane quadrant
    const int hh = lane >> 4;            // half of the keys / accumulator columns
    const int r = quad * 32 + sub * 16 + (lane & 15);  // row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32 + sub * 16) << 16;
    const uint32_t tA = tbase + tt * 256 + 128 + lane_off;
    float4* Fs = reinterpret_cast<float4*>(smem + C::oF) + ((tt * 2 + hh) * kRows + r) * (C::kFRow / 4);
    const float kLog2e = 1.4426950408889634f;
    // Arithmetic on pairs of fp32 (sm_100 f32x2 instructions: two lanes per
    // instruction, each rounded exactly like the scalar form).
    const float2 kNegMagic2 = make_float2(-kMagicF, -kMagicF);
    // Byte-lane magics: fp32 values in [2^23, 2^24) with a zero low byte whose
    // bits K0..K3 satisfy K0 + K1 2^8 + K2 2^16 + K3 2^24 = 0 mod 2^32, so
    // t0 + t1 2^8 + t2 2^16 + t3 2^24 of the rounded sums is the packed word.
    const float2 kMagLo = make_float2(8388608.0f, 11862016.0f);   // bits 0x4B000000, 0x4B350000
    const float2 kMagHi = make_float2(8421376.0f, kMagicF);       // bits 0x4B008000, 0x4B400000
    constexpr int kPMode = MODE & 3;
    constexpr bool kLf = (MODE & 4) != 0;
    constexpr float kLevels = kPMode == 2 ? 7.0f : 15.0f;  // code for P = 1
    constexpr int kZero = kPMode == 2 ? 0 : 8;              // zero point of the stored codes
    const float2 kLv2 = make_float2(kLevels, kLevels);
    uint32_t g = 0;
    bool ok = true;
    float2 F2[kFr / 2];  // F[2i], F[2i+1] of this thread's columns
    // F += coef * (integer accumulator A); with reset, A is then set back to
    // zero (its bits to 1.5 * 2^23).
    //
    // Without reset, A keeps accumulating across a change of the row maximum:
    // with segments s_k of P.V results between changes, A_k = s_1 + ... + s_k
    // and segment weights w_k, sum_k w_k s_k = sum_k (w_k - w_(k+1)) A_k plus
    // w_last A_last, so each change adds (w_old - w_new) A to F and the final
    // fold adds w_last A.  This needs no TMEM store at a change.
    auto fold = [&](float coef, bool reset, int dump_t, bool dump_now) {
      const float2 w2 = make_float2(coef, coef);
#pragma unroll
      for (int c = 0; c < kHD; c += 32) {
        uint32_t a[32];
        tmem_ld_h<32, kHD>(tA + c, a);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int col = c + 4 * q;
          const float2 lo = __fadd2_rn(make_float2(__uint_as_float(a[4 * q]), __uint_as_float(a[4 * q + 1])), kNegMagic2);
          const float2 hi = __fadd2_rn(make_float2(__uint_as_float(a[4 * q + 2]), __uint_as_float(a[4 * q + 3])), kNegMagic2);
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
        if (DUMP && dump_now && prm.dump_acc) {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            prm.dump_acc[(static_cast<size_t>(r) * nb + dump_t) * D + wide_to_dim(hh * kHD + c + i)] =
                (static_cast<int>(a[i]) - static_cast<int>(kMagic)) / 16;
        }
        if (reset) {
          uint32_t m[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) m[i] = kMagic;
          tmem_st_h<32, kHD>(tA + c, m);
        }
      }
    };
    // The P.V accumulator starts at the bits of 1.5 * 2^23 (integer zero).
    {
      uint32_t m[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) m[i] = kMagic;
#pragma unroll
      for (int c = 0; c < kHD; c += 32) tmem_st_h<32, kHD>(tA + c, m);
    }
    uint32_t li = 0;
    for (int item = blockIdx.x; item < prm.nitems && ok; item += gridDim.x, ++li) {
      const int bh = item / prm.npairs, pair = item % prm.npairs;
      const int qtile = pair * 2 + tt;
      const int row = qtile * kRows + r;
      const bool row_ok = row < prm.N;
      float sq_row = 0.0f;
      if constexpr (kFQ) {
        const uint32_t slot = li & 1;
        if (!(ok = wait_at(B.sq_full + slot, (li >> 1) & 1, abort_flag, 21u, li))) break;
        sq_row = reinterpret_cast<const float*>(smem + C::oSq)[(slot * kTiles + tt) * kRows + r];
        __syncwarp();
        if (lane == 0) mbar_arrive(B.sq_empty + slot);
      } else if (row_ok) {
        sq_row = prm.sq[static_cast<size_t>(bh) * prm.N + row];
      }
      const float ci = row_ok ? __fmul_rn(sq_row, prm.inv_sqrt_d) : 0.0f;
      const float cpi = __fmul_rn(ci, kLog2e);
      const float2 cpi2 = make_float2(cpi, cpi);
      const bool dump_tile = DUMP && bh == prm.dump_bh && qtile == prm.dump_tile && row_ok;
#pragma unroll
      for (int i = 0; i < kFr / 2; ++i) F2[i] = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int q = 0; q < (kHD - kFr) / 4; ++q) Fs[q] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      float m_run = -INFINITY, m_ref = 0.0f, w = 1.0f, Lf = 0.0f;
      int Lrun = 0;   // code sum of the row since the last fold (denominator)
      float Lrun_e = 0.0f;  // fp32 sum of exp(S - m) since the last fold (fp32 denominator)
      int Labs = 0;   // code sum of the row since the last reset of A (magnitude bound)
      for (int t = 0; t < nb; ++t, ++g) {
        const uint32_t buf = g & 1;
        const uint32_t tS = tbase + tt * 256 + buf * 64 + lane_off;
        if (!(ok = wait_at(B.s_full + tt * 2 + buf, (g >> 1) & 1, abort_flag, 10u, g))) break;
        __syncwarp();
        tc_fence_after();
        const int ks = g % C::kKS;
        if (!(ok = wait_at(B.kw_full + ks, (g / C::kKS) & 1, abort_flag, 11u, g))) break;
        const float4* ksc = reinterpret_cast<const float4*>(smem + C::oKsc) + ks * (BN / 4) + hh * (kHK / 4);
        const int nvalid = min(BN, prm.N - t * BN);
        // v = S_int * s_k for this thread's half of the block, in registers
        // (256 S_int is exact in fp32 and s_k/256 a power-of-two scaling, so v
        // is S_int * s_k rounded once).  Keys past N give NaN, which fmaxf skips.
        uint32_t raw[kHK];
        tmem_ld_h<kHK, kHK>(tS, raw);
        if (dump_tile && prm.dump_s) {
          for (int j = 0; j < kHK; ++j)
            if (hh * kHK + j < nvalid)
              prm.dump_s[static_cast<size_t>(r) * prm.N + t * BN + hh * kHK + j] = static_cast<int32_t>(raw[j]) / 256;
        }
        float2 v2[kHK / 2];
#pragma unroll
        for (int j = 0; j < kHK; j += 4) {
          const float4 sc = ksc[j / 4];
          if constexpr (kS8) {  // S is already the exact fp32 value of S_int
            v2[j / 2] = __fmul2_rn(make_float2(__uint_as_float(raw[j]), __uint_as_float(raw[j + 1])),
                                   make_float2(sc.x, sc.y));
            v2[j / 2 + 1] = __fmul2_rn(make_float2(__uint_as_float(raw[j + 2]), __uint_as_float(raw[j + 3])),
                                       make_float2(sc.z, sc.w));
          } else {
            v2[j / 2] = __fmul2_rn(make_float2(static_cast<float>(static_cast<int>(raw[j])),
                                               static_cast<float>(static_cast<int>(raw[j + 1]))),
                                   make_float2(sc.x, sc.y));
            v2[j / 2 + 1] = __fmul2_rn(make_float2(static_cast<float>(static_cast<int>(raw[j + 2])),
                                                   static_cast<float>(static_cast<int>(raw[j + 3]))),
                                       make_float2(sc.z, sc.w));
          }
        }
        float vmax = tree_max<kHK>(reinterpret_cast<const float*>(v2));
        vmax = fmaxf(vmax, __shfl_xor_sync(0xFFFFFFFFu, vmax, 16));  // the row's other half
        const float m_blk = __fmul_rn(vmax, ci);
        const float m_new = fmaxf(m_run, m_blk);
        const bool grow = m_new > m_run;
        const float Mp = __fmul_rn(kPMode == 1 ? m_blk : m_new, kLog2e);  // the max the codes use
        const float2 nMp2 = make_float2(-Mp, -Mp);
        // P code c + 8 = rint(15 exp2(y)): adding 15 e to a magic in [2^23, 2^24)
        // with a zero low byte rounds it to an integer that lands in the low
        // byte of the sum's bits.
        uint32_t words[kHK / 4];
        float2 esum = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int q = 0; q < kHK / 4; ++q) {
          const float2 x01 = __ffma2_rn(v2[2 * q], cpi2, nMp2);
          const float2 x23 = __ffma2_rn(v2[2 * q + 1], cpi2, nMp2);
          float2 e01 = make_float2(ex2_approx(x01.x), ex2_approx(x01.y));
          float2 e23 = make_float2(ex2_approx(x23.x), ex2_approx(x23.y));
          const float2 t01 = __ffma2_rn(kLv2, e01, kMagLo);
          const float2 t23 = __ffma2_rn(kLv2, e23, kMagHi);
          if constexpr (kLf) {
            if (nvalid < BN) {  // keys past N (NaN scores) do not count
              const int j = hh * kHK + 4 * q;
              e01 = make_float2(j < nvalid ? e01.x : 0.0f, j + 1 < nvalid ? e01.y : 0.0f);
              e23 = make_float2(j + 2 < nvalid ? e23.x : 0.0f, j + 3 < nvalid ? e23.y : 0.0f);
            }
            esum = __fadd2_rn(esum, __fadd2_rn(e01, e23));
          }
          // Integer multiply-adds (FMA pipe) instead of byte permutes (ALU).
          // Keys past N give NaN bits; they form a suffix of the word, and
          // the carries of their garbage only reach higher (also masked) bytes.
          const uint32_t lo = __float_as_uint(t01.y) * 256u + __float_as_uint(t01.x);
          const uint32_t hi = __float_as_uint(t23.y) * 256u + __float_as_uint(t23.x);
          words[q] = hi * 65536u + lo;
        }
        if (nvalid < BN) {  // last, ragged block: codes of keys past N are 0
#pragma unroll
          for (int q = 0; q < kHK / 4; ++q) {
            const int lim = nvalid - hh * kHK - 4 * q;
            words[q] &= lim >= 4 ? 0xFFFFFFFFu : (lim <= 0 ? 0u : (0xFFFFFFFFu >> (8 * (4 - lim))));
          }
        }
        // Sum of the row's codes (+8 each): bytes are at most 15, so plain
        // word additions of up to 16 words cannot carry between bytes.
        uint32_t wsum = 0;
#pragma unroll
        for (int q = 0; q < kHK / 4; ++q) wsum += words[q];
        int lq = static_cast<int>(__dp4a(wsum, 0x01010101u, 0u));  // unsigned bytes
        lq += __shfl_xor_sync(0xFFFFFFFFu, lq, 16);
        float le = 0.0f;
        if constexpr (kLf) {
          le = esum.x + esum.y;
          le += __shfl_xor_sync(0xFFFFFFFFu, le, 16);
        }
        // P codes over the S columns they came from: word q of half hh is
        // column hh * BN / 8 + q; P.V reads kKeysPV keys, those past BN are 0.
        tmem_st_h<kHK / 4, kHK / 4>(tS, words);
        if constexpr (C::kKeysPV > BN) {
          constexpr int kZ = (C::kKeysPV - BN) / 8;
          uint32_t zw[kZ];
#pragma unroll
          for (int q = 0; q < kZ; ++q) zw[q] = 0u;
          tmem_st_h<kZ, kZ>(tS + BN / 4, zw);
        }
        if (dump_tile && prm.dump_p) {
          for (int j = 0; j < kHK; ++j)
            if (hh * kHK + j < nvalid)
              prm.dump_p[static_cast<size_t>(r) * prm.N + t * BN + hh * kHK + j] =
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
        // Block-local codes: every block has its own weight exp(m_block - m_ref).
        if constexpr (kPMode == 1) w_new = t == 0 ? 1.0f : ex2_approx(__fmul_rn(m_blk - m_ref, kLog2e));
        const bool change = grow || (kPMode == 1 && w_new != w);
        // Fold when a row's maximum grows (its earlier codes used the old
        // maximum); reset A when its magnitude bound nears the exact range of
        // the read-back (|A| < 2^22).
        const bool near_bound = (Labs + 15 * BN) * 112 >= (1 << 22) - 4096;
        // Both votes are taken by every lane before either is used.
        const bool reset = __any_sync(0xFFFFFFFFu, (t > 0) && (near_bound || DUMP));
        const bool any_change = __any_sync(0xFFFFFFFFu, (t > 0) && change);
        if (reset || any_change) {
          if (!(ok = wait_at(B.pv_done + tt * 2 + ((g - 1) & 1), ((g - 1) >> 1) & 1, abort_flag, 12u, g))) break;
          __syncwarp();
          tc_fence_after();
          if (sc != 1.0f) {  // new reference maximum: rescale F and the denominator
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
          fold(reset ? w : w - w_new, reset, t - 1, dump_tile);
          Lf = fmaf(w, kLf ? Lrun_e : static_cast<float>(Lrun), Lf);
          Lrun = 0;
          Lrun_e = 0.0f;
          if (reset) Labs = 0;
        }
        w = w_new;
        Labs += lq;
        Lrun += lq;
        Lrun_e += le;
        m_run = m_new;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(B.p_full + tt * 2 + buf);
          mbar_arrive(B.kw_empty + ks);
        }
      }
      if (!ok) break;
      // Last block: fold the accumulator (and reset it), normalise, store.
      if (!(ok = wait_at(B.pv_done + tt * 2 + ((g - 1) & 1), ((g - 1) >> 1) & 1, abort_flag, 13u, g))) break;
      __syncwarp();
      tc_fence_after();
      fold(w, true, nb - 1, dump_tile);
      Lf = fmaf(w, kLf ? Lrun_e : static_cast<float>(Lrun), Lf);
      if (row_ok) {
        // O = (s_v / L) (acc / 16) / l with L the code levels; l is the code
        // sum / L, or the fp32 sum of exp.
        const float inv = 1.0f / (kLf ? 16.0f * kLevels * Lf : 16.0f * Lf);
        const float* sv = prm.sv + static_cast<size_t>(bh) * D;
        const float* Fsf = reinterpret_cast<const float*>(Fs);
        __nv_bfloat16* orow = prm.out + (static_cast<size_t>(bh) * prm.N + row) * D;
        auto fget = [&](int i) -> float {  // column i of this thread's half
          return i < kFr ? ((i & 1) ? F2[i >> 1].y : F2[i >> 1].x) : Fsf[i - kFr];
        };
        // Widened positions hh * D/2 + c + (4a + b) and + 16 hold channels
        // d = hh * D/2 + c + 8a + 2b and d + 1 (packed layout); in the s8
        // layout position p is channel p.
#pragma unroll
        for (int c = 0; c < kHD; c += 32) {
          const int c0 = hh * kHD + c;
          uint32_t pk[16];
#pragma unroll
          for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) {
              const int d = kS8 ? c0 + 2 * (4 * a + b) : c0 + 8 * a + 2 * b;
              const float f0 = kS8 ? fget(c + 2 * (4 * a + b)) : fget(c + 4 * a + b);
              const float f1 = kS8 ? fget(c + 2 * (4 * a + b) + 1) : fget(c + 16 + 4 * a + b);
              const __nv_bfloat162 h2 = __floats2bfloat162_rn(f0 * __ldg(sv + d) * inv, f1 * __ldg(sv + d + 1) * inv);
              pk[4 * a + b] = *reinterpret_cast<const uint32_t*>(&h2);
            }
          uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
          for (int u = 0; u < 4; ++u) dst[u] = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
        }
        if (prm.lse && hh == 0)
          prm.lse[static_cast<size_t>(bh) * prm.N + row] = m_ref + logf(kLf ? Lf : Lf * (1.0f / kLevels));
      }
    }
    if (!ok) set_status(kStatusTimeout);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, 512);
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 get_encoder() {
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

// 3D map over packed codes [BH, N, D/2] bytes; box = rows x D/2; zero fill past N.
bool make_code_map(CUtensorMap* m, const void* base, int BH, int N, int D, int rows) {
  auto enc = get_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D / 2), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D / 2), static_cast<cuuint64_t>(N) * (D / 2)};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(D / 2), static_cast<cuuint32_t>(rows), 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3D map over s8 codes [BH, N, D] bytes; box = rows x D, swizzled like the
// widened operand tiles (128B for D = 128, 64B for D = 64); zero fill past N.
bool make_s8_map(CUtensorMap* m, const void* base, int BH, int N, int D, int rows) {
  auto enc = get_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(N) * D};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(D), static_cast<cuuint32_t>(rows), 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, int BN, bool DUMP, int MODE>
cudaError_t launch_cfg(const ra_problem& p, const uint8_t* q4, const uint8_t* k4, const uint8_t* v4,
                       const AttnParams& prm, cudaStream_t st) {
  using C = Cfg<D, BN>;
  CUtensorMap mq, mk, mv;
  const int BH = p.B * p.H;
  if constexpr ((MODE & 16) != 0) {
    if (!make_s8_map(&mq, q4, BH, p.N, D, kRows) || !make_s8_map(&mk, k4, BH, p.N, D, BN) ||
        !make_s8_map(&mv, v4, BH, p.N, D, BN))
      return cudaErrorInvalidValue;
  } else if (!make_code_map(&mq, q4, BH, p.N, D, kRows) || !make_code_map(&mk, k4, BH, p.N, D, BN) ||
             !make_code_map(&mv, v4, BH, p.N, D, BN)) {
    return cudaErrorInvalidValue;
  }
  auto kern = attn_int4_kernel<D, BN, DUMP, MODE>;
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

cudaError_t launch_attn_int4(const ra_problem& p, const uint8_t* q4, const float* sq, const uint8_t* k4,
                             const float* sk, const uint8_t* v4, const float* sv, void* out, float* lse,
                             const AttnDump* dump, int mode, cudaStream_t st, int* unsupported,
                             const FusedQ* fq) {
  AttnParams prm{};
  prm.N = p.N;
  prm.BH = p.B * p.H;
  prm.nblocks = (p.N + p.block_k - 1) / p.block_k;
  prm.npairs = (p.N + 2 * kRows - 1) / (2 * kRows);
  prm.nitems = prm.BH * prm.npairs;
  prm.inv_sqrt_d = static_cast<float>(1.0 / sqrt(static_cast<double>(p.D)));
  prm.sq = sq; prm.sk = sk; prm.sv = sv;
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.lse = lse;
  const bool dmp = dump != nullptr;
  if (dmp) {
    prm.dump_bh = dump->bh; prm.dump_tile = dump->q_tile;
    prm.dump_s = dump->s; prm.dump_p = dump->p; prm.dump_acc = dump->acc;
  }
  *unsupported = 0;
  if (fq) {
    // Fused Q: block_k = 64, the method's P codes and denominator, no dump.
    // The unused Q tensor map is encoded over the K codes (never loaded).
    if (p.block_k != 64 || mode != 0 || dmp) {
      *unsupported = 1;
      return cudaSuccess;
    }
    prm.qraw = fq->q; prm.qdtype = fq->dtype; prm.pos = fq->pos; prm.tab = fq->tab;
    prm.rot = p.rot; prm.seg = seg_info(p);
    return p.D == 128 ? launch_cfg<128, 64, false, 8>(p, k4, k4, v4, prm, st)
                      : launch_cfg<64, 64, false, 8>(p, k4, k4, v4, prm, st);
  }
  if (mode == 16) {
    // s8 code layout: block_k = 64, the method's P codes and denominator, no dump.
    if (p.block_k != 64 || dmp) {
      *unsupported = 1;
      return cudaSuccess;
    }
    return p.D == 128 ? launch_cfg<128, 64, false, 16>(p, q4, k4, v4, prm, st)
                      : launch_cfg<64, 64, false, 16>(p, q4, k4, v4, prm, st);
  }
  if (p.block_k == 128)
    return launch_attn_int4_pair(p, q4, sq, k4, sk, v4, sv, out, lse, dump, mode, st, unsupported);
#define RA_CASE(DD, BB, MM)                                                                          \
  if (p.D == DD && p.block_k == BB && mode == MM)                                                    \
    return dmp ? launch_cfg<DD, BB, true, MM>(p, q4, k4, v4, prm, st)                                \
               : launch_cfg<DD, BB, false, MM>(p, q4, k4, v4, prm, st);
  RA_CASE(128, 64, 0)
  RA_CASE(128, 32, 0)
  RA_CASE(128, 16, 0)
  RA_CASE(64, 64, 0)
  RA_CASE(64, 32, 0)
  RA_CASE(64, 16, 0)
  // Ablation modes: block_k = 64 only.
  RA_CASE(128, 64, 1)
  RA_CASE(128, 64, 2)
  RA_CASE(128, 64, 4)
  RA_CASE(128, 64, 5)
  RA_CASE(128, 64, 6)
  RA_CASE(64, 64, 1)
  RA_CASE(64, 64, 2)
  RA_CASE(64, 64, 4)
  RA_CASE(64, 64, 5)
  RA_CASE(64, 64, 6)
#undef RA_CASE
  *unsupported = 1;
  return cudaSuccess;
}

cudaError_t read_attn_int4_diag(uint32_t* out) {
  uint32_t zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(out, g_attn_diag, sizeof(uint32_t));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_attn_diag, &zero, sizeof(uint32_t));
}

cudaError_t read_attn_int4_status(uint32_t* out) {
  uint32_t zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(out, g_attn_status, sizeof(uint32_t));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_attn_status, &zero, sizeof(uint32_t));
}

}  // namespace ra
