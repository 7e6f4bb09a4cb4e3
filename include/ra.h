/*
 * ra.h -- C ABI of the RotateAttention INT4 attention forward for NVIDIA B200
 * (sm_100a).
 *
 * Method: "RotateAttention: RoPE-Aware Rotation and Range Rectification for
 * INT4 Quantized Attention in Video Generation" (arXiv 2607.02584).  Page
 * references below are to the papernotes.org note on that paper ("overall
 * framework", "key design 1-3") and to the gecl reading notes ("Method",
 * "Key Insight").
 *
 * Conventions shared by every entry point
 *   - Tensors are dense, row-major, in DEVICE memory unless stated otherwise:
 *     [B, H, N, D] means D fastest, then N, H, B.  Every device pointer must be
 *     16-byte aligned.
 *   - The caller owns every buffer.  The library never allocates or frees
 *     device memory; scratch space is passed in as `workspace`.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) and returns after enqueueing the work.
 *   - Arguments are validated on the host before anything is launched; an
 *     invalid argument returns RA_ERR_INVALID_ARG and launches nothing.
 *     A configuration the kernels do not implement returns RA_ERR_UNSUPPORTED.
 *     A failed CUDA runtime call returns RA_ERR_CUDA.
 *   - Faults found by the kernels themselves (a position outside the grid, an
 *     internal wait that ran past its bound) are recorded in a device status
 *     word and reported by the next ra_sync_status() call, as
 *     RA_ERR_INVALID_ARG or RA_ERR_TIMEOUT.  No kernel traps.
 *   - No exception crosses this interface.
 *
 * Packed INT4 codes: two 4-bit two's-complement codes per byte, element 2t in
 * the low nibble and 2t+1 in the high nibble.
 */
#ifndef RA_H_
#define RA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  RA_OK = 0,
  RA_ERR_INVALID_ARG = 1,
  RA_ERR_UNSUPPORTED = 2,
  RA_ERR_CUDA = 3,
  RA_ERR_TIMEOUT = 4
} ra_status;

/* RoPE-aware rotation (papernotes page, key design 1). */
typedef enum {
  RA_ROT_NONE = 0,         /* 3D RoPE only */
  RA_ROT_INTERLEAVED = 1,  /* H2 blocks on adjacent channel pairs, fused into the RoPE tables */
  RA_ROT_HALF = 2,         /* per segment: pair channel i with i + Dj/2, then H2 blocks */
  RA_ROT_FULL = 3          /* the whole row times H_D / sqrt(D) (Sylvester Hadamard), after
                              RoPE: the pages' full-rotation ablation (papernotes page,
                              ablation on rotation granularity) */
} ra_rot_mode;

typedef enum { RA_DT_F32 = 0, RA_DT_BF16 = 1 } ra_dtype;

/*
 * Problem description (papernotes page, key design 1: the head dimension is
 * split D = Df + Dh + Dw into frame / height / width RoPE segments).
 *   B, H, N, D   batch, heads, tokens, head dimension.  D is 64 or 128; N >= 1.
 *   seg[3]       Df, Dh, Dw: even, >= 2, summing to D.
 *   grid[3]      extents of the frame / height / width token grid.  Every
 *                position pos[n][j] must lie in [0, grid[j]).
 *   theta        RoPE base; segment j, pair k rotates by pos_j * theta^(-2k/Dj).
 *   rot          ra_rot_mode.
 *   block_q      query rows per tile: 16, 32, 64 or 128.  It does not change any
 *                result (rows are independent).
 *   block_k      keys per softmax block: 16, 32, 64 or 128.  It is part of the
 *                method: the running row maximum that the P codes use is
 *                updated once per block_k keys, and the V column sums are
 *                per block_k keys.  ra_attn_int4 implements all four; 128
 *                runs on a pair of SMs per 256-row query tile (a cluster of
 *                two CTAs sharing one MMA), the others on one SM per two
 *                128-row tiles.
 */
typedef struct {
  int B, H, N, D;
  int seg[3];
  int grid[3];
  float theta;
  int rot;
  int block_q, block_k;
} ra_problem;

/* Human-readable name of a status code (static string, never NULL). */
const char* ra_status_string(ra_status s);

/* Bytes of workspace ra_rope_rotate_quant needs for problem p (0 if p is invalid). */
size_t ra_workspace_bytes(const ra_problem* p);

/*
 * Fused prologue: 3D RoPE + RoPE-aware rotation of Q and K, K smoothing,
 * per-token INT4 of Q and K, per-channel INT4 of V, per-block V column sums.
 * papernotes page: "overall framework" (smoothing, rotation, quantised V) and
 * key design 1 (RoPE-aware rotation, fused into the RoPE tables for the
 * interleaved mode); gecl notes "Key Insight" (per-token INT4 for Q and K).
 *
 *   in_dtype       RA_DT_BF16 or RA_DT_F32: element type of q, k, v.
 *   q, k, v        [B, H, N, D] inputs.  V is used as given (the offline V
 *                  Hadamard of key design 3 belongs to the weights).
 *   pos            [N, 3] int32 (frame, row, col) grid position of each token.
 *   q4, k4, v4     [B, H, N, D/2] packed INT4 codes (output).
 *   sq, sk         [B, H, N] fp32 per-token scales amax/7 (output).
 *   k_mean         [B, H, D] fp32 mean over tokens of the rotated K (output).
 *   sv             [B, H, D] fp32 per-channel V scales amax/7 (output).
 *   v_colsum       [B, H, ceil(N/block_k), D] int32: sum of the V codes of each
 *                  key block (output); the P.V zero-point correction is
 *                  8 * v_colsum.
 *   workspace      device scratch of at least ra_workspace_bytes(p) bytes,
 *                  16-byte aligned; its contents on entry do not matter.
 * q, q4 and sq may all be NULL together: K and V only, for ra_attn_int4_qfused,
 * which quantises Q itself (any other mix of NULLs is RA_ERR_INVALID_ARG).
 * Quantisation: s = fl(amax/7), code = clamp(rint(x * fl(7/amax)), -7, 7) with
 * the product taken exactly and ties to even; amax = 0 gives s = 0 and codes 0.
 */
ra_status ra_rope_rotate_quant(const ra_problem* p, int in_dtype,
                               const void* q, const void* k, const void* v,
                               const int32_t* pos,
                               uint8_t* q4, float* sq, uint8_t* k4, float* sk,
                               float* k_mean, uint8_t* v4, float* sv, int32_t* v_colsum,
                               void* workspace, size_t ws_bytes, void* stream);

/*
 * INT4 attention forward from the prologue's codes (papernotes page,
 * flowchart D-F and key design 2):
 *   S = (S_int * s_k[j]) * (s_q[i] / sqrt(D)), S_int = sum_d q4[i,d] k4[j,d] (exact);
 *   online softmax with the running row maximum m, updated per block_k keys;
 *   range-rectified P codes c = clamp(rint(15 exp(S - m)), 0, 15) - 8;
 *   INT4 P.V with the zero-point correction 8 * colsum(V block) folded into the
 *   integer accumulator: acc = sum_j (c_ij + 8) v4[j, d];
 *   O = sum_t alpha-chain (s_v/15) acc_t / sum_t alpha-chain sum_j (c_ij + 8)/15.
 *   out   [B, H, N, D] bf16 (output).
 *   lse   nullable [B, H, N] fp32: m + ln(l) with l the denominator above.
 */
ra_status ra_attn_int4(const ra_problem* p,
                       const uint8_t* q4, const float* sq,
                       const uint8_t* k4, const float* sk,
                       const uint8_t* v4, const float* sv,
                       void* out, float* lse, void* stream);

/*
 * The byte code layout: the same INT4 codes with one code per byte, channels
 * in natural order, [B, H, N, D] bytes: q8 and k8 hold the FP8 E4M3 value
 * equal to the code (every integer in [-7, 7] is exact in E4M3), v8 the int8
 * value 16 x code (the code in the high nibble).  On sm_100a the tensor cores
 * have no 4-bit integer kind, so packed nibbles must be widened to bytes
 * before every MMA; in this layout the attention kernel loads Q, K and V tiles
 * by TMA straight into its MMA operands and skips the widening (twice the code
 * bytes in HBM), and Q K^T runs as an FP8 MMA with an fp32 accumulator, which
 * is exact here (|S_int| <= 49 D < 2^13) and spares the softmax its integer
 * conversion.  ra_rope_rotate_quant_s8 takes the arguments of
 * ra_rope_rotate_quant (q, q8, sq may be NULL together) and writes q8, k8, v8
 * in this layout; every other output is identical.  ra_attn_int4_s8 takes the
 * arguments of ra_attn_int4 with these codes; its out and lse equal
 * ra_attn_int4's on the packed codes bit for bit.  Implemented for
 * block_k = 64 (D = 64 or 128), the method's P codes and denominator; other
 * block sizes return RA_ERR_UNSUPPORTED.
 */
ra_status ra_rope_rotate_quant_s8(const ra_problem* p, int in_dtype,
                                  const void* q, const void* k, const void* v,
                                  const int32_t* pos,
                                  uint8_t* q8, float* sq, uint8_t* k8, float* sk,
                                  float* k_mean, int8_t* v8, float* sv, int32_t* v_colsum,
                                  void* workspace, size_t ws_bytes, void* stream);
ra_status ra_attn_int4_s8(const ra_problem* p,
                          const uint8_t* q8, const float* sq,
                          const uint8_t* k8, const float* sk,
                          const int8_t* v8, const float* sv,
                          void* out, float* lse, void* stream);

/*
 * INT4 attention with Q's prologue fused into the attention kernel (the
 * papernotes page, highlights: the rotation rides on the elementwise RoPE
 * pass at no extra memory traffic).  Instead of q4/sq, the kernel's code-
 * widening warps read the raw Q, apply the same RoPE, rotation and per-token
 * INT4 quantisation as ra_rope_rotate_quant (bit-identical codes and scales)
 * and write the codes straight into the MMA's operand tiles; Q's codes never
 * reach HBM.  K and V come from ra_rope_rotate_quant called with q, q4 and sq
 * NULL.  Results equal ra_attn_int4 on the codes of the full prologue, bit for
 * bit.
 *   in_dtype   RA_DT_BF16 or RA_DT_F32: element type of q.
 *   q          [B, H, N, D] raw Q (before RoPE).
 *   pos        [N, 3] int32 grid positions (the same array as the prologue's).
 *   k4, sk, v4, sv   as for ra_attn_int4 (from the K/V-only prologue).
 *   workspace  device scratch of at least ra_workspace_bytes(p) bytes (the
 *              RoPE table of p->rot is built in it; it may be the prologue's).
 *   out, lse   as for ra_attn_int4.
 * Implemented for block_k = 64 (D = 64 or 128) and the method's P codes and
 * denominator; other block sizes return RA_ERR_UNSUPPORTED.
 */
ra_status ra_attn_int4_qfused(const ra_problem* p, int in_dtype, const void* q, const int32_t* pos,
                              const uint8_t* k4, const float* sk, const uint8_t* v4, const float* sv,
                              void* workspace, size_t ws_bytes, void* out, float* lse, void* stream);

/*
 * Test entry on raw codes: runs the INT4 attention kernel of ra_attn_int4 on
 * given codes and scales (no prologue), writing out / lse for every row like
 * ra_attn_int4, and dumps the integer intermediates of one 128-row query tile
 * (tile q_tile of head (b, h)):
 *   s_dump    [128, N] int32   S_int = sum_d q4[i,d] k4[j,d]
 *   p_dump    [128, N] int8    P codes c in [-8, 7]
 *   acc_dump  [128, ceil(N/block_k), D] int32  per-block P.V accumulator
 *             sum_j (c_ij + 8) v4[j, d]  (= sum_j c_ij v4[j,d] + 8 colsum)
 * Rows past N in the tile are left unwritten.  Dump pointers may be NULL.
 * For block_k = 128 the dump variant only adds reads and stores: its out and
 * lse equal those of ra_attn_int4 bit for bit.  For smaller blocks it folds
 * the integer accumulator into the output after every block (the same values
 * up to fp32 rounding order).
 */
ra_status ra_test_int4_codes(const ra_problem* p,
                             const uint8_t* q4, const float* sq,
                             const uint8_t* k4, const float* sk,
                             const uint8_t* v4, const float* sv,
                             int b, int h, int q_tile,
                             int32_t* s_dump, int8_t* p_dump, int32_t* acc_dump,
                             void* out, float* lse, void* stream);

/*
 * Ablation switches of the INT4 attention.  The method's choices (papernotes
 * page, key design 2) are the defaults; the alternatives it is compared with
 * can be measured with the same kernels:
 *   p_mode  RA_P_RANGE      range-rectified codes against the running maximum
 *                           (default, as ra_attn_int4);
 *           RA_P_LOCAL_MAX  the same codes against each key block's own
 *                           maximum; block t then enters the output and the
 *                           denominator with the weight exp(m_block - m);
 *           RA_P_SYMMETRIC  SageAttention-style codes c = rint(7 exp(S - m))
 *                           in [0, 7] (levels 0..7 only), no zero point:
 *                           acc = sum_j c_ij v4[j, d], dequantised as c / 7.
 *   l_mode  RA_L_CODES      denominator = sum of the dequantised codes (default);
 *           RA_L_FP32       denominator = fp32 sum of exp(S - m_c), m_c the
 *                           maximum the codes are taken against.
 * opts == NULL selects the defaults.  A mode other than the defaults is
 * implemented for block_k = 64 and 128 (RA_ERR_UNSUPPORTED otherwise); an out
 * of range mode is RA_ERR_INVALID_ARG.  All other arguments as ra_attn_int4 /
 * ra_test_int4_codes; in the test entry p_dump holds the stored codes (c in
 * [-8, 7], or [0, 7] for RA_P_SYMMETRIC) and acc_dump the accumulator
 * sum_j (c_ij + zero point) v4[j, d].
 */
typedef enum { RA_P_RANGE = 0, RA_P_LOCAL_MAX = 1, RA_P_SYMMETRIC = 2 } ra_p_mode;
typedef enum { RA_L_CODES = 0, RA_L_FP32 = 1 } ra_l_mode;
typedef struct {
  int p_mode;  /* ra_p_mode */
  int l_mode;  /* ra_l_mode */
} ra_attn_opts;

ra_status ra_attn_int4_opts(const ra_problem* p, const ra_attn_opts* opts,
                            const uint8_t* q4, const float* sq,
                            const uint8_t* k4, const float* sk,
                            const uint8_t* v4, const float* sv,
                            void* out, float* lse, void* stream);
ra_status ra_test_int4_codes_opts(const ra_problem* p, const ra_attn_opts* opts,
                                  const uint8_t* q4, const float* sq,
                                  const uint8_t* k4, const float* sk,
                                  const uint8_t* v4, const float* sv,
                                  int b, int h, int q_tile,
                                  int32_t* s_dump, int8_t* p_dump, int32_t* acc_dump,
                                  void* out, float* lse, void* stream);

/*
 * 3D RoPE only (no rotation, no quantisation) of Q and K, output bf16: the
 * input of the bf16 fallback path (papernotes page, key design 3: sensitive
 * layers and steps keep full-precision attention; rotation does not change
 * QK^T, so the fallback skips it).
 *   q, k         [B, H, N, D] in in_dtype;  q_roped, k_roped [B, H, N, D] bf16.
 *   workspace    device scratch of at least ra_workspace_bytes(p) bytes (holds
 *                the RoPE table).
 */
ra_status ra_rope_bf16(const ra_problem* p, int in_dtype, const void* q, const void* k,
                       const int32_t* pos, void* q_roped, void* k_roped,
                       void* workspace, size_t ws_bytes, void* stream);

/*
 * bf16 FlashAttention forward, the selective-precision fallback (papernotes
 * page, key design 3).  softmax(q k^T / sqrt(D)) v with fp32 accumulation.
 *   q, k, v  [B, H, N, D] bf16;  out [B, H, N, D] bf16;  lse nullable [B, H, N].
 */
ra_status ra_attn_bf16_fallback(const ra_problem* p, const void* q, const void* k,
                                const void* v, void* out, float* lse, void* stream);

/*
 * Allocation-free prologue.  (The paper has no counterpart; this is a
 * deployment convenience.)  Same computation, arguments and results as
 * ra_rope_rotate_quant, without the workspace arguments: it is meant for
 * callers that cannot allocate device memory when they run it, such as an
 * inference-engine plugin whose execute step may not call the allocator, or a
 * service with a fixed device-memory budget reserved at start-up.
 *
 * The scratch space is a fixed array of RA_STATIC_SCRATCH_BYTES inside the
 * library's device memory; every GPU that loads the library holds it until the
 * process exits.  The entry point never allocates or frees memory.
 *   - Problems whose ra_workspace_bytes(p) exceeds RA_STATIC_SCRATCH_BYTES
 *     return RA_ERR_UNSUPPORTED and launch nothing (32 MiB covers, e.g.,
 *     B*H*ceil(N/256) <= ~21000 at D = 128).
 *   - The first call on a device looks up the array's device address, with
 *     that device current; make that first call before any stream capture.
 *     The address is kept per device together with the CUDA context it was
 *     found in; after a device reset (a new primary context) the next call
 *     looks it up again.
 *   - All calls on a device share the one array: calls whose work may overlap
 *     on the GPU (different streams without ordering between them) race on it.
 *     Calls ordered on one stream are safe; the array keeps the last call's
 *     contents, and nothing in it needs to start at zero.
 */
#define RA_STATIC_SCRATCH_BYTES ((size_t)32 << 20)
ra_status ra_rope_rotate_quant_noalloc(const ra_problem* p, int in_dtype,
                                       const void* q, const void* k, const void* v,
                                       const int32_t* pos,
                                       uint8_t* q4, float* sq, uint8_t* k4, float* sk,
                                       float* k_mean, uint8_t* v4, float* sv, int32_t* v_colsum,
                                       void* stream);

/*
 * Synchronises `stream`, then reads and clears the device status word of the
 * current device.  Returns RA_OK, RA_ERR_INVALID_ARG (a kernel saw a position
 * outside the grid), RA_ERR_TIMEOUT (an internal wait ran past its bound) or
 * RA_ERR_CUDA.
 */
ra_status ra_sync_status(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* RA_H_ */
