// C ABI of the RotateAttention INT4 forward: argument validation, workspace
// sizing, dispatch to the kernel units, device status.  See include/ra.h.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "ra_internal.h"

namespace {

using ra::WorkspaceLayout;

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned16_or_null(const void* p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Problem checks shared by every entry point.  block_k 128 is a valid problem
// (the prologue handles it) that the attention kernel reports as unsupported.
bool valid_problem(const ra_problem* p) {
  if (!p) return false;
  if (p->B < 1 || p->H < 1 || p->N < 1 || p->N > (1 << 24)) return false;
  if (p->D != 64 && p->D != 128) return false;
  if (static_cast<long long>(p->B) * p->H * p->N * p->D >= (1LL << 31)) return false;
  int sum = 0;
  for (int j = 0; j < 3; ++j) {
    if (p->seg[j] < 2 || (p->seg[j] & 1)) return false;
    if (p->grid[j] < 1 || p->grid[j] > (1 << 20)) return false;
    sum += p->seg[j];
  }
  if (sum != p->D) return false;
  if (!(p->theta > 0.0f) || !std::isfinite(p->theta)) return false;
  if (p->rot < RA_ROT_NONE || p->rot > RA_ROT_FULL) return false;
  const int bq = p->block_q, bk = p->block_k;
  if (bq != 16 && bq != 32 && bq != 64 && bq != 128) return false;
  if (bk != 16 && bk != 32 && bk != 64 && bk != 128) return false;
  return true;
}

ra_status from_cuda(cudaError_t e) { return e == cudaSuccess ? RA_OK : RA_ERR_CUDA; }

}  // namespace

extern "C" {

const char* ra_status_string(ra_status s) {
  switch (s) {
    case RA_OK: return "ok";
    case RA_ERR_INVALID_ARG: return "invalid argument";
    case RA_ERR_UNSUPPORTED: return "unsupported configuration";
    case RA_ERR_CUDA: return "CUDA runtime error";
    case RA_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

size_t ra_workspace_bytes(const ra_problem* p) {
  if (!valid_problem(p)) return 0;
  return ra::workspace_layout(*p).total;
}

static ra_status rope_rotate_quant(const ra_problem* p, int in_dtype, const void* q, const void* k,
                                   const void* v, const int32_t* pos, uint8_t* q4, float* sq, uint8_t* k4,
                                   float* sk, float* k_mean, uint8_t* v4, float* sv, int32_t* v_colsum,
                                   void* workspace, size_t ws_bytes, void* stream, bool s8);

ra_status ra_rope_rotate_quant(const ra_problem* p, int in_dtype, const void* q, const void* k,
                               const void* v, const int32_t* pos, uint8_t* q4, float* sq, uint8_t* k4,
                               float* sk, float* k_mean, uint8_t* v4, float* sv, int32_t* v_colsum,
                               void* workspace, size_t ws_bytes, void* stream) {
  return rope_rotate_quant(p, in_dtype, q, k, v, pos, q4, sq, k4, sk, k_mean, v4, sv, v_colsum, workspace,
                           ws_bytes, stream, false);
}

ra_status ra_rope_rotate_quant_s8(const ra_problem* p, int in_dtype, const void* q, const void* k,
                                  const void* v, const int32_t* pos, uint8_t* q8, float* sq, uint8_t* k8,
                                  float* sk, float* k_mean, int8_t* v8, float* sv, int32_t* v_colsum,
                                  void* workspace, size_t ws_bytes, void* stream) {
  return rope_rotate_quant(p, in_dtype, q, k, v, pos, q8, sq, k8, sk, k_mean, reinterpret_cast<uint8_t*>(v8), sv,
                           v_colsum,
                           workspace, ws_bytes, stream, true);
}

static ra_status rope_rotate_quant(const ra_problem* p, int in_dtype, const void* q, const void* k,
                                   const void* v, const int32_t* pos, uint8_t* q4, float* sq, uint8_t* k4,
                                   float* sk, float* k_mean, uint8_t* v4, float* sv, int32_t* v_colsum,
                                   void* workspace, size_t ws_bytes, void* stream, bool s8) {
  if (!valid_problem(p) || (in_dtype != RA_DT_F32 && in_dtype != RA_DT_BF16)) return RA_ERR_INVALID_ARG;
  // Q, q4 and sq are either all given or all NULL (K and V only).
  const bool no_q = !q && !q4 && !sq;
  const void* ptrs[] = {k, v, pos, k4, sk, k_mean, v4, sv, v_colsum, workspace};
  for (const void* x : ptrs)
    if (!aligned16(x)) return RA_ERR_INVALID_ARG;
  if (!no_q && (!aligned16(q) || !aligned16(q4) || !aligned16(sq))) return RA_ERR_INVALID_ARG;
  if (ws_bytes < ra::workspace_layout(*p).total) return RA_ERR_INVALID_ARG;
  return from_cuda(ra::launch_prologue(*p, in_dtype, q, k, v, pos, q4, sq, k4, sk, k_mean, v4, sv, v_colsum,
                                       workspace, static_cast<cudaStream_t>(stream), s8));
}

ra_status ra_attn_int4_s8(const ra_problem* p, const uint8_t* q8, const float* sq, const uint8_t* k8,
                          const float* sk, const int8_t* v8, const float* sv, void* out, float* lse,
                          void* stream) {
  if (!valid_problem(p)) return RA_ERR_INVALID_ARG;
  const void* ptrs[] = {q8, sq, k8, sk, v8, sv, out};
  for (const void* x : ptrs)
    if (!aligned16(x)) return RA_ERR_INVALID_ARG;
  if (!aligned16_or_null(lse)) return RA_ERR_INVALID_ARG;
  if (p->block_k != 64) return RA_ERR_UNSUPPORTED;
  int unsupported = 0;
  cudaError_t e = ra::launch_attn_int4(*p, q8, sq, k8, sk, reinterpret_cast<const uint8_t*>(v8), sv, out, lse,
                                       nullptr, 16,
                                       static_cast<cudaStream_t>(stream), &unsupported);
  if (unsupported) return RA_ERR_UNSUPPORTED;
  return from_cuda(e);
}

ra_status ra_attn_int4_qfused(const ra_problem* p, int in_dtype, const void* q, const int32_t* pos,
                              const uint8_t* k4, const float* sk, const uint8_t* v4, const float* sv,
                              void* workspace, size_t ws_bytes, void* out, float* lse, void* stream) {
  if (!valid_problem(p) || (in_dtype != RA_DT_F32 && in_dtype != RA_DT_BF16)) return RA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, pos, k4, sk, v4, sv, workspace, out};
  for (const void* x : ptrs)
    if (!aligned16(x)) return RA_ERR_INVALID_ARG;
  if (!aligned16_or_null(lse)) return RA_ERR_INVALID_ARG;
  if (ws_bytes < ra::workspace_layout(*p).total) return RA_ERR_INVALID_ARG;
  if (p->block_k != 64) return RA_ERR_UNSUPPORTED;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  ra::FusedQ fq;
  fq.q = q;
  fq.dtype = in_dtype;
  fq.pos = pos;
  cudaError_t e = ra::launch_rope_table(*p, workspace, &fq.tab, st);
  if (e != cudaSuccess) return from_cuda(e);
  int unsupported = 0;
  e = ra::launch_attn_int4(*p, nullptr, nullptr, k4, sk, v4, sv, out, lse, nullptr, 0, st, &unsupported, &fq);
  if (unsupported) return RA_ERR_UNSUPPORTED;
  return from_cuda(e);
}

// Kernel mode bits from the ablation options (0 = the method's defaults).
static bool attn_mode(const ra_attn_opts* o, int* mode) {
  if (!o) { *mode = 0; return true; }
  if (o->p_mode < RA_P_RANGE || o->p_mode > RA_P_SYMMETRIC || o->l_mode < RA_L_CODES || o->l_mode > RA_L_FP32)
    return false;
  *mode = o->p_mode | (o->l_mode == RA_L_FP32 ? 4 : 0);
  return true;
}

ra_status ra_attn_int4(const ra_problem* p, const uint8_t* q4, const float* sq, const uint8_t* k4,
                       const float* sk, const uint8_t* v4, const float* sv, void* out, float* lse,
                       void* stream) {
  return ra_attn_int4_opts(p, nullptr, q4, sq, k4, sk, v4, sv, out, lse, stream);
}

ra_status ra_attn_int4_opts(const ra_problem* p, const ra_attn_opts* opts, const uint8_t* q4, const float* sq,
                            const uint8_t* k4, const float* sk, const uint8_t* v4, const float* sv, void* out,
                            float* lse, void* stream) {
  int mode = 0;
  if (!valid_problem(p) || !attn_mode(opts, &mode)) return RA_ERR_INVALID_ARG;
  const void* ptrs[] = {q4, sq, k4, sk, v4, sv, out};
  for (const void* x : ptrs)
    if (!aligned16(x)) return RA_ERR_INVALID_ARG;
  if (!aligned16_or_null(lse)) return RA_ERR_INVALID_ARG;
  int unsupported = 0;
  cudaError_t e = ra::launch_attn_int4(*p, q4, sq, k4, sk, v4, sv, out, lse, nullptr, mode,
                                       static_cast<cudaStream_t>(stream), &unsupported);
  if (unsupported) return RA_ERR_UNSUPPORTED;
  return from_cuda(e);
}

ra_status ra_test_int4_codes(const ra_problem* p, const uint8_t* q4, const float* sq, const uint8_t* k4,
                             const float* sk, const uint8_t* v4, const float* sv, int b, int h, int q_tile,
                             int32_t* s_dump, int8_t* p_dump, int32_t* acc_dump, void* out, float* lse,
                             void* stream) {
  return ra_test_int4_codes_opts(p, nullptr, q4, sq, k4, sk, v4, sv, b, h, q_tile, s_dump, p_dump, acc_dump,
                                 out, lse, stream);
}

ra_status ra_test_int4_codes_opts(const ra_problem* p, const ra_attn_opts* opts, const uint8_t* q4,
                                  const float* sq, const uint8_t* k4, const float* sk, const uint8_t* v4,
                                  const float* sv, int b, int h, int q_tile, int32_t* s_dump, int8_t* p_dump,
                                  int32_t* acc_dump, void* out, float* lse, void* stream) {
  int mode = 0;
  if (!valid_problem(p) || !attn_mode(opts, &mode)) return RA_ERR_INVALID_ARG;
  const void* ptrs[] = {q4, sq, k4, sk, v4, sv, out};
  for (const void* x : ptrs)
    if (!aligned16(x)) return RA_ERR_INVALID_ARG;
  if (!aligned16_or_null(lse) || !aligned16_or_null(s_dump) || !aligned16_or_null(p_dump) ||
      !aligned16_or_null(acc_dump))
    return RA_ERR_INVALID_ARG;
  const int ntiles = (p->N + 127) / 128;
  if (b < 0 || b >= p->B || h < 0 || h >= p->H || q_tile < 0 || q_tile >= ntiles) return RA_ERR_INVALID_ARG;
  ra::AttnDump d;
  d.bh = b * p->H + h;
  d.q_tile = q_tile;
  d.s = s_dump;
  d.p = p_dump;
  d.acc = acc_dump;
  int unsupported = 0;
  cudaError_t e = ra::launch_attn_int4(*p, q4, sq, k4, sk, v4, sv, out, lse, &d, mode,
                                       static_cast<cudaStream_t>(stream), &unsupported);
  if (unsupported) return RA_ERR_UNSUPPORTED;
  return from_cuda(e);
}

ra_status ra_rope_bf16(const ra_problem* p, int in_dtype, const void* q, const void* k, const int32_t* pos,
                       void* q_roped, void* k_roped, void* workspace, size_t ws_bytes, void* stream) {
  if (!valid_problem(p) || (in_dtype != RA_DT_F32 && in_dtype != RA_DT_BF16)) return RA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, pos, q_roped, k_roped, workspace};
  for (const void* x : ptrs)
    if (!aligned16(x)) return RA_ERR_INVALID_ARG;
  if (ws_bytes < ra::workspace_layout(*p).total) return RA_ERR_INVALID_ARG;
  return from_cuda(ra::launch_rope_bf16(*p, in_dtype, q, k, pos, q_roped, k_roped, workspace,
                                        static_cast<cudaStream_t>(stream)));
}

ra_status ra_attn_bf16_fallback(const ra_problem* p, const void* q, const void* k, const void* v, void* out,
                                float* lse, void* stream) {
  if (!valid_problem(p)) return RA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, out};
  for (const void* x : ptrs)
    if (!aligned16(x)) return RA_ERR_INVALID_ARG;
  if (!aligned16_or_null(lse)) return RA_ERR_INVALID_ARG;
  int unsupported = 0;
  cudaError_t e = ra::launch_attn_bf16(*p, q, k, v, out, lse, static_cast<cudaStream_t>(stream), &unsupported);
  if (unsupported) return RA_ERR_UNSUPPORTED;
  return from_cuda(e);
}

ra_status ra_sync_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return RA_ERR_CUDA;
  uint32_t a = 0, b = 0, c = 0, d = 0;
  if (ra::read_prologue_status(&a) != cudaSuccess || ra::read_attn_int4_status(&b) != cudaSuccess ||
      ra::read_attn_bf16_status(&c) != cudaSuccess || ra::read_attn_pair_status(&d) != cudaSuccess)
    return RA_ERR_CUDA;
  const uint32_t s = a | b | c | d;
  if (s & 2u) return RA_ERR_TIMEOUT;
  if (s & 1u) return RA_ERR_INVALID_ARG;
  return RA_OK;
}

}  // extern "C"
