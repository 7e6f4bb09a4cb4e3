// Internal interface between the C ABI (ra_host.cu) and the kernel units.
#pragma once

#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "../../include/ra.h"

namespace ra {

struct WorkspaceLayout {
  size_t tab, tab0, ksum, vmax, vinv, total;
};

size_t rope_table_len(const ra_problem& p);
int prologue_nchunk(const ra_problem& p);
WorkspaceLayout workspace_layout(const ra_problem& p);

cudaError_t launch_prologue(const ra_problem& p, int dtype, const void* q, const void* k, const void* v,
                            const int32_t* pos, uint8_t* q4, float* sq, uint8_t* k4, float* sk,
                            float* k_mean, uint8_t* v4, float* sv, int32_t* colsum, void* ws,
                            cudaStream_t st, bool s8 = false);
cudaError_t launch_rope_bf16(const ra_problem& p, int dtype, const void* q, const void* k,
                             const int32_t* pos, void* qo, void* ko, void* ws, cudaStream_t st);
cudaError_t read_prologue_status(uint32_t* out);
// The RoPE table of p.rot in the workspace's table slot; *tab receives its address.
cudaError_t launch_rope_table(const ra_problem& p, void* ws, const float2** tab, cudaStream_t st);

// INT4 attention.  dump_* select the tile whose intermediates are written when
// the dump pointers are non-null (dump variant of the kernel).
struct AttnDump {
  int bh = -1, q_tile = -1;
  int32_t* s = nullptr;
  int8_t* p = nullptr;
  int32_t* acc = nullptr;
};
// Fused-Q input of the attention: the raw Q, the positions and the RoPE table
// (of the problem's rotation mode); the kernel's widening warps apply the
// prologue's RoPE, rotation and per-token quantisation to Q themselves.
struct FusedQ {
  const void* q = nullptr;
  int dtype = 0;
  const int32_t* pos = nullptr;
  const float2* tab = nullptr;
};
cudaError_t launch_attn_int4(const ra_problem& p, const uint8_t* q4, const float* sq, const uint8_t* k4,
                             const float* sk, const uint8_t* v4, const float* sv, void* out, float* lse,
                             const AttnDump* dump, int mode, cudaStream_t st, int* unsupported,
                             const FusedQ* fq = nullptr);
cudaError_t read_attn_int4_status(uint32_t* out);
// block_k = 128: the CTA-pair kernel (ra_attn_int4_pair.cu).
cudaError_t launch_attn_int4_pair(const ra_problem& p, const uint8_t* q4, const float* sq, const uint8_t* k4,
                                  const float* sk, const uint8_t* v4, const float* sv, void* out, float* lse,
                                  const AttnDump* dump, int mode, cudaStream_t st, int* unsupported);
cudaError_t read_attn_pair_status(uint32_t* out);
cudaError_t read_attn_pair_diag(uint32_t* out);
cudaError_t read_attn_int4_diag(uint32_t* out);  // first timed-out wait site (diagnosis)

cudaError_t launch_attn_bf16(const ra_problem& p, const void* q, const void* k, const void* v, void* out,
                             float* lse, cudaStream_t st, int* unsupported);
cudaError_t read_attn_bf16_status(uint32_t* out);

}  // namespace ra
