// bf16 FlashAttention forward (selective-precision fallback) on sm_100a.
#include <cuda_runtime.h>

#include <cstdint>

#include "ra_common.cuh"
#include "ra_internal.h"

namespace ra {
namespace {
__device__ uint32_t g_bf16_status = 0;
}  // namespace

cudaError_t launch_attn_bf16(const ra_problem&, const void*, const void*, const void*, void*, float*,
                             cudaStream_t, int* unsupported) {
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
