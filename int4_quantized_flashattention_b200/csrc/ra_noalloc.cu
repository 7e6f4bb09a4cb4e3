// Allocation-free variant of the fused prologue (ra_rope_rotate_quant_noalloc).
//
// Some callers cannot allocate device memory when they run the prologue: an
// inference-engine plugin whose execute step may not call the allocator, or a
// service that reserves a fixed device-memory budget at start-up and forbids
// allocation afterwards.  For them this entry point takes no workspace
// argument: the scratch space lives in a fixed-size array in the library's
// own device memory, which every GPU that loads the library holds until the
// process exits.
#include <cuda_runtime.h>

#include <mutex>

#include "ra_internal.h"

namespace {

constexpr size_t kScratchBytes = RA_STATIC_SCRATCH_BYTES;

// The scratch array.  In host code this name only stands for the symbol; its
// device address is obtained with cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 256;
std::mutex g_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once per
// device (the first call on a device does it, with that device current).
ra_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return RA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return RA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return RA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return RA_OK;
}

}  // namespace

extern "C" ra_status ra_rope_rotate_quant_noalloc(const ra_problem* p, int in_dtype, const void* q,
                                                  const void* k, const void* v, const int32_t* pos,
                                                  uint8_t* q4, float* sq, uint8_t* k4, float* sk,
                                                  float* k_mean, uint8_t* v4, float* sv, int32_t* v_colsum,
                                                  void* stream) {
  const size_t need = ra_workspace_bytes(p);
  if (need == 0) return RA_ERR_INVALID_ARG;
  if (need > kScratchBytes) return RA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  const ra_status st = scratch_address(&scratch);
  if (st != RA_OK) return st;
  // Every scratch byte the prologue reads is written earlier in the same call,
  // so the previous call's contents need no clearing.
  return ra_rope_rotate_quant(p, in_dtype, q, k, v, pos, q4, sq, k4, sk, k_mean, v4, sv, v_colsum, scratch,
                              kScratchBytes, stream);
}
