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

// Looked-up addresses, one per device, each with the context it belongs to:
// a device reset (or any other teardown of the primary context) reloads the
// library's device code, and the array may then live at another address, so
// an entry is only used while its context is the current one.
constexpr int kMaxDevices = 256;
struct Entry {
  void* ctx = nullptr;
  void* addr = nullptr;
};
std::mutex g_mutex;
Entry g_entries[kMaxDevices];

// The current context of the calling thread (driver entry point, fetched once).
void* current_context() {
  using Fn = int (*)(void**);
  static Fn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<Fn>(p);
  }
  void* ctx = nullptr;
  if (fn == nullptr || fn(&ctx) != 0) return nullptr;
  return ctx;
}

// Device address of the scratch array on the current device and context,
// looked up with that device current on the first call in a context.
ra_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return RA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return RA_ERR_UNSUPPORTED;
  void* ctx = current_context();   // NULL before the runtime has made a context current
  std::lock_guard<std::mutex> lock(g_mutex);
  Entry& e = g_entries[dev];
  if (ctx == nullptr || e.addr == nullptr || e.ctx != ctx) {
    // The lookup itself makes the device's primary context current if needed.
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return RA_ERR_CUDA;
    e.addr = p;
    e.ctx = current_context();
  }
  *out = e.addr;
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
