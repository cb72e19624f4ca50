// attn_decode_splitkv_noalloc: the split-KV decode for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc or any allocator: a plugin inside a
// serving process whose device memory is all handed out by the host
// application's own pool, or a latency-critical decode loop where an
// allocation (which may synchronise the device) is not allowed.  They can
// still pass their inputs and outputs, so this entry point takes its split
// workspace from a fixed array in device memory that the library itself
// declares.  That array exists on every GPU that loads the library and stays
// there until the process exits.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "attn.h"
#include "host_once.h"

namespace {

constexpr size_t kNoAllocWorkspaceBytes = 32u << 20;  // 32 MiB

// The shared scratch.  In host code this name is only a stand-in for the
// symbol, not a device address: the address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_workspace[kNoAllocWorkspaceBytes];

attn::PerContextOnce g_setup;
void* g_workspace_ptr[attn::kMaxDevices] = {};

// Once per device (and again in a new context, e.g. after cudaDeviceReset),
// with that device current: the device address of the array.
attn_status_t workspace_for_current_device(void** out) {
  const cudaError_t e = attn::once_per_context(g_setup, [](int dev) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_workspace) != cudaSuccess || ptr == nullptr) {
      g_workspace_ptr[dev] = nullptr;
      return cudaErrorInvalidSymbol;
    }
    g_workspace_ptr[dev] = ptr;
    return cudaSuccess;
  });
  if (e == cudaErrorInvalidDevice) return ATTN_ERR_UNSUPPORTED;
  if (e != cudaSuccess) return ATTN_ERR_CUDA;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_setup.mu);
  *out = g_workspace_ptr[dev];
  return *out ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace

extern "C" {

attn_status_t attn_decode_splitkv_noalloc(const void* q, const void* k_cache,
                                          const void* v_cache, void* o, float* lse,
                                          const int32_t* kv_lens, int B, int Hq, int Hkv, int Lq,
                                          int Lk_max, int d, float scale, int num_splits,
                                          void* stream) {
  const size_t need = attn_decode_workspace_size(B, Hq, Hkv, Lq, Lk_max, d, num_splits);
  if (need == 0) return ATTN_ERR_INVALID_ARG;
  if (need > kNoAllocWorkspaceBytes) return ATTN_ERR_WORKSPACE;
  if (!q || !k_cache || !v_cache || !o || !lse || !kv_lens) return ATTN_ERR_INVALID_ARG;
  void* ws = nullptr;
  attn_status_t st = workspace_for_current_device(&ws);
  if (st != ATTN_OK) return st;
  return attn_decode_splitkv(q, k_cache, v_cache, o, lse, kv_lens, B, Hq, Hkv, Lq, Lk_max, d,
                             scale, num_splits, ws, kNoAllocWorkspaceBytes, stream);
}

}  // extern "C"
