// One-time, per-device host set-up (a kernel's shared-memory opt-in, the
// device address of a __device__ symbol) that stays valid only as long as the
// CUDA context it was done in: after cudaDeviceReset the device gets a new
// context, the old function attributes are gone and symbols may move.  The
// set-up is therefore keyed by the context's unique id (cuCtxGetId) and
// redone when it changes; concurrent first callers are serialised.
#pragma once

#include <cuda_runtime.h>

#include <mutex>

namespace attn {

constexpr int kMaxDevices = 64;

// Unique id of the calling thread's current CUDA context, or 0 when there is
// none yet (the set-up then runs again on the next call).
unsigned long long current_context_id();

struct PerContextOnce {
  std::mutex mu;
  unsigned long long ctx[kMaxDevices] = {};
  cudaError_t result[kMaxDevices] = {};
};

// Runs setup(dev) for the current device once per context; returns its result.
template <class F>
cudaError_t once_per_context(PerContextOnce& st, F&& setup) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  const unsigned long long id = current_context_id();
  std::lock_guard<std::mutex> lock(st.mu);
  if (id == 0 || st.ctx[dev] != id) {
    st.result[dev] = setup(dev);
    st.ctx[dev] = id;
  }
  return st.result[dev];
}

}  // namespace attn
