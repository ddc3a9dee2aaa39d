// Adapter gradients for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc: a host framework that owns every byte of device memory
// through its own pool and forbids other allocations, a runtime that works from a fixed memory
// plan decided ahead of time, or a latency-critical loop that must not pay cudaMalloc/cudaFree
// (cudaFree synchronises the whole device).  qlr_backward_lora needs a scratch workspace for its
// split reductions; this entry point takes the scratch from a fixed array compiled into the
// library instead, so the caller passes only inputs and outputs.
//
// The array lives in device global memory of every GPU that loads the library, until the process
// exits.  Its device address is looked up with cudaGetSymbolAddress once per device, on the first
// call made while that device is current.  Every call shares the one array, which keeps whatever
// the last call left in it; the split partial sums stored there are fully overwritten before they
// are read, so nothing has to start at zero.  Calls that may run at the same time on the GPU (on
// different streams, or from different host threads) race on the array and must be serialised.
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"

namespace {

static __device__ __align__(256) uint8_t g_noalloc_scratch[QLR_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

// Device address of g_noalloc_scratch on the current device (nullptr if it cannot be resolved).
void* scratch_address() {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace

extern "C" int qlr_backward_lora_noalloc(const qlr_qweight* w, const uint16_t* X, const uint16_t* dY,
                                         const uint16_t* T_save, const uint16_t* B, int64_t M, int r, float s,
                                         int pooled, float* dA, float* dB, uint16_t* dT_out, int32_t* status,
                                         void* stream) {
  const size_t need = qlr_backward_lora_workspace_bytes(w, M, r, pooled);
  if (need > QLR_NOALLOC_SCRATCH_BYTES) return QLR_ERR_WORKSPACE;  // larger than the built-in scratch
  void* scratch = need ? scratch_address() : nullptr;
  if (need && !scratch) return QLR_ERR_CUDA;
  return qlr_backward_lora(w, X, dY, T_save, B, M, r, s, pooled, dA, dB, dT_out, scratch,
                           need ? QLR_NOALLOC_SCRATCH_BYTES : 0, status, stream);
}
