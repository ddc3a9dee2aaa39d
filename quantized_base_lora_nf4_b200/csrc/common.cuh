// Shared declarations of the library's kernels and host helpers.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/qlr.h"

namespace qlr {

struct Levels {
  float v[16];
};

void nf_levels_f32(int k, float* out);
Levels levels_for(int bits);

// Nearest-level decision of the NF-k quantiser as a table over 33 cells of width 1/16 on [-1, 1]:
// cell k = round-half-even(16 u) + 16, code(u) = base[k] + (u >= t[k]) (t[k] = +inf: no threshold).
struct NfTable {
  float t[33];
  int32_t base[33];
};
// Builds the table of levels_for(bits) (cached); false when a cell would hold two thresholds.
bool nf_decision_table(int bits, NfTable* out);

// Status sink used when the caller passes no status word.
int32_t* status_or_sink(int32_t* status);

// Bound (SM clock cycles) given to the pipeline waits of the kernels launched next (qlr_set_wait_limit).
long long wait_limit_cycles();

__device__ __forceinline__ void report(int32_t* status, int32_t code) { atomicExch(status, code); }

// ---- launch wrappers (quantize.cu) ----
cudaError_t launch_quantize_nfk(const float* W, int64_t n_elems, int bits, int block, int dq_block,
                                const qlr_qweight* out, int32_t* status, cudaStream_t st);
cudaError_t launch_quantize_int4g(const float* W, int64_t N, int64_t K, int group, const qlr_qweight* out,
                                  int32_t* status, cudaStream_t st);
cudaError_t launch_dequant(const qlr_qweight* w, uint16_t* out, cudaStream_t st);
cudaError_t launch_merge(const qlr_qweight* w, const uint16_t* A, const uint16_t* B, int r, float s,
                         cudaStream_t st);

// ---- elementwise (elementwise.cu) ----
cudaError_t launch_swiglu_fwd(const uint16_t* G, const uint16_t* U, uint16_t* H, int64_t n, cudaStream_t st);
cudaError_t launch_swiglu_bwd(const uint16_t* dH, const uint16_t* G, const uint16_t* U, uint16_t* dG,
                              uint16_t* dU, int64_t n, cudaStream_t st);
cudaError_t launch_expand_adapter(const uint16_t* A, int r, int64_t K, int L, uint16_t* Aexp, cudaStream_t st);
// The pooled adapter (pooled.cu): T_save = bf16(s P(X) A^T) and dA = dT^T P(X) straight from X.
bool pooled_adapter_supported(int64_t K, int L, int r);
cudaError_t launch_pooled_lora_down(const uint16_t* X, int64_t M, int64_t K, int L, const uint16_t* A, int r, float s,
                                    uint16_t* T, cudaStream_t st);
size_t pooled_dA_workspace_bytes(int64_t M, int64_t K, int L, int r);
cudaError_t launch_pooled_dA(const uint16_t* X, int64_t M, int64_t K, int L, const uint16_t* dT, int r, float* dA,
                             float* part, cudaStream_t st);

// The rank-r products T = bf16(s X A^T) (A [r, K]) and dT = bf16(s dY B) (B [K, r], w_is_k_by_r), r = 16, 32
// or 64, at 1024 or more tokens in one launch: clusters of 4 CTAs split K and sum their partial tiles in
// shared memory in a fixed order (skinny.cu).  No workspace.
bool skinny_supported(int64_t M, int64_t K, int r);
cudaError_t launch_skinny(const uint16_t* X, int64_t M, int64_t K, const uint16_t* W, bool w_is_k_by_r, int r, float s,
                          uint16_t* out, int32_t* status, long long wait_cycles, cudaStream_t st);

// T = bf16(s X A^T) for 1..16 tokens without pooling: one fixed-order reduction kernel, no workspace.
bool lora_down_small_supported(int64_t M);
cudaError_t launch_lora_down_small(const uint16_t* X, int64_t M, int64_t K, const uint16_t* A, int r, float s,
                                   uint16_t* T, cudaStream_t st);

int device_sm_count();

// Decode-shape forward (1..16 tokens) of a 4-bit NF weight with double quantisation (decode.cu).
bool decode_supported(const qlr_qweight* w, int64_t M);
cudaError_t launch_decode(const qlr_qweight* w, const uint16_t* X, int64_t M, const uint16_t* B, int r,
                          const uint16_t* T_save, uint16_t* Y, int32_t* status, cudaStream_t st);

// Counts kernel launches issued by this library (reported by qlr_launch_count).
void count_launch(int n = 1);

// Raises a kernel's dynamic shared-memory limit to `bytes` on the current device, once per (kernel,
// device): the attribute belongs to the device that is current when it is set, so a process that
// drives several GPUs needs it on each.
cudaError_t ensure_max_dynamic_smem_fn(const void* kern, int bytes);
template <typename Kern>
cudaError_t ensure_max_dynamic_smem(Kern kern, int bytes) {
  return ensure_max_dynamic_smem_fn(reinterpret_cast<const void*>(kern), bytes);
}

// Launches a hot-path kernel with programmatic stream serialisation, so that its launch and set-up
// overlap the tail of the previous kernel on the stream; the kernel itself calls pdl_wait before it
// reads or writes global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  count_launch();
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace qlr
