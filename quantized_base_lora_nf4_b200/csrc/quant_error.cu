// Squared reconstruction error of NF-k quantisation, ||W - dequant(Q(W))||_F^2: the per-option input of
// LQ-LoRA's budgeted allocation (qlr_lqlora_allocate).  The weight is quantised into the caller's
// workspace with the library's quantiser; the error is summed in fp64 with a fixed thread-to-element
// mapping and fixed reduction trees, so it is deterministic.
#include "common.cuh"
#include "nfk.cuh"

namespace qlr {

namespace {

constexpr int kErrCtas = 1024;

__device__ __forceinline__ double block_sum(double v, double* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  double t = 0.0;
  if (threadIdx.x == 0)
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) t += red[w];
  return t;
}

__global__ void __launch_bounds__(256) sq_error_kernel(const float* __restrict__ W, int64_t n, const nfk::View v,
                                                       double* __restrict__ partial) {
  __shared__ double red[8];
  double acc = 0.0;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const double d = static_cast<double>(W[i]) - static_cast<double>(nfk::dequant_at(v, i));  // exact
    acc += d * d;
  }
  const double t = block_sum(acc, red);
  if (threadIdx.x == 0) partial[blockIdx.x] = t;
}

__global__ void __launch_bounds__(256) sum_partials_kernel(const double* __restrict__ partial, int n,
                                                           double* __restrict__ out) {
  __shared__ double red[8];
  double acc = 0.0;
  for (int i = threadIdx.x; i < n; i += blockDim.x) acc += partial[i];
  const double t = block_sum(acc, red);
  if (threadIdx.x == 0) *out = t;
}

inline size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

}  // namespace qlr

using namespace qlr;

extern "C" size_t qlr_nf_quant_error_workspace_bytes(int64_t N, int64_t K, int bits, int block, int dq_block) {
  size_t total = 0;
  for (int part : {QLR_PART_CODES, dq_block ? QLR_PART_C1_FP8 : QLR_PART_C1, QLR_PART_S2}) {
    if (part == QLR_PART_S2 && !dq_block) continue;
    const int64_t b = qlr_qweight_part_bytes(QLR_FMT_NFK, N, K, bits, block, dq_block, 0, part);
    if (b < 0) return 0;
    total += al256(static_cast<size_t>(b));
  }
  return total + al256(kErrCtas * sizeof(double));
}

extern "C" int qlr_nf_quant_error(const float* W, int64_t N, int64_t K, int bits, int block, int dq_block,
                                  double* err_out, void* workspace, size_t workspace_bytes, int32_t* status,
                                  void* stream) {
  if (!W || !err_out || N <= 0 || K <= 0) return QLR_ERR_ARG;
  const size_t need = qlr_nf_quant_error_workspace_bytes(N, K, bits, block, dq_block);
  if (need == 0) return QLR_ERR_ARG;  // bits, block or dq_block not supported
  if ((N * K) % 128) return QLR_ERR_SHAPE;
  if (!workspace || workspace_bytes < need) return QLR_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) || (reinterpret_cast<uintptr_t>(W) & 15u) ||
      (reinterpret_cast<uintptr_t>(err_out) & 7u))
    return QLR_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the quantised weight lives in the workspace
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  qlr_qweight q{};
  q.fmt = QLR_FMT_NFK;
  q.N = N;
  q.K = K;
  q.bits = bits;
  q.block = block;
  q.dq_block = dq_block;
  size_t off = 0;
  q.codes = ws;
  off += al256(static_cast<size_t>(qlr_qweight_part_bytes(QLR_FMT_NFK, N, K, bits, block, dq_block, 0, QLR_PART_CODES)));
  if (dq_block) {
    q.c1_fp8 = ws + off;
    off += al256(static_cast<size_t>(qlr_qweight_part_bytes(QLR_FMT_NFK, N, K, bits, block, dq_block, 0, QLR_PART_C1_FP8)));
    q.s2 = reinterpret_cast<float*>(ws + off);
    off += al256(static_cast<size_t>(qlr_qweight_part_bytes(QLR_FMT_NFK, N, K, bits, block, dq_block, 0, QLR_PART_S2)));
  } else {
    q.c1 = reinterpret_cast<float*>(ws + off);
    off += al256(static_cast<size_t>(qlr_qweight_part_bytes(QLR_FMT_NFK, N, K, bits, block, dq_block, 0, QLR_PART_C1)));
  }
  double* partial = reinterpret_cast<double*>(ws + off);
  int32_t* stat = status_or_sink(status);
  if (launch_quantize_nfk(W, N * K, bits, block, dq_block, &q, stat, st) != cudaSuccess) return QLR_ERR_CUDA;
  count_launch(2);
  sq_error_kernel<<<kErrCtas, 256, 0, st>>>(W, N * K, nfk::view_of(&q), partial);
  sum_partials_kernel<<<1, 256, 0, st>>>(partial, kErrCtas, err_out);
  return cudaGetLastError() == cudaSuccess ? QLR_OK : QLR_ERR_CUDA;
}
