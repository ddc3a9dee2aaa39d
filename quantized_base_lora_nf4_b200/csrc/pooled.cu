// The pooled adapter of QA-LoRA (abstract: the adapter's input is reduced group-wise, "decreasing the
// degrees of freedom of adaptation", so that the product B A can later be merged into the group
// zero points).  With P(X)[m, g] = mean of X[m, gL .. gL + L - 1] (the group of L inputs that shares a
// scale and zero point), the two adapter products that involve P(X) are small dense problems over
// the pooled input instead of full-K GEMMs:
//   T_save = bf16(s P(X) A^T)     [M, r], reduction over the K / L groups
//   dA     = dT^T P(X)            [r, K / L] fp32, reduction over the M tokens
// Both kernels read X once (16-byte loads), pool in fp32 and reduce in a fixed order.
#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx.cuh"

namespace qlr {

namespace {

__device__ __forceinline__ float lo_bf(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float hi_bf(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ float sum8(const uint4 q) {
  return ((lo_bf(q.x) + hi_bf(q.x)) + (lo_bf(q.y) + hi_bf(q.y))) + ((lo_bf(q.z) + hi_bf(q.z)) + (lo_bf(q.w) + hi_bf(q.w)));
}

// T_save: one warp per token.  Lanes walk the token's row in 16-byte chunks, the L / 8 lanes of a group
// combine their sums with shuffles, the group means go to shared memory, and lane j then forms
// T[m, j] = bf16(s sum_g mean_g A[j, g]) against the adapter staged (fp32, [G][r]) in shared memory.
template <int L>
__global__ void __launch_bounds__(256) pooled_lora_down_kernel(const uint16_t* __restrict__ X, int64_t M, int64_t K,
                                                               const uint16_t* __restrict__ A, int r, float s,
                                                               uint16_t* __restrict__ T) {
  constexpr int LPG = L / 8;  // lanes per group
  extern __shared__ float smem_f[];
  const int G = static_cast<int>(K / L);
  float* sA = smem_f;                    // [G][r]
  float* sXp = smem_f + G * r;           // [8 warps][G]
  pdl_launch_dependents();
  pdl_wait();
  for (int i = threadIdx.x; i < G * r; i += blockDim.x) {
    const int g = i / r, j = i - g * r;
    sA[i] = __uint_as_float(static_cast<uint32_t>(A[static_cast<int64_t>(j) * G + g]) << 16);
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* xp = sXp + warp * G;
  const int64_t n8 = K / 8;
  for (int64_t m = static_cast<int64_t>(blockIdx.x) * 8 + warp; m < M; m += static_cast<int64_t>(gridDim.x) * 8) {
    const uint4* xr = reinterpret_cast<const uint4*>(X + m * K);
#pragma unroll 4
    for (int64_t c0 = 0; c0 < n8; c0 += 32) {
      const int64_t i = c0 + lane;
      float v = i < n8 ? sum8(__ldg(xr + i)) : 0.f;
#pragma unroll
      for (int o = LPG / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (i < n8 && (lane & (LPG - 1)) == 0) xp[i / LPG] = v * (1.0f / L);  // L is a power of two: exact
    }
    __syncwarp();
    for (int j = lane; j < r; j += 32) {
      float acc = 0.f;
      for (int g = 0; g < G; ++g) acc = fmaf(xp[g], sA[g * r + j], acc);
      T[m * r + j] = static_cast<uint16_t>(pack_bf16x2_rn(s * acc, 0.f) & 0xFFFFu);
    }
    __syncwarp();
  }
}

// dA: one CTA per group g.  Thread t takes tokens t, t + 256, ...: the group mean of X[m] times the
// token's dT row, accumulated in fp32 registers, then summed over the CTA in a fixed order.
template <int L, int R>
__global__ void __launch_bounds__(256) pooled_dA_kernel(const uint16_t* __restrict__ X, int64_t M, int64_t K,
                                                        const uint16_t* __restrict__ dT, float* __restrict__ dA) {
  __shared__ float red[8][R];
  pdl_launch_dependents();
  pdl_wait();
  const int G = static_cast<int>(K / L), g = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float acc[R];
#pragma unroll
  for (int j = 0; j < R; ++j) acc[j] = 0.f;
  constexpr int kUnroll = L >= 128 ? 2 : 4;  // tokens in flight per thread (X loads of L / 8 chunks each)
#pragma unroll kUnroll
  for (int64_t m = threadIdx.x; m < M; m += 256) {
    const uint4* xr = reinterpret_cast<const uint4*>(X + m * K + static_cast<int64_t>(g) * L);
    float xs = 0.f;
#pragma unroll
    for (int c = 0; c < L / 8; ++c) xs += sum8(__ldg(xr + c));
    xs *= 1.0f / L;
    const uint4* tr = reinterpret_cast<const uint4*>(dT + m * R);
#pragma unroll
    for (int c = 0; c < R / 8; ++c) {
      const uint4 q = __ldg(tr + c);
      acc[8 * c + 0] = fmaf(lo_bf(q.x), xs, acc[8 * c + 0]);
      acc[8 * c + 1] = fmaf(hi_bf(q.x), xs, acc[8 * c + 1]);
      acc[8 * c + 2] = fmaf(lo_bf(q.y), xs, acc[8 * c + 2]);
      acc[8 * c + 3] = fmaf(hi_bf(q.y), xs, acc[8 * c + 3]);
      acc[8 * c + 4] = fmaf(lo_bf(q.z), xs, acc[8 * c + 4]);
      acc[8 * c + 5] = fmaf(hi_bf(q.z), xs, acc[8 * c + 5]);
      acc[8 * c + 6] = fmaf(lo_bf(q.w), xs, acc[8 * c + 6]);
      acc[8 * c + 7] = fmaf(hi_bf(q.w), xs, acc[8 * c + 7]);
    }
  }
#pragma unroll
  for (int j = 0; j < R; ++j) {
    float v = acc[j];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[warp][j] = v;
  }
  __syncthreads();
  if (threadIdx.x < R) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) t += red[w][threadIdx.x];
    dA[static_cast<int64_t>(threadIdx.x) * G + g] = t;
  }
}

size_t lora_down_smem(int64_t K, int L, int r) { return static_cast<size_t>(K / L) * (r + 8) * 4; }

template <int L>
cudaError_t launch_down_L(const uint16_t* X, int64_t M, int64_t K, const uint16_t* A, int r, float s, uint16_t* T,
                          cudaStream_t st) {
  const size_t smem = lora_down_smem(K, L, r);
  if (smem > 48 * 1024) {
    const cudaError_t e =
        cudaFuncSetAttribute(pooled_lora_down_kernel<L>, cudaFuncAttributeMaxDynamicSharedMemorySize, 160 * 1024);
    if (e != cudaSuccess) return e;
  }
  int64_t grid = (M + 7) / 8;
  const int64_t cap = static_cast<int64_t>(device_sm_count()) * 4;
  if (grid > cap) grid = cap;
  return launch_pdl(pooled_lora_down_kernel<L>, dim3(static_cast<unsigned>(grid)), dim3(256), smem, st, X, M, K, A, r,
                    s, T);
}

template <int L>
cudaError_t launch_dA_L(const uint16_t* X, int64_t M, int64_t K, const uint16_t* dT, int r, float* dA, cudaStream_t st) {
  const dim3 grid(static_cast<unsigned>(K / L)), block(256);
  switch (r) {
    case 8: return launch_pdl(pooled_dA_kernel<L, 8>, grid, block, 0, st, X, M, K, dT, dA);
    case 16: return launch_pdl(pooled_dA_kernel<L, 16>, grid, block, 0, st, X, M, K, dT, dA);
    case 32: return launch_pdl(pooled_dA_kernel<L, 32>, grid, block, 0, st, X, M, K, dT, dA);
    case 64: return launch_pdl(pooled_dA_kernel<L, 64>, grid, block, 0, st, X, M, K, dT, dA);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

bool pooled_adapter_supported(int64_t K, int L, int r) {
  return (L == 32 || L == 64 || L == 128) && K % L == 0 && (r == 8 || r == 16 || r == 32 || r == 64) &&
         lora_down_smem(K, L, r) <= 160 * 1024;
}

cudaError_t launch_pooled_lora_down(const uint16_t* X, int64_t M, int64_t K, int L, const uint16_t* A, int r, float s,
                                    uint16_t* T, cudaStream_t st) {
  switch (L) {
    case 32: return launch_down_L<32>(X, M, K, A, r, s, T, st);
    case 64: return launch_down_L<64>(X, M, K, A, r, s, T, st);
    case 128: return launch_down_L<128>(X, M, K, A, r, s, T, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_pooled_dA(const uint16_t* X, int64_t M, int64_t K, int L, const uint16_t* dT, int r, float* dA,
                             cudaStream_t st) {
  switch (L) {
    case 32: return launch_dA_L<32>(X, M, K, dT, r, dA, st);
    case 64: return launch_dA_L<64>(X, M, K, dT, r, dA, st);
    case 128: return launch_dA_L<128>(X, M, K, dT, r, dA, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace qlr
