// The pooled adapter of QA-LoRA (abstract: the adapter's input is reduced group-wise, which gives the
// adaptation fewer degrees of freedom, so that the product B A can later be merged into the group
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

// T_save: one CTA per pair of tokens, K / 16 threads per token (each owns 4 consecutive 16-byte
// chunks = 32 inputs, all loaded before any arithmetic).  The L / 32 threads of a group combine their
// sums with shuffles and the group means go to shared memory; then 8 threads per output T[m, j]
// split the K / L-long dot product with A and combine it with shuffles, in a fixed order.
constexpr int kDownTok = 2;

template <int L>
__global__ void __launch_bounds__(256) pooled_lora_down_kernel(const uint16_t* __restrict__ X, int64_t M, int64_t K,
                                                               const uint16_t* __restrict__ A, int r, float s,
                                                               uint16_t* __restrict__ T) {
  constexpr int TPG = L / 32;  // threads per group (1, 2 or 4)
  extern __shared__ float smem_f[];
  const int G = static_cast<int>(K / L);
  const int tpt = static_cast<int>(K / 32);  // threads per token
  float* sXp = smem_f;                       // [kDownTok][G]
  pdl_launch_dependents();
  pdl_wait();
  const int64_t m0 = static_cast<int64_t>(blockIdx.x) * kDownTok;
  // pooling: thread i of token tk sums inputs [32 i, 32 i + 32) of row m0 + tk
  // the loop bound is uniform over the CTA so that every lane reaches the shuffles; a group's TPG
  // threads are adjacent lanes and never straddle the end (tpt is a multiple of TPG)
  for (int base = 0; base < kDownTok * tpt; base += blockDim.x) {
    const int i = base + threadIdx.x;
    const bool in = i < kDownTok * tpt;
    const int tk = in ? i / tpt : 0, c = in ? i - tk * tpt : 0;
    float v = 0.f;
    if (in && m0 + tk < M) {
      const uint4* xr = reinterpret_cast<const uint4*>(X + (m0 + tk) * K) + 4 * c;
      const uint4 q0 = __ldg(xr), q1 = __ldg(xr + 1), q2 = __ldg(xr + 2), q3 = __ldg(xr + 3);
      v = (sum8(q0) + sum8(q1)) + (sum8(q2) + sum8(q3));
    }
#pragma unroll
    for (int o = TPG / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (in && (c & (TPG - 1)) == 0) sXp[tk * G + c / TPG] = v * (1.0f / L);  // L is a power of two: exact
  }
  __syncthreads();
  // T[m0 + tk, j]: 8 threads per output, group g = sub, sub + 8, ...
  const int sub = threadIdx.x & 7;
  for (int o = threadIdx.x >> 3; o < kDownTok * r; o += blockDim.x >> 3) {
    const int tk = o / r, j = o - tk * r;
    const float* xp = sXp + tk * G;
    const uint16_t* arow = A + static_cast<int64_t>(j) * G;
    float acc = 0.f;
    for (int g = sub; g < G; g += 8) acc = fmaf(xp[g], __uint_as_float(static_cast<uint32_t>(__ldg(arow + g)) << 16), acc);
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    acc += __shfl_xor_sync(0xffffffffu, acc, 4);
    if (sub == 0 && m0 + tk < M)
      T[(m0 + tk) * r + j] = static_cast<uint16_t>(pack_bf16x2_rn(s * acc, 0.f) & 0xFFFFu);
  }
}

// dA, first pass: one CTA per block of 16 tokens pools their rows (coalesced, as above) into shared
// memory with their dT rows, and writes the block's partial dA[j, g] = sum_m dT[m, j] mean_g(X[m]).
constexpr int kDaTok = 16;

template <int L>
__global__ void __launch_bounds__(256) pooled_dA_partial_kernel(const uint16_t* __restrict__ X, int64_t M, int64_t K,
                                                                const uint16_t* __restrict__ dT, int r,
                                                                float* __restrict__ part) {
  constexpr int TPG = L / 32;
  extern __shared__ float smem_f[];
  const int G = static_cast<int>(K / L);
  const int tpt = static_cast<int>(K / 32);
  float* sXp = smem_f;                  // [kDaTok][G]
  float* sdT = smem_f + kDaTok * G;     // [kDaTok][r]
  pdl_launch_dependents();
  pdl_wait();
  const int64_t m0 = static_cast<int64_t>(blockIdx.x) * kDaTok;
#pragma unroll 4
  for (int base = 0; base < kDaTok * tpt; base += blockDim.x) {  // uniform bound: see above
    const int i = base + threadIdx.x;
    const bool in = i < kDaTok * tpt;
    const int tk = in ? i / tpt : 0, c = in ? i - tk * tpt : 0;
    float v = 0.f;
    if (in && m0 + tk < M) {
      const uint4* xr = reinterpret_cast<const uint4*>(X + (m0 + tk) * K) + 4 * c;
      const uint4 q0 = __ldg(xr), q1 = __ldg(xr + 1), q2 = __ldg(xr + 2), q3 = __ldg(xr + 3);
      v = (sum8(q0) + sum8(q1)) + (sum8(q2) + sum8(q3));
    }
#pragma unroll
    for (int o = TPG / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (in && (c & (TPG - 1)) == 0) sXp[tk * G + c / TPG] = v * (1.0f / L);
  }
  for (int i = threadIdx.x; i < kDaTok * r; i += blockDim.x) {
    const int tk = i / r;
    sdT[i] = (m0 + tk < M) ? __uint_as_float(static_cast<uint32_t>(dT[m0 * r + i]) << 16) : 0.f;
  }
  __syncthreads();
  float* out = part + static_cast<int64_t>(blockIdx.x) * r * G;
  for (int o = threadIdx.x; o < r * G; o += blockDim.x) {
    const int j = o / G, g = o - j * G;
    float acc = 0.f;
#pragma unroll
    for (int tk = 0; tk < kDaTok; ++tk) acc = fmaf(sdT[tk * r + j], sXp[tk * G + g], acc);
    out[o] = acc;
  }
}

// dA, second pass: dA[j, g] = sum over the token blocks of the partials.  A CTA takes 32 consecutive
// outputs; warp w sums the blocks w, w + 8, ... (coalesced rows of 32 partials, several loads in
// flight) and the eight warp sums are added in warp order, so the result is deterministic.
__global__ void __launch_bounds__(256) pooled_dA_reduce_kernel(const float* __restrict__ part, int nblk, int n,
                                                               float* __restrict__ dA) {
  __shared__ float red[8][32];
  pdl_launch_dependents();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int o = blockIdx.x * 32 + lane;
  float acc = 0.f;
  if (o < n) {
#pragma unroll 4
    for (int b = warp; b < nblk; b += 8) acc += part[static_cast<int64_t>(b) * n + o];
  }
  red[warp][lane] = acc;
  __syncthreads();
  if (warp == 0 && o < n) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) t += red[w][lane];
    dA[o] = t;
  }
}

size_t lora_down_smem(int64_t K, int L) { return static_cast<size_t>(K / L) * kDownTok * 4; }
size_t dA_smem(int64_t K, int L, int r) { return (static_cast<size_t>(K / L) + r) * kDaTok * 4; }

template <typename Kern>
cudaError_t allow_smem(Kern kern, size_t smem) {
  if (smem <= 48 * 1024) return cudaSuccess;
  return ensure_max_dynamic_smem(kern, static_cast<int>(smem));
}

template <int L>
cudaError_t launch_down_L(const uint16_t* X, int64_t M, int64_t K, const uint16_t* A, int r, float s, uint16_t* T,
                          cudaStream_t st) {
  const size_t smem = lora_down_smem(K, L);
  cudaError_t e = allow_smem(pooled_lora_down_kernel<L>, smem);
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>((M + kDownTok - 1) / kDownTok);
  return launch_pdl(pooled_lora_down_kernel<L>, dim3(grid), dim3(256), smem, st, X, M, K, A, r, s, T);
}

template <int L>
cudaError_t launch_dA_L(const uint16_t* X, int64_t M, int64_t K, const uint16_t* dT, int r, float* dA, float* part,
                        cudaStream_t st) {
  const size_t smem = dA_smem(K, L, r);
  cudaError_t e = allow_smem(pooled_dA_partial_kernel<L>, smem);
  if (e != cudaSuccess) return e;
  const int nblk = static_cast<int>((M + kDaTok - 1) / kDaTok);
  e = launch_pdl(pooled_dA_partial_kernel<L>, dim3(static_cast<unsigned>(nblk)), dim3(256), smem, st, X, M, K, dT, r,
                 part);
  if (e != cudaSuccess) return e;
  const int n = static_cast<int>(r * (K / L));
  return launch_pdl(pooled_dA_reduce_kernel, dim3(static_cast<unsigned>((n + 31) / 32)), dim3(256), 0, st,
                    static_cast<const float*>(part), nblk, n, dA);
}

}  // namespace

bool pooled_adapter_supported(int64_t K, int L, int r) {
  return (L == 32 || L == 64 || L == 128) && K % L == 0 && (r == 8 || r == 16 || r == 32 || r == 64) &&
         dA_smem(K, L, r) <= 160 * 1024;
}

size_t pooled_dA_workspace_bytes(int64_t M, int64_t K, int L, int r) {
  return static_cast<size_t>((M + kDaTok - 1) / kDaTok) * r * (K / L) * 4;
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
                             float* part, cudaStream_t st) {
  switch (L) {
    case 32: return launch_dA_L<32>(X, M, K, dT, r, dA, part, st);
    case 64: return launch_dA_L<64>(X, M, K, dT, r, dA, part, st);
    case 128: return launch_dA_L<128>(X, M, K, dT, r, dA, part, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace qlr
