// Memory-bound helpers: SwiGLU forward/backward, QA-LoRA group pooling of the adapter input,
// the expanded adapter used by the input gradient, and the fixed-order reduction of split
// partial sums.  Vectorised 16-byte loads/stores; grids sized in multiples of the SM count.
#include <cuda_bf16.h>

#include "common.cuh"
#include "gemm.cuh"
#include "ptx.cuh"

namespace qlr {

namespace {

__device__ __forceinline__ float lo_f(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float hi_f(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ float sigmoidf_(float g) { return 1.0f / (1.0f + expf(-g)); }

__global__ void swiglu_fwd_kernel(const uint4* __restrict__ G, const uint4* __restrict__ U, uint4* __restrict__ H,
                                  int64_t n8) {
  pdl_launch_dependents();
  pdl_wait();
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4 g = G[i], u = U[i];
    const uint32_t gv[4] = {g.x, g.y, g.z, g.w}, uv[4] = {u.x, u.y, u.z, u.w};
    uint32_t hv[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float g0 = lo_f(gv[j]), g1 = hi_f(gv[j]);
      const float h0 = g0 * sigmoidf_(g0) * lo_f(uv[j]);
      const float h1 = g1 * sigmoidf_(g1) * hi_f(uv[j]);
      hv[j] = pack_bf16x2_rn(h0, h1);
    }
    H[i] = make_uint4(hv[0], hv[1], hv[2], hv[3]);
  }
}

__global__ void swiglu_bwd_kernel(const uint4* __restrict__ dH, const uint4* __restrict__ G, const uint4* __restrict__ U,
                                  uint4* __restrict__ dG, uint4* __restrict__ dU, int64_t n8) {
  pdl_launch_dependents();
  pdl_wait();
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4 d = dH[i], g = G[i], u = U[i];
    const uint32_t dv[4] = {d.x, d.y, d.z, d.w}, gv[4] = {g.x, g.y, g.z, g.w}, uv[4] = {u.x, u.y, u.z, u.w};
    uint32_t og[4], ou[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float rg[2], ru[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float dh = h ? hi_f(dv[j]) : lo_f(dv[j]);
        const float gg = h ? hi_f(gv[j]) : lo_f(gv[j]);
        const float uu = h ? hi_f(uv[j]) : lo_f(uv[j]);
        const float sg = sigmoidf_(gg);
        rg[h] = dh * uu * sg * (1.0f + gg * (1.0f - sg));
        ru[h] = dh * gg * sg;
      }
      og[j] = pack_bf16x2_rn(rg[0], rg[1]);
      ou[j] = pack_bf16x2_rn(ru[0], ru[1]);
    }
    dG[i] = make_uint4(og[0], og[1], og[2], og[3]);
    dU[i] = make_uint4(ou[0], ou[1], ou[2], ou[3]);
  }
}

// Aexp[j, k] = bf16( A[j, k / L] / L ): the adapter seen by the un-pooled input.
__global__ void expand_kernel(const uint16_t* __restrict__ A, int r, int64_t K, int L, uint16_t* __restrict__ Aexp) {
  pdl_launch_dependents();
  pdl_wait();
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= r * K) return;
  const int64_t j = i / K, k = i % K;
  const float v = bf16_bits_to_f32(A[j * (K / L) + k / L]) / static_cast<float>(L);
  Aexp[i] = static_cast<uint16_t>(pack_bf16x2_rn(v, 0.f) & 0xFFFFu);
}

// Split-order sum of an adapter GEMM's parts + its output transform, one thread per output element.
__global__ void adapter_reduce_kernel(const AdapterParams p, int bn) {
  pdl_launch_dependents();
  pdl_wait();
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t split_stride = static_cast<int64_t>(p.m_tiles) * 128 * bn;
  if (i >= static_cast<int64_t>(p.Mm) * p.r) return;
  int64_t m, j;
  if (p.out_mode == ADAPTER_COLS_F32) {  // consecutive threads walk output columns (coalesced stores)
    j = i / p.Mm;
    m = i % p.Mm;
  } else {
    m = i / p.r;
    j = i % p.r;
  }
  float acc = 0.f;
  for (int s = 0; s < p.splits; ++s) acc += p.part[s * split_stride + m * bn + j];
  if (p.out_mode == ADAPTER_ROWS_BF16)
    static_cast<uint16_t*>(p.out)[m * p.ld_out + j] = static_cast<uint16_t>(pack_bf16x2_rn(p.scale * acc, 0.f) & 0xFFFFu);
  else if (p.out_mode == ADAPTER_ROWS_F32)
    static_cast<float*>(p.out)[m * p.ld_out + j] = acc;
  else
    static_cast<float*>(p.out)[j * p.ld_out + m] = acc;
}

// The pooled transposed output out[j, g] = (sum of the L rows of group g) / L: a block of 256 threads
// covers 256 consecutive rows of one column j; each thread sums its row's splits, warps add their 32
// rows by shuffles, and the group totals combine the warp sums (L = 32, 64 or 128 divides 256).
__global__ void adapter_reduce_pooled_kernel(const AdapterParams p, int bn) {
  __shared__ float warp_sum[8];
  pdl_launch_dependents();
  pdl_wait();
  const int64_t split_stride = static_cast<int64_t>(p.m_tiles) * 128 * bn;
  const int64_t blocks_per_col = (p.Mm + 255) / 256;
  const int64_t j = blockIdx.x / blocks_per_col;
  const int64_t m = (blockIdx.x % blocks_per_col) * 256 + threadIdx.x;
  float v = 0.f;
  if (m < p.Mm)
    for (int s = 0; s < p.splits; ++s) v += p.part[s * split_stride + m * bn + j];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) warp_sum[threadIdx.x >> 5] = v;
  __syncthreads();
  const int L = p.pool_L, wpg = L / 32;
  if (threadIdx.x < 256 / L) {
    float g = 0.f;
    for (int w = 0; w < wpg; ++w) g += warp_sum[threadIdx.x * wpg + w];
    const int64_t og = ((blockIdx.x % blocks_per_col) * 256) / L + threadIdx.x;
    if (og * L < p.Mm) static_cast<float*>(p.out)[j * p.ld_out + og] = g / static_cast<float>(L);
  }
}

unsigned grid_for(int64_t n_items, int threads) {
  const int64_t want = (n_items + threads - 1) / threads;
  const int64_t cap = static_cast<int64_t>(device_sm_count()) * 8;
  return static_cast<unsigned>(want < 1 ? 1 : (want > cap ? cap : want));
}

}  // namespace

cudaError_t launch_adapter_reduce(const AdapterParams& p, int bn, cudaStream_t st) {
  if (p.out_mode == ADAPTER_COLS_F32 && p.pool_L > 1) {
    const int64_t blocks = (static_cast<int64_t>(p.Mm) + 255) / 256 * p.r;
    return launch_pdl(adapter_reduce_pooled_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st, p, bn);
  }
  const int64_t n = static_cast<int64_t>(p.Mm) * p.r;
  if (n == 0) return cudaSuccess;
  return launch_pdl(adapter_reduce_kernel, dim3(static_cast<unsigned>((n + 255) / 256)), dim3(256), 0, st, p, bn);
}

cudaError_t launch_swiglu_fwd(const uint16_t* G, const uint16_t* U, uint16_t* H, int64_t n, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const int64_t n8 = n / 8;
  return launch_pdl(swiglu_fwd_kernel, dim3(grid_for(n8, 256)), dim3(256), 0, st, reinterpret_cast<const uint4*>(G),
                    reinterpret_cast<const uint4*>(U), reinterpret_cast<uint4*>(H), n8);
}

cudaError_t launch_swiglu_bwd(const uint16_t* dH, const uint16_t* G, const uint16_t* U, uint16_t* dG, uint16_t* dU,
                              int64_t n, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const int64_t n8 = n / 8;
  return launch_pdl(swiglu_bwd_kernel, dim3(grid_for(n8, 256)), dim3(256), 0, st, reinterpret_cast<const uint4*>(dH),
                    reinterpret_cast<const uint4*>(G), reinterpret_cast<const uint4*>(U), reinterpret_cast<uint4*>(dG),
                    reinterpret_cast<uint4*>(dU), n8);
}

cudaError_t launch_expand_adapter(const uint16_t* A, int r, int64_t K, int L, uint16_t* Aexp, cudaStream_t st) {
  const int64_t n = static_cast<int64_t>(r) * K;
  return launch_pdl(expand_kernel, dim3(static_cast<unsigned>((n + 255) / 256)), dim3(256), 0, st, A, r, K, L, Aexp);
}

}  // namespace qlr
