// Memory-bound helpers: SwiGLU forward/backward, QA-LoRA group pooling of the adapter input,
// the expanded adapter used by the input gradient, and the fixed-order reduction of split
// partial sums.  Vectorised 16-byte loads/stores; grids sized in multiples of the SM count.
#include <cuda_bf16.h>

#include "common.cuh"
#include "gemm.cuh"
#include "ptx.cuh"
#include "swiglu.cuh"

namespace qlr {

namespace {

__device__ __forceinline__ float lo_f(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float hi_f(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

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
      hv[j] = pack_bf16x2_rn(swiglu_h(lo_f(gv[j]), lo_f(uv[j])), swiglu_h(hi_f(gv[j]), hi_f(uv[j])));
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
        swiglu_grads(dh, gg, uu, rg[h], ru[h]);
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

// Split-order sum of an adapter GEMM's parts + its output transform, row outputs (T_save, dT: bf16 scaled;
// dB: fp32): a thread sums four consecutive columns of one row, every split's 16 bytes loaded before any
// addition, and adds them in split order (deterministic, and the same sums as one column per thread).
__global__ void __launch_bounds__(256) adapter_reduce_rows_kernel(const AdapterParams p, int bn) {
  pdl_launch_dependents();
  pdl_wait();
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int q = p.r / 4;  // float4 groups per row
  if (i >= static_cast<int64_t>(p.Mm) * q) return;
  const int64_t m = i / q;
  const int j = static_cast<int>(i - m * q) * 4;
  const int64_t split_stride = static_cast<int64_t>(p.m_tiles) * 128 * bn;
  const float* src = p.part + m * bn + j;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  int s = 0;
  for (; s + 4 <= p.splits; s += 4) {  // four splits' loads in flight, summed in order
    float4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = __ldg(reinterpret_cast<const float4*>(src + (s + u) * split_stride));
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      acc.x += v[u].x;
      acc.y += v[u].y;
      acc.z += v[u].z;
      acc.w += v[u].w;
    }
  }
  for (; s < p.splits; ++s) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(src + s * split_stride));
    acc.x += v.x;
    acc.y += v.y;
    acc.z += v.z;
    acc.w += v.w;
  }
  if (p.out_mode == ADAPTER_ROWS_BF16) {
    uint2 w;
    w.x = pack_bf16x2_rn(p.scale * acc.x, p.scale * acc.y);
    w.y = pack_bf16x2_rn(p.scale * acc.z, p.scale * acc.w);
    *reinterpret_cast<uint2*>(static_cast<uint16_t*>(p.out) + m * p.ld_out + j) = w;
  } else {
    *reinterpret_cast<float4*>(static_cast<float*>(p.out) + m * p.ld_out + j) = acc;
  }
}

// The transposed output out[j, m] (dA^T, unpooled): a CTA takes 32 rows m, sums their splits (coalesced
// 16-byte loads of whole rows, split order), turns the 32 x r tile in shared memory and writes each column
// j as 32 consecutive floats.
__global__ void __launch_bounds__(256) adapter_reduce_cols_kernel(const AdapterParams p, int bn) {
  __shared__ float tile[32][65];
  pdl_launch_dependents();
  pdl_wait();
  const int64_t m0 = static_cast<int64_t>(blockIdx.x) * 32;
  const int64_t split_stride = static_cast<int64_t>(p.m_tiles) * 128 * bn;
  const int q = p.r / 4;
  for (int e = threadIdx.x; e < 32 * q; e += blockDim.x) {
    const int row = e / q, j = (e - row * q) * 4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (m0 + row < p.Mm) {
      const float* src = p.part + (m0 + row) * bn + j;
      for (int s = 0; s < p.splits; ++s) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(src + s * split_stride));
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
      }
    }
    tile[row][j] = acc.x;
    tile[row][j + 1] = acc.y;
    tile[row][j + 2] = acc.z;
    tile[row][j + 3] = acc.w;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < 32 * p.r; e += blockDim.x) {
    const int j = e >> 5, row = e & 31;
    if (m0 + row < p.Mm) static_cast<float*>(p.out)[static_cast<int64_t>(j) * p.ld_out + m0 + row] = tile[row][j];
  }
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

// Adapter down-projection for a few tokens: T[m, j] = bf16(s * sum_k X[m, k] A[j, k]), m < M <= 16.
// One CTA per (adapter row j, pair of tokens); each thread takes 8 inputs per pass, sums them in fp32,
// and the partial sums are combined in a fixed order (within each warp, then over the warps), so the
// result does not depend on scheduling.  Used instead of the split-K tensor-core GEMM, whose 128-token
// tiles, partial sums and reduction launch cost more than the whole product at these sizes.
constexpr int kSmallTokens = 16;
constexpr int kSmallPerCta = 2;

__global__ void __launch_bounds__(256) lora_down_small_kernel(const uint16_t* __restrict__ X, int M, int64_t K,
                                                              const uint16_t* __restrict__ A, int r, float s,
                                                              uint16_t* __restrict__ T) {
  __shared__ float part[8][kSmallPerCta];
  pdl_launch_dependents();
  pdl_wait();
  const int j = blockIdx.x % r, m0 = (blockIdx.x / r) * kSmallPerCta;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float acc[kSmallPerCta];
#pragma unroll
  for (int m = 0; m < kSmallPerCta; ++m) acc[m] = 0.f;
  const uint4* a = reinterpret_cast<const uint4*>(A + static_cast<int64_t>(j) * K);
  const int64_t n8 = K / 8;
  for (int64_t c = threadIdx.x; c < n8; c += 256) {
    const uint4 av = __ldg(a + c);
    const float af[8] = {lo_f(av.x), hi_f(av.x), lo_f(av.y), hi_f(av.y), lo_f(av.z), hi_f(av.z), lo_f(av.w), hi_f(av.w)};
#pragma unroll
    for (int m = 0; m < kSmallPerCta; ++m) {
      if (m0 + m < M) {
        const uint4 xv = __ldg(reinterpret_cast<const uint4*>(X + static_cast<int64_t>(m0 + m) * K) + c);
        float d = af[0] * lo_f(xv.x);
        d = fmaf(af[1], hi_f(xv.x), d);
        d = fmaf(af[2], lo_f(xv.y), d);
        d = fmaf(af[3], hi_f(xv.y), d);
        d = fmaf(af[4], lo_f(xv.z), d);
        d = fmaf(af[5], hi_f(xv.z), d);
        d = fmaf(af[6], lo_f(xv.w), d);
        d = fmaf(af[7], hi_f(xv.w), d);
        acc[m] += d;
      }
    }
  }
#pragma unroll
  for (int m = 0; m < kSmallPerCta; ++m) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], o);
    if (lane == 0) part[warp][m] = acc[m];
  }
  __syncthreads();
  if (threadIdx.x < kSmallPerCta && m0 + threadIdx.x < M) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) t += part[w][threadIdx.x];
    T[static_cast<int64_t>(m0 + threadIdx.x) * r + j] = static_cast<uint16_t>(pack_bf16x2_rn(s * t, 0.f) & 0xFFFFu);
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
  if (p.Mm == 0) return cudaSuccess;
  if (p.out_mode == ADAPTER_COLS_F32) {
    const int64_t blocks = (static_cast<int64_t>(p.Mm) + 31) / 32;
    return launch_pdl(adapter_reduce_cols_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st, p, bn);
  }
  const int64_t n = static_cast<int64_t>(p.Mm) * (p.r / 4);
  return launch_pdl(adapter_reduce_rows_kernel, dim3(static_cast<unsigned>((n + 255) / 256)), dim3(256), 0, st, p, bn);
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

bool lora_down_small_supported(int64_t M) { return M >= 1 && M <= kSmallTokens; }

cudaError_t launch_lora_down_small(const uint16_t* X, int64_t M, int64_t K, const uint16_t* A, int r, float s,
                                   uint16_t* T, cudaStream_t st) {
  const unsigned grid = static_cast<unsigned>(r * ((M + kSmallPerCta - 1) / kSmallPerCta));
  return launch_pdl(lora_down_small_kernel, dim3(grid), dim3(256), 0, st, X, static_cast<int>(M), K, A, r, s, T);
}

cudaError_t launch_expand_adapter(const uint16_t* A, int r, int64_t K, int L, uint16_t* Aexp, cudaStream_t st) {
  const int64_t n = static_cast<int64_t>(r) * K;
  return launch_pdl(expand_kernel, dim3(static_cast<unsigned>((n + 255) / 256)), dim3(256), 0, st, A, r, K, L, Aexp);
}

}  // namespace qlr
