// Quantisers (NF-k + double quantisation, group-wise INT4), whole-matrix dequantisation and
// the QA-LoRA zero-point merge.  All memory-bound; one pass over the weight each.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "ptx.cuh"

namespace qlr {

namespace {

constexpr int kQuantThreads = 256;  // 8 warps; one CTA per group of 256 first-level blocks

__device__ __forceinline__ int nearest_level(float u, const Levels& lv, int nlev) {
  // first index of the minimum of fp32 |u - level|
  float best = fabsf(__fsub_rn(u, lv.v[0]));
  int bi = 0;
#pragma unroll
  for (int i = 1; i < 16; ++i) {
    if (i < nlev) {
      const float d = fabsf(__fsub_rn(u, lv.v[i]));
      if (d < best) {
        best = d;
        bi = i;
      }
    }
  }
  return bi;
}

// NF-k blockwise quantisation (QLoRA explainer: "Background: what is quantization?",
// "Innovation 1: 4-bit NormalFloat (NF4)", "Innovation 2: Double Quantization").
// A warp handles units of 128 consecutive elements; lane j holds elements j + 32e (e < 4),
// so every load is one coalesced 128-byte line and bit planes fall out of warp ballots.
__global__ void __launch_bounds__(kQuantThreads) quantize_nfk_kernel(
    const float* __restrict__ W, int64_t n_blocks, int bits, int block, int dq_block, Levels lv,
    int zero_code, uint8_t* __restrict__ codes, float* __restrict__ c1_out, uint8_t* __restrict__ c1_fp8,
    float* __restrict__ s2_out, int32_t* status) {
  __shared__ float s_c1[256];
  __shared__ float s_red[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t blk0 = static_cast<int64_t>(blockIdx.x) * 256;
  const int nblk = static_cast<int>((n_blocks - blk0) < 256 ? (n_blocks - blk0) : 256);
  const int nlev = 1 << bits;
  const int blocks_per_unit = 128 / block;  // 2 (block 64) or 1 (block 128)
  const int n_units = nblk / blocks_per_unit;
  bool bad = false;
  for (int u = warp; u < n_units; u += 8) {
    const int64_t b_first = blk0 + static_cast<int64_t>(u) * blocks_per_unit;
    const int64_t e0 = b_first * block;  // first element of the unit
    float x[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      x[e] = __ldg(W + e0 + 32 * e + lane);
      bad |= !isfinite(x[e]);
    }
    // block absmax: elements 32e+lane belong to block (32e)/block of the unit
    float m0 = fmaxf(fabsf(x[0]), fabsf(x[1]));
    float m1 = fmaxf(fabsf(x[2]), fabsf(x[3]));
    if (block == 128) {
      m0 = fmaxf(m0, m1);
      m1 = m0;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, o));
      m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, o));
    }
    if (lane == 0) {
      s_c1[u * blocks_per_unit] = m0;
      if (blocks_per_unit == 2) s_c1[u * blocks_per_unit + 1] = m1;
    }
    int code[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float c1 = (block == 128 || e < 2) ? m0 : m1;
      code[e] = (c1 == 0.f) ? zero_code : nearest_level(__fdiv_rn(x[e], c1), lv, nlev);
    }
    // pack
    if (bits == 4) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int nb = __shfl_down_sync(0xffffffffu, code[e], 1);
        if ((lane & 1) == 0) codes[(e0 + 32 * e + lane) >> 1] = static_cast<uint8_t>(code[e] | (nb << 4));
      }
    } else if (bits == 2) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c1v = __shfl_down_sync(0xffffffffu, code[e], 1);
        const int c2v = __shfl_down_sync(0xffffffffu, code[e], 2);
        const int c3v = __shfl_down_sync(0xffffffffu, code[e], 3);
        if ((lane & 3) == 0)
          codes[(e0 + 32 * e + lane) >> 2] = static_cast<uint8_t>(code[e] | (c1v << 2) | (c2v << 4) | (c3v << 6));
      }
    } else {  // bits == 3: three bit planes per 32 codes
      uint32_t* words = reinterpret_cast<uint32_t*>(codes);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t p0 = __ballot_sync(0xffffffffu, code[e] & 1);
        const uint32_t p1 = __ballot_sync(0xffffffffu, (code[e] >> 1) & 1);
        const uint32_t p2 = __ballot_sync(0xffffffffu, (code[e] >> 2) & 1);
        if (lane == 0) {
          const int64_t g = (e0 + 32 * e) >> 5;
          words[3 * g + 0] = p0;
          words[3 * g + 1] = p1;
          words[3 * g + 2] = p2;
        }
      }
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) report(status, QLR_ERR_NONFINITE);
  __syncthreads();
  if (dq_block == 0) {
    for (int t = threadIdx.x; t < nblk; t += kQuantThreads) c1_out[blk0 + t] = s_c1[t];
    return;
  }
  // second level: one fp32 constant per dq_block first-level constants (dq_block == 256 here)
  float m = (threadIdx.x < nblk) ? s_c1[threadIdx.x] : 0.f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) s_red[warp] = m;
  __syncthreads();
  float gmax = s_red[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) gmax = fmaxf(gmax, s_red[w]);
  const float s2 = __fdiv_rn(gmax, 448.0f);
  if (threadIdx.x == 0) s2_out[blockIdx.x] = s2;
  if (threadIdx.x < nblk) {
    const float ratio = (s2 == 0.f) ? 0.f : __fdiv_rn(s_c1[threadIdx.x], s2);
    c1_fp8[blk0 + threadIdx.x] = static_cast<uint8_t>(__nv_cvt_float_to_fp8(ratio, __NV_SATFINITE, __NV_E4M3));
  }
}

// Group-wise INT4 with fp16 scale and zero point (QA-LoRA abstract).  One warp per group
// of `group` consecutive inputs of one row; lane j holds elements j + 32e.
template <int G>
__global__ void __launch_bounds__(256) quantize_int4g_kernel(const float* __restrict__ W, int64_t n_groups,
                                                               uint8_t* __restrict__ codes, __half* __restrict__ scale,
                                                               __half* __restrict__ zero, int32_t* status) {
  constexpr int E = G / 32;
  const int lane = threadIdx.x & 31;
  const int64_t gw = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (gw >= n_groups) return;
  const float* src = W + gw * G;
  float x[E];
  float lo = 0.f, hi = 0.f;
  bool bad = false;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    x[e] = __ldg(src + 32 * e + lane);
    bad |= !isfinite(x[e]);
    lo = fminf(lo, x[e]);
    hi = fmaxf(hi, x[e]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) report(status, QLR_ERR_NONFINITE);
  const __half sc16 = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), 15.0f));
  const float sc = __half2float(sc16);
  float z = 0.f;
  if (sc > 0.f) z = __fadd_rn(fminf(fmaxf(rintf(__fdiv_rn(-lo, sc)), 0.f), 15.f), 0.0f);  // +0, never -0
#pragma unroll
  for (int e = 0; e < E; ++e) {
    int c = 0;
    if (sc > 0.f) c = static_cast<int>(fminf(fmaxf(rintf(__fadd_rn(__fdiv_rn(x[e], sc), z)), 0.f), 15.f));
    const int nb = __shfl_down_sync(0xffffffffu, c, 1);
    if ((lane & 1) == 0) codes[(gw * G + 32 * e + lane) >> 1] = static_cast<uint8_t>(c | (nb << 4));
  }
  if (lane == 0) {
    scale[gw] = sc16;
    zero[gw] = __float2half_rn(z);
  }
}

__device__ __forceinline__ float e4m3_to_f32(uint8_t b) {
  const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(b), __NV_E4M3);
  return __half2float(__half(h));
}

__device__ __forceinline__ uint32_t unpack_code(const uint8_t* codes, int bits, int64_t idx) {
  if (bits == 4) return (codes[idx >> 1] >> ((idx & 1) * 4)) & 0xF;
  if (bits == 2) return (codes[idx >> 2] >> ((idx & 3) * 2)) & 0x3;
  const uint32_t* w = reinterpret_cast<const uint32_t*>(codes) + 3 * (idx >> 5);
  const int t = static_cast<int>(idx & 31);
  return ((w[0] >> t) & 1) | (((w[1] >> t) & 1) << 1) | (((w[2] >> t) & 1) << 2);
}

// Whole-matrix dequantisation, thread per 32 consecutive elements (one block or group).
__global__ void dequant_nfk_kernel(const uint8_t* __restrict__ codes, const float* __restrict__ c1,
                                   const uint8_t* __restrict__ c1_fp8, const float* __restrict__ s2, int bits,
                                   int block, int dq_block, Levels lv, int64_t n_chunks, uint16_t* __restrict__ out) {
  const int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (c >= n_chunks) return;
  const int64_t e0 = c * 32;
  const int64_t b = e0 / block;
  const float scale = dq_block ? __fmul_rn(e4m3_to_f32(c1_fp8[b]), s2[b / dq_block]) : c1[b];
  uint32_t pk[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float v0 = __fmul_rn(lv.v[unpack_code(codes, bits, e0 + 2 * i)], scale);
    const float v1 = __fmul_rn(lv.v[unpack_code(codes, bits, e0 + 2 * i + 1)], scale);
    pk[i] = pack_bf16x2_rn(v0, v1);
  }
  uint4* dst = reinterpret_cast<uint4*>(out + e0);
#pragma unroll
  for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
}

__global__ void dequant_int4g_kernel(const uint8_t* __restrict__ codes, const __half* __restrict__ scale,
                                     const __half* __restrict__ zero, int group, int64_t n_chunks,
                                     uint16_t* __restrict__ out) {
  const int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (c >= n_chunks) return;
  const int64_t e0 = c * 32;
  const int64_t g = e0 / group;
  const float sc = __half2float(scale[g]);
  const float z = __half2float(zero[g]);
  uint32_t pk[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t byte = codes[(e0 >> 1) + i];
    const float v0 = __fmul_rn(__fsub_rn(static_cast<float>(byte & 0xF), z), sc);
    const float v1 = __fmul_rn(__fsub_rn(static_cast<float>(byte >> 4), z), sc);
    pk[i] = pack_bf16x2_rn(v0, v1);
  }
  uint4* dst = reinterpret_cast<uint4*>(out + e0);
#pragma unroll
  for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
}

// QA-LoRA merge: zero' = fp16(zero - s (B A)[o, g] / (L scale)), fp64 throughout.
__global__ void merge_kernel(const uint16_t* __restrict__ A, const uint16_t* __restrict__ B, int r, float s,
                             int64_t N, int64_t G, int L, const __half* __restrict__ scale, __half* __restrict__ zero) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= N * G) return;
  const int64_t o = i / G, g = i % G;
  const double sc = static_cast<double>(__half2float(scale[i]));
  if (sc == 0.0) return;
  double ba = 0.0;
  for (int j = 0; j < r; ++j)
    ba += static_cast<double>(bf16_bits_to_f32(B[o * r + j])) * static_cast<double>(bf16_bits_to_f32(A[j * G + g]));
  const double t = static_cast<double>(s) * ba;
  const double den = static_cast<double>(L) * sc;
  const double zp = static_cast<double>(__half2float(zero[i])) - t / den;
  zero[i] = __double2half(zp);
}

}  // namespace

cudaError_t launch_quantize_nfk(const float* W, int64_t n_elems, int bits, int block, int dq_block,
                                const qlr_qweight* out, int32_t* status, cudaStream_t st) {
  const int64_t n_blocks = n_elems / block;
  const int64_t grid = (n_blocks + 255) / 256;
  Levels lv = levels_for(bits);
  int zc = 0;
  for (int i = 0; i < (1 << bits); ++i)
    if (lv.v[i] == 0.f) zc = i;
  count_launch();
  quantize_nfk_kernel<<<static_cast<unsigned>(grid), kQuantThreads, 0, st>>>(
      W, n_blocks, bits, block, dq_block, lv, zc, out->codes, out->c1, out->c1_fp8, out->s2, status);
  return cudaGetLastError();
}

cudaError_t launch_quantize_int4g(const float* W, int64_t N, int64_t K, int group, const qlr_qweight* out,
                                  int32_t* status, cudaStream_t st) {
  const int64_t n_groups = N * (K / group);
  const int64_t grid = (n_groups * 32 + 255) / 256;
  __half* sc = reinterpret_cast<__half*>(out->scale);
  __half* z = reinterpret_cast<__half*>(out->zero);
  switch (group) {
    case 32: count_launch(); quantize_int4g_kernel<32><<<static_cast<unsigned>(grid), 256, 0, st>>>(W, n_groups, out->codes, sc, z, status); break;
    case 64: count_launch(); quantize_int4g_kernel<64><<<static_cast<unsigned>(grid), 256, 0, st>>>(W, n_groups, out->codes, sc, z, status); break;
    case 128: count_launch(); quantize_int4g_kernel<128><<<static_cast<unsigned>(grid), 256, 0, st>>>(W, n_groups, out->codes, sc, z, status); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_dequant(const qlr_qweight* w, uint16_t* out, cudaStream_t st) {
  const int64_t n_chunks = w->N * w->K / 32;
  const unsigned grid = static_cast<unsigned>((n_chunks + 255) / 256);
  if (w->fmt == QLR_FMT_NFK) {
    count_launch();
    dequant_nfk_kernel<<<grid, 256, 0, st>>>(w->codes, w->c1, w->c1_fp8, w->s2, w->bits, w->block, w->dq_block,
                                            levels_for(w->bits), n_chunks, out);
  } else {
    count_launch();
    dequant_int4g_kernel<<<grid, 256, 0, st>>>(w->codes, reinterpret_cast<const __half*>(w->scale),
                                              reinterpret_cast<const __half*>(w->zero), w->group, n_chunks, out);
  }
  return cudaGetLastError();
}

cudaError_t launch_merge(const qlr_qweight* w, const uint16_t* A, const uint16_t* B, int r, float s,
                         cudaStream_t st) {
  const int64_t G = w->K / w->group;
  const int64_t n = w->N * G;
  count_launch();
  merge_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(
      A, B, r, s, w->N, G, w->group, reinterpret_cast<const __half*>(w->scale), reinterpret_cast<__half*>(w->zero));
  return cudaGetLastError();
}

}  // namespace qlr
