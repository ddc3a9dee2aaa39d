// Quantisers (NF-k + double quantisation, group-wise INT4), whole-matrix dequantisation and
// the QA-LoRA zero-point merge.  All memory-bound; one pass over the weight each.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "ptx.cuh"

namespace qlr {

namespace {

// First index of the minimum of fp32 |u - level| over the ascending levels s_lv[0 .. 2^bits - 1], with
// s_lv[0] = -1 <= u <= 1 = s_lv[last].  A binary search finds the largest i with s_lv[i] <= u; only
// levels i and i + 1 can then be nearest (for j < i, u - s_lv[j] > u - s_lv[i] and fp32 rounding is
// monotone; a rounding tie would need an ulp of at least the level spacing, impossible for |u| <= 1),
// and a tie between the two goes to i, the lower index.
__device__ __forceinline__ int nearest_level(float u, const float* s_lv, int bits) {
  int i = 0;
  for (int step = 1 << (bits - 1); step > 0; step >>= 1)
    if (u >= s_lv[i + step]) i += step;
  const int last = (1 << bits) - 1;
  if (i == last) return last;
  const float d0 = fabsf(__fsub_rn(u, s_lv[i]));
  const float d1 = fabsf(__fsub_rn(u, s_lv[i + 1]));
  return d1 < d0 ? i + 1 : i;
}

// NF-k blockwise quantisation (QLoRA explainer: "Background: what is quantization?",
// "Innovation 1: 4-bit NormalFloat (NF4)", "Innovation 2: Double Quantization").
// One CTA per group of 256 first-level blocks (the double-quantisation group).  Each thread owns
// 8 consecutive inputs per chunk (two 16-byte loads); every load of the CTA is issued before any
// arithmetic, the BLOCK / 8 threads of a block combine their absmax with shuffles, and the codes
// of a thread leave as one 32-bit (k = 4) or 16-bit (k = 2) store, or as 3-bit planes assembled over
// four adjacent lanes (32 codes).
constexpr int kNfThreads = 512;

template <int BLOCK>
__global__ void __launch_bounds__(kNfThreads) quantize_nfk_kernel(
    const float* __restrict__ W, int64_t n_blocks, int bits, int dq_block, Levels lv, int zero_code,
    uint8_t* __restrict__ codes, float* __restrict__ c1_out, uint8_t* __restrict__ c1_fp8,
    float* __restrict__ s2_out, int32_t* status) {
  constexpr int TPB = BLOCK / 8;                         // threads per block: 8 or 16
  constexpr int CH = 256 * BLOCK / (kNfThreads * 8);     // chunks per thread: 4 or 8
  __shared__ float s_c1[256];
  __shared__ float s_red[kNfThreads / 32];
  __shared__ float s_lv[16];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid < 16) s_lv[tid] = lv.v[tid];
  const int64_t blk0 = static_cast<int64_t>(blockIdx.x) * 256;
  const int nblk = static_cast<int>((n_blocks - blk0) < 256 ? (n_blocks - blk0) : 256);
  const int64_t e0 = blk0 * BLOCK;  // first input of this CTA
  const float4* src = reinterpret_cast<const float4*>(W + e0);
  float4 v[CH][2];
#pragma unroll
  for (int c = 0; c < CH; ++c) {
    const int e = c * kNfThreads + tid;  // 8-input chunk index within the CTA
    if (e / TPB < nblk) {
      v[c][0] = __ldg(src + 2 * e);
      v[c][1] = __ldg(src + 2 * e + 1);
    } else {
      v[c][0] = v[c][1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  __syncthreads();  // s_lv
  bool bad = false;
#pragma unroll
  for (int c = 0; c < CH; ++c) {
    const int e = c * kNfThreads + tid;
    const int lb = e / TPB;           // block within the CTA (uniform over the block's threads)
    const bool valid = lb < nblk;
    const float x[8] = {v[c][0].x, v[c][0].y, v[c][0].z, v[c][0].w, v[c][1].x, v[c][1].y, v[c][1].z, v[c][1].w};
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      bad |= !isfinite(x[i]);
      m = fmaxf(m, fabsf(x[i]));
    }
#pragma unroll
    for (int o = TPB / 2; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (valid && (tid & (TPB - 1)) == 0) s_c1[lb] = m;
    int code[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) code[i] = (m == 0.f) ? zero_code : nearest_level(__fdiv_rn(x[i], m), s_lv, bits);
    const int64_t chunk = blk0 * TPB + e;  // global 8-input chunk index
    if (bits == 4) {
      uint32_t word = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) word |= static_cast<uint32_t>(code[i]) << (4 * i);
      if (valid) reinterpret_cast<uint32_t*>(codes)[chunk] = word;
    } else if (bits == 2) {
      uint32_t half = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) half |= static_cast<uint32_t>(code[i]) << (2 * i);
      if (valid) reinterpret_cast<uint16_t*>(codes)[chunk] = static_cast<uint16_t>(half);
    } else {  // bits == 3: lanes 4q .. 4q+3 hold 32 consecutive codes; plane word p, bit t = bit p of code t
      const int q = lane & 3;
      uint32_t pl[3];
#pragma unroll
      for (int p = 0; p < 3; ++p) {
        uint32_t b = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) b |= ((static_cast<uint32_t>(code[i]) >> p) & 1u) << i;
        b <<= 8 * q;
        b |= __shfl_xor_sync(0xffffffffu, b, 1);
        b |= __shfl_xor_sync(0xffffffffu, b, 2);
        pl[p] = b;
      }
      if (valid && q == 0) {
        uint32_t* words = reinterpret_cast<uint32_t*>(codes) + 3 * (chunk >> 2);
        words[0] = pl[0];
        words[1] = pl[1];
        words[2] = pl[2];
      }
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) report(status, QLR_ERR_NONFINITE);
  __syncthreads();
  if (dq_block == 0) {
    if (tid < nblk) c1_out[blk0 + tid] = s_c1[tid];
    return;
  }
  // second level: one fp32 constant per 256 first-level constants
  float mm = (tid < nblk) ? s_c1[tid] : 0.f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mm = fmaxf(mm, __shfl_xor_sync(0xffffffffu, mm, o));
  if (lane == 0) s_red[warp] = mm;
  __syncthreads();
  float gmax = s_red[0];
#pragma unroll
  for (int w = 1; w < kNfThreads / 32; ++w) gmax = fmaxf(gmax, s_red[w]);
  const float s2 = __fdiv_rn(gmax, 448.0f);
  if (tid == 0) s2_out[blockIdx.x] = s2;
  if (tid < nblk) {
    const float ratio = (s2 == 0.f) ? 0.f : __fdiv_rn(s_c1[tid], s2);
    c1_fp8[blk0 + tid] = static_cast<uint8_t>(__nv_cvt_float_to_fp8(ratio, __NV_SATFINITE, __NV_E4M3));
  }
}

// Group-wise INT4 with fp16 scale and zero point (QA-LoRA abstract).  Each thread holds 8
// consecutive inputs (two 16-byte loads) and writes their 8 codes as one 32-bit word; the G / 8
// threads of a group (adjacent lanes) combine their ranges with shuffles.
template <int G>
__global__ void __launch_bounds__(256) quantize_int4g_kernel(const float* __restrict__ W, int64_t n_groups,
                                                               uint8_t* __restrict__ codes, __half* __restrict__ scale,
                                                               __half* __restrict__ zero, int32_t* status) {
  constexpr int TPG = G / 8;  // threads per group: 4, 8 or 16 (a group never straddles a warp)
  const int lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const bool valid = t < n_groups * TPG;  // whole groups only: validity is uniform within a group
  float x[8];
  if (valid) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(W) + 2 * t);
    const float4 b = __ldg(reinterpret_cast<const float4*>(W) + 2 * t + 1);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] = 0.f;
  }
  float lo = 0.f, hi = 0.f;
  bool bad = false;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    bad |= !isfinite(x[e]);
    lo = fminf(lo, x[e]);
    hi = fmaxf(hi, x[e]);
  }
#pragma unroll
  for (int o = TPG / 2; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) report(status, QLR_ERR_NONFINITE);
  if (!valid) return;
  const __half sc16 = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), 15.0f));
  const float sc = __half2float(sc16);
  float z = 0.f;
  if (sc > 0.f) z = __fadd_rn(fminf(fmaxf(rintf(__fdiv_rn(-lo, sc)), 0.f), 15.f), 0.0f);  // +0, never -0
  uint32_t word = 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    int c = 0;
    if (sc > 0.f) c = static_cast<int>(fminf(fmaxf(rintf(__fadd_rn(__fdiv_rn(x[e], sc), z)), 0.f), 15.f));
    word |= static_cast<uint32_t>(c) << (4 * e);  // element 2j in the low nibble of byte j
  }
  reinterpret_cast<uint32_t*>(codes)[t] = word;
  if ((lane & (TPG - 1)) == 0) {
    const int64_t g = t / TPG;
    scale[g] = sc16;
    zero[g] = __float2half_rn(z);
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
  if (block == 64)
    quantize_nfk_kernel<64><<<static_cast<unsigned>(grid), kNfThreads, 0, st>>>(
        W, n_blocks, bits, dq_block, lv, zc, out->codes, out->c1, out->c1_fp8, out->s2, status);
  else
    quantize_nfk_kernel<128><<<static_cast<unsigned>(grid), kNfThreads, 0, st>>>(
        W, n_blocks, bits, dq_block, lv, zc, out->codes, out->c1, out->c1_fp8, out->s2, status);
  return cudaGetLastError();
}

cudaError_t launch_quantize_int4g(const float* W, int64_t N, int64_t K, int group, const qlr_qweight* out,
                                  int32_t* status, cudaStream_t st) {
  const int64_t n_groups = N * (K / group);
  const int64_t grid = (n_groups * (group / 8) + 255) / 256;  // one thread per 8 inputs
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
