// Element-wise view of an NF-k weight for the offline kernels (LQ-LoRA initialisation, quantisation
// error): the code of element i of the row-major flattened matrix and its dequantised value, the bf16
// weight the layer uses: bf16(level[code] * scale), scale = fp32(E4M3(c1_8)) * s2 (fp32 products), or
// the fp32 block absmax without double quantisation.
#pragma once
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "ptx.cuh"

namespace qlr {
namespace nfk {

__device__ __forceinline__ float bf16_round(float x) {
  return __uint_as_float((pack_bf16x2_rn(x, 0.f) & 0xFFFFu) << 16);
}

// packed layouts: k = 4 two codes per byte (low nibble first); k = 2 four per byte (code 4j + t at
// bits 2t); k = 3 per 32 codes three 32-bit bit planes
__device__ __forceinline__ uint32_t code_at(const uint8_t* codes, int bits, int64_t i) {
  if (bits == 4) return (codes[i >> 1] >> ((i & 1) * 4)) & 0xFu;
  if (bits == 2) return (codes[i >> 2] >> ((i & 3) * 2)) & 0x3u;
  const uint32_t* w = reinterpret_cast<const uint32_t*>(codes) + 3 * (i >> 5);
  const int t = static_cast<int>(i & 31);
  return ((w[0] >> t) & 1u) | (((w[1] >> t) & 1u) << 1) | (((w[2] >> t) & 1u) << 2);
}

struct View {
  const uint8_t* codes;
  const float* c1;
  const uint8_t* c1_fp8;
  const float* s2;
  int bits, block_shift, dq;
  Levels lv;
};

__device__ __forceinline__ float dequant_at(const View& v, int64_t i) {
  const int64_t b = i >> v.block_shift;
  float scale;
  if (v.dq) {
    const __half_raw hr = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(v.c1_fp8[b]), __NV_E4M3);
    scale = __fmul_rn(__half2float(__half(hr)), v.s2[b >> 8]);
  } else {
    scale = v.c1[b];
  }
  return bf16_round(__fmul_rn(v.lv.v[code_at(v.codes, v.bits, i)], scale));
}

inline View view_of(const qlr_qweight* w) {
  View v;
  v.codes = w->codes;
  v.c1 = w->c1;
  v.c1_fp8 = w->c1_fp8;
  v.s2 = w->s2;
  v.bits = w->bits;
  v.block_shift = w->block == 128 ? 7 : 6;
  v.dq = w->dq_block ? 1 : 0;
  v.lv = levels_for(w->bits);
  return v;
}

}  // namespace nfk
}  // namespace qlr
