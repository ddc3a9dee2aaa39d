// Device building blocks shared by the tcgen05 GEMM kernels: the dequantiser (2-, 3- and 4-bit codes
// unpacked to 4-bit fields, a 16-entry bf16 table per block or group, byte-permute lookups) and the
// epilogue stores.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "gemm.cuh"
#include "ptx.cuh"
#include "swiglu.cuh"

namespace qlr {
namespace eng {

__device__ __forceinline__ float e4m3_to_f32(uint8_t b) {
  const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(b), __NV_E4M3);
  return __half2float(__half(h));
}

struct Lut {
  uint32_t l0, l1, l2, l3, h0, h1, h2, h3;
};

__device__ __forceinline__ Lut make_lut(const float (&v)[16]) {
  uint32_t p[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) p[j] = pack_bf16x2_rn(v[2 * j], v[2 * j + 1]);
  Lut t;
  t.l0 = prmt(p[0], p[1], 0x6420);
  t.h0 = prmt(p[0], p[1], 0x7531);
  t.l1 = prmt(p[2], p[3], 0x6420);
  t.h1 = prmt(p[2], p[3], 0x7531);
  t.l2 = prmt(p[4], p[5], 0x6420);
  t.h2 = prmt(p[4], p[5], 0x7531);
  t.l3 = prmt(p[6], p[7], 0x6420);
  t.h3 = prmt(p[6], p[7], 0x7531);
  return t;
}

// 4 codes (low 16 bits of w, code i at bits 4i..4i+3) -> two bf16x2 words (code 0 in the low half).
__device__ __forceinline__ void lut4(const Lut& t, uint32_t w, uint32_t& o0, uint32_t& o1) {
  const uint32_t sel = w & 0x7777u;
  const uint32_t sel2 = ((w >> 1) & 0x4444u) | 0x3210u;
  const uint32_t lo = prmt(prmt(t.l0, t.l1, sel), prmt(t.l2, t.l3, sel), sel2);
  const uint32_t hi = prmt(prmt(t.h0, t.h1, sel), prmt(t.h2, t.h3, sel), sel2);
  o0 = prmt(lo, hi, 0x5140);
  o1 = prmt(lo, hi, 0x7362);
}

__device__ __forceinline__ uint4 lut8(const Lut& t, uint32_t w) {
  uint4 r;
  lut4(t, w, r.x, r.y);
  lut4(t, w >> 16, r.z, r.w);
  return r;
}

// The first eight entries of a table, for codes below 8 (2- and 3-bit codes unpacked to 4-bit fields):
// each 4-bit field is itself a byte-permute selector (its top bit, the sign-replicate flag, is clear),
// so one permute per byte plane and the two interleaves give 4 codes.
struct Lut8 {
  uint32_t l0, l1, h0, h1;
};

__device__ __forceinline__ Lut8 make_lut8(const float (&v)[8]) {
  uint32_t p[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) p[j] = pack_bf16x2_rn(v[2 * j], v[2 * j + 1]);
  return Lut8{prmt(p[0], p[1], 0x6420), prmt(p[2], p[3], 0x6420), prmt(p[0], p[1], 0x7531),
              prmt(p[2], p[3], 0x7531)};
}

__device__ __forceinline__ uint4 lut8_small(const Lut8& t, uint32_t w) {
  uint4 r;
  const uint32_t lo0 = prmt(t.l0, t.l1, w), hi0 = prmt(t.h0, t.h1, w);
  const uint32_t w1 = w >> 16;
  const uint32_t lo1 = prmt(t.l0, t.l1, w1), hi1 = prmt(t.h0, t.h1, w1);
  r.x = prmt(lo0, hi0, 0x5140);
  r.y = prmt(lo0, hi0, 0x7362);
  r.z = prmt(lo1, hi1, 0x5140);
  r.w = prmt(lo1, hi1, 0x7362);
  return r;
}

// Per-thread scale data of one 64-code run, loaded one stage ahead of its use so the global-memory
// latency overlaps the dequantisation of the previous stage.
//   NF with double quantisation: a = E4M3 byte of the block, b = bits of its fp32 second-level constant;
//   NF without:                  a = bits of the fp32 block absmax;
//   INT4 group:                  a = fp16 scales of the run's group(s), b = fp16 zero points.
struct DqConst {
  uint32_t a, b;
};

__device__ __forceinline__ DqConst load_dq_const(const DqParams& dq, int64_t row, int64_t col, bool valid) {
  DqConst c{0u, 0u};
  if (!valid) return c;
  const int64_t u = row * dq.units_per_row + (col >> dq.unit_shift);  // block (NF) or group (INT4) index
  if (dq.fmt == QLR_FMT_NFK) {
    if (dq.dq_block) {
      c.a = __ldg(dq.c1_fp8 + u);
      c.b = __float_as_uint(__ldg(dq.s2 + (u >> dq.dq_shift)));
    } else {
      c.a = __float_as_uint(__ldg(dq.c1 + u));
    }
  } else if (dq.group == 32) {  // two groups per run; u is even, so the pair is one aligned 32-bit word
    c.a = __ldg(reinterpret_cast<const uint32_t*>(dq.scale + u));
    c.b = __ldg(reinterpret_cast<const uint32_t*>(dq.zero + u));
  } else {
    c.a = __ldg(reinterpret_cast<const unsigned short*>(dq.scale + u));
    c.b = __ldg(reinterpret_cast<const unsigned short*>(dq.zero + u));
  }
  return c;
}

__device__ __forceinline__ Lut nf_lut_c(const DqParams& dq, const DqConst& c) {
  const float scale = dq.dq_block ? __fmul_rn(e4m3_to_f32(static_cast<uint8_t>(c.a)), __uint_as_float(c.b))
                                  : __uint_as_float(c.a);
  float v[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __fmul_rn(dq.lv.v[i], scale);
  return make_lut(v);
}

// The 2^bits <= 8 levels of a 2- or 3-bit NF block (entries past the last level are never selected).
__device__ __forceinline__ Lut8 nf_lut8_c(const DqParams& dq, const DqConst& c) {
  const float scale = dq.dq_block ? __fmul_rn(e4m3_to_f32(static_cast<uint8_t>(c.a)), __uint_as_float(c.b))
                                  : __uint_as_float(c.a);
  float v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __fmul_rn(dq.lv.v[i], scale);
  return make_lut8(v);
}

__device__ __forceinline__ Lut int4_lut_c(uint32_t sc_bits16, uint32_t z_bits16) {
  const float sc = __half2float(__ushort_as_half(static_cast<unsigned short>(sc_bits16)));
  const float z = __half2float(__ushort_as_half(static_cast<unsigned short>(z_bits16)));
  float v[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __fmul_rn(__fsub_rn(static_cast<float>(i), z), sc);
  return make_lut(v);
}

// 2-bit fields i = 0..7 of a 16-bit word -> 4-bit fields (field i at bits 4i..4i+3).
__device__ __forceinline__ uint32_t spread2to4(uint32_t x) {
  x = (x | (x << 8)) & 0x00FF00FFu;
  x = (x | (x << 4)) & 0x0F0F0F0Fu;
  return (x | (x << 2)) & 0x33333333u;
}

// bits t = 0..7 of a byte -> bit 4t.
__device__ __forceinline__ uint32_t spread1to4(uint32_t x) {
  x = (x | (x << 12)) & 0x000F000Fu;
  x = (x | (x << 6)) & 0x03030303u;
  return (x | (x << 3)) & 0x11111111u;
}

// The 64 codes of one run, unpacked to eight words of eight 4-bit codes (code 8q + i at bits 4i of
// word q).  Packed layouts (little-endian): k = 4 two codes per byte, low nibble first (32 bytes,
// 16-byte aligned); k = 2 four codes per byte, code 4j + t at bits 2t (16 bytes, 16-byte aligned);
// k = 3 bit planes, per 32 codes three 32-bit words, word p holding bit p of code t at bit t (24 bytes,
// 8-byte aligned).
__device__ __forceinline__ void load_codes64(const uint8_t* src, int bits, uint32_t (&w)[8]) {
  if (bits == 4) {
    const uint4 c0 = reinterpret_cast<const uint4*>(src)[0], c1 = reinterpret_cast<const uint4*>(src)[1];
    w[0] = c0.x; w[1] = c0.y; w[2] = c0.z; w[3] = c0.w;
    w[4] = c1.x; w[5] = c1.y; w[6] = c1.z; w[7] = c1.w;
  } else if (bits == 2) {
    const uint4 c = *reinterpret_cast<const uint4*>(src);
    const uint32_t q[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      w[2 * i] = spread2to4(q[i] & 0xFFFFu);
      w[2 * i + 1] = spread2to4(q[i] >> 16);
    }
  } else {
    const uint2 a = reinterpret_cast<const uint2*>(src)[0], b = reinterpret_cast<const uint2*>(src)[1],
                c = reinterpret_cast<const uint2*>(src)[2];
    const uint32_t pl[2][3] = {{a.x, a.y, b.x}, {b.y, c.x, c.y}};
#pragma unroll
    for (int gi = 0; gi < 2; ++gi)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int sh = 8 * j;
        w[4 * gi + j] = spread1to4((pl[gi][0] >> sh) & 0xFFu) | (spread1to4((pl[gi][1] >> sh) & 0xFFu) << 1) |
                        (spread1to4((pl[gi][2] >> sh) & 0xFFu) << 2);
      }
  }
}

// Dequantise 64 consecutive codes (one run of a row of W, `bits` wide, its scale data in `c`) into
// the eight 16-byte chunks of one 128-byte swizzled shared-memory row at `dst_row` (`sw` = row index
// for the swizzle).  SMALL: the weight is 2- or 3-bit NF, looked up in the table's first eight entries
// (a separate instantiation, so the 4-bit and INT4 code paths stay as compact as before).
template <bool SMALL>
__device__ __forceinline__ void dequant_row64(const DqParams& dq, const uint8_t* codes_smem, int bits, const DqConst& c,
                                              bool valid, uint8_t* dst_row, int sw) {
  if (!valid) {
#pragma unroll
    for (int k = 0; k < 8; ++k) *reinterpret_cast<uint4*>(dst_row + ((k ^ sw) << 4)) = make_uint4(0, 0, 0, 0);
    return;
  }
  uint32_t w[8];
  load_codes64(codes_smem, bits, w);
  if constexpr (SMALL) {
    const Lut8 t = nf_lut8_c(dq, c);
#pragma unroll
    for (int k = 0; k < 8; ++k) *reinterpret_cast<uint4*>(dst_row + ((k ^ sw) << 4)) = lut8_small(t, w[k]);
    return;
  }
  if (dq.fmt == QLR_FMT_NFK) {
    const Lut t = nf_lut_c(dq, c);
#pragma unroll
    for (int k = 0; k < 8; ++k) *reinterpret_cast<uint4*>(dst_row + ((k ^ sw) << 4)) = lut8(t, w[k]);
  } else if (dq.group == 32) {
    const Lut t0 = int4_lut_c(c.a & 0xFFFFu, c.b & 0xFFFFu);
#pragma unroll
    for (int k = 0; k < 4; ++k) *reinterpret_cast<uint4*>(dst_row + ((k ^ sw) << 4)) = lut8(t0, w[k]);
    const Lut t1 = int4_lut_c(c.a >> 16, c.b >> 16);
#pragma unroll
    for (int k = 4; k < 8; ++k) *reinterpret_cast<uint4*>(dst_row + ((k ^ sw) << 4)) = lut8(t1, w[k]);
  } else {
    const Lut t0 = int4_lut_c(c.a, c.b);
#pragma unroll
    for (int k = 0; k < 8; ++k) *reinterpret_cast<uint4*>(dst_row + ((k ^ sw) << 4)) = lut8(t0, w[k]);
  }
}

// Writes one 32-column chunk of an fp32 accumulator row as bf16 into out^T (out row = D column),
// transposing through a per-warp 32 x 32 bf16 staging tile so that every global store is 16 bytes wide.
__device__ __forceinline__ void store_chunk_bf16_t(const uint32_t (&v)[32], uint16_t* stg, int lane, int dcol0,
                                                   int drow0, const GemmParams& p) {
#pragma unroll
  for (int jj = 0; jj < 32; ++jj)
    stg[jj * 32 + lane] = static_cast<uint16_t>(pack_bf16x2_rn(__uint_as_float(v[jj]), 0.f) & 0xFFFFu);
  __syncwarp();
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const int idx = t * 32 + lane;
    const int jj = idx >> 2, part = idx & 3;
    const int orow = dcol0 + jj;              // output row (D column)
    const int ocol = drow0 + part * 8;        // output column (D row)
    if (orow < p.Nn && ocol < p.Mm) {
      const uint4 val = *reinterpret_cast<const uint4*>(stg + jj * 32 + part * 8);
      *reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + static_cast<int64_t>(orow) * p.ldo + ocol) = val;
    }
  }
  __syncwarp();
}

// As store_chunk_bf16_t, staged in fp32 for the outputs that need the unrounded value or more than a store
// (a thread handles 8 consecutive outputs of one row): with `accumulate` the previous bf16 value is added to
// the fp32 result before its one rounding; EPI_SWIGLU_FWD stores the result U and H = silu(G) U;
// EPI_SWIGLU_BWD treats the result as dH and stores dG and dU instead.
// The staging tile keeps row jj's column c at jj * 32 + (c ^ 4 (jj mod 8)): the XOR moves whole 16-byte
// groups, so both the column writes (one row per loop step, a lane per column) and the 16-byte row reads
// spread over all 32 banks.
template <int EPI>
__device__ __forceinline__ void store_chunk_f32_t(const uint32_t (&v)[32], float* stg, int lane, int dcol0, int drow0,
                                                  const GemmParams& p) {
#pragma unroll
  for (int jj = 0; jj < 32; ++jj) stg[jj * 32 + (lane ^ ((jj & 7) << 2))] = __uint_as_float(v[jj]);
  __syncwarp();
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const int idx = t * 32 + lane;
    const int jj = idx >> 2, part = idx & 3;
    const int orow = dcol0 + jj;              // output row (D column)
    const int ocol = drow0 + part * 8;        // output column (D row)
    if (orow < p.Nn && ocol < p.Mm) {
      const int sw = (jj & 7) << 2;
      const float4 f0 = *reinterpret_cast<const float4*>(stg + jj * 32 + ((part * 8) ^ sw));
      const float4 f1 = *reinterpret_cast<const float4*>(stg + jj * 32 + ((part * 8 + 4) ^ sw));
      float f[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
      const int64_t off = static_cast<int64_t>(orow) * p.ldo + ocol;
      uint16_t* dst = static_cast<uint16_t*>(p.out) + off;
      if (EPI == EPI_STORE && p.accumulate) {
        const uint4 o4 = *reinterpret_cast<const uint4*>(dst);
        const uint32_t ov[4] = {o4.x, o4.y, o4.z, o4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          f[2 * e] = __fadd_rn(f[2 * e], bf16_bits_to_f32(ov[e] & 0xFFFFu));
          f[2 * e + 1] = __fadd_rn(f[2 * e + 1], bf16_bits_to_f32(ov[e] >> 16));
        }
      }
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) w[e] = pack_bf16x2_rn(f[2 * e], f[2 * e + 1]);
      if (EPI == EPI_STORE) {
        *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
      } else if (EPI == EPI_SWIGLU_FWD) {  // w = U; H = silu(G) U
        *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
        const uint4 g4 = *reinterpret_cast<const uint4*>(p.aux_g + off);
        const uint32_t gv[4] = {g4.x, g4.y, g4.z, g4.w};
        uint32_t hv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          hv[e] = pack_bf16x2_rn(swiglu_h(bf16_bits_to_f32(gv[e] & 0xFFFFu), bf16_bits_to_f32(w[e] & 0xFFFFu)),
                                 swiglu_h(bf16_bits_to_f32(gv[e] >> 16), bf16_bits_to_f32(w[e] >> 16)));
        *reinterpret_cast<uint4*>(p.aux_out + off) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
      } else {  // w = dH (bf16, as a stored dH would be); dG to out, dU to aux_out
        const uint4 g4 = *reinterpret_cast<const uint4*>(p.aux_g + off);
        const uint4 u4 = *reinterpret_cast<const uint4*>(p.aux_u + off);
        const uint32_t gv[4] = {g4.x, g4.y, g4.z, g4.w}, uv[4] = {u4.x, u4.y, u4.z, u4.w};
        uint32_t og[4], ou[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float g0, u0, g1, u1;
          swiglu_grads(bf16_bits_to_f32(w[e] & 0xFFFFu), bf16_bits_to_f32(gv[e] & 0xFFFFu),
                       bf16_bits_to_f32(uv[e] & 0xFFFFu), g0, u0);
          swiglu_grads(bf16_bits_to_f32(w[e] >> 16), bf16_bits_to_f32(gv[e] >> 16), bf16_bits_to_f32(uv[e] >> 16), g1,
                       u1);
          og[e] = pack_bf16x2_rn(g0, g1);
          ou[e] = pack_bf16x2_rn(u0, u1);
        }
        *reinterpret_cast<uint4*>(dst) = make_uint4(og[0], og[1], og[2], og[3]);
        *reinterpret_cast<uint4*>(p.aux_out + off) = make_uint4(ou[0], ou[1], ou[2], ou[3]);
      }
    }
  }
  __syncwarp();
}

}  // namespace eng
}  // namespace qlr
