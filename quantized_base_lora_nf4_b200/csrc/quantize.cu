// Quantisers (NF-k + double quantisation, group-wise INT4), whole-matrix dequantisation and
// the QA-LoRA zero-point merge.  All memory-bound; one pass over the weight each.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include <cmath>
#include <cstring>
#include <limits>
#include <mutex>

#include "common.cuh"
#include "ptx.cuh"

namespace qlr {

namespace {

// u = fp32(x / m) for every x of one block or group with a single correctly rounded reciprocal
// y = RN(1/m) per block: q = RN(x y) lies within an ulp of x / m, the remainder x - q m is exact in one
// fma, and RN(q + (x - q m) y) is the correctly rounded quotient (P. Markstein, "Computation of
// elementary functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990).  The
// argument needs every intermediate in the normal range: callers take this path only for divisors in
// [2^-64, 2^64] (and, for the INT4 groups, |x| < 2^64), where quotients of magnitude 2^-24 and up --
// the only ones whose exact value can change a code -- keep every step normal.
constexpr float kDivLo = 0x1p-64f, kDivHi = 0x1p64f;

__device__ __forceinline__ float div_rn_by(float x, float m, float y) {
  const float q = __fmul_rn(x, y);
  const float rem = fmaf(-q, m, x);
  return fmaf(rem, y, q);
}

// Nearest NF level of u in [-1, 1] from the host-built decision table (common.cuh): the cell
// k = round-half-even(16 u) + 16 is the integer part of fma(u, 16, 1.5 * 2^23 + 16), and the cell holds
// at most one threshold.  A NaN u (non-finite input, reported separately) lands in the last cell.
__device__ __forceinline__ int nf_code(float u, const float2* s_tab) {
  const float t = fmaf(u, 16.0f, 12582928.0f);
  const uint32_t k = min(__float_as_uint(t) - 0x4B400000u, 32u);
  const float2 e = s_tab[k];
  return __float_as_int(e.y) + (u >= e.x ? 1 : 0);
}

// NF-k blockwise quantisation (QLoRA explainer: "Background: what is quantization?",
// "Innovation 1: 4-bit NormalFloat (NF4)", "Innovation 2: Double Quantization").
// One CTA of 4 BLOCK threads per group of 256 first-level blocks (the double-quantisation group).  A
// thread owns 8 consecutive inputs per chunk (two 16-byte loads) and walks 8 chunks, one at a time with
// the next already in flight (32 registers: 2048 threads per SM); the BLOCK / 8 threads of a block combine their absmax with shuffles,
// and the codes of a thread leave as one 32-bit (k = 4) or 16-bit (k = 2) store, or as 3-bit planes
// assembled over four adjacent lanes (32 codes).
constexpr int kNfUnroll = 1;  // chunks per thread per step

template <int BLOCK, int BITS>
__global__ void __launch_bounds__(4 * BLOCK, 2048 / (4 * BLOCK)) quantize_nfk_kernel(
    const float* __restrict__ W, int64_t n_blocks, int dq_block, const __grid_constant__ NfTable tab, int zero_code,
    uint8_t* __restrict__ codes, float* __restrict__ c1_out, uint8_t* __restrict__ c1_fp8,
    float* __restrict__ s2_out, int32_t* status) {
  constexpr int kNfThreads = 4 * BLOCK;
  constexpr int TPB = BLOCK / 8;                         // threads per block: 8 or 16
  constexpr int NCH = 256 * BLOCK / (kNfThreads * 8);    // chunks per thread: 8
  constexpr int NIT = NCH / kNfUnroll;
  __shared__ float s_c1[256];
  __shared__ float s_red[kNfThreads / 32];
  static_assert(kNfThreads >= 256, "one thread per first-level constant of the group");
  __shared__ float2 s_tab[33];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid < 33) s_tab[tid] = make_float2(tab.t[tid], __int_as_float(tab.base[tid]));
  const int64_t blk0 = static_cast<int64_t>(blockIdx.x) * 256;
  const int nblk = static_cast<int>((n_blocks - blk0) < 256 ? (n_blocks - blk0) : 256);
  const float4* src = reinterpret_cast<const float4*>(W + blk0 * BLOCK);
  auto load = [&](int c, float4 (&v)[2]) {
    const int e = c * kNfThreads + tid;  // 8-input chunk index within the CTA
    if (e / TPB < nblk) {
      v[0] = __ldg(src + 2 * e);
      v[1] = __ldg(src + 2 * e + 1);
    } else {
      v[0] = v[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  bool bad = false;
  auto quantize_chunk = [&](int c, const float4 (&v)[2]) {
    const int e = c * kNfThreads + tid;
    const int lb = e / TPB;           // block within the CTA (uniform over the block's threads)
    const bool valid = lb < nblk;
    const float x[8] = {v[0].x, v[0].y, v[0].z, v[0].w, v[1].x, v[1].y, v[1].z, v[1].w};
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      bad |= !isfinite(x[i]);
      m = fmaxf(m, fabsf(x[i]));
    }
#pragma unroll
    for (int o = TPB / 2; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (valid && (tid & (TPB - 1)) == 0) s_c1[lb] = m;
    float u[8];
    if (m >= kDivLo && m <= kDivHi) {
      const float y = __frcp_rn(m);
#pragma unroll
      for (int i = 0; i < 8; ++i) u[i] = div_rn_by(x[i], m, y);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) u[i] = __fdiv_rn(x[i], m);
    }
    int code[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) code[i] = (m == 0.f) ? zero_code : nf_code(u[i], s_tab);
    const int64_t chunk = blk0 * TPB + e;  // global 8-input chunk index
    if constexpr (BITS == 4) {
      uint32_t word = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) word |= static_cast<uint32_t>(code[i]) << (4 * i);
      if (valid) reinterpret_cast<uint32_t*>(codes)[chunk] = word;
    } else if constexpr (BITS == 2) {
      uint32_t half = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) half |= static_cast<uint32_t>(code[i]) << (2 * i);
      if (valid) reinterpret_cast<uint16_t*>(codes)[chunk] = static_cast<uint16_t>(half);
    } else {  // 3 bits: lanes 4q .. 4q+3 hold 32 consecutive codes; plane word p, bit t = bit p of code t
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
  };
  float4 cur[kNfUnroll][2], nxt[kNfUnroll][2];
#pragma unroll
  for (int j = 0; j < kNfUnroll; ++j) load(j, cur[j]);
  __syncthreads();  // s_tab
#pragma unroll
  for (int it = 0; it < NIT; ++it) {
    if (it + 1 < NIT) {
#pragma unroll
      for (int j = 0; j < kNfUnroll; ++j) load((it + 1) * kNfUnroll + j, nxt[j]);
    }
#pragma unroll
    for (int j = 0; j < kNfUnroll; ++j) quantize_chunk(it * kNfUnroll + j, cur[j]);
    if (it + 1 < NIT) {
#pragma unroll
      for (int j = 0; j < kNfUnroll; ++j) {
        cur[j][0] = nxt[j][0];
        cur[j][1] = nxt[j][1];
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
  // x / sc through one reciprocal per group (div_rn_by); a group with an input of magnitude 2^64 or more,
  // or whose fp16 scale overflowed, takes the plain division
  float u[8];
  if (sc <= 65504.f && fmaxf(-lo, hi) < kDivHi) {
    const float y = sc > 0.f ? __frcp_rn(sc) : 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) u[e] = div_rn_by(x[e], sc, y);
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) u[e] = __fdiv_rn(x[e], sc);
  }
  uint32_t word = 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    int c = 0;
    if (sc > 0.f) c = static_cast<int>(fminf(fmaxf(rintf(__fadd_rn(u[e], z)), 0.f), 15.f));
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

namespace {

template <int BLOCK>
cudaError_t launch_nfk_block(const float* W, int64_t n_blocks, int bits, int dq_block, const NfTable& tab, int zc,
                             const qlr_qweight* out, int32_t* status, cudaStream_t st) {
  const unsigned grid = static_cast<unsigned>((n_blocks + 255) / 256);
  count_launch();
  switch (bits) {
    case 2:
      quantize_nfk_kernel<BLOCK, 2><<<grid, 4 * BLOCK, 0, st>>>(W, n_blocks, dq_block, tab, zc, out->codes, out->c1,
                                                                 out->c1_fp8, out->s2, status);
      break;
    case 3:
      quantize_nfk_kernel<BLOCK, 3><<<grid, 4 * BLOCK, 0, st>>>(W, n_blocks, dq_block, tab, zc, out->codes, out->c1,
                                                                 out->c1_fp8, out->s2, status);
      break;
    default:
      quantize_nfk_kernel<BLOCK, 4><<<grid, 4 * BLOCK, 0, st>>>(W, n_blocks, dq_block, tab, zc, out->codes, out->c1,
                                                                 out->c1_fp8, out->s2, status);
      break;
  }
  return cudaGetLastError();
}

}  // namespace

// ---- the nearest-level decision table (host) ---------------------------------------------------
namespace {

uint32_t bits_of(float f) {
  uint32_t b;
  std::memcpy(&b, &f, 4);
  return b;
}
float float_of(uint32_t b) {
  float f;
  std::memcpy(&f, &b, 4);
  return f;
}
// fp32 values in increasing order as integers (-0 and +0 both map to 0)
int64_t ordinal(float f) {
  const uint32_t b = bits_of(f);
  return (b >> 31) ? -static_cast<int64_t>(b & 0x7FFFFFFFu) : static_cast<int64_t>(b);
}
float from_ordinal(int64_t o) {
  return o < 0 ? float_of(static_cast<uint32_t>(-o) | 0x80000000u) : float_of(static_cast<uint32_t>(o));
}
// the rule itself: first index of the smallest fp32 |u - level|
int nearest_by_rule(float u, const float* lv, int n) {
  int best = 0;
  float bd = std::fabs(u - lv[0]);
  for (int j = 1; j < n; ++j) {
    const float d = std::fabs(u - lv[j]);
    if (d < bd) {
      bd = d;
      best = j;
    }
  }
  return best;
}
// the device's cell of u (same fma, correctly rounded on both sides)
int cell_of(float u) { return static_cast<int>(bits_of(std::fma(u, 16.0f, 12582928.0f)) - 0x4B400000u); }
// smallest u of [-1, 1] where a predicate that is false below some point and true above it holds
template <class Pred>
int64_t first_true(Pred pred) {
  int64_t lo = ordinal(-1.0f), hi = ordinal(1.0f);
  while (lo < hi) {
    const int64_t mid = lo + (hi - lo) / 2;
    if (pred(from_ordinal(mid)))
      hi = mid;
    else
      lo = mid + 1;
  }
  return lo;
}

// Levels i and i + 1 differ by far more than the rounding of |u - level| on [-1, 1], so the rule's
// choice never decreases as u grows and is fixed by the smallest u reaching each code (its thresholds).
bool build_decision_table(int bits, NfTable* tab) {
  const Levels lv = levels_for(bits);
  const int n = 1 << bits;
  int64_t thr[16];
  for (int i = 1; i < n; ++i) thr[i] = first_true([&](float u) { return nearest_by_rule(u, lv.v, n) >= i; });
  for (int k = 0; k <= 32; ++k) {
    const int64_t lo = first_true([&](float u) { return cell_of(u) >= k; });
    const int64_t hi = k == 32 ? ordinal(1.0f) : first_true([&](float u) { return cell_of(u) >= k + 1; }) - 1;
    tab->base[k] = nearest_by_rule(from_ordinal(lo), lv.v, n);
    tab->t[k] = std::numeric_limits<float>::infinity();
    int inside = 0;
    for (int i = 1; i < n; ++i)
      if (thr[i] > lo && thr[i] <= hi) {
        tab->t[k] = from_ordinal(thr[i]);
        ++inside;
      }
    if (inside > 1) return false;
  }
  return true;
}

}  // namespace

bool nf_decision_table(int bits, NfTable* out) {
  static std::mutex mu;
  static NfTable cache[5];
  static int state[5] = {0, 0, 0, 0, 0};  // 0 not built, 1 built, -1 not representable
  if (bits < 2 || bits > 4 || !out) return false;
  std::lock_guard<std::mutex> lock(mu);
  if (state[bits] == 0) state[bits] = build_decision_table(bits, &cache[bits]) ? 1 : -1;
  if (state[bits] < 0) return false;
  *out = cache[bits];
  return true;
}

cudaError_t launch_quantize_nfk(const float* W, int64_t n_elems, int bits, int block, int dq_block,
                                const qlr_qweight* out, int32_t* status, cudaStream_t st) {
  const int64_t n_blocks = n_elems / block;
  NfTable tab;
  if (bits < 2 || bits > 4 || !nf_decision_table(bits, &tab)) return cudaErrorInvalidValue;
  Levels lv = levels_for(bits);
  int zc = 0;
  for (int i = 0; i < (1 << bits); ++i)
    if (lv.v[i] == 0.f) zc = i;
  return block == 64 ? launch_nfk_block<64>(W, n_blocks, bits, dq_block, tab, zc, out, status, st)
                     : launch_nfk_block<128>(W, n_blocks, bits, dq_block, tab, zc, out, status, st);
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
