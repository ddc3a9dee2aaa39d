// Decode-shape forward (1..16 tokens) of the NF4 layer: Y = X dequant(W)^T + T_save B^T.
//
// At a few tokens the layer is a matrix-vector product bound by the HBM read of the packed 4-bit
// codes (QLoRA explainer, "The complete QLoRA forward pass": each frozen NF4 block is dequantised to
// bf16 on the fly and multiplied by the input).  One warp owns 16 weight rows and streams their codes
// across all of K with 8-byte loads kept several steps in flight; CTAs of four warps (64 rows) give
// 448 CTAs for a 28672-row weight, about three per SM.
//
// Per 128-wide reduction step a lane loads, for rows g and g+8 of its group, 16 codes of each of the
// step's two 64-code halves.  Codes become bf16 NF4 levels through a byte-permute table lookup and
// feed mma.sync m16n8k16 (weight rows on the M side, tokens on the N side, fp32 accumulate); the
// reduction index is permuted consistently for the weight and the input, and every MMA stays inside
// one block, so each block's partial dot products are scaled by the block's constant
// fp32(E4M3(c1_8)) * s2 (or c1) once and added to the accumulator.  The effective weight is therefore
// bf16(level) * scale, rounded once less than the bf16(level * scale) the tensor-core GEMMs use.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "ptx.cuh"

namespace qlr {

namespace {

constexpr int kDecodeWarps = 4;  // 64 weight rows per CTA
constexpr int kInFlight = 4;     // 128-wide reduction steps loaded ahead

struct DecodeParams {
  const uint8_t* codes;
  const float* c1;
  const uint8_t* c1_fp8;
  const float* s2;
  int block, dq_block;
  int block_shift, dq_shift;  // log2 of the block and double-quantisation sizes
  int64_t N, K;
  int M;
  const uint16_t* X;       // [M, K] bf16
  const uint16_t* B;       // [N, r] bf16
  const uint16_t* T_save;  // [M, r] bf16
  int r;
  uint16_t* Y;             // [M, N] bf16
  Levels lv;
};

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

struct Lut16 {
  uint32_t l0, l1, l2, l3, h0, h1, h2, h3;
};

// 4 codes (low 16 bits of w) -> two bf16x2 words, code 0 in the low half of the first.
__device__ __forceinline__ void lut4(const Lut16& t, uint32_t w, uint32_t& o0, uint32_t& o1) {
  const uint32_t sel = w & 0x7777u;
  const uint32_t sel2 = ((w >> 1) & 0x4444u) | 0x3210u;
  const uint32_t lo = prmt(prmt(t.l0, t.l1, sel), prmt(t.l2, t.l3, sel), sel2);
  const uint32_t hi = prmt(prmt(t.h0, t.h1, sel), prmt(t.h2, t.h3, sel), sel2);
  o0 = prmt(lo, hi, 0x5140);
  o1 = prmt(lo, hi, 0x7362);
}

__device__ __forceinline__ float block_scale(const DecodeParams& p, int64_t b) {
  if (p.dq_block) {
    const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(__ldg(p.c1_fp8 + b)), __NV_E4M3);
    return __fmul_rn(__half2float(__half(h)), __ldg(p.s2 + (b >> p.dq_shift)));
  }
  return __ldg(p.c1 + b);
}

// NT: token tiles of 8 (1: M <= 8, 2: M <= 16).
template <int NT>
__global__ void __launch_bounds__(kDecodeWarps * 32) decode_kernel(const DecodeParams p) {
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int64_t row0 = (static_cast<int64_t>(blockIdx.x) * kDecodeWarps + (threadIdx.x >> 5)) * 16;
  if (row0 >= p.N) return;
  const int64_t ra = row0 + g, rb = row0 + g + 8;  // this lane's two weight rows
  const bool va = ra < p.N, vb = rb < p.N;

  Lut16 lut;
  {
    uint32_t pk[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) pk[j] = pack_bf16x2_rn(p.lv.v[2 * j], p.lv.v[2 * j + 1]);
    lut.l0 = prmt(pk[0], pk[1], 0x6420); lut.h0 = prmt(pk[0], pk[1], 0x7531);
    lut.l1 = prmt(pk[2], pk[3], 0x6420); lut.h1 = prmt(pk[2], pk[3], 0x7531);
    lut.l2 = prmt(pk[4], pk[5], 0x6420); lut.h2 = prmt(pk[4], pk[5], 0x7531);
    lut.l3 = prmt(pk[6], pk[7], 0x6420); lut.h3 = prmt(pk[6], pk[7], 0x7531);
  }

  const int64_t row_bytes = p.K / 2;
  // lane (g, t): 8 bytes (16 codes) of each 64-code half, at byte offset 32h + 8t of the step
  const uint2* pa = reinterpret_cast<const uint2*>(p.codes + ra * row_bytes) + t;
  const uint2* pb = reinterpret_cast<const uint2*>(p.codes + rb * row_bytes) + t;
  const int nsteps = static_cast<int>(p.K / 128);
  const int64_t blocks_per_row = p.K / p.block;

  float acc[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;

  uint2 buf[kInFlight][2][2];  // [step][half][row a / row b]
#pragma unroll
  for (int s = 0; s < kInFlight; ++s) {
    if (s < nsteps) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        buf[s][h][0] = va ? __ldg(pa + s * 8 + 4 * h) : make_uint2(0, 0);
        buf[s][h][1] = vb ? __ldg(pb + s * 8 + 4 * h) : make_uint2(0, 0);
      }
    }
  }

  for (int s0 = 0; s0 < nsteps; s0 += kInFlight) {
#pragma unroll
    for (int u = 0; u < kInFlight; ++u) {
      const int s = s0 + u;
      if (s >= nsteps) break;
      uint2 cur[2][2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        cur[h][0] = buf[u][h][0];
        cur[h][1] = buf[u][h][1];
      }
      const int sn = s + kInFlight;  // refill this slot kInFlight steps ahead
      if (sn < nsteps) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          buf[u][h][0] = va ? __ldg(pa + sn * 8 + 4 * h) : make_uint2(0, 0);
          buf[u][h][1] = vb ? __ldg(pb + sn * 8 + 4 * h) : make_uint2(0, 0);
        }
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int64_t k0 = static_cast<int64_t>(s) * 128 + 64 * h;  // first k of this half
        // codes of this lane: row a/b, k = k0 + 16 t + i (i < 16); MMA m (< 4) takes i = 4m .. 4m+3
        float part[NT][4];
#pragma unroll
        for (int n = 0; n < NT; ++n) part[n][0] = part[n][1] = part[n][2] = part[n][3] = 0.f;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const uint32_t wa = (m < 2 ? cur[h][0].x : cur[h][0].y) >> (16 * (m & 1));
          const uint32_t wb = (m < 2 ? cur[h][1].x : cur[h][1].y) >> (16 * (m & 1));
          uint32_t a[4];
          lut4(lut, wa, a[0], a[2]);  // row g: slots (2t,2t+1) <- codes 0,1; (2t+8,2t+9) <- codes 2,3
          lut4(lut, wb, a[1], a[3]);  // row g+8
#pragma unroll
          for (int n = 0; n < NT; ++n) {
            const int tok = 8 * n + g;
            uint32_t b0 = 0, b1 = 0;
            if (tok < p.M) {
              const uint2 xv =
                  __ldg(reinterpret_cast<const uint2*>(p.X + static_cast<int64_t>(tok) * p.K + k0 + 16 * t + 4 * m));
              b0 = xv.x;
              b1 = xv.y;
            }
            mma_bf16_16816(part[n], a, b0, b1);
          }
        }
        const int64_t bidx = k0 >> p.block_shift;
        const float sa = va ? block_scale(p, ra * blocks_per_row + bidx) : 0.f;
        const float sb = vb ? block_scale(p, rb * blocks_per_row + bidx) : 0.f;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          acc[n][0] = fmaf(sa, part[n][0], acc[n][0]);
          acc[n][1] = fmaf(sa, part[n][1], acc[n][1]);
          acc[n][2] = fmaf(sb, part[n][2], acc[n][2]);
          acc[n][3] = fmaf(sb, part[n][3], acc[n][3]);
        }
      }
    }
  }

  // adapter term: rows of B (16 x r) times T_save^T (r x tokens), r/16 more MMAs
  for (int kr = 0; kr < p.r; kr += 16) {
    uint32_t a[4];
    const uint32_t* ba = reinterpret_cast<const uint32_t*>(p.B + ra * p.r + kr);
    const uint32_t* bb = reinterpret_cast<const uint32_t*>(p.B + rb * p.r + kr);
    const bool hi_ok = kr + 8 < p.r;  // r = 8: the upper eight slots are zero
    a[0] = va ? __ldg(ba + t) : 0u;
    a[1] = vb ? __ldg(bb + t) : 0u;
    a[2] = (va && hi_ok) ? __ldg(ba + t + 4) : 0u;
    a[3] = (vb && hi_ok) ? __ldg(bb + t + 4) : 0u;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const int tok = 8 * n + g;
      uint32_t b0 = 0, b1 = 0;
      if (tok < p.M) {
        const uint32_t* tp = reinterpret_cast<const uint32_t*>(p.T_save + static_cast<int64_t>(tok) * p.r + kr);
        b0 = __ldg(tp + t);
        b1 = hi_ok ? __ldg(tp + t + 4) : 0u;
      }
      mma_bf16_16816(acc[n], a, b0, b1);
    }
  }

#pragma unroll
  for (int n = 0; n < NT; ++n) {
    const int tok0 = 8 * n + 2 * t;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int tok = tok0 + e;
      if (tok < p.M) {
        if (va) p.Y[static_cast<int64_t>(tok) * p.N + ra] = static_cast<uint16_t>(pack_bf16x2_rn(acc[n][e], 0.f) & 0xFFFFu);
        if (vb) p.Y[static_cast<int64_t>(tok) * p.N + rb] = static_cast<uint16_t>(pack_bf16x2_rn(acc[n][2 + e], 0.f) & 0xFFFFu);
      }
    }
  }
}

}  // namespace

cudaError_t launch_decode(const qlr_qweight* w, const uint16_t* X, int64_t M, const uint16_t* B, int r,
                          const uint16_t* T_save, uint16_t* Y, cudaStream_t st) {
  DecodeParams p;
  p.codes = w->codes;
  p.c1 = w->c1;
  p.c1_fp8 = w->c1_fp8;
  p.s2 = w->s2;
  p.block = w->block;
  p.dq_block = w->dq_block;
  p.block_shift = w->block == 128 ? 7 : 6;
  p.dq_shift = 8;
  p.N = w->N;
  p.K = w->K;
  p.M = static_cast<int>(M);
  p.X = X;
  p.B = B;
  p.T_save = T_save;
  p.r = r;
  p.Y = Y;
  p.lv = levels_for(4);
  const unsigned grid = static_cast<unsigned>((w->N + 16 * kDecodeWarps - 1) / (16 * kDecodeWarps));
  count_launch();
  if (M <= 8)
    decode_kernel<1><<<grid, kDecodeWarps * 32, 0, st>>>(p);
  else
    decode_kernel<2><<<grid, kDecodeWarps * 32, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace qlr
