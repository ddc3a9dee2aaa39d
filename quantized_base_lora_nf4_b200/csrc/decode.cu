// Decode-shape forward (1..16 tokens) of the NF4 + double-quantised layer: Y = X dequant(W)^T + T_save B^T.
//
// At a few tokens the layer is a matrix-vector product bound by the HBM read of the packed 4-bit
// codes (QLoRA explainer, "The complete QLoRA forward pass": each frozen NF4 block is dequantised to
// bf16 on the fly and multiplied by the input).  A CTA owns 64 weight rows: a producer warp streams
// every 128-wide reduction step -- the rows' codes (64 x 64 bytes, 64-byte swizzle) and the input
// tile (16 tokens x 128, 128-byte swizzle) -- by TMA into a ring of 5-6 shared-memory slots, and four
// compute warps (16 rows each) consume it.  The block constants of the 64 rows are staged in shared
// memory once.  448 CTAs of 160 threads cover a 28672-row weight in one wave.
//
// Per step a lane takes, for rows g and g+8 of its warp, 16 codes of each of the step's two 64-code
// halves.  Codes become bf16 NF4 levels through a byte-permute table lookup and
// feed mma.sync m16n8k16 (weight rows on the M side, tokens on the N side, fp32 accumulate); the
// reduction index is permuted consistently for the weight and the input, and every MMA stays inside
// one block, so each block's partial dot products are scaled by the block's constant
// fp32(E4M3(c1_8)) * s2 (or c1) once and added to the accumulator.  The effective weight is therefore
// bf16(level) * scale, rounded once less than the bf16(level * scale) the tensor-core GEMMs use.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include <mutex>

#include "common.cuh"
#include "gemm.cuh"
#include "ptx.cuh"

namespace qlr {

namespace {

constexpr int kComputeWarps = 4;                 // 64 weight rows per CTA, 16 per warp
constexpr int kThreads = (kComputeWarps + 1) * 32;  // + one TMA producer warp

struct DecodeParams {
  const uint8_t* c1_fp8;
  const float* s2;
  int block_shift;          // log2 of the block (64 or 128)
  int64_t N, K;
  int M;
  const uint16_t* B;        // [N, r] bf16
  const uint16_t* T_save;   // [M, r] bf16
  int r;
  uint16_t* Y;              // [M, N] bf16
  Levels lv;
  int32_t* status;
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

template <int NT>
struct DCfg {
  static constexpr int kCodes = 64 * 64;            // [64 rows][64 bytes] of codes per step
  static constexpr int kXHalf = 8 * NT * 128;        // [8 NT tokens][64 bf16] per half step
  static constexpr int kSlot = kCodes + 2 * kXHalf;  // 1 KB multiple
  static constexpr int kSlots = NT == 1 ? 6 : 5;
};

// Shared-memory bytes after the ring: E4M3 bytes of 64 rows, the s2 values they use, barriers.
inline int decode_scale_bytes(int64_t bpr) { return static_cast<int>((64 * bpr + 1023) / 1024 * 1024) + 2048; }

struct alignas(8) DBars {
  uint64_t full[8];
  uint64_t empty[8];
  int abort_flag;
};

// NT: token tiles of 8 (1: M <= 8, 2: M <= 16).
template <int NT>
__global__ void __launch_bounds__(kThreads) decode_kernel(const __grid_constant__ DecodeParams p,
                                                          const __grid_constant__ CUtensorMap tm_codes,
                                                          const __grid_constant__ CUtensorMap tm_x) {
  using C = DCfg<NT>;
  constexpr int NSL = C::kSlots;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  const int64_t bpr = p.K >> p.block_shift;      // blocks per row
  uint8_t* s_c8 = smem + NSL * C::kSlot;        // [64 rows][blocks per row] E4M3 bytes
  float* s_s2 = reinterpret_cast<float*>(s_c8 + (64 * bpr + 1023) / 1024 * 1024);  // <= 64 bpr / 256 + 2 values
  DBars* bars = reinterpret_cast<DBars*>(reinterpret_cast<uint8_t*>(s_s2) + 1024);
  volatile int* abort_flag = &bars->abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * 64;
  const int nsteps = static_cast<int>(p.K / 128);
  const int64_t s2_first = (row0 * bpr) >> 8;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSL; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], kComputeWarps);
    }
    bars->abort_flag = 0;
    fence_barrier_init();
  }
  // block constants of this CTA's 64 rows, once
  {
    const int64_t rows = (p.N - row0) < 64 ? (p.N - row0) : 64;
    const int64_t n8 = rows * bpr;
    for (int64_t i = threadIdx.x; i < n8; i += kThreads) s_c8[i] = __ldg(p.c1_fp8 + row0 * bpr + i);
    const int64_t n2 = (((row0 + rows) * bpr - 1) >> 8) - s2_first + 1;
    for (int64_t i = threadIdx.x; i < n2; i += kThreads) s_s2[i] = __ldg(p.s2 + s2_first + i);
  }
  __syncthreads();

  if (warp == kComputeWarps) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_codes);
      tma_prefetch_desc(&tm_x);
      int s = 0;
      for (; s < nsteps; ++s) {
        const int sl = s % NSL;
        if (!mbar_wait(&bars->empty[sl], ((s / NSL) & 1) ^ 1, abort_flag)) break;
        uint8_t* slot = ring + sl * C::kSlot;
        mbar_arrive_expect_tx(&bars->full[sl], C::kSlot);
        tma_load_2d(slot, &tm_codes, s * 64, static_cast<int32_t>(row0), &bars->full[sl]);
        tma_load_2d(slot + C::kCodes, &tm_x, s * 128, 0, &bars->full[sl]);
        tma_load_2d(slot + C::kCodes + C::kXHalf, &tm_x, s * 128 + 64, 0, &bars->full[sl]);
      }
      const int first = s > NSL ? s - NSL : 0;  // drain the loads still in flight
      for (int q = first; q < s; ++q) {
        volatile int never = 0;
        mbar_wait(&bars->full[q % NSL], (q / NSL) & 1, &never);
      }
    }
  } else {
    // ------------------------------------------------------------------ compute warps
    const int g = lane >> 2, t = lane & 3;
    const int lr_a = warp * 16 + g, lr_b = lr_a + 8;     // local rows 0..63
    const int64_t ra = row0 + lr_a, rb = row0 + lr_b;
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
    auto scale = [&](int lr, int64_t b) -> float {  // fp32(E4M3(c1_8)) * s2 of block b of local row lr
      const __half_raw hr =
          __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(s_c8[lr * bpr + b]), __NV_E4M3);
      return __fmul_rn(__half2float(__half(hr)), s_s2[(((row0 + lr) * bpr + b) >> 8) - s2_first]);
    };
    float acc[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
    for (int s = 0; s < nsteps; ++s) {
      const int sl = s % NSL;
      const bool ok = mbar_wait(&bars->full[sl], (s / NSL) & 1, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      const uint8_t* codes = ring + sl * C::kSlot;
      const uint8_t* xs = codes + C::kCodes;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        // 64-byte swizzled code rows: 16-byte chunk c of row r sits at chunk c ^ ((r >> 1) & 3)
        const int c = 2 * h + (t >> 1);
        const uint2 wa = *reinterpret_cast<const uint2*>(codes + lr_a * 64 + ((c ^ ((lr_a >> 1) & 3)) << 4) + 8 * (t & 1));
        const uint2 wb = *reinterpret_cast<const uint2*>(codes + lr_b * 64 + ((c ^ ((lr_b >> 1) & 3)) << 4) + 8 * (t & 1));
        const uint8_t* xh = xs + h * C::kXHalf;
        float part[NT][4];
#pragma unroll
        for (int n = 0; n < NT; ++n) part[n][0] = part[n][1] = part[n][2] = part[n][3] = 0.f;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          // this lane's codes: k = 128 s + 64 h + 16 t + i; MMA m takes i = 4m .. 4m+3
          uint32_t a[4];
          lut4(lut, (m < 2 ? wa.x : wa.y) >> (16 * (m & 1)), a[0], a[2]);
          lut4(lut, (m < 2 ? wb.x : wb.y) >> (16 * (m & 1)), a[1], a[3]);
#pragma unroll
          for (int n = 0; n < NT; ++n) {
            // 128-byte swizzled input rows: X[tok][16 t + 4 m .. +3] at chunk (2t + m/2) ^ (tok & 7)
            const int tok = 8 * n + g;
            const int ch = (2 * t + (m >> 1)) ^ (tok & 7);
            const uint2 xv = *reinterpret_cast<const uint2*>(xh + tok * 128 + (ch << 4) + 8 * (m & 1));
            mma_bf16_16816(part[n], a, xv.x, xv.y);
          }
        }
        const int64_t b = (static_cast<int64_t>(s) * 128 + 64 * h) >> p.block_shift;
        const float sa = va ? scale(lr_a, b) : 0.f;
        const float sb = vb ? scale(lr_b, b) : 0.f;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          acc[n][0] = fmaf(sa, part[n][0], acc[n][0]);
          acc[n][1] = fmaf(sa, part[n][1], acc[n][1]);
          acc[n][2] = fmaf(sb, part[n][2], acc[n][2]);
          acc[n][3] = fmaf(sb, part[n][3], acc[n][3]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->empty[sl]);
    }

    // adapter term: rows of B (16 x r) times T_save^T (r x tokens), r/16 more MMAs
    for (int kr = 0; kr < p.r; kr += 16) {
      const bool hi_ok = kr + 8 < p.r;  // r = 8: the upper eight slots are zero
      const uint32_t* ba = reinterpret_cast<const uint32_t*>(p.B + ra * p.r + kr);
      const uint32_t* bb = reinterpret_cast<const uint32_t*>(p.B + rb * p.r + kr);
      uint32_t a[4];
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
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int tok = 8 * n + 2 * t + e;
        if (tok < p.M) {
          if (va) p.Y[static_cast<int64_t>(tok) * p.N + ra] = static_cast<uint16_t>(pack_bf16x2_rn(acc[n][e], 0.f) & 0xFFFFu);
          if (vb) p.Y[static_cast<int64_t>(tok) * p.N + rb] = static_cast<uint16_t>(pack_bf16x2_rn(acc[n][2 + e], 0.f) & 0xFFFFu);
        }
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && bars->abort_flag) report(p.status, QLR_ERR_TIMEOUT);
}

template <int NT>
cudaError_t launch_decode_variant(const DecodeParams& p, const CUtensorMap& tc, const CUtensorMap& tx,
                                  cudaStream_t st) {
  using C = DCfg<NT>;
  const int smem = C::kSlots * C::kSlot + decode_scale_bytes(p.K >> p.block_shift) + 1024;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [&] {
    attr_err = cudaFuncSetAttribute(decode_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
  });
  if (attr_err != cudaSuccess) return attr_err;
  const unsigned grid = static_cast<unsigned>((p.N + 63) / 64);
  count_launch();
  decode_kernel<NT><<<grid, kThreads, smem, st>>>(p, tc, tx);
  return cudaGetLastError();
}

}  // namespace

bool decode_supported(const qlr_qweight* w, int64_t M) {
  return M >= 1 && M <= 16 && w->fmt == QLR_FMT_NFK && w->bits == 4 && w->dq_block == 256 && w->K % 128 == 0 &&
         w->K <= 32768;
}

cudaError_t launch_decode(const qlr_qweight* w, const uint16_t* X, int64_t M, const uint16_t* B, int r,
                          const uint16_t* T_save, uint16_t* Y, int32_t* status, cudaStream_t st) {
  DecodeParams p;
  p.c1_fp8 = w->c1_fp8;
  p.s2 = w->s2;
  p.block_shift = w->block == 128 ? 7 : 6;
  p.N = w->N;
  p.K = w->K;
  p.M = static_cast<int>(M);
  p.B = B;
  p.T_save = T_save;
  p.r = r;
  p.Y = Y;
  p.lv = levels_for(4);
  p.status = status;
  const int nt = M <= 8 ? 1 : 2;
  CUtensorMap tc, tx;
  if (make_tmap(&tc, w->codes, 1, w->N, w->K / 2, 64, 64, 64)) return cudaErrorInvalidValue;
  if (make_tmap(&tx, X, 2, M, w->K, 8 * nt, 64, 128)) return cudaErrorInvalidValue;
  return nt == 1 ? launch_decode_variant<1>(p, tc, tx, st) : launch_decode_variant<2>(p, tc, tx, st);
}

}  // namespace qlr
