// Decode-shape forward (1..16 tokens) of the NF4 + double-quantised layer: Y = X dequant(W)^T + T_save B^T.
//
// At a few tokens the layer is a matrix-vector product bound by the HBM read of the packed 4-bit
// codes (QLoRA explainer, "The complete QLoRA forward pass": each frozen NF4 block is dequantised to
// bf16 on the fly and multiplied by the input).  One persistent CTA per SM owns a contiguous range of
// 16-row units (12 or 13 for a 28672-row weight on 148 SMs) and one compute warp per unit; a producer
// warp streams every 256-wide reduction step -- one box of all the CTA's codes (16 rows x 128 bytes per
// unit, 128-byte swizzle) and the input tile as four quarters of tokens x 64 (128-byte swizzle) -- by TMA
// into a ring of shared-memory slots that all compute warps consume in step.  A warp takes the whole
// step of its unit (16 MMAs at up to 8 tokens), so the per-step costs (the slot wait and release, the
// block scales) are paid once per 4096 weights.
//
// A code byte (two 4-bit codes) becomes the bf16 pair (level[lo], level[hi]) with one shared-memory
// load from a 256-entry table replicated per lane (conflict-free), which is exactly one mma.sync
// m16n8k16 A-register.  The weight rows are the MMA's M side, tokens its N side, fp32 accumulate;
// the reduction index is permuted consistently for weight and input, every MMA stays inside one
// block, and each block's partial sums are scaled once by fp32(E4M3(c1_8)) * s2.  The effective weight
// is bf16(level) * scale: one rounding fewer than the bf16(level * scale) of the tensor-core GEMMs.
// The adapter term T_save B^T seeds the accumulators before the first step, so its global loads overlap
// the first ring fills.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "gemm.cuh"
#include "ptx.cuh"

namespace qlr {

namespace {

constexpr int kMaxUnits = 14;                        // 16-row units per CTA
constexpr int kComputeWarps = kMaxUnits;             // one per unit
constexpr int kThreads = (kComputeWarps + 1) * 32;   // + one TMA producer warp

struct DecodeParams {
  const uint8_t* c1_fp8;
  const float* s2;
  int block_shift;          // log2 of the block (64 or 128)
  int64_t N, K;
  int M;
  int units;                // ceil(N / 16)
  int nu_lo;                // every CTA owns nu_lo or nu_lo + 1 (<= kMaxUnits) units
  const uint16_t* B;        // [N, r] bf16
  const uint16_t* T_save;   // [M, r] bf16
  int r;
  uint16_t* Y;              // [M, N] bf16
  Levels lv;
  int32_t* status;
  long long wait_cycles;    // bound of every pipeline wait (SM clock cycles)
};

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// One step = 256 reduction inputs: per unit 16 rows x 128 code bytes (128-byte swizzle), and the input
// tile as four quarters of [8 NT tokens][64 bf16].
template <int NT>
struct DCfg {
  static constexpr int kUnitCodes = 16 * 128;
  static constexpr int kXQ = 8 * NT * 128;
  static constexpr int kSlot = kMaxUnits * kUnitCodes + 4 * kXQ;  // 32 KB (NT = 1) or 36 KB (NT = 2)
  static constexpr int kHighSlots = NT == 1 ? 3 : 2;              // slots from 128 KB up
};

// Shared-memory map, as shared-window addresses.  The dequantisation table sits at 64 KB so that one
// byte permute of (code word, 4 lane | 64 KB) yields the address of a table entry; each 256-byte entry
// uses its first 128 bytes, and the E4M3 block constants of CTA row lr fill the second half of entry lr
// when a row has at most 128 of them, their 4-byte words XOR-swizzled by lr mod 32 so that the rows a warp
// reads at the same block index sit in different banks (rows 256 bytes apart would share one).  Below the table: the barriers, the s2 values (and the E4M3
// constants of longer rows), and one more ring slot ending at 64 KB when it fits; the other slots start
// at 128 KB.
constexpr uint32_t kLutAddr = 0x10000;   // [256 code bytes][256 B: 32 lanes x bf16x2 | E4M3 row]
constexpr uint32_t kRingAddr = 0x20000;
constexpr uint32_t kBarBytes = 1024;

struct alignas(8) DBars {
  uint64_t full[6];
  uint64_t empty[6];
  int abort_flag;
};

// Below-table layout for a window whose barriers start at bars_addr (<= 1 KB on every launch).
struct DLayout {
  uint32_t s2_addr, c8_addr, c8_stride, const_end;
  bool c8_swizzled;  // in the table's free halves: byte b of row lr at b ^ 4 (lr mod 32)
};
__host__ __device__ inline DLayout decode_layout(uint32_t bars_addr, int64_t bpr) {
  DLayout L;
  L.s2_addr = bars_addr + kBarBytes;
  const uint32_t s2_bytes = static_cast<uint32_t>(((16ull * kMaxUnits * bpr) / 256 + 4) * 4 + 15) & ~15u;
  if (bpr <= 128) {
    L.c8_addr = kLutAddr + 128;
    L.c8_stride = 256;
    L.c8_swizzled = true;
    L.const_end = L.s2_addr + s2_bytes;
  } else {
    L.c8_addr = L.s2_addr + s2_bytes;
    L.c8_stride = static_cast<uint32_t>(bpr + 4);
    L.c8_swizzled = false;
    L.const_end = L.c8_addr + 16u * kMaxUnits * L.c8_stride;
  }
  return L;
}

// The dynamic window starts at some address of at most 1 KB (reserved shared memory), so a window of
// kRingAddr + the high slots reaches past the ring whatever that start is.
inline size_t decode_smem_bytes(int nt) {
  return kRingAddr + static_cast<size_t>(nt == 1 ? DCfg<1>::kHighSlots * DCfg<1>::kSlot
                                                 : DCfg<2>::kHighSlots * DCfg<2>::kSlot);
}

// The table is written once before the first barrier and only read afterwards, so its loads may be
// scheduled freely (no volatile); the ring loads stay ordered after their barrier waits.
__device__ __forceinline__ uint32_t lds_table(uint32_t addr) {
  uint32_t v;
  asm("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint2 lds_v2(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint32_t lds_u8(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ float lds_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v));
}
__device__ __forceinline__ void sts_u8(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.u8 [%0], %1;" ::"r"(addr), "r"(v));
}

// NT: token tiles of 8 (1: M <= 8, 2: M <= 16).
template <int NT>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const __grid_constant__ DecodeParams p,
                                                             const __grid_constant__ CUtensorMap tm_codes_lo,
                                                             const __grid_constant__ CUtensorMap tm_codes_hi,
                                                             const __grid_constant__ CUtensorMap tm_x) {
  using C = DCfg<NT>;
  constexpr int kMaxSlots = C::kHighSlots + 1;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t base = smem_u32(smem_raw);
  const int64_t bpr = p.K >> p.block_shift;  // blocks per row
  const uint32_t bars_addr = (base + 1023u) & ~1023u;
  const DLayout lay = decode_layout(bars_addr, bpr);
  if (lay.const_end > kLutAddr) {  // the window starts higher than assumed
    if (threadIdx.x == 0) report(p.status, QLR_ERR_UNSUPPORTED);
    return;
  }
  // one more slot below the table when the constants leave room for it
  const uint32_t low_slot = kLutAddr - C::kSlot;
  const int nslots = lay.const_end <= low_slot ? kMaxSlots : C::kHighSlots;
  auto slot_addr = [&](int sl) { return sl < C::kHighSlots ? kRingAddr + sl * C::kSlot : low_slot; };
  auto gen = [&](uint32_t addr) { return smem_raw + (addr - base); };  // generic pointer of a shared address
  DBars* bars = reinterpret_cast<DBars*>(gen(bars_addr));
  uint32_t* lut = reinterpret_cast<uint32_t*>(gen(kLutAddr));
  volatile int* abort_flag = &bars->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // this CTA's contiguous range of 16-row units
  const int u_begin = static_cast<int>((static_cast<int64_t>(blockIdx.x) * p.units) / gridDim.x);
  const int u_end = static_cast<int>((static_cast<int64_t>(blockIdx.x + 1) * p.units) / gridDim.x);
  const int nsteps = static_cast<int>(p.K / 256);

  pdl_launch_dependents();
  pdl_wait();
  if (threadIdx.x == 0) {
    for (int s = 0; s < nslots; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], kComputeWarps);
    }
    bars->abort_flag = 0;
    fence_barrier_init();
  }
  // code byte e -> (bf16 level[e & 15], bf16 level[e >> 4]), one copy per lane at 64 KB + 256 e + 4 lane
  for (int i = threadIdx.x; i < 256 * 32; i += kThreads) {
    const int e = i >> 5;
    lut[e * 64 + (i & 31)] = pack_bf16x2_rn(p.lv.v[e & 15], p.lv.v[e >> 4]);
  }

  __syncthreads();  // barriers and table ready

  const int nu = u_end - u_begin;  // nu_lo or nu_lo + 1, at most kMaxUnits (host grid sizing)
  const int64_t prow0 = static_cast<int64_t>(u_begin) * 16;
  const int prows = static_cast<int>(static_cast<int64_t>(nu) * 16 < p.N - prow0 ? nu * 16 : p.N - prow0);
  const int64_t s2_first = (prow0 * bpr) >> 8;

  if (warp == kComputeWarps) {
    // ---------------------------------------------------------------- TMA producer
    // one box of all this CTA's rows (16 nu x 128 B of codes) and four input quarters per step
    if (lane == 0) {
      const CUtensorMap* tm_codes = nu == p.nu_lo ? &tm_codes_lo : &tm_codes_hi;
      tma_prefetch_desc(tm_codes);
      tma_prefetch_desc(&tm_x);
      int sl = 0;
      uint32_t ph = 0;  // ring slot and the parity of its current fill
      for (int s = 0; s < nsteps; ++s) {
        if (!mbar_wait(&bars->empty[sl], ph ^ 1, abort_flag, p.wait_cycles)) break;
        uint8_t* slot = gen(slot_addr(sl));
        mbar_arrive_expect_tx(&bars->full[sl], nu * C::kUnitCodes + 4 * C::kXQ);
        tma_load_2d(slot, tm_codes, s * 128, static_cast<int32_t>(prow0), &bars->full[sl]);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          tma_load_2d(slot + kMaxUnits * C::kUnitCodes + q * C::kXQ, &tm_x, s * 256 + 64 * q, 0, &bars->full[sl]);
        if (++sl == nslots) {
          sl = 0;
          ph ^= 1;
        }
      }
      // after an abort, the copies still in flight must land before the CTA may exit: wait for the
      // last fill of every slot (one outstanding fill per slot at most)
      if (*abort_flag) {
        for (int k = 0; k < nslots; ++k) {
          if (--sl < 0) {
            sl = nslots - 1;
            ph ^= 1;
          }
          mbar_drain(&bars->full[sl], ph);
        }
      }
    }
  } else {
    // ---------------------------------------------------------------- compute warps
    const int g = lane >> 2, t = lane & 3;
    const int unit = warp;
    const bool active = unit < nu;
    // MMA row g reads weight row pi(g): rows 0, 2, 4, 6 for g = 0..3 and 1, 3, 5, 7 for g = 4..7, which spreads
    // each half-warp's code loads over all 32 banks under the 128-byte swizzle
    const int pg = ((g & 3) << 1) | (g >> 2);
    const int lr_a = unit * 16 + pg, lr_b = lr_a + 8;  // rows of this CTA, 0 .. 16 nu - 1
    const int64_t ra = prow0 + lr_a, rb = prow0 + lr_b;
    const bool va = active && ra < p.N, vb = active && rb < p.N;

    // stage the block constants of this CTA's rows: every load of a thread issued before its stores
    {
      const int64_t g0 = prow0 * bpr;  // first E4M3 byte of the CTA
      if ((bpr & 3) == 0) {
        constexpr int kRowsPerWarp = (16 * kMaxUnits + kComputeWarps - 1) / kComputeWarps;  // 16
        for (int cb = 4 * lane; cb < bpr; cb += 128) {
          uint32_t v[kRowsPerWarp];
#pragma unroll
          for (int j = 0; j < kRowsPerWarp; ++j) {
            const int lr = warp + j * kComputeWarps;
            v[j] = lr < prows ? __ldg(reinterpret_cast<const uint32_t*>(p.c1_fp8 + g0 + lr * bpr + cb)) : 0u;
          }
#pragma unroll
          for (int j = 0; j < kRowsPerWarp; ++j) {
            const int lr = warp + j * kComputeWarps;
            if (lr < prows) sts_u32(lay.c8_addr + lr * lay.c8_stride + (cb ^ (lay.c8_swizzled ? (lr & 31) << 2 : 0)), v[j]);
          }
        }
      } else {
        for (int lr = warp; lr < prows; lr += kComputeWarps)
          for (int b = lane; b < bpr; b += 32)
            sts_u8(lay.c8_addr + lr * lay.c8_stride + (b ^ (lay.c8_swizzled ? (lr & 31) << 2 : 0)),
                   __ldg(p.c1_fp8 + g0 + lr * bpr + b));
      }
      const int n2 = static_cast<int>((((prow0 + prows) * bpr - 1) >> 8) - s2_first + 1);
      float* s_s2 = reinterpret_cast<float*>(gen(lay.s2_addr));
      for (int i = threadIdx.x; i < n2; i += kComputeWarps * 32) s_s2[i] = __ldg(p.s2 + s2_first + i);
    }

    float acc[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
    // adapter term first: rows of B (16 x r) times T_save^T (r x tokens), r/16 MMAs per token tile
    if (active) {
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
    }
    named_bar_sync(1, kComputeWarps * 32);  // constants staged

    const uint32_t lut_lane = kLutAddr | (4u * lane);
    // per-lane parts of the shared addresses that do not change from step to step: quarter q of a row is
    // 16-byte chunks 2q, 2q + 1 (lane t reads 8 bytes of chunk 2q + t/2), XOR-swizzled by the row index mod 8
    // (rows pg and pg + 8 have the same index mod 8, so one swizzled chunk offset serves both); the chunk of
    // quarter q is that of quarter 0 XOR 2q
    const uint32_t code_a = unit * C::kUnitCodes + pg * 128 + 8 * (t & 1) +
                            static_cast<uint32_t>(((t >> 1) ^ (pg & 7)) << 4);
    const uint32_t code_b = code_a + 8 * 128;
    // lane t computes the scales of row (t odd ? b : a) in quarters t / 2 and 2 + t / 2; the other lanes of
    // the row pair fetch them by shuffle
    const bool v_own = (t & 1) ? vb : va;
    const int lr_own = (t & 1) ? lr_b : lr_a;
    const uint32_t c8_own = lay.c8_addr + lr_own * lay.c8_stride;
    const uint32_t c8_x = lay.c8_swizzled ? static_cast<uint32_t>(lr_own & 31) << 2 : 0u;
    const uint32_t s2_own = lr_own * static_cast<uint32_t>(bpr) + static_cast<uint32_t>((prow0 * bpr) & 255);
    const int bshift = p.block_shift;
    // the input fragments for this lane: X[tok][64 q + 16 t .. +15], two swizzled 16-byte chunks per quarter
    uint32_t x_off[NT][2];
    bool x_ok[NT];
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const int tok = 8 * n + g;
      x_ok[n] = tok < p.M;  // rows past the last token are zero; skipping them saves shared-memory wavefronts
      x_off[n][0] = kMaxUnits * C::kUnitCodes + tok * 128 + (((2 * t) ^ (tok & 7)) << 4);
      x_off[n][1] = kMaxUnits * C::kUnitCodes + tok * 128 + (((2 * t + 1) ^ (tok & 7)) << 4);
    }
    auto load_x = [&](uint32_t slot, int q, uint4 (&xv)[NT][2]) {
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        if (x_ok[n]) {
          xv[n][0] = lds_v4(slot + x_off[n][0] + q * C::kXQ);
          xv[n][1] = lds_v4(slot + x_off[n][1] + q * C::kXQ);
        } else {
          xv[n][0] = xv[n][1] = make_uint4(0u, 0u, 0u, 0u);
        }
      }
    };
    // one quarter: 4 MMAs per token tile on unscaled levels, then the block scale applied once
    auto quarter = [&](const uint2 wa, const uint2 wb, const uint4 (&xv)[NT][2], float sa, float sb) {
      float part[NT][4];
#pragma unroll
      for (int n = 0; n < NT; ++n) part[n][0] = part[n][1] = part[n][2] = part[n][3] = 0.f;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        // this lane's codes: k = 256 s + 64 q + 16 t + i; MMA m takes i = 4m .. 4m+3 (bytes 2m, 2m+1)
        const uint32_t qa = m < 2 ? wa.x : wa.y, qb = m < 2 ? wb.x : wb.y;
        // byte permute: address bytes 0, 2, 3 from (4 lane | 64 KB), byte 1 = the code byte
        constexpr uint32_t kSelLo[2] = {0x7604u, 0x7624u}, kSelHi[2] = {0x7614u, 0x7634u};
        uint32_t af[4];
        af[0] = lds_table(__byte_perm(qa, lut_lane, kSelLo[m & 1]));
        af[2] = lds_table(__byte_perm(qa, lut_lane, kSelHi[m & 1]));
        af[1] = lds_table(__byte_perm(qb, lut_lane, kSelLo[m & 1]));
        af[3] = lds_table(__byte_perm(qb, lut_lane, kSelHi[m & 1]));
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          const uint4 x4 = xv[n][m >> 1];
          mma_bf16_16816(part[n], af, (m & 1) ? x4.z : x4.x, (m & 1) ? x4.w : x4.y);
        }
      }
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        acc[n][0] = fmaf(sa, part[n][0], acc[n][0]);
        acc[n][1] = fmaf(sa, part[n][1], acc[n][1]);
        acc[n][2] = fmaf(sb, part[n][2], acc[n][2]);
        acc[n][3] = fmaf(sb, part[n][3], acc[n][3]);
      }
    };

    int sl = 0;
    uint32_t ph = 0;  // ring slot and the parity of its current fill
    for (int s = 0; s < nsteps; ++s) {
      const bool ok = mbar_wait(&bars->full[sl], ph, abort_flag, p.wait_cycles);
      if (!__all_sync(0xffffffffu, ok)) break;
      const uint32_t slot = slot_addr(sl);  // codes [unit][16 rows][128 B], then the input quarters
      if (active) {
        uint2 wa[4], wb[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          wa[q] = lds_v2(slot + (code_a ^ (static_cast<uint32_t>(q) << 5)));
          wb[q] = lds_v2(slot + (code_b ^ (static_cast<uint32_t>(q) << 5)));
        }
        // the scales of this lane's row in quarters t / 2 (h = 0) and 2 + t / 2 (h = 1)
        float my_scale[2] = {0.f, 0.f};
        if (v_own) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t b = static_cast<uint32_t>((s * 256 + 64 * (2 * h + (t >> 1))) >> bshift);
            const __half_raw hr =
                __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(lds_u8(c8_own + (b ^ c8_x))), __NV_E4M3);
            my_scale[h] = __fmul_rn(__half2float(__half(hr)), lds_f32(lay.s2_addr + ((s2_own + b) >> 8) * 4));
          }
        }
        if (NT == 1) {  // copy every quarter's input to registers and free the slot before the arithmetic
          uint4 xv[4][NT][2];
#pragma unroll
          for (int q = 0; q < 4; ++q) load_x(slot, q, xv[q]);
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->empty[sl]);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float sa = __shfl_sync(0xffffffffu, my_scale[q >> 1], (lane & ~3) + 2 * (q & 1));
            const float sb = __shfl_sync(0xffffffffu, my_scale[q >> 1], (lane & ~3) + 2 * (q & 1) + 1);
            quarter(wa[q], wb[q], xv[q], sa, sb);
          }
        } else {  // 16 tokens: one quarter's input at a time; free the slot afterwards
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 xv[NT][2];
            load_x(slot, q, xv);
            const float sa = __shfl_sync(0xffffffffu, my_scale[q >> 1], (lane & ~3) + 2 * (q & 1));
            const float sb = __shfl_sync(0xffffffffu, my_scale[q >> 1], (lane & ~3) + 2 * (q & 1) + 1);
            quarter(wa[q], wb[q], xv, sa, sb);
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->empty[sl]);
        }
      } else {
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->empty[sl]);
      }
      if (++sl == nslots) {
        sl = 0;
        ph ^= 1;
      }
    }
    if (active) {
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
  }
  __syncthreads();
  if (threadIdx.x == 0 && bars->abort_flag) report(p.status, QLR_ERR_TIMEOUT);
}

template <int NT>
cudaError_t launch_decode_variant(const DecodeParams& p, int grid, const CUtensorMap& tc_lo, const CUtensorMap& tc_hi,
                                  const CUtensorMap& tx, cudaStream_t st) {
  const size_t smem = decode_smem_bytes(NT);
  const cudaError_t attr_err = ensure_max_dynamic_smem(decode_kernel<NT>, 227 * 1024);
  if (attr_err != cudaSuccess) return attr_err;
  return launch_pdl(decode_kernel<NT>, dim3(grid), dim3(kThreads), smem, st, p, tc_lo, tc_hi, tx);
}

}  // namespace

bool decode_supported(const qlr_qweight* w, int64_t M) {
  if (M < 1 || M > 16 || w->fmt != QLR_FMT_NFK || w->bits != 4 || w->dq_block != 256 || w->K % 256) return false;
  // the constants fit below the table when the window starts within its first kilobyte
  return decode_layout(1024, w->K / w->block).const_end <= kLutAddr && decode_smem_bytes(M <= 8 ? 1 : 2) <= 227 * 1024;
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
  p.units = static_cast<int>((w->N + 15) / 16);
  // one CTA per SM, each owning a contiguous run of units; more CTAs only when a run would exceed kMaxUnits
  const int sms = device_sm_count();
  int grid = p.units < sms ? p.units : sms;
  if (grid < (p.units + kMaxUnits - 1) / kMaxUnits) grid = (p.units + kMaxUnits - 1) / kMaxUnits;
  p.nu_lo = p.units / grid;
  const int nu_hi = std::min({p.nu_lo + 1, kMaxUnits, p.units});
  p.B = B;
  p.T_save = T_save;
  p.r = r;
  p.Y = Y;
  p.lv = levels_for(4);
  p.status = status;
  p.wait_cycles = wait_limit_cycles();
  const int nt = M <= 8 ? 1 : 2;
  CUtensorMap tc_lo, tc_hi, tx;
  if (make_tmap(&tc_lo, w->codes, 1, w->N, w->K / 2, 16 * p.nu_lo, 128, 128)) return cudaErrorInvalidValue;
  if (make_tmap(&tc_hi, w->codes, 1, w->N, w->K / 2, 16 * nu_hi, 128, 128)) return cudaErrorInvalidValue;
  if (make_tmap(&tx, X, 2, M, w->K, 8 * nt, 64, 128)) return cudaErrorInvalidValue;
  return nt == 1 ? launch_decode_variant<1>(p, grid, tc_lo, tc_hi, tx, st)
                 : launch_decode_variant<2>(p, grid, tc_lo, tc_hi, tx, st);
}

}  // namespace qlr
