// tcgen05 GEMM engine for sm_100a.
//
// One persistent CTA per SM walks a static list of output tiles (128 x BN).  Warp roles:
//   warp 0        TMA producer: fills a ring of shared-memory stages (A tile, B tile, and for the
//                 fused quantised paths a tile of packed 4-bit codes instead of A);
//   warp 1        allocates TMEM and issues tcgen05.mma (one elected lane), committing each stage
//                 back to the producer and each finished tile to the epilogue;
//   warps 2..5    epilogue: TMEM -> registers -> (bf16, transposed through shared memory) -> global;
//   warps 6..13   (fused paths only) dequantise the codes of a stage into the bf16 A tile, laid out
//                 in the canonical 128-byte-swizzled UMMA layout, K-major (forward) or MN-major
//                 (input gradient).  Two groups of four warps take alternate stages.
// Two TMEM accumulators (2 x BN fp32 columns) let the epilogue of one tile overlap the main loop
// of the next.  A "tail" segment appends extra reduction columns with their own operands: the
// LoRA term s T B^T in the forward and dT A in the input gradient, folded into the same
// accumulator instead of running as a separate GEMM.
//
// Dequantisation of 64 codes of one row (one NF block or two INT4 groups) builds a 16-entry bf16
// table from the block's scale once, then maps 8 codes per 32-bit word to 4 bf16 pairs with byte
// permutes (prmt), so every element costs under three integer ops and no shared-memory lookup.
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "gemm.cuh"
#include "ptx.cuh"

namespace qlr {

namespace {

constexpr int kThreadsPlain = 192;  // producer, MMA, 4 epilogue warps
constexpr int kThreadsDq = 448;     // + 8 dequantiser warps

template <int BN, bool DQ>
struct Cfg {
  static constexpr int kA = 16384;
  static constexpr int kB = BN * 128;
  static constexpr int kC = DQ ? 4096 : 0;
  static constexpr int kStage = ((kA + kB + kC) + 1023) / 1024 * 1024;
  static constexpr int kStaging = 4 * 32 * 32 * 2;
  static constexpr int kBudget = 227 * 1024 - kStaging - 2048;
  static constexpr int kStagesRaw = kBudget / kStage;
  static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
  static constexpr int kAcc = (2 * BN <= 512) ? 2 : 1;
  static constexpr int kTmemCols = (kAcc * BN <= 32) ? 32 : (kAcc * BN <= 64) ? 64 : (kAcc * BN <= 128) ? 128
                                   : (kAcc * BN <= 256) ? 256 : 512;
  static constexpr int kSmem = kStages * kStage + kStaging + 2048;
  static_assert(kStages >= 2, "not enough shared memory for two stages");
};

struct alignas(8) Bars {
  uint64_t full_tma[8];
  uint64_t full_a[8];
  uint64_t empty[8];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

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

__device__ __forceinline__ Lut nf_lut(const DqParams& dq, int64_t block_index) {
  float scale;
  if (dq.dq_block) {
    scale = __fmul_rn(e4m3_to_f32(__ldg(dq.c1_fp8 + block_index)), __ldg(dq.s2 + block_index / dq.dq_block));
  } else {
    scale = __ldg(dq.c1 + block_index);
  }
  float v[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __fmul_rn(dq.lv.v[i], scale);
  return make_lut(v);
}

__device__ __forceinline__ Lut int4_lut(const DqParams& dq, int64_t group_index) {
  const float sc = __half2float(dq.scale[group_index]);
  const float z = __half2float(dq.zero[group_index]);
  float v[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __fmul_rn(__fsub_rn(static_cast<float>(i), z), sc);
  return make_lut(v);
}

// Dequantise 64 consecutive 4-bit codes of row `row`, starting at column `col` of W, into the eight
// 16-byte chunks of one 128-byte swizzled shared-memory row at `dst_row` (row index `sw` for the swizzle).
__device__ __forceinline__ void dequant_row64(const DqParams& dq, const uint8_t* codes_smem, int64_t row, int64_t col,
                                              bool valid, uint8_t* dst_row, int sw) {
  const uint4* src = reinterpret_cast<const uint4*>(codes_smem);
  const uint4 c0 = src[0], c1 = src[1];
  const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
  if (!valid) {
#pragma unroll
    for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(dst_row + ((c ^ sw) << 4)) = make_uint4(0, 0, 0, 0);
    return;
  }
  if (dq.fmt == QLR_FMT_NFK) {
    const Lut t = nf_lut(dq, (row * dq.K + col) / dq.block);
#pragma unroll
    for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(dst_row + ((c ^ sw) << 4)) = lut8(t, w[c]);
  } else {
    const int64_t g0 = row * (dq.K / dq.group) + col / dq.group;
    if (dq.group == 32) {
      const Lut t0 = int4_lut(dq, g0);
#pragma unroll
      for (int c = 0; c < 4; ++c) *reinterpret_cast<uint4*>(dst_row + ((c ^ sw) << 4)) = lut8(t0, w[c]);
      const Lut t1 = int4_lut(dq, g0 + 1);
#pragma unroll
      for (int c = 4; c < 8; ++c) *reinterpret_cast<uint4*>(dst_row + ((c ^ sw) << 4)) = lut8(t1, w[c]);
    } else {
      const Lut t0 = int4_lut(dq, g0);
#pragma unroll
      for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(dst_row + ((c ^ sw) << 4)) = lut8(t0, w[c]);
    }
  }
}

template <int A_SRC, int B_SRC, int BN, int OUT, int TAIL_A_MN>
__global__ void __launch_bounds__((A_SRC >= A_DQ_K) ? kThreadsDq : kThreadsPlain, 1)
    gemm_kernel(const __grid_constant__ GemmParams p, const __grid_constant__ GemmMaps maps) {
  constexpr bool DQ = (A_SRC >= A_DQ_K);
  using C = Cfg<BN, DQ>;
  constexpr int NS = C::kStages;
  constexpr uint32_t kIdescMain = idesc_bf16(128, BN, (A_SRC == A_TMA_MN || A_SRC == A_DQ_MN) ? 1u : 0u,
                                             B_SRC == B_TMA_MN ? 1u : 0u);
  constexpr uint32_t kIdescTail = idesc_bf16(128, BN, TAIL_A_MN ? 1u : 0u, 0u);

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* staging = smem + NS * C::kStage;
  Bars* bars = reinterpret_cast<Bars*>(staging + C::kStaging);
  volatile int* abort_flag = &bars->abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bars->full_tma[s], 1);
      mbar_init(&bars->full_a[s], 128);
      mbar_init(&bars->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&bars->acc_full[a], 1);
      mbar_init(&bars->acc_empty[a], 128);
    }
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&maps.a);
    tma_prefetch_desc(&maps.b);
    tma_prefetch_desc(&maps.a_tail);
    tma_prefetch_desc(&maps.b_tail);
    tma_prefetch_desc(&maps.codes);
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = bars->tmem_base;

  const int tiles_per_split = p.m_tiles * p.n_tiles;
  const int n_tiles_total = tiles_per_split * p.splits;
  const int steps_per_split = (p.n_main + p.splits - 1) / p.splits;

  auto tile_coords = [&](int tile, int& split, int& m0, int& n0, int& kb, int& nmain, int& ntail) {
    split = tile / tiles_per_split;
    const int rem = tile % tiles_per_split;
    m0 = (rem / p.n_tiles) * 128;
    n0 = (rem % p.n_tiles) * BN;
    kb = split * steps_per_split;
    const int ke = min(p.n_main, kb + steps_per_split);
    nmain = max(0, ke - kb);
    ntail = (split == p.splits - 1) ? p.n_tail : 0;
  };

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t j = 0;
      for (int tile = blockIdx.x; tile < n_tiles_total && !*abort_flag; tile += gridDim.x) {
        int split, m0, n0, kb, nmain, ntail;
        tile_coords(tile, split, m0, n0, kb, nmain, ntail);
        for (int ks = 0; ks < nmain + ntail; ++ks, ++j) {
          const int s = j % NS;
          const uint32_t ph = (j / NS) & 1;
          if (!mbar_wait(&bars->empty[s], ph ^ 1, abort_flag)) break;
          uint8_t* st_a = smem + s * C::kStage;
          uint8_t* st_b = st_a + C::kA;
          uint8_t* st_c = st_b + C::kB;
          uint64_t* fb = &bars->full_tma[s];
          if (ks < nmain) {
            const int k0 = (kb + ks) * 64;
            uint32_t bytes = C::kB;
            if (A_SRC == A_TMA_K) {
              tma_load_2d(st_a, &maps.a, k0, m0, fb);
              bytes += C::kA;
            } else if (A_SRC == A_TMA_MN) {
              tma_load_2d(st_a, &maps.a, m0, k0, fb);
              tma_load_2d(st_a + 8192, &maps.a, m0 + 64, k0, fb);
              bytes += C::kA;
            } else if (A_SRC == A_DQ_K) {
              bytes += 4096;
            } else {
              bytes += 4096;
            }
            mbar_arrive_expect_tx(fb, bytes);
            if (A_SRC == A_DQ_K) tma_load_2d(st_c, &maps.codes, k0 / 2, m0, fb);
            if (A_SRC == A_DQ_MN) tma_load_2d(st_c, &maps.codes, m0 / 2, k0, fb);
            if (B_SRC == B_TMA_K) {
              tma_load_2d(st_b, &maps.b, k0, n0, fb);
            } else {
              const int atom_bytes = 64 * p.b_atom * 2;
              for (int a = 0; a < BN / p.b_atom; ++a)
                tma_load_2d(st_b + a * atom_bytes, &maps.b, n0 + a * p.b_atom, k0, fb);
            }
          } else {
            const int kt = (ks - nmain) * 64;
            mbar_arrive_expect_tx(fb, C::kA + C::kB);
            if (TAIL_A_MN) {
              tma_load_2d(st_a, &maps.a_tail, m0, kt, fb);
              tma_load_2d(st_a + 8192, &maps.a_tail, m0 + 64, kt, fb);
            } else {
              tma_load_2d(st_a, &maps.a_tail, kt, m0, fb);
            }
            tma_load_2d(st_b, &maps.b_tail, kt, n0, fb);
          }
        }
      }
      // drain: wait (bounded, regardless of abort) for the loads of the last NS issued stages
      const uint32_t first = j > NS ? j - NS : 0;
      for (uint32_t q = first; q < j; ++q) {
        volatile int never = 0;
        mbar_wait(&bars->full_tma[q % NS], (q / NS) & 1, &never);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t j = 0;
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < n_tiles_total && ok; tile += gridDim.x, ++it) {
        int split, m0, n0, kb, nmain, ntail;
        tile_coords(tile, split, m0, n0, kb, nmain, ntail);
        const int acc = it % C::kAcc;
        const uint32_t aph = (it / C::kAcc) & 1;
        if (!mbar_wait(&bars->acc_empty[acc], aph ^ 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int ks = 0; ks < nmain + ntail; ++ks, ++j) {
          const int s = j % NS;
          const uint32_t ph = (j / NS) & 1;
          const bool tail = ks >= nmain;
          if (!mbar_wait(&bars->full_tma[s], ph, abort_flag)) { ok = false; break; }
          if (DQ) {  // dequantisers arrive for every stage (tail stages carry no work for them)
            if (!mbar_wait(&bars->full_a[s], ph, abort_flag)) { ok = false; break; }
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * C::kStage);
          const uint32_t b_addr = a_addr + C::kA;
          int nsub = 4;
          if (tail) {
            const int rem = p.r_tail - (ks - nmain) * 64;
            nsub = rem >= 64 ? 4 : (rem + 15) / 16;
          }
          for (int kk = 0; kk < nsub; ++kk) {
            uint64_t ad, bd;
            const bool a_mn = tail ? (TAIL_A_MN != 0) : (A_SRC == A_TMA_MN || A_SRC == A_DQ_MN);
            if (a_mn)
              ad = smem_desc(a_addr + kk * 2048, 8192, 1024, kSw128);
            else
              ad = smem_desc(a_addr + kk * 32, 16, 1024, kSw128);
            if (!tail && B_SRC == B_TMA_MN) {
              const uint32_t rb = p.b_atom * 2;
              const uint32_t lay = rb == 128 ? kSw128 : (rb == 64 ? kSw64 : kSw32);
              bd = smem_desc(b_addr + kk * 16 * rb, 64 * rb, 8 * rb, lay);
            } else {
              bd = smem_desc(b_addr + kk * 32, 16, 1024, kSw128);
            }
            umma_bf16_ss(d_tmem, ad, bd, tail ? kIdescTail : kIdescMain, (ks > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&bars->empty[s]);
        }
        if (!ok) break;
        umma_commit(&bars->acc_full[acc]);
      }
      // make sure every issued MMA has retired before TMEM is released
      umma_commit(&bars->drain);
      volatile int never = 0;
      mbar_wait(&bars->drain, 0, &never);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    uint16_t* stg = reinterpret_cast<uint16_t*>(staging) + q * 32 * 32;
    int it = 0;
    for (int tile = blockIdx.x; tile < n_tiles_total; tile += gridDim.x, ++it) {
      int split, m0, n0, kb, nmain, ntail;
      tile_coords(tile, split, m0, n0, kb, nmain, ntail);
      const int acc = it % C::kAcc;
      const uint32_t aph = (it / C::kAcc) & 1;
      const bool got = mbar_wait(&bars->acc_full[acc], aph, abort_flag);
      __syncwarp();
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const int row = m0 + q * 32 + lane;  // D row (MMA M index)
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem_base + acc * BN + c * 32 + ((q * 32) << 16), v);
        tmem_ld_wait();
        if (OUT == OUT_F32_D) {
          float* o = static_cast<float*>(p.out) +
                     (static_cast<int64_t>(split) * p.m_tiles * 128 + row) * p.ldo + n0 + c * 32;
#pragma unroll
          for (int i = 0; i < 8; ++i)
            reinterpret_cast<float4*>(o)[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                                          __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
        } else {
          // stage D[row, n0 + 32c + jj] as [jj][lane] bf16, then write 16-byte pieces of out rows
#pragma unroll
          for (int jj = 0; jj < 32; ++jj)
            stg[jj * 32 + lane] = static_cast<uint16_t>(pack_bf16x2_rn(__uint_as_float(v[jj]), 0.f) & 0xFFFFu);
          __syncwarp();
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int idx = t * 32 + lane;
            const int jj = idx >> 2, part = idx & 3;
            const int orow = n0 + c * 32 + jj;           // output row (D column)
            const int ocol = m0 + q * 32 + part * 8;     // output column (D row)
            if (orow < p.Nn && ocol < p.Mm) {
              uint4 val = *reinterpret_cast<const uint4*>(stg + jj * 32 + part * 8);
              uint16_t* dst = static_cast<uint16_t*>(p.out) + static_cast<int64_t>(orow) * p.ldo + ocol;
              if (p.accumulate) {
                const uint4 old = *reinterpret_cast<const uint4*>(dst);
                uint32_t* nv = reinterpret_cast<uint32_t*>(&val);
                const uint32_t* ov = reinterpret_cast<const uint32_t*>(&old);
#pragma unroll
                for (int e = 0; e < 4; ++e)
                  nv[e] = pack_bf16x2_rn(bf16_bits_to_f32(nv[e] & 0xFFFFu) + bf16_bits_to_f32(ov[e] & 0xFFFFu),
                                         bf16_bits_to_f32(nv[e] >> 16) + bf16_bits_to_f32(ov[e] >> 16));
              }
              *reinterpret_cast<uint4*>(dst) = val;
            }
          }
          __syncwarp();
        }
      }
      tc_fence_before();
      mbar_arrive(&bars->acc_empty[acc]);
    }
  } else if (DQ) {
    // ------------------------------------------------------------------ dequantisers
    const int dt = threadIdx.x - 6 * 32;  // 0..255
    const int grp = dt >> 7;
    const int t = dt & 127;
    uint32_t j = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < n_tiles_total && ok; tile += gridDim.x) {
      int split, m0, n0, kb, nmain, ntail;
      tile_coords(tile, split, m0, n0, kb, nmain, ntail);
      for (int ks = 0; ks < nmain + ntail; ++ks, ++j) {
        if (static_cast<int>(j & 1) != grp) continue;
        const int s = j % NS;
        const uint32_t ph = (j / NS) & 1;
        if (!mbar_wait(&bars->full_tma[s], ph, abort_flag)) { ok = false; break; }
        if (ks >= nmain) {  // tail stage: operands came by TMA; only keep the barrier phases in step
          mbar_arrive(&bars->full_a[s]);
          continue;
        }
        uint8_t* st_a = smem + s * C::kStage;
        const uint8_t* st_c = st_a + C::kA + C::kB;
        const int k0 = (kb + ks) * 64;
        if (A_SRC == A_DQ_K) {
          // row t of the W tile: W[m0 + t, k0 .. k0 + 63] -> K-major row t
          const int64_t row = m0 + t;
          dequant_row64(p.dq, st_c + t * 32, row, k0, row < p.dq.N, st_a + t * 128, t & 7);
        } else {
          // W[k0 + nr, m0 + 64h .. +63] -> MN-major atom h, K-row nr
          const int nr = t >> 1, h = t & 1;
          const int64_t row = k0 + nr;
          const int64_t col = m0 + 64 * h;
          dequant_row64(p.dq, st_c + nr * 64 + h * 32, row, col, row < p.dq.N && col < p.dq.K,
                        st_a + h * 8192 + nr * 128, nr & 7);
        }
        fence_proxy_async_smem();
        mbar_arrive(&bars->full_a[s]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
  if (threadIdx.x == 0 && bars->abort_flag) report(p.status, QLR_ERR_TIMEOUT);
}

template <int A_SRC, int B_SRC, int BN, int OUT, int TAIL_A_MN>
cudaError_t launch_variant(const GemmParams& p, const GemmMaps& maps, cudaStream_t st) {
  constexpr bool DQ = (A_SRC >= A_DQ_K);
  using C = Cfg<BN, DQ>;
  auto kern = gemm_kernel<A_SRC, B_SRC, BN, OUT, TAIL_A_MN>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [&] {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem + 1024);
  });
  if (attr_err != cudaSuccess) return attr_err;
  const int tiles = p.m_tiles * p.n_tiles * p.splits;
  const int grid = tiles < device_sm_count() ? tiles : device_sm_count();
  count_launch();
  kern<<<grid, DQ ? kThreadsDq : kThreadsPlain, C::kSmem + 1024, st>>>(p, maps);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm(int a_src, int b_src, int bn, int out_mode, int tail_a_mn, const GemmParams& p,
                        const GemmMaps& maps, cudaStream_t st) {
  // forward (fused dequant, K-major W tile) and input gradient (fused dequant, MN-major W tile)
  if (a_src == A_DQ_K && b_src == B_TMA_K && bn == 256 && out_mode == OUT_BF16_T && !tail_a_mn)
    return launch_variant<A_DQ_K, B_TMA_K, 256, OUT_BF16_T, 0>(p, maps, st);
  if (a_src == A_DQ_K && b_src == B_TMA_K && bn == 64 && out_mode == OUT_BF16_T && !tail_a_mn)
    return launch_variant<A_DQ_K, B_TMA_K, 64, OUT_BF16_T, 0>(p, maps, st);
  if (a_src == A_DQ_MN && b_src == B_TMA_K && bn == 256 && out_mode == OUT_BF16_T && tail_a_mn)
    return launch_variant<A_DQ_MN, B_TMA_K, 256, OUT_BF16_T, 1>(p, maps, st);
  if (a_src == A_DQ_MN && b_src == B_TMA_K && bn == 64 && out_mode == OUT_BF16_T && tail_a_mn)
    return launch_variant<A_DQ_MN, B_TMA_K, 64, OUT_BF16_T, 1>(p, maps, st);
  // adapter GEMMs (split reductions into fp32 partials)
  if (a_src == A_TMA_K && b_src == B_TMA_K && out_mode == OUT_F32_D) {  // T = X A^T
    if (bn == 32) return launch_variant<A_TMA_K, B_TMA_K, 32, OUT_F32_D, 0>(p, maps, st);
    if (bn == 64) return launch_variant<A_TMA_K, B_TMA_K, 64, OUT_F32_D, 0>(p, maps, st);
  }
  if (a_src == A_TMA_K && b_src == B_TMA_MN && out_mode == OUT_F32_D) {  // dT = dY B
    if (bn == 32) return launch_variant<A_TMA_K, B_TMA_MN, 32, OUT_F32_D, 0>(p, maps, st);
    if (bn == 64) return launch_variant<A_TMA_K, B_TMA_MN, 64, OUT_F32_D, 0>(p, maps, st);
  }
  if (a_src == A_TMA_MN && b_src == B_TMA_MN && out_mode == OUT_F32_D) {  // dB = dY^T T, dA^T = X^T dT
    if (bn == 32) return launch_variant<A_TMA_MN, B_TMA_MN, 32, OUT_F32_D, 0>(p, maps, st);
    if (bn == 64) return launch_variant<A_TMA_MN, B_TMA_MN, 64, OUT_F32_D, 0>(p, maps, st);
  }
  return cudaErrorNotSupported;
}

// ---- tensor maps ---------------------------------------------------------------------------------
namespace {
PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}
}  // namespace

int make_tmap(CUtensorMap* m, const void* base, int elem_bytes, uint64_t rows, uint64_t cols, uint32_t box_rows,
              uint32_t box_cols, int swizzle_bytes) {
  auto enc = get_encode();
  if (!enc) return QLR_ERR_CUDA;
  const CUtensorMapDataType dt =
      elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * static_cast<uint64_t>(elem_bytes)};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_NONE;
  if (swizzle_bytes == 128) sw = CU_TENSOR_MAP_SWIZZLE_128B;
  if (swizzle_bytes == 64) sw = CU_TENSOR_MAP_SWIZZLE_64B;
  if (swizzle_bytes == 32) sw = CU_TENSOR_MAP_SWIZZLE_32B;
  const CUresult r = enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? QLR_OK : QLR_ERR_CUDA;
}

}  // namespace qlr
