// Fused dequantise + tcgen05 GEMM for sm_100a: the frozen 4-bit weight never reaches global memory
// in bf16 (QLoRA explainer, "The QLoRA recipe", stage 3: each frozen block is dequantised to bf16 on
// the fly and multiplied by the input; "Background: how LoRA works": the adapter term is added).
//
//   forward         D = Y^T [N, M]:  A = dequant(W) tile, K-major  (W rows on the 128 TMEM lanes)
//                                    B = X tile [tokens, 64], K-major
//                   tail (r extra reduction columns): A = B_lora rows, B = T_save = s P(X) A^T
//   input gradient  D = dX^T [K, M]: A = dequant(W)^T tile, MN-major (W rows are the reduction)
//                                    B = dY tile, K-major
//                   tail: A = A_lora (or its group expansion) rows, B = dT
//
// Three decoupled shared-memory rings keep the dequantiser off the activation stream's latency:
//   codes ring (8 x 4 KB)   filled by TMA from a dedicated producer warp, far ahead of use;
//   A ring     (3-4 x 16 KB) written by the dequantiser warps in the canonical 128-byte-swizzled
//                            UMMA layout (they also copy the tail's weight-side rows);
//   B ring     (4-8 stages)  activation tiles by TMA.
// Warp roles (Roles below): 1 TMEM allocator + MMA issuer, 2..5 epilogue, one activation and one codes
// producer, and eight warps in two groups of dequantisers taking alternate reduction steps.  Two TMEM
// accumulators (2 x BN fp32 columns) overlap each tile's epilogue with the next tile's main loop.
// Every wait is bounded; a wait that runs out aborts the CTA and reports QLR_ERR_TIMEOUT.
#include <mutex>
#include <type_traits>

#include "engine.cuh"

namespace qlr {

namespace {

constexpr int kThreadsFused = 480;
// Warp roles.  A warp runs on scheduler (warp % 4).  Warp 1 allocates TMEM and issues the MMAs from
// one thread; epilogue warps 2..5 read TMEM lane quadrants 2, 3, 0, 1 (a warp may only read the
// quadrant warp % 4).  With 2 x BN-token tiles (MMA-heavy: each dequantised stage feeds two MMA
// groups) the issuer's scheduler holds only light roles, the two TMA producers and one epilogue warp,
// so the dequantisers' integer work does not delay the next MMAs.  With BN-token tiles the
// dequantisation per MMA doubles and the eight dequantiser warps are spread two per scheduler instead.
constexpr int kIssuerWarp = 1;
// Warps in a dequantiser group (128 tile rows) and in the epilogue (four TMEM lane quadrants).  Each of
// these warps signals its part of a stage or tile with one barrier arrival from lane 0 after a warp
// sync: 32 arrivals at one shared-memory address would be serialised by the memory pipe.
constexpr int kGroupWarps = 4;
template <bool PAIR>
struct Roles {
  static constexpr int kActWarp = PAIR ? 9 : 0;
  static constexpr int kCodesWarp = PAIR ? 13 : 14;
  // dequantiser slot of a warp (slot / 4 = group, slot % 4 = 32-row block), -1 for other roles
  __device__ __forceinline__ static int dq_slot(int warp) {
    if (!PAIR) return warp >= 6 && warp <= 13 ? warp - 6 : -1;
    switch (warp) {
      case 0: return 0;
      case 6: return 1;
      case 7: return 2;
      case 8: return 3;
      case 10: return 4;
      case 11: return 5;
      case 12: return 6;
      case 14: return 7;
      default: return -1;
    }
  }
};

template <int BN>
struct FCfg {
  static constexpr int kA = 16384;
  static constexpr int kB = BN * 128;
  static constexpr int kC = kCodeRingBytes / kCodeRingSlots;
  static constexpr int NSA = BN >= 256 ? 3 : 4;
  static constexpr int NSC = kCodeRingSlots;
  static constexpr int kStaging = 4 * 32 * 32 * 4;  // per epilogue warp a 32 x 32 fp32 tile
  static constexpr int kFixed = kStaging + 2048;
  static constexpr int kBudget = 227 * 1024 - kFixed - NSA * kA - NSC * kC;
  static constexpr int NSB = (kBudget / kB) > 8 ? 8 : (kBudget / kB);
  static constexpr int kOffA = NSB * kB;
  static constexpr int kOffC = kOffA + NSA * kA;
  static constexpr int kOffStaging = kOffC + NSC * kC;
  static constexpr int kOffBars = kOffStaging + kStaging;
  static constexpr int kSmem = kOffBars + 2048;
  static constexpr int kTmemCols = (2 * BN <= 128) ? 128 : (2 * BN <= 256) ? 256 : 512;
  static_assert(NSB >= 2, "not enough shared memory");
  static_assert(kSmem + 1024 <= 227 * 1024, "shared memory budget");
};

struct alignas(8) FBars {
  uint64_t b_full[8], b_empty[8];
  uint64_t a_full[4], a_empty[4];
  uint64_t c_full[kCodeRingSlots], c_empty[kCodeRingSlots];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

// Copies 64 bf16 of one row of the tail's weight-side operand (zero outside the matrix) into one
// 128-byte swizzled shared-memory row.
__device__ __forceinline__ void copy_row64(const uint16_t* src_row, bool row_ok, int64_t col0, int64_t ncols,
                                           uint8_t* dst_row, int sw) {
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint4 v = make_uint4(0, 0, 0, 0);
    if (row_ok && col0 + 8 * c < ncols) v = __ldg(reinterpret_cast<const uint4*>(src_row + col0 + 8 * c));
    *reinterpret_cast<uint4*>(dst_row + ((c ^ sw) << 4)) = v;
  }
}

// As copy_row64 for the input gradient's pooled adapter: column k of the row is bf16(A[j, k / L] / L).
__device__ __forceinline__ void copy_row64_pooled(const uint16_t* src_row, bool row_ok, int64_t col0, int64_t ncols,
                                                  int L, uint8_t* dst_row, int sw) {
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint4 v = make_uint4(0, 0, 0, 0);
    const int64_t k = col0 + 8 * c;
    if (row_ok && k < ncols) {
      const float a = __fdiv_rn(bf16_bits_to_f32(src_row[k / L]), static_cast<float>(L));
      const uint32_t pair = pack_bf16x2_rn(a, a);
      v = make_uint4(pair, pair, pair, pair);
    }
    *reinterpret_cast<uint4*>(dst_row + ((c ^ sw) << 4)) = v;
  }
}

// PAIR: one tile covers 2 x BN tokens with both TMEM accumulators, so every dequantised weight
// stage feeds twice the MMA work (the epilogue then does not overlap the next tile's main loop).
// EPI: EPI_STORE (with a run-time accumulate flag), EPI_SWIGLU_FWD or EPI_SWIGLU_BWD (see GemmParams).
// SMALL: the weight is 2- or 3-bit NF (the dequantisers' eight-entry lookup).
template <int A_SRC, int BN, bool PAIR, int EPI, bool SMALL>
__global__ void __launch_bounds__(kThreadsFused, 1)
    fused_kernel(const __grid_constant__ GemmParams p, const __grid_constant__ GemmMaps maps) {
  using C = FCfg<BN>;
  constexpr int TOK = PAIR ? 2 * BN : BN;    // tokens per tile
  constexpr int HALVES = PAIR ? 2 : 1;      // activation stages per reduction step
  constexpr bool MN = (A_SRC == A_DQ_MN);
  constexpr uint32_t kIdesc = idesc_bf16(128, BN, MN ? 1u : 0u, 0u);
  constexpr int NSA = C::NSA, NSB = C::NSB, NSC = C::NSC;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring_b = smem;
  uint8_t* ring_a = smem + C::kOffA;
  uint8_t* ring_c = smem + C::kOffC;
  uint8_t* staging = smem + C::kOffStaging;
  FBars* bars = reinterpret_cast<FBars*>(smem + C::kOffBars);
  volatile int* abort_flag = &bars->abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSB; ++s) {
      mbar_init(&bars->b_full[s], 1);
      mbar_init(&bars->b_empty[s], 1);
    }
    for (int s = 0; s < NSA; ++s) {
      mbar_init(&bars->a_full[s], kGroupWarps);
      mbar_init(&bars->a_empty[s], 1);
    }
    for (int s = 0; s < NSC; ++s) {
      mbar_init(&bars->c_full[s], 1);
      mbar_init(&bars->c_empty[s], kGroupWarps * p.code_steps);  // every step of a box is one dequantiser group
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&bars->acc_full[a], 1);
      mbar_init(&bars->acc_empty[a], kGroupWarps);
    }
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    fence_barrier_init();
  }
  constexpr int kActWarp = Roles<PAIR>::kActWarp, kCodesWarp = Roles<PAIR>::kCodesWarp;
  if (warp == kActWarp && lane == 0) {
    tma_prefetch_desc(&maps.b);
    tma_prefetch_desc(&maps.b_tail);
  }
  if (warp == kCodesWarp && lane == 0) tma_prefetch_desc(&maps.codes);
  // everything above touches only shared memory and kernel parameters; from here on the previous
  // kernel's results are needed (and its TMEM must be free)
  pdl_launch_dependents();
  pdl_wait();
  if (warp == kIssuerWarp) {
    tmem_alloc(&bars->tmem_base, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = bars->tmem_base;

  // Work items: tiles of 128 weight rows x TOK tokens in row-major tile order.  With token pairs, the tiles
  // from p.full_items on (the last, partial wave of a launch with more tiles than CTAs) are each split
  // into two items of BN tokens, one per half, so that they spread over more CTAs.
  const int n_items = p.n_items;
  const int nmain = p.n_main, ntail = p.n_tail, nsteps = nmain + ntail;
  auto item_of = [&](int item, int& m0, int& n0, int& halves) {
    int tile = item, half = 0;
    halves = HALVES;
    if (PAIR && item >= p.full_items) {
      const int hi = item - p.full_items;
      tile = p.full_items + (hi >> 1);
      half = hi & 1;
      halves = 1;
    }
    m0 = (tile / p.n_tiles) * 128;
    n0 = (tile % p.n_tiles) * TOK + half * BN;
  };

  if (warp == kActWarp) {
    // ------------------------------------------------------------------ activation producer
    if (lane == 0) {
      uint32_t j = 0;
      for (int item = blockIdx.x; item < n_items && !*abort_flag; item += gridDim.x) {
        int m0, n0, halves;
        item_of(item, m0, n0, halves);
        bool ok = true;
        auto loads = [&](auto nh_tag) {
          constexpr int NH = decltype(nh_tag)::value;
          for (int ks = 0; ks < nsteps && ok; ++ks) {
#pragma unroll
            for (int h = 0; h < NH; ++h) {
              const int s = j % NSB;
              if (!mbar_wait(&bars->b_empty[s], ((j / NSB) & 1) ^ 1, abort_flag, p.wait_cycles)) { ok = false; break; }
              uint64_t* fb = &bars->b_full[s];
              mbar_arrive_expect_tx(fb, C::kB);
              if (ks < nmain)
                tma_load_2d(ring_b + s * C::kB, &maps.b, ks * 64, n0 + h * BN, fb);
              else
                tma_load_2d(ring_b + s * C::kB, &maps.b_tail, (ks - nmain) * 64, n0 + h * BN, fb);
              ++j;
            }
          }
        };
        if (halves == HALVES)
          loads(std::integral_constant<int, HALVES>{});
        else
          loads(std::integral_constant<int, 1>{});
      }
      const uint32_t first = j > NSB ? j - NSB : 0;
      for (uint32_t q = first; q < j; ++q) {
        mbar_drain(&bars->b_full[q % NSB], (q / NSB) & 1);
      }
    }
  } else if (warp == kCodesWarp) {
    // ------------------------------------------------------------------ codes producer
    if (lane == 0) {
      const int lg = p.code_slots_log2, ncs = 1 << lg, kb = p.code_bits;
      const uint32_t mask = static_cast<uint32_t>(ncs - 1);
      uint32_t jc = 0;  // boxes
      for (int item = blockIdx.x; item < n_items && !*abort_flag; item += gridDim.x) {
        int m0, n0, halves;
        item_of(item, m0, n0, halves);
        for (int ks = 0; ks < nmain; ks += p.code_steps, ++jc) {
          const int s = static_cast<int>(jc & mask);
          if (!mbar_wait(&bars->c_empty[s], ((jc >> lg) & 1) ^ 1, abort_flag, p.wait_cycles)) break;
          uint64_t* fb = &bars->c_full[s];
          mbar_arrive_expect_tx(fb, p.code_box_bytes);
          if (!MN)  // [128 W rows][8 kb bytes per step]
            tma_load_2d(ring_c + s * p.code_box_bytes, &maps.codes, ks * 8 * kb, m0, fb);
          else      // [64 W rows][16 kb bytes: 128 codes]
            tma_load_2d(ring_c + s * p.code_box_bytes, &maps.codes, m0 / 8 * kb, ks * 64, fb);
        }
      }
      const uint32_t first = jc > static_cast<uint32_t>(ncs) ? jc - ncs : 0;
      for (uint32_t q = first; q < jc; ++q) {
        mbar_drain(&bars->c_full[q & mask], (q >> lg) & 1);
      }
    }
  } else if (warp == kIssuerWarp) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t j = 0, jb = 0;  // A-ring steps, B-ring stages
      int it = 0;
      // descriptors of ring slot 0; a slot or a 16-wide reduction slice is a fixed address offset, which
      // adds to the descriptor's address field (addr >> 4) without carrying out of it
      const uint64_t a_desc0 = MN ? smem_desc(smem_u32(ring_a), 8192, 1024, kSw128)
                                  : smem_desc(smem_u32(ring_a), 16, 1024, kSw128);
      const uint64_t b_desc0 = smem_desc(smem_u32(ring_b), 16, 1024, kSw128);
      constexpr uint32_t kAk = MN ? (2048 >> 4) : (32 >> 4), kBk = 32 >> 4;
      bool ok = true;
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x, ++it) {
        int m0, n0, halves;
        item_of(item, m0, n0, halves);
        const int acc = PAIR ? 0 : (it & 1);
        const uint32_t acc_par = PAIR ? ((it & 1) ^ 1) : (((it >> 1) & 1) ^ 1);
        if (!mbar_wait(&bars->acc_empty[acc], acc_par, abort_flag, p.wait_cycles)) break;
        tc_fence_after();
        // the step loop with the activation stages per step (halves) as a compile-time count: a split tail
        // item runs the one-stage copy, everything else the unrolled full one
        auto steps = [&](auto nh_tag) {
          constexpr int NH = decltype(nh_tag)::value;
          for (int ks = 0; ks < nsteps && ok; ++ks, ++j) {
            const int sa = j % NSA;
            if (!mbar_wait(&bars->a_full[sa], (j / NSA) & 1, abort_flag, p.wait_cycles)) { ok = false; break; }
            const uint64_t ad0 = a_desc0 + static_cast<uint32_t>((sa * C::kA) >> 4);
            int nsub = 4;
            if (ks >= nmain) {
              const int rem = p.r_tail - (ks - nmain) * 64;
              nsub = rem >= 64 ? 4 : (rem + 15) / 16;
            }
#pragma unroll
            for (int h = 0; h < NH; ++h) {
              const int sb = jb % NSB;
              if (!mbar_wait(&bars->b_full[sb], (jb / NSB) & 1, abort_flag, p.wait_cycles)) { ok = false; break; }
              tc_fence_after();
              const uint64_t bd0 = b_desc0 + static_cast<uint32_t>((sb * C::kB) >> 4);
              const uint32_t d_tmem = tmem_base + (PAIR ? h : acc) * BN;
              if (nsub == 4) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                  umma_bf16_ss(d_tmem, ad0 + kk * kAk, bd0 + kk * kBk, kIdesc, (ks > 0 || kk > 0) ? 1u : 0u);
              } else {
                for (int kk = 0; kk < nsub; ++kk)
                  umma_bf16_ss(d_tmem, ad0 + kk * kAk, bd0 + kk * kBk, kIdesc, (ks > 0 || kk > 0) ? 1u : 0u);
              }
              umma_commit(&bars->b_empty[sb]);
              ++jb;
            }
            if (!ok) break;
            umma_commit(&bars->a_empty[sa]);
          }
        };
        if (halves == HALVES)
          steps(std::integral_constant<int, HALVES>{});
        else
          steps(std::integral_constant<int, 1>{});
        if (!ok) break;
        umma_commit(&bars->acc_full[acc]);
      }
      umma_commit(&bars->drain);
      mbar_drain(&bars->drain, 0);
    }
  } else if (warp >= 2 && warp <= 5) {
    // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;
    uint16_t* stg = reinterpret_cast<uint16_t*>(staging) + q * 32 * 32;
    float* stgf = reinterpret_cast<float*>(staging) + q * 32 * 32;
    int it = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++it) {
      int m0, n0, halves;
      item_of(item, m0, n0, halves);
      const int acc = PAIR ? 0 : (it & 1);
      const uint32_t acc_par = PAIR ? (it & 1) : ((it >> 1) & 1);
      const bool got = mbar_wait_pause(&bars->acc_full[acc], acc_par, abort_flag, p.wait_cycles);
      __syncwarp();
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < halves * BN / 32; ++c) {  // PAIR: accumulator columns 0..2*BN-1 are tokens n0 .. n0+2*BN-1
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem_base + (PAIR ? 0 : acc * BN) + c * 32 + ((q * 32) << 16), v);
        tmem_ld_wait();
        if (EPI == EPI_STORE && !p.accumulate)
          eng::store_chunk_bf16_t(v, stg, lane, n0 + c * 32, m0 + q * 32, p);
        else
          eng::store_chunk_f32_t<EPI>(v, stgf, lane, n0 + c * 32, m0 + q * 32, p);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->acc_empty[acc]);
    }
  } else {
    // ------------------------------------------------------------------ dequantisers (warps 6..13)
    const int slot = Roles<PAIR>::dq_slot(warp);
    const int grp = slot >> 2;
    const int t = (slot & 3) * 32 + lane;
    auto run_of = [&](int m0, int k0, int64_t& row, int64_t& col, bool& valid) {
      if (!MN) {  // row t of the W tile: W[m0 + t, k0 .. k0 + 63] -> K-major row t
        row = m0 + t;
        col = k0;
        valid = row < p.dq.N;
      } else {  // W[k0 + nr, m0 + 64h .. +63] -> MN-major atom h, reduction row nr (nr = t % 64, h = t / 64,
                // so 8 consecutive threads store 8 consecutive swizzled rows without bank conflicts)
        row = k0 + (t & 63);
        col = m0 + 64 * (t >> 6);
        valid = row < p.dq.N && col < p.dq.K;
      }
    };
    // cursor over the CTA's step sequence; j counts every step, jc the main (dequantised) ones
    int item = blockIdx.x, ks = 0;
    int tm0 = 0;
    auto item_m0 = [&](int it_) {
      int m0, n0, halves;
      item_of(it_, m0, n0, halves);
      return m0;
    };
    if (item < n_items) tm0 = item_m0(item);
    uint32_t j = 0, jc = 0;
    auto seek = [&]() -> bool {  // advance to the next step with (j & 1) == grp
      while (item < n_items) {
        if (ks >= nsteps) {
          item += gridDim.x;
          ks = 0;
          if (item < n_items) tm0 = item_m0(item);
          continue;
        }
        if (static_cast<int>(j & 1) == grp) return true;
        if (ks < nmain) ++jc;
        ++ks;
        ++j;
      }
      return false;
    };
    auto prefetch = [&]() -> eng::DqConst {
      eng::DqConst c{0u, 0u};
      if (ks < nmain) {
        int64_t row, col;
        bool valid;
        run_of(tm0, ks * 64, row, col, valid);
        c = eng::load_dq_const(p.dq, row, col, valid);
      }
      return c;
    };
    bool have = seek();
    eng::DqConst cur = have ? prefetch() : eng::DqConst{0u, 0u};
    while (have) {
      const int c_m0 = tm0, c_ks = ks;
      const uint32_t c_j = j, c_jc = jc;
      if (ks < nmain) ++jc;
      ++ks;
      ++j;
      const bool have_next = seek();
      const eng::DqConst nxt = have_next ? prefetch() : eng::DqConst{0u, 0u};

      const int sa = c_j % NSA;
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->a_empty[sa], ((c_j / NSA) & 1) ^ 1, abort_flag, p.wait_cycles)))
        break;
      uint8_t* st_a = ring_a + sa * C::kA;
      if (c_ks < nmain) {
        const int kb = p.code_bits, lg = p.code_slots_log2;
        const uint32_t box = p.code_steps == 2 ? c_jc >> 1 : c_jc, sub = p.code_steps == 2 ? (c_jc & 1) : 0;
        const int sc = static_cast<int>(box & ((1u << lg) - 1u));
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->c_full[sc], (box >> lg) & 1, abort_flag, p.wait_cycles))) break;
        const uint8_t* st_c = ring_c + sc * p.code_box_bytes;
        int64_t row, col;
        bool valid;
        run_of(c_m0, c_ks * 64, row, col, valid);
        if (!MN) {  // row t: 8 kb bytes per step, code_steps steps per box row
          eng::dequant_row64<SMALL>(p.dq, st_c + t * 8 * kb * p.code_steps + sub * 8 * kb, kb, cur, valid, st_a + t * 128,
                             t & 7);
        } else {    // reduction row nr: 16 kb bytes (128 codes), half h
          const int nr = t & 63, h = t >> 6;
          eng::dequant_row64<SMALL>(p.dq, st_c + nr * 16 * kb + h * 8 * kb, kb, cur, valid, st_a + h * 8192 + nr * 128,
                             nr & 7);
        }
        __syncwarp();  // the warp's code reads are done
        if (lane == 0) mbar_arrive(&bars->c_empty[sc]);
      } else {
        const int kt = (c_ks - nmain) * 64;
        if (!MN) {  // B_lora[m0 + t, kt .. kt + 63]
          const int64_t row = c_m0 + t;
          copy_row64(p.tail_a + row * p.tail_a_cols, row < p.tail_a_rows, kt, p.tail_a_cols, st_a + t * 128, t & 7);
        } else {    // A[kt + nr, m0 + 64h .. +63] (or the group expansion of the pooled adapter)
          const int nr = t & 63, h = t >> 6;
          const int64_t row = kt + nr;
          const uint16_t* src = p.tail_a + row * p.tail_a_cols;
          if (p.tail_pool_L > 1)
            copy_row64_pooled(src, row < p.tail_a_rows, c_m0 + 64 * h, p.dq.K, p.tail_pool_L,
                              st_a + h * 8192 + nr * 128, nr & 7);
          else
            copy_row64(src, row < p.tail_a_rows, c_m0 + 64 * h, p.tail_a_cols, st_a + h * 8192 + nr * 128, nr & 7);
        }
      }
      fence_proxy_async_smem();  // each thread's tile stores, before the MMA reads them
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->a_full[sa]);
      cur = nxt;
      have = have_next;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kIssuerWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
  if (threadIdx.x == 0 && bars->abort_flag) report(p.status, QLR_ERR_TIMEOUT);
}

template <int A_SRC, int BN, bool PAIR, int EPI, bool SMALL>
cudaError_t launch_fused_variant(const GemmParams& p, const GemmMaps& maps, cudaStream_t st) {
  using C = FCfg<BN>;
  auto kern = fused_kernel<A_SRC, BN, PAIR, EPI, SMALL>;
  const cudaError_t attr_err = ensure_max_dynamic_smem(kern, C::kSmem + 1024);
  if (attr_err != cudaSuccess) return attr_err;
  const int items = p.n_items;
  const int grid = items < device_sm_count() ? items : device_sm_count();
  return launch_pdl(kern, dim3(grid), dim3(kThreadsFused), C::kSmem + 1024, st, p, maps);
}

}  // namespace

namespace {
template <int A_SRC, int EPI, bool SMALL>
cudaError_t launch_fused_epi(int bn, const GemmParams& p, const GemmMaps& maps, cudaStream_t st) {
  if (bn == 512) return launch_fused_variant<A_SRC, 256, true, EPI, SMALL>(p, maps, st);
  if (bn == 256) return launch_fused_variant<A_SRC, 256, false, EPI, SMALL>(p, maps, st);
  if (bn == 64) return launch_fused_variant<A_SRC, 64, false, EPI, SMALL>(p, maps, st);
  return cudaErrorNotSupported;
}
}  // namespace

// bn = tokens per tile: 512 (paired 256-column accumulators), 256 or 64; the epilogue mode is p.epi (the
// SwiGLU forward only with the forward, the SwiGLU backward only with the input gradient).
// 2- and 3-bit NF weights with the plain epilogue take the eight-entry lookup instantiation, every other
// case the general one.
cudaError_t launch_fused(int a_src, int bn, const GemmParams& p, const GemmMaps& maps, cudaStream_t st) {
  if (p.splits != 1) return cudaErrorNotSupported;
  const bool small = p.dq.fmt == QLR_FMT_NFK && p.code_bits < 4;
  if (a_src == A_DQ_K) {
    if (p.epi == EPI_STORE)
      return small ? launch_fused_epi<A_DQ_K, EPI_STORE, true>(bn, p, maps, st)
                   : launch_fused_epi<A_DQ_K, EPI_STORE, false>(bn, p, maps, st);
    if (p.epi == EPI_SWIGLU_FWD) return launch_fused_epi<A_DQ_K, EPI_SWIGLU_FWD, false>(bn, p, maps, st);
  }
  if (a_src == A_DQ_MN) {
    if (p.epi == EPI_STORE)
      return small ? launch_fused_epi<A_DQ_MN, EPI_STORE, true>(bn, p, maps, st)
                   : launch_fused_epi<A_DQ_MN, EPI_STORE, false>(bn, p, maps, st);
    if (p.epi == EPI_SWIGLU_BWD) return launch_fused_epi<A_DQ_MN, EPI_SWIGLU_BWD, false>(bn, p, maps, st);
  }
  return cudaErrorNotSupported;
}

}  // namespace qlr
