// tcgen05 GEMM engine for sm_100a: both operands by TMA (the adapter GEMMs of the layer).
//
// One persistent CTA per SM walks a static list of output tiles (128 x BN, optionally split along
// the reduction).  Warp roles:
//   warp 0        TMA producer: fills a ring of shared-memory stages (A tile + B tile);
//   warp 1        allocates TMEM and issues tcgen05.mma (one elected lane), committing each stage
//                 back to the producer and each finished tile to the epilogue;
//   warps 2..5    epilogue: TMEM -> registers -> global (fp32 partials, or bf16 through a
//                 transposing shared-memory tile).
// Operands may be K-major or MN-major (128/64/32-byte swizzle), so the same kernel computes
// T = X A^T, dT = dY B, dB = dY^T T and dA^T = X^T dT straight from the row-major tensors.
// Two TMEM accumulators let the epilogue of one tile overlap the main loop of the next.
// The fused dequantising kernels live in fused.cu.
#include <cudaTypedefs.h>

#include <mutex>

#include "engine.cuh"

namespace qlr {

namespace {

constexpr int kThreadsPlain = 192;  // producer, MMA, 4 epilogue warps

template <int BN>
struct Cfg {
  static constexpr int kA = 16384;
  static constexpr int kB = BN * 128;
  static constexpr int kStage = ((kA + kB) + 1023) / 1024 * 1024;
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
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

template <int A_SRC, int B_SRC, int BN, int OUT>
__global__ void __launch_bounds__(kThreadsPlain, 1)
    gemm_kernel(const __grid_constant__ GemmParams p, const __grid_constant__ GemmMaps maps) {
  using C = Cfg<BN>;
  constexpr int NS = C::kStages;
  constexpr uint32_t kIdesc = idesc_bf16(128, BN, A_SRC == A_TMA_MN ? 1u : 0u, B_SRC == B_TMA_MN ? 1u : 0u);

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* staging = smem + NS * C::kStage;
  Bars* bars = reinterpret_cast<Bars*>(staging + C::kStaging);
  volatile int* abort_flag = &bars->abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bars->full[s], 1);
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

  auto tile_coords = [&](int tile, int& split, int& m0, int& n0, int& kb, int& nmain) {
    split = tile / tiles_per_split;
    const int rem = tile % tiles_per_split;
    m0 = (rem / p.n_tiles) * 128;
    n0 = (rem % p.n_tiles) * BN;
    kb = split * steps_per_split;
    const int ke = min(p.n_main, kb + steps_per_split);
    nmain = max(0, ke - kb);
  };

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t j = 0;
      for (int tile = blockIdx.x; tile < n_tiles_total && !*abort_flag; tile += gridDim.x) {
        int split, m0, n0, kb, nmain;
        tile_coords(tile, split, m0, n0, kb, nmain);
        for (int ks = 0; ks < nmain; ++ks, ++j) {
          const int s = j % NS;
          const uint32_t ph = (j / NS) & 1;
          if (!mbar_wait(&bars->empty[s], ph ^ 1, abort_flag)) break;
          uint8_t* st_a = smem + s * C::kStage;
          uint8_t* st_b = st_a + C::kA;
          uint64_t* fb = &bars->full[s];
          const int k0 = (kb + ks) * 64;
          mbar_arrive_expect_tx(fb, C::kA + C::kB);
          if (A_SRC == A_TMA_K) {
            tma_load_2d(st_a, &maps.a, k0, m0, fb);
          } else {
            tma_load_2d(st_a, &maps.a, m0, k0, fb);
            tma_load_2d(st_a + 8192, &maps.a, m0 + 64, k0, fb);
          }
          if (B_SRC == B_TMA_K) {
            tma_load_2d(st_b, &maps.b, k0, n0, fb);
          } else {
            const int atom_bytes = 64 * p.b_atom * 2;
            for (int a = 0; a < BN / p.b_atom; ++a) tma_load_2d(st_b + a * atom_bytes, &maps.b, n0 + a * p.b_atom, k0, fb);
          }
        }
      }
      // drain: wait (bounded, regardless of abort) for the loads of the last NS issued stages
      const uint32_t first = j > NS ? j - NS : 0;
      for (uint32_t q = first; q < j; ++q) {
        volatile int never = 0;
        mbar_wait(&bars->full[q % NS], (q / NS) & 1, &never);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t j = 0;
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < n_tiles_total && ok; tile += gridDim.x, ++it) {
        int split, m0, n0, kb, nmain;
        tile_coords(tile, split, m0, n0, kb, nmain);
        const int acc = it % C::kAcc;
        const uint32_t aph = (it / C::kAcc) & 1;
        if (!mbar_wait(&bars->acc_empty[acc], aph ^ 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int ks = 0; ks < nmain; ++ks, ++j) {
          const int s = j % NS;
          const uint32_t ph = (j / NS) & 1;
          if (!mbar_wait(&bars->full[s], ph, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * C::kStage);
          const uint32_t b_addr = a_addr + C::kA;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = (A_SRC == A_TMA_MN) ? smem_desc(a_addr + kk * 2048, 8192, 1024, kSw128)
                                                    : smem_desc(a_addr + kk * 32, 16, 1024, kSw128);
            uint64_t bd;
            if (B_SRC == B_TMA_MN) {
              const uint32_t rb = p.b_atom * 2;
              const uint32_t lay = rb == 128 ? kSw128 : (rb == 64 ? kSw64 : kSw32);
              bd = smem_desc(b_addr + kk * 16 * rb, 64 * rb, 8 * rb, lay);
            } else {
              bd = smem_desc(b_addr + kk * 32, 16, 1024, kSw128);
            }
            umma_bf16_ss(d_tmem, ad, bd, kIdesc, (ks > 0 || kk > 0) ? 1u : 0u);
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
  } else {
    // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    uint16_t* stg = reinterpret_cast<uint16_t*>(staging) + q * 32 * 32;
    int it = 0;
    for (int tile = blockIdx.x; tile < n_tiles_total; tile += gridDim.x, ++it) {
      int split, m0, n0, kb, nmain;
      tile_coords(tile, split, m0, n0, kb, nmain);
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
          eng::store_chunk_bf16_t(v, stg, lane, n0 + c * 32, m0 + q * 32, p);
        }
      }
      tc_fence_before();
      mbar_arrive(&bars->acc_empty[acc]);
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

template <int A_SRC, int B_SRC, int BN, int OUT>
cudaError_t launch_variant(const GemmParams& p, const GemmMaps& maps, cudaStream_t st) {
  using C = Cfg<BN>;
  auto kern = gemm_kernel<A_SRC, B_SRC, BN, OUT>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [&] {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem + 1024);
  });
  if (attr_err != cudaSuccess) return attr_err;
  const int tiles = p.m_tiles * p.n_tiles * p.splits;
  const int grid = tiles < device_sm_count() ? tiles : device_sm_count();
  count_launch();
  kern<<<grid, kThreadsPlain, C::kSmem + 1024, st>>>(p, maps);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm(int a_src, int b_src, int bn, int out_mode, int tail_a_mn, const GemmParams& p,
                        const GemmMaps& maps, cudaStream_t st) {
  (void)tail_a_mn;
  if (a_src == A_DQ_K || a_src == A_DQ_MN) return launch_fused(a_src, bn, p, maps, st);
  if (out_mode != OUT_F32_D) return cudaErrorNotSupported;
  if (a_src == A_TMA_K && b_src == B_TMA_K) {  // T = X A^T
    if (bn == 32) return launch_variant<A_TMA_K, B_TMA_K, 32, OUT_F32_D>(p, maps, st);
    if (bn == 64) return launch_variant<A_TMA_K, B_TMA_K, 64, OUT_F32_D>(p, maps, st);
  }
  if (a_src == A_TMA_K && b_src == B_TMA_MN) {  // dT = dY B
    if (bn == 32) return launch_variant<A_TMA_K, B_TMA_MN, 32, OUT_F32_D>(p, maps, st);
    if (bn == 64) return launch_variant<A_TMA_K, B_TMA_MN, 64, OUT_F32_D>(p, maps, st);
  }
  if (a_src == A_TMA_MN && b_src == B_TMA_MN) {  // dB = dY^T T, dA^T = X^T dT
    if (bn == 32) return launch_variant<A_TMA_MN, B_TMA_MN, 32, OUT_F32_D>(p, maps, st);
    if (bn == 64) return launch_variant<A_TMA_MN, B_TMA_MN, 64, OUT_F32_D>(p, maps, st);
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
