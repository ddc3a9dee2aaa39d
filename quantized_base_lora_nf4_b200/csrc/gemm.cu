// tcgen05 GEMM engine for sm_100a: the rank-r adapter GEMMs of the layer (both operands by TMA).
//
//   T   = s P(X) A^T   D[M, r]  = X [M, K]  (K-major)  x  A (or its group expansion) [r, K] (K-major)
//   dT  = s dY B       D[M, r]  = dY [M, N] (K-major)  x  B [N, r] (MN-major)
//   dB  = dY^T T       D[N, r]  = dY^T (MN-major)      x  T_save [M, r] (MN-major)
//   dA^T = X^T dT      D[K, r]  = X^T (MN-major)       x  dT [M, r] (MN-major), pooled by group for QA-LoRA
//
// One persistent CTA per SM walks a static list of (tile, split) work items; a tile is 128 rows x BN.
// Warp roles: 0 TMA producer (ring of A+B stages), 1 TMEM allocator + single-thread tcgen05.mma
// issuer, 2..5 epilogue.  Two TMEM accumulators overlap an item's epilogue with the next item's main
// loop.  Without a split the epilogue applies the output transform directly; with one, each item's
// fp32 tile goes to the workspace and a reduction kernel (elementwise.cu) sums the parts in
// split order (deterministic) and applies the transform with one thread per output.
#include <cudaTypedefs.h>

#include <mutex>

#include "engine.cuh"

namespace qlr {

namespace {

constexpr int kThreadsAdapter = 192;

template <int BN>
struct ACfg {
  static constexpr int kA = 16384;
  static constexpr int kB = BN * 128;
  static constexpr int kStage = ((kA + kB) + 1023) / 1024 * 1024;
  static constexpr int kStages = 8;
  static constexpr int kSmem = kStages * kStage + 2048;
  static constexpr int kTmemCols = (2 * BN <= 64) ? 64 : 128;
};

struct alignas(8) ABars {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int ep_ok[4];
  float chunk[4 * 64];
};

// Output transform of one finished row (`acc` = the BN fp32 values of D row m0 + row).
template <int BN>
__device__ __forceinline__ void adapter_store(const AdapterParams& p, float (&acc)[BN], int m0, int row, int lane,
                                              int q, ABars* bars) {
  const int grow = m0 + row;
  if (p.out_mode == ADAPTER_ROWS_BF16) {
    if (grow < p.Mm) {
      uint16_t* o = static_cast<uint16_t*>(p.out) + static_cast<int64_t>(grow) * p.ld_out;
#pragma unroll
      for (int j = 0; j < BN; j += 8) {
        if (j < p.r) {
          uint4 w;
          w.x = pack_bf16x2_rn(p.scale * acc[j], p.scale * acc[j + 1]);
          w.y = pack_bf16x2_rn(p.scale * acc[j + 2], p.scale * acc[j + 3]);
          w.z = pack_bf16x2_rn(p.scale * acc[j + 4], p.scale * acc[j + 5]);
          w.w = pack_bf16x2_rn(p.scale * acc[j + 6], p.scale * acc[j + 7]);
          *reinterpret_cast<uint4*>(o + j) = w;
        }
      }
    }
  } else if (p.out_mode == ADAPTER_ROWS_F32) {
    if (grow < p.Mm) {
      float* o = static_cast<float*>(p.out) + static_cast<int64_t>(grow) * p.ld_out;
#pragma unroll
      for (int j = 0; j < BN; j += 4)
        if (j < p.r) *reinterpret_cast<float4*>(o + j) = make_float4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]);
    }
  } else if (p.pool_L <= 1) {  // out[j, m]
    if (grow < p.Mm) {
      float* o = static_cast<float*>(p.out);
#pragma unroll
      for (int j = 0; j < BN; ++j)
        if (j < p.r) o[static_cast<int64_t>(j) * p.ld_out + grow] = acc[j];
    }
  } else {  // out[j, m / L]: sum 32-row chunks per warp, then groups of L rows
#pragma unroll
    for (int j = 0; j < BN; ++j) {
      float v = grow < p.Mm ? acc[j] : 0.f;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) bars->chunk[q * BN + j] = v;
    }
    named_bar_sync(1, 128);
    const int per_group = p.pool_L / 32;
    const int n_groups = 128 / p.pool_L;
    for (int tid = row; tid < n_groups * p.r; tid += 128) {  // row doubles as a 0..127 thread index
      const int g = tid / p.r, j = tid % p.r;
      float v = 0.f;
      for (int c = 0; c < per_group; ++c) v += bars->chunk[(g * per_group + c) * BN + j];
      const int64_t og = (m0 / p.pool_L) + g;
      if (og * p.pool_L < p.Mm)
        static_cast<float*>(p.out)[static_cast<int64_t>(j) * p.ld_out + og] = v / static_cast<float>(p.pool_L);
    }
    named_bar_sync(1, 128);
  }
}

template <int A_SRC, int B_SRC, int BN>
__global__ void __launch_bounds__(kThreadsAdapter, 1)
    adapter_kernel(const __grid_constant__ AdapterParams p, const __grid_constant__ GemmMaps maps) {
  using C = ACfg<BN>;
  constexpr int NS = C::kStages;
  constexpr uint32_t kIdesc = idesc_bf16(128, BN, A_SRC == A_TMA_MN ? 1u : 0u, B_SRC == B_TMA_MN ? 1u : 0u);

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  ABars* bars = reinterpret_cast<ABars*>(smem + NS * C::kStage);
  volatile int* abort_flag = &bars->abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int S = p.splits;
  const int n_items = p.m_tiles * S;
  const int sps = (p.n_steps + S - 1) / S;
  auto item_coords = [&](int item, int& tile, int& split, int& kb, int& nsteps) {
    split = item / p.m_tiles;
    tile = item % p.m_tiles;
    kb = split * sps;
    nsteps = max(0, min(p.n_steps, kb + sps) - kb);
  };

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
  // everything above touches only shared memory and kernel parameters; from here on the previous
  // kernel's results are needed (and its TMEM must be free)
  pdl_launch_dependents();
  pdl_wait();
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t j = 0;
      for (int item = blockIdx.x; item < n_items && !*abort_flag; item += gridDim.x) {
        int tile, split, kb, nsteps;
        item_coords(item, tile, split, kb, nsteps);
        const int m0 = tile * 128;
        for (int ks = 0; ks < nsteps; ++ks, ++j) {
          const int s = j % NS;
          if (!mbar_wait(&bars->empty[s], ((j / NS) & 1) ^ 1, abort_flag, p.wait_cycles)) break;
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
            tma_load_2d(st_b, &maps.b, k0, 0, fb);
          } else {
            const int atom_bytes = 64 * p.b_atom * 2;
            for (int a = 0; a < BN / p.b_atom; ++a) tma_load_2d(st_b + a * atom_bytes, &maps.b, a * p.b_atom, k0, fb);
          }
        }
      }
      const uint32_t first = j > NS ? j - NS : 0;
      for (uint32_t qq = first; qq < j; ++qq) {
        mbar_drain(&bars->full[qq % NS], (qq / NS) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t j = 0;
      int it = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x, ++it) {
        int tile, split, kb, nsteps;
        item_coords(item, tile, split, kb, nsteps);
        const int acc = it & 1;
        if (!mbar_wait(&bars->acc_empty[acc], ((it >> 1) & 1) ^ 1, abort_flag, p.wait_cycles)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int ks = 0; ks < nsteps; ++ks, ++j) {
          const int s = j % NS;
          if (!mbar_wait(&bars->full[s], (j / NS) & 1, abort_flag, p.wait_cycles)) { ok = false; break; }
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
              bd = smem_desc(b_addr + kk * 16 * rb, 64 * rb, 8 * rb, rb == 128 ? kSw128 : kSw64);
            } else {
              bd = smem_desc(b_addr + kk * 32, 16, 1024, kSw128);
            }
            umma_bf16_ss(d_tmem, ad, bd, kIdesc, (ks > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&bars->empty[s]);
        }
        if (!ok) break;
        umma_commit(&bars->acc_full[acc]);  // also for an empty item: the epilogue then reads zeros
      }
      umma_commit(&bars->drain);
      mbar_drain(&bars->drain, 0);
    }
  } else {
    // ------------------------------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;
    const int row = q * 32 + lane;
    int it = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++it) {
      int tile, split, kb, nsteps;
      item_coords(item, tile, split, kb, nsteps);
      const int m0 = tile * 128;
      const int acc = it & 1;
      const bool got = mbar_wait(&bars->acc_full[acc], (it >> 1) & 1, abort_flag, p.wait_cycles);
      __syncwarp();
      bool all_got = __all_sync(0xffffffffu, got);
      if (S == 1 && p.out_mode == ADAPTER_COLS_F32 && p.pool_L > 1) {
        // the pooled store synchronises the four epilogue warps on a named barrier, so they must leave
        // the loop together: one joint decision after an abort
        if (lane == 0) bars->ep_ok[q] = all_got ? 1 : 0;
        named_bar_sync(1, 128);
        all_got = bars->ep_ok[0] && bars->ep_ok[1] && bars->ep_ok[2] && bars->ep_ok[3];
        named_bar_sync(1, 128);
      }
      if (!all_got) break;
      tc_fence_after();
      float v[BN];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t u[32];
        tmem_ld_32x32b_x32(tmem_base + acc * BN + c * 32 + ((q * 32) << 16), u);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) v[c * 32 + i] = nsteps > 0 ? __uint_as_float(u[i]) : 0.f;
      }
      tc_fence_before();
      mbar_arrive(&bars->acc_empty[acc]);  // the accumulator is free for the next item
      if (S == 1) {
        adapter_store<BN>(p, v, m0, row, lane, q, bars);
        continue;
      }
      float* mine = p.part + (static_cast<int64_t>(split) * p.m_tiles * 128 + m0 + row) * BN;
#pragma unroll
      for (int i = 0; i < BN / 4; ++i)
        reinterpret_cast<float4*>(mine)[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
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

template <int A_SRC, int B_SRC, int BN>
cudaError_t launch_adapter_variant(const AdapterParams& p, const GemmMaps& maps, cudaStream_t st) {
  using C = ACfg<BN>;
  auto kern = adapter_kernel<A_SRC, B_SRC, BN>;
  const cudaError_t attr_err = ensure_max_dynamic_smem(kern, C::kSmem + 1024);
  if (attr_err != cudaSuccess) return attr_err;
  const int items = p.m_tiles * p.splits;
  const int grid = items < device_sm_count() ? items : device_sm_count();
  return launch_pdl(kern, dim3(grid), dim3(kThreadsAdapter), C::kSmem + 1024, st, p, maps);
}

}  // namespace

cudaError_t launch_adapter(int a_src, int b_src, int bn, const AdapterParams& p, const GemmMaps& maps,
                           cudaStream_t st) {
  if (p.splits < 1 || p.splits > 64) return cudaErrorInvalidValue;
  if (a_src == A_TMA_K && b_src == B_TMA_K) {  // T = X A^T
    if (bn == 32) return launch_adapter_variant<A_TMA_K, B_TMA_K, 32>(p, maps, st);
    if (bn == 64) return launch_adapter_variant<A_TMA_K, B_TMA_K, 64>(p, maps, st);
  }
  if (a_src == A_TMA_K && b_src == B_TMA_MN) {  // dT = dY B
    if (bn == 32) return launch_adapter_variant<A_TMA_K, B_TMA_MN, 32>(p, maps, st);
    if (bn == 64) return launch_adapter_variant<A_TMA_K, B_TMA_MN, 64>(p, maps, st);
  }
  if (a_src == A_TMA_MN && b_src == B_TMA_MN) {  // dB = dY^T T, dA^T = X^T dT
    if (bn == 32) return launch_adapter_variant<A_TMA_MN, B_TMA_MN, 32>(p, maps, st);
    if (bn == 64) return launch_adapter_variant<A_TMA_MN, B_TMA_MN, 64>(p, maps, st);
  }
  return cudaErrorNotSupported;
}

cudaError_t launch_gemm(int a_src, int b_src, int bn, int out_mode, int tail_a_mn, const GemmParams& p,
                        const GemmMaps& maps, cudaStream_t st) {
  (void)b_src;
  (void)out_mode;
  (void)tail_a_mn;
  if (a_src == A_DQ_K || a_src == A_DQ_MN) return launch_fused(a_src, bn, p, maps, st);
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
