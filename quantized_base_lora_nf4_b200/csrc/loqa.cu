// LoQA: gradients of the loss with respect to the group-wise INT4 scale and zero point (LoQA abstract: the
// scale and the zero point of the quantiser are fine-tuned; read on the QA-LoRA group-wise INT4 format).
//
// With W[o, k] = s[o, g] (c[o, k] - z[o, g]) (g = k / L) and G = dY^T X the gradient with respect to W,
//   dscale[o, g] = sum_{k in g} G[o, k] (c[o, k] - z[o, g]),   dzero[o, g] = -s[o, g] sum_{k in g} G[o, k].
// G is a full N x K x M contraction; it never reaches global memory.  A persistent tcgen05 GEMM computes
// 128 x 256 tiles of G in TMEM (weight rows o on the 128 lanes, inputs k on 256 columns, the tokens as the
// reduction) from two MN-major TMA operands -- dY^T straight from dY [M, N] and X^T straight from X [M, K],
// both row-major, 128-byte swizzled -- and the epilogue reduces each row's 256 columns group by group with
// the row's 4-bit codes, writing only the [N, K / L] gradients.
//
// Warp roles: 0 TMA producer, 1 TMEM allocator + single-thread MMA issuer, 2..5 epilogue (a warp reads TMEM
// lane quadrant warp % 4).  Two 256-column accumulators overlap a tile's epilogue with the next tile's main
// loop.  Every wait is bounded (QLR_ERR_TIMEOUT in the status word).
#include <cuda_fp16.h>

#include "engine.cuh"

namespace qlr {

namespace {

constexpr int kThreadsLoqa = 192;
constexpr int kLoqaBN = 256;                     // inputs k per tile
constexpr int kLoqaA = 16384;                    // dY^T stage: 128 rows o x 64 tokens (two 64-wide atoms)
constexpr int kLoqaB = kLoqaBN * 128;            // X^T stage: 256 inputs k x 64 tokens (four 64-wide atoms)
constexpr int kLoqaStage = kLoqaA + kLoqaB;      // 48 KB
constexpr int kLoqaStages = 4;
constexpr int kLoqaSmem = kLoqaStages * kLoqaStage + 1024;

struct LoqaParams {
  int N, K, M, L, G;        // G = K / L groups per row
  int o_tiles, k_tiles, n_steps;
  const uint8_t* codes;     // [N, K / 2] packed 4-bit codes
  const __half* scale;      // [N, G]
  const __half* zero;       // [N, G]
  float* dscale;            // [N, G]
  float* dzero;             // [N, G]
  int32_t* status;
  long long wait_cycles;
};

struct alignas(8) LBars {
  uint64_t full[kLoqaStages], empty[kLoqaStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

__global__ void __launch_bounds__(kThreadsLoqa, 1)
    loqa_grad_kernel(const __grid_constant__ LoqaParams p, const __grid_constant__ CUtensorMap tm_dy,
                     const __grid_constant__ CUtensorMap tm_x) {
  constexpr int NS = kLoqaStages;
  constexpr uint32_t kIdesc = idesc_bf16(128, kLoqaBN, 1u, 1u);  // both operands MN-major
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  LBars* bars = reinterpret_cast<LBars*>(smem + NS * kLoqaStage);
  volatile int* abort_flag = &bars->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = p.o_tiles * p.k_tiles;

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
    tma_prefetch_desc(&tm_dy);
    tma_prefetch_desc(&tm_x);
  }
  pdl_launch_dependents();
  pdl_wait();
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, 512);
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
        const int o0 = (item / p.k_tiles) * 128, k0 = (item % p.k_tiles) * kLoqaBN;
        for (int ks = 0; ks < p.n_steps; ++ks, ++j) {
          const int s = j % NS;
          if (!mbar_wait(&bars->empty[s], ((j / NS) & 1) ^ 1, abort_flag, p.wait_cycles)) break;
          uint8_t* st_a = smem + s * kLoqaStage;
          uint8_t* st_b = st_a + kLoqaA;
          uint64_t* fb = &bars->full[s];
          const int t0 = ks * 64;
          mbar_arrive_expect_tx(fb, kLoqaStage);
          // [64 tokens][64 rows o] boxes: token rows of 128 bytes, the canonical MN-major 128-byte atoms
          tma_load_2d(st_a, &tm_dy, o0, t0, fb);
          tma_load_2d(st_a + 8192, &tm_dy, o0 + 64, t0, fb);
#pragma unroll
          for (int a = 0; a < kLoqaBN / 64; ++a) tma_load_2d(st_b + a * 8192, &tm_x, k0 + 64 * a, t0, fb);
        }
      }
      const uint32_t first = j > NS ? j - NS : 0;
      for (uint32_t q = first; q < j; ++q) mbar_drain(&bars->full[q % NS], (q / NS) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t j = 0;
      int it = 0;
      bool ok = true;
      const uint64_t a_desc0 = smem_desc(smem_u32(smem), 8192, 1024, kSw128);
      const uint64_t b_desc0 = smem_desc(smem_u32(smem + kLoqaA), 8192, 1024, kSw128);
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x, ++it) {
        const int acc = it & 1;
        if (!mbar_wait(&bars->acc_empty[acc], ((it >> 1) & 1) ^ 1, abort_flag, p.wait_cycles)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kLoqaBN;
        for (int ks = 0; ks < p.n_steps; ++ks, ++j) {
          const int s = j % NS;
          if (!mbar_wait(&bars->full[s], (j / NS) & 1, abort_flag, p.wait_cycles)) { ok = false; break; }
          tc_fence_after();
          const uint32_t soff = static_cast<uint32_t>((s * kLoqaStage) >> 4);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)  // 16 tokens = two 8-row groups of 1024 bytes per MMA
            umma_bf16_ss(d_tmem, a_desc0 + soff + kk * (2048 >> 4), b_desc0 + soff + kk * (2048 >> 4), kIdesc,
                         (ks > 0 || kk > 0) ? 1u : 0u);
          umma_commit(&bars->empty[s]);
        }
        if (!ok) break;
        umma_commit(&bars->acc_full[acc]);
      }
      umma_commit(&bars->drain);
      mbar_drain(&bars->drain, 0);
    }
  } else {
    // ------------------------------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;
    int it = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++it) {
      const int o0 = (item / p.k_tiles) * 128, k0 = (item % p.k_tiles) * kLoqaBN;
      const int acc = it & 1;
      const bool got = mbar_wait(&bars->acc_full[acc], (it >> 1) & 1, abort_flag, p.wait_cycles);
      __syncwarp();
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const int o = o0 + q * 32 + lane;
      const bool row_ok = o < p.N;
      const uint8_t* crow = p.codes + static_cast<int64_t>(o) * (p.K / 2);
      float s0 = 0.f, s1 = 0.f;
#pragma unroll 1
      for (int c = 0; c < kLoqaBN / 32; ++c) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem_base + acc * kLoqaBN + c * 32 + ((q * 32) << 16), v);
        tmem_ld_wait();
        const int k = k0 + 32 * c;
        if (row_ok && k < p.K) {
          const uint4 cw = __ldg(reinterpret_cast<const uint4*>(crow + k / 2));
          const uint32_t w[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float g = __uint_as_float(v[e]);
            const float code = static_cast<float>((w[e >> 3] >> (4 * (e & 7))) & 0xFu);  // element 2j: low nibble
            s0 = __fadd_rn(s0, g);
            s1 = __fmaf_rn(g, code, s1);
          }
          if ((k + 32) % p.L == 0) {  // the group ends with this chunk
            const int64_t gi = static_cast<int64_t>(o) * p.G + (k + 32) / p.L - 1;
            const float sc = __half2float(p.scale[gi]), z = __half2float(p.zero[gi]);
            p.dscale[gi] = __fmaf_rn(-z, s0, s1);
            p.dzero[gi] = -sc * s0;
            s0 = s1 = 0.f;
          }
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
    tmem_dealloc(tmem_base, 512);
  }
  if (threadIdx.x == 0 && bars->abort_flag) report(p.status, QLR_ERR_TIMEOUT);
}

}  // namespace

}  // namespace qlr

using namespace qlr;

extern "C" int qlr_loqa_grad(const qlr_qweight* w, const uint16_t* X, const uint16_t* dY, int64_t M, float* dscale,
                             float* dzero, int32_t* status, void* stream) {
  if (!w || !dscale || !dzero || M < 0) return QLR_ERR_ARG;
  if (w->fmt != QLR_FMT_INT4G || !w->codes || !w->scale || !w->zero) return QLR_ERR_ARG;
  if (w->group != 32 && w->group != 64 && w->group != 128) return QLR_ERR_ARG;
  const int64_t N = w->N, K = w->K;
  if (N <= 0 || K <= 0 || K % w->group || N % 8) return QLR_ERR_SHAPE;
  if (N > (int64_t(1) << 30) || K > (int64_t(1) << 30) || M > (int64_t(1) << 30)) return QLR_ERR_SHAPE;
  auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (!al16(w->codes) || !al16(dscale) || !al16(dzero)) return QLR_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t G = K / w->group;
  if (M == 0) {  // no tokens: the gradients are zero
    if (cudaMemsetAsync(dscale, 0, size_t(N) * G * 4, st) != cudaSuccess) return QLR_ERR_CUDA;
    return cudaMemsetAsync(dzero, 0, size_t(N) * G * 4, st) == cudaSuccess ? QLR_OK : QLR_ERR_CUDA;
  }
  if (!X || !dY) return QLR_ERR_ARG;
  if (!al16(X) || !al16(dY)) return QLR_ERR_ALIGN;
  CUtensorMap tm_dy, tm_x;
  if (make_tmap(&tm_dy, dY, 2, M, N, 64, 64, 128)) return QLR_ERR_CUDA;
  if (make_tmap(&tm_x, X, 2, M, K, 64, 64, 128)) return QLR_ERR_CUDA;
  LoqaParams p;
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.M = static_cast<int>(M);
  p.L = w->group;
  p.G = static_cast<int>(G);
  p.o_tiles = static_cast<int>((N + 127) / 128);
  p.k_tiles = static_cast<int>((K + kLoqaBN - 1) / kLoqaBN);
  p.n_steps = static_cast<int>((M + 63) / 64);
  p.codes = w->codes;
  p.scale = reinterpret_cast<const __half*>(w->scale);
  p.zero = reinterpret_cast<const __half*>(w->zero);
  p.dscale = dscale;
  p.dzero = dzero;
  p.status = status_or_sink(status);
  p.wait_cycles = wait_limit_cycles();
  const cudaError_t e = ensure_max_dynamic_smem(loqa_grad_kernel, kLoqaSmem + 1024);
  if (e != cudaSuccess) return QLR_ERR_CUDA;
  const int items = p.o_tiles * p.k_tiles;
  const int grid = items < device_sm_count() ? items : device_sm_count();
  return launch_pdl(loqa_grad_kernel, dim3(grid), dim3(kThreadsLoqa), kLoqaSmem + 1024, st, p, tm_dy, tm_x) ==
                 cudaSuccess
             ? QLR_OK
             : QLR_ERR_CUDA;
}
