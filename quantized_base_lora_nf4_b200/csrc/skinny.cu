// The adapter products of rank r = 16, 32 or 64 at many tokens in one launch (QLoRA explainer,
// "Background: how LoRA works": the adapter's down-projection; its gradient dT = s dY B for the backward):
//     OUT[m, j] = bf16( s * sum_k X[m, k] W(k, j) ),   X [M, K] bf16 row-major, j < r,
// with W(k, j) = A[j, k] (A [r, K] row-major: T_save = bf16(s X A^T)) or W(k, j) = B[k, j] (B [K, r]
// row-major: dT = bf16(s dY B)).
//
// The reduction is long (K = 4096 .. 11008) and the output narrow, so a launch must split K to keep
// every SM streaming.  Here a cluster of 4 CTAs owns 64 tokens, each CTA a quarter of K: a TMA producer
// warp streams [64 tokens x 64 k] tiles of X and [r x 64 k] tiles of W into an 8-stage ring, four warps
// multiply them with mma.sync (16 tokens x r outputs each, fp32 accumulate), and the four fp32
// partial tiles are summed in shared memory across the cluster (CTA c sums rows 16c .. 16c+15 over the
// ranks in order 0..3, a fixed order), scaled and written as bf16.  No partial sums reach global memory
// and no second launch is needed.
#include <cuda_bf16.h>

#include "cluster.cuh"
#include "common.cuh"
#include "gemm.cuh"
#include "ptx.cuh"

namespace qlr {

namespace {

constexpr int kSkCluster = 4;                    // CTAs per cluster (quarters of K)
constexpr int kSkRows = 64;                      // tokens per cluster
constexpr int kSkStages = 8;
constexpr int kSkTile = 64 * 128;                // one [64 x 64] bf16 tile, 128-byte rows
constexpr int kSkStage = 2 * kSkTile;            // X tile + W tile (r x 64 bf16, at most as large)
constexpr int kSkPartStride = 72;                // fp32 row stride of the partial tile (bank spread)
constexpr int kSkPartBytes = kSkRows * kSkPartStride * 4;
constexpr int kSkThreads = 5 * 32;               // 4 MMA warps + 1 TMA warp
constexpr int kSkSmem = 1024 + kSkStages * kSkStage + kSkPartBytes + 256;

struct SkinnyParams {
  int64_t M, K;
  int kc;                 // reduction columns per CTA (a multiple of 64)
  float s;
  uint16_t* out;          // [M, 64] bf16
  int32_t* status;
  long long wait_cycles;  // bound of every pipeline wait (SM clock cycles)
};

struct alignas(8) SkBars {
  uint64_t full[kSkStages], empty[kSkStages];
  int abort_flag;
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// byte offset of 16-byte chunk `ch` of row `row` in a tile of RB-byte rows written by TMA with the RB-byte
// swizzle (RB = 128, 64 or 32): the chunk bits of the offset are XORed with the bits from 7 up
template <int RB>
__device__ __forceinline__ uint32_t swz(int row, int ch) {
  const int off = row * RB + ch * 16;
  return static_cast<uint32_t>(off ^ (((off >> 7) & (RB / 16 - 1)) << 4));
}

// TRANS_W: W is B [K, R] (a tile holds 64 k rows of R outputs, 2R-byte rows) rather than A [R, K] (R output
// rows of 64 k).
template <bool TRANS_W, int R>
__global__ void __launch_bounds__(kSkThreads, 1) skinny_kernel(const __grid_constant__ SkinnyParams p,
                                                               const __grid_constant__ CUtensorMap tm_x,
                                                               const __grid_constant__ CUtensorMap tm_w) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  float* part = reinterpret_cast<float*>(smem + kSkStages * kSkStage);
  SkBars* bars = reinterpret_cast<SkBars*>(smem + kSkStages * kSkStage + kSkPartBytes);
  volatile int* abort_flag = &bars->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int64_t m0 = static_cast<int64_t>(blockIdx.x / kSkCluster) * kSkRows;
  const int64_t k_begin = static_cast<int64_t>(rank) * p.kc;
  const int64_t k_len = p.K - k_begin < p.kc ? (p.K - k_begin > 0 ? p.K - k_begin : 0) : p.kc;
  const int nsteps = static_cast<int>((k_len + 63) / 64);
  // the clusters walk their quarter of K from different starting points, so that they do not all read
  // the same tile of the (shared) weight-side operand at the same time
  const int rot = nsteps > 0 ? static_cast<int>((blockIdx.x / kSkCluster) % nsteps) : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSkStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 4);
    }
    bars->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
  }
  pdl_launch_dependents();
  pdl_wait();
  __syncthreads();

  float acc[R / 8][4];
#pragma unroll
  for (int n = 0; n < R / 8; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;

  if (warp == 4) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int s = 0;
      for (; s < nsteps; ++s) {
        const int st = s % kSkStages;
        if (!mbar_wait(&bars->empty[st], ((s / kSkStages) & 1) ^ 1, abort_flag, p.wait_cycles)) break;
        uint8_t* dst = ring + st * kSkStage;
        const int32_t k = static_cast<int32_t>(k_begin + 64 * ((s + rot) % nsteps));
        mbar_arrive_expect_tx(&bars->full[st], kSkTile + 128 * R);
        tma_load_2d(dst, &tm_x, k, static_cast<int32_t>(m0), &bars->full[st]);
        if (TRANS_W)
          tma_load_2d(dst + kSkTile, &tm_w, 0, k, &bars->full[st]);
        else
          tma_load_2d(dst + kSkTile, &tm_w, k, 0, &bars->full[st]);
      }
      // after an abort the fills still in flight must land before the shared memory is reused or freed
      if (*abort_flag)
        for (int q = s > kSkStages ? s - kSkStages : 0; q < s; ++q)
          mbar_drain(&bars->full[q % kSkStages], (q / kSkStages) & 1);
    }
  } else {
    // ------------------------------------------------------------------ MMA warps: tokens 16 warp .. +15
    const int g = lane >> 2, t = lane & 3, q8 = lane >> 3;
    const uint32_t ring0 = smem_u32(ring);
    for (int s = 0; s < nsteps; ++s) {
      const int st = s % kSkStages;
      const bool ok = mbar_wait(&bars->full[st], (s / kSkStages) & 1, abort_flag, p.wait_cycles);
      if (!__all_sync(0xffffffffu, ok)) break;
      const uint32_t xt = ring0 + st * kSkStage, wt = xt + kSkTile;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        uint32_t a[4];
        const int ar = 16 * warp + (lane & 15);
        ldsm_x4(xt + swz<128>(ar, 2 * kk + (lane >> 4)), a);
#pragma unroll
        for (int np = 0; np < R / 16; ++np) {  // output tiles 2 np, 2 np + 1 (8 outputs each)
          uint32_t b[4];
          if (TRANS_W) {  // tile rows are k: transpose while loading
            const int kr = 16 * kk + (lane & 7) + ((q8 & 1) << 3);
            ldsm_x4_t(wt + swz<2 * R>(kr, 2 * np + (q8 >> 1)), b);
          } else {        // tile rows are outputs j
            const int jr = 16 * np + (lane & 7) + ((q8 >> 1) << 3);
            ldsm_x4(wt + swz<128>(jr, 2 * kk + (q8 & 1)), b);
          }
          mma_16816(acc[2 * np], a, b[0], b[1]);
          mma_16816(acc[2 * np + 1], a, b[2], b[3]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->empty[st]);
    }
    // this CTA's partial tile: rows g, g + 8 of the warp's 16, columns 8 n + 2 t, + 1
#pragma unroll
    for (int n = 0; n < R / 8; ++n) {
      float* r0 = part + (16 * warp + g) * kSkPartStride + 8 * n + 2 * t;
      *reinterpret_cast<float2*>(r0) = make_float2(acc[n][0], acc[n][1]);
      *reinterpret_cast<float2*>(r0 + 8 * kSkPartStride) = make_float2(acc[n][2], acc[n][3]);
    }
  }
  cluster_sync_all();  // every partial tile of the cluster written
  if (threadIdx.x < 2 * R) {
    // rank c sums rows 16 c .. 16 c + 15 over the four partial tiles in rank order: 8 outputs a thread
    const int row = 16 * static_cast<int>(rank) + static_cast<int>(threadIdx.x) / (R / 8);
    const int col = (static_cast<int>(threadIdx.x) % (R / 8)) * 8;
    const uint32_t local = smem_u32(part + row * kSkPartStride + col);
    float sum[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (uint32_t q = 0; q < kSkCluster; ++q) {
      const uint32_t ra = map_rank(local, q);
      const float4 u = ld_cluster_v4(ra), v = ld_cluster_v4(ra + 16);
      sum[0] += u.x; sum[1] += u.y; sum[2] += u.z; sum[3] += u.w;
      sum[4] += v.x; sum[5] += v.y; sum[6] += v.z; sum[7] += v.w;
    }
    const int64_t m = m0 + row;
    if (m < p.M) {
      uint4 o;
      o.x = pack_bf16x2_rn(__fmul_rn(p.s, sum[0]), __fmul_rn(p.s, sum[1]));
      o.y = pack_bf16x2_rn(__fmul_rn(p.s, sum[2]), __fmul_rn(p.s, sum[3]));
      o.z = pack_bf16x2_rn(__fmul_rn(p.s, sum[4]), __fmul_rn(p.s, sum[5]));
      o.w = pack_bf16x2_rn(__fmul_rn(p.s, sum[6]), __fmul_rn(p.s, sum[7]));
      *reinterpret_cast<uint4*>(p.out + m * R + col) = o;
    }
  }
  cluster_sync_all();  // no CTA leaves while another still reads its partial tile
  if (threadIdx.x == 0 && bars->abort_flag) report(p.status, QLR_ERR_TIMEOUT);
}

template <bool TRANS_W, int R>
cudaError_t launch_skinny_variant(const SkinnyParams& p, const CUtensorMap& tx, const CUtensorMap& tw, int grid,
                                  cudaStream_t st) {
  auto kern = skinny_kernel<TRANS_W, R>;
  const cudaError_t e = ensure_max_dynamic_smem(kern, kSkSmem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kSkThreads);
  cfg.dynamicSmemBytes = kSkSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kSkCluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  count_launch();
  return cudaLaunchKernelEx(&cfg, kern, p, tx, tw);
}

}  // namespace

bool skinny_supported(int64_t M, int64_t K, int r) {
  return (r == 16 || r == 32 || r == 64) && M >= 1024 && K % 64 == 0;
}

cudaError_t launch_skinny(const uint16_t* X, int64_t M, int64_t K, const uint16_t* W, bool w_is_k_by_r, int r, float s,
                          uint16_t* out, int32_t* status, long long wait_cycles, cudaStream_t st) {
  CUtensorMap tx, tw;
  if (make_tmap(&tx, X, 2, M, K, kSkRows, 64, 128)) return cudaErrorInvalidValue;
  if (w_is_k_by_r ? make_tmap(&tw, W, 2, K, r, 64, r, 2 * r) : make_tmap(&tw, W, 2, r, K, r, 64, 128))
    return cudaErrorInvalidValue;
  SkinnyParams p;
  p.M = M;
  p.K = K;
  p.kc = static_cast<int>(((K / 64 + kSkCluster - 1) / kSkCluster) * 64);
  p.s = s;
  p.out = out;
  p.status = status;
  p.wait_cycles = wait_cycles;
  const int grid = static_cast<int>((M + kSkRows - 1) / kSkRows) * kSkCluster;
  switch (r) {
    case 16: return w_is_k_by_r ? launch_skinny_variant<true, 16>(p, tx, tw, grid, st)
                                : launch_skinny_variant<false, 16>(p, tx, tw, grid, st);
    case 32: return w_is_k_by_r ? launch_skinny_variant<true, 32>(p, tx, tw, grid, st)
                                : launch_skinny_variant<false, 32>(p, tx, tw, grid, st);
    case 64: return w_is_k_by_r ? launch_skinny_variant<true, 64>(p, tx, tw, grid, st)
                                : launch_skinny_variant<false, 64>(p, tx, tw, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace qlr
