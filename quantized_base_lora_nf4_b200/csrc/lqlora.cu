// LQ-LoRA initialisation (LQ-LoRA abstract: an iterative method splits each pretrained matrix into a
// low-rank part kept in high precision plus a quantised part that is cheap to store; the
// quantised part stays frozen and the low-rank part is the trainable adapter).  Read as the
// alternation
//     Q_0 = 0;  for t = 1..T:  L_t = rank-r truncated SVD of (W - dequant(Q_{t-1})),
//                              Q_t = NF-k quantisation of (W - L_t)
// with the adapter A = bf16(sqrt(S_r) V_r^T), B = bf16(U_r sqrt(S_r) / s), so s B A = L_T.
//
// Residuals, the rank-r subtraction, the factor split and the quantisation run in this library's
// kernels; the SVD is cuSOLVER's gesvd (a library factorisation), loaded with dlopen on first use so
// that the library itself has no link-time dependency on it.  An offline, once-per-weight step.
#include <cuda_fp8.h>
#include <cusolverDn.h>
#include <dlfcn.h>

#include <mutex>

#include "common.cuh"
#include "nfk.cuh"
#include "ptx.cuh"

namespace qlr {

namespace {

// ---- cuSOLVER, resolved at run time ------------------------------------------------------------
struct Solver {
  decltype(&cusolverDnCreate) create = nullptr;
  decltype(&cusolverDnDestroy) destroy = nullptr;
  decltype(&cusolverDnSetStream) set_stream = nullptr;
  decltype(&cusolverDnSgesvd_bufferSize) buffer_size = nullptr;
  decltype(&cusolverDnSgesvd) gesvd = nullptr;
  bool ok = false;
};

const Solver& solver() {
  static Solver s;
  static std::once_flag once;
  std::call_once(once, [] {
    void* h = dlopen("libcusolver.so.11", RTLD_NOW | RTLD_LOCAL);
    if (!h) h = dlopen("libcusolver.so", RTLD_NOW | RTLD_LOCAL);
    if (!h) return;
    s.create = reinterpret_cast<decltype(s.create)>(dlsym(h, "cusolverDnCreate"));
    s.destroy = reinterpret_cast<decltype(s.destroy)>(dlsym(h, "cusolverDnDestroy"));
    s.set_stream = reinterpret_cast<decltype(s.set_stream)>(dlsym(h, "cusolverDnSetStream"));
    s.buffer_size = reinterpret_cast<decltype(s.buffer_size)>(dlsym(h, "cusolverDnSgesvd_bufferSize"));
    s.gesvd = reinterpret_cast<decltype(s.gesvd)>(dlsym(h, "cusolverDnSgesvd"));
    s.ok = s.create && s.destroy && s.set_stream && s.buffer_size && s.gesvd;
  });
  return s;
}

// ---- kernels -----------------------------------------------------------------------------------
// R = W - dequant(Q): the weight the quantised layer actually uses
__global__ void residual_kernel(const float* __restrict__ W, int64_t n, const nfk::View v, float* __restrict__ R) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    R[i] = __fsub_rn(W[i], nfk::dequant_at(v, i));
}

// column-major copy (N x K, leading dimension N) of the row-major N x K matrix R
__global__ void transpose_kernel(const float* __restrict__ R, int64_t N, int64_t K, float* __restrict__ T) {
  __shared__ float tile[32][33];
  const int64_t i0 = static_cast<int64_t>(blockIdx.y) * 32, k0 = static_cast<int64_t>(blockIdx.x) * 32;
  for (int y = threadIdx.y; y < 32; y += blockDim.y) {
    const int64_t i = i0 + y, k = k0 + threadIdx.x;
    if (i < N && k < K) tile[y][threadIdx.x] = R[i * K + k];
  }
  __syncthreads();
  for (int y = threadIdx.y; y < 32; y += blockDim.y) {
    const int64_t k = k0 + y, i = i0 + threadIdx.x;
    if (i < N && k < K) T[k * N + i] = tile[threadIdx.x][y];
  }
}

// Ur[i][c] = U_R[i][c] sqrt(S[c]) (N x r), Vr[c][k] = sqrt(S[c]) V_R^T[c][k] (r x K), both row-major.
// wide (K >= N): gesvd factored R^T (K x N) = U' S V'^T, so U_R = V' (from VT, ld N), V_R^T = U'^T (from U, ld K);
// else: gesvd factored R (N x K) = U S V^T, so U_R = U (ld N), V_R^T = VT (ld K).
__global__ void factors_kernel(const float* __restrict__ U, const float* __restrict__ VT, const float* __restrict__ S,
                               int64_t N, int64_t K, int r, int wide, float* __restrict__ Ur, float* __restrict__ Vr) {
  const int64_t nu = N * r, total = nu + static_cast<int64_t>(r) * K;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    if (e < nu) {
      const int64_t i = e / r;
      const int c = static_cast<int>(e - i * r);
      const float u = wide ? VT[c + i * N] : U[i + c * N];
      Ur[e] = u * sqrtf(S[c]);
    } else {
      const int64_t f = e - nu;
      const int c = static_cast<int>(f / K);
      const int64_t k = f - static_cast<int64_t>(c) * K;
      const float v = wide ? U[k + static_cast<int64_t>(c) * K] : VT[c + k * K];
      Vr[f] = sqrtf(S[c]) * v;
    }
  }
}

// Rp = W - Ur Vr (fp32, the r products summed in order c = 0 .. r-1): 64 x 64 output tiles with the
// two factor tiles in shared memory, 16 outputs per thread.
constexpr int kLrTile = 64;

__global__ void __launch_bounds__(256) lowrank_sub_kernel(const float* __restrict__ W, const float* __restrict__ Ur,
                                                          const float* __restrict__ Vr, int64_t N, int64_t K, int r,
                                                          float* __restrict__ Rp) {
  __shared__ float su[kLrTile][65];   // [row][c], r <= 64
  __shared__ float sv[64][kLrTile];   // [c][col]
  const int64_t i0 = static_cast<int64_t>(blockIdx.y) * kLrTile, k0 = static_cast<int64_t>(blockIdx.x) * kLrTile;
  for (int e = threadIdx.x; e < kLrTile * r; e += blockDim.x) {
    const int row = e / r, c = e - row * r;
    su[row][c] = (i0 + row < N) ? Ur[(i0 + row) * r + c] : 0.f;
  }
  for (int e = threadIdx.x; e < r * kLrTile; e += blockDim.x) {
    const int c = e / kLrTile, col = e - c * kLrTile;
    sv[c][col] = (k0 + col < K) ? Vr[static_cast<int64_t>(c) * K + k0 + col] : 0.f;
  }
  __syncthreads();
  const int col = threadIdx.x & 63, rq = threadIdx.x >> 6;  // 4 row groups of 16 rows
#pragma unroll 4
  for (int rr = 0; rr < 16; ++rr) {
    const int row = rq * 16 + rr;
    const int64_t i = i0 + row, k = k0 + col;
    if (i < N && k < K) {
      float acc = 0.f;
      for (int c = 0; c < r; ++c) acc = fmaf(su[row][c], sv[c][col], acc);
      Rp[i * K + k] = __fsub_rn(W[i * K + k], acc);
    }
  }
}

// A = bf16(Vr) [r, K], B = bf16(Ur / s) [N, r]
__global__ void adapter_out_kernel(const float* __restrict__ Ur, const float* __restrict__ Vr, int64_t N, int64_t K,
                                   int r, float s, uint16_t* __restrict__ A, uint16_t* __restrict__ B) {
  const int64_t na = static_cast<int64_t>(r) * K, total = na + N * r;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    if (e < na)
      A[e] = static_cast<uint16_t>(pack_bf16x2_rn(Vr[e], 0.f) & 0xFFFFu);
    else
      B[e - na] = static_cast<uint16_t>(pack_bf16x2_rn(__fdiv_rn(Ur[e - na], s), 0.f) & 0xFFFFu);
  }
}

unsigned grid_of(int64_t n) {
  const int64_t want = (n + 255) / 256, cap = static_cast<int64_t>(device_sm_count()) * 16;
  return static_cast<unsigned>(want < 1 ? 1 : (want > cap ? cap : want));
}

inline size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

struct LqLayout {
  size_t R, T, S, U, VT, Ur, Vr, rwork, info, work, total;
};

LqLayout lq_layout(int64_t N, int64_t K, int r, int lwork) {
  const int64_t m = N > K ? N : K, n = N > K ? K : N;
  LqLayout L;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += al256(bytes);
    return at;
  };
  L.R = take(static_cast<size_t>(N) * K * 4);
  L.T = take(N > K ? static_cast<size_t>(N) * K * 4 : 0);
  L.S = take(static_cast<size_t>(n) * 4);
  L.U = take(static_cast<size_t>(m) * n * 4);
  L.VT = take(static_cast<size_t>(n) * n * 4);
  L.Ur = take(static_cast<size_t>(N) * r * 4);
  L.Vr = take(static_cast<size_t>(r) * K * 4);
  L.rwork = take(static_cast<size_t>(n) * 4);
  L.info = take(4);
  L.work = take(static_cast<size_t>(lwork) * 4);
  L.total = off;
  return L;
}

// One solver handle per device, created on the first call made while that device is current and kept for
// the life of the process (the handle's own small device allocation happens once, not per call).
cusolverDnHandle_t device_handle() {
  static std::mutex mu;
  static cusolverDnHandle_t handles[64] = {nullptr};
  const Solver& sv = solver();
  if (!sv.ok) return nullptr;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!handles[dev] && sv.create(&handles[dev]) != CUSOLVER_STATUS_SUCCESS) handles[dev] = nullptr;
  return handles[dev];
}

int gesvd_lwork(int64_t N, int64_t K, int* lwork) {
  const Solver& sv = solver();
  if (!sv.ok) return QLR_ERR_UNSUPPORTED;
  cusolverDnHandle_t h = device_handle();
  if (!h) return QLR_ERR_CUDA;
  const int m = static_cast<int>(N > K ? N : K), n = static_cast<int>(N > K ? K : N);
  return sv.buffer_size(h, m, n, lwork) == CUSOLVER_STATUS_SUCCESS ? QLR_OK : QLR_ERR_CUDA;
}

int check_lq_args(int64_t N, int64_t K, int bits, int block, int dq_block, int r, int iters) {
  if (N <= 0 || K <= 0 || bits < 2 || bits > 4 || (block != 64 && block != 128) || (dq_block != 0 && dq_block != 256))
    return QLR_ERR_ARG;
  if (r < 1 || r > 64 || r > N || r > K || iters < 0 || iters > 64) return QLR_ERR_ARG;
  if ((N * K) % 128 || N > (1 << 20) || K > (1 << 20)) return QLR_ERR_SHAPE;
  return QLR_OK;
}

}  // namespace

}  // namespace qlr

using namespace qlr;

extern "C" size_t qlr_lqlora_init_workspace_bytes(int64_t N, int64_t K, int r) {
  if (N <= 0 || K <= 0 || r < 1 || r > 64) return 0;
  int lwork = 0;
  if (gesvd_lwork(N, K, &lwork) != QLR_OK) return 0;
  return lq_layout(N, K, r, lwork).total;
}

extern "C" int qlr_lqlora_init(const float* W, int64_t N, int64_t K, int bits, int block, int dq_block, int r, float s,
                               int iters, qlr_qweight* out, uint16_t* A, uint16_t* B, void* workspace,
                               size_t workspace_bytes, int32_t* status, void* stream) {
  int rc = check_lq_args(N, K, bits, block, dq_block, r, iters);
  if (rc) return rc;
  if (!W || !out || !A || !B || !(s > 0.f)) return QLR_ERR_ARG;
  if (out->fmt != QLR_FMT_NFK || out->bits != bits || out->block != block || out->dq_block != dq_block ||
      out->N != N || out->K != K || !out->codes || (dq_block ? (!out->c1_fp8 || !out->s2) : !out->c1))
    return QLR_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(W) | reinterpret_cast<uintptr_t>(A) | reinterpret_cast<uintptr_t>(B)) & 15u)
    return QLR_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t* stat = status_or_sink(status);
  if (iters == 0) {  // plain quantisation, zero adapter
    if (cudaMemsetAsync(A, 0, static_cast<size_t>(r) * K * 2, st) != cudaSuccess ||
        cudaMemsetAsync(B, 0, static_cast<size_t>(N) * r * 2, st) != cudaSuccess)
      return QLR_ERR_CUDA;
    return launch_quantize_nfk(W, N * K, bits, block, dq_block, out, stat, st) == cudaSuccess ? QLR_OK : QLR_ERR_CUDA;
  }
  const Solver& sv = solver();
  if (!sv.ok) return QLR_ERR_UNSUPPORTED;
  int lwork = 0;
  if ((rc = gesvd_lwork(N, K, &lwork))) return rc;
  const LqLayout L = lq_layout(N, K, r, lwork);
  if (!workspace || workspace_bytes < L.total) return QLR_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return QLR_ERR_ALIGN;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* R = reinterpret_cast<float*>(ws + L.R);
  float* T = reinterpret_cast<float*>(ws + L.T);
  float* S = reinterpret_cast<float*>(ws + L.S);
  float* U = reinterpret_cast<float*>(ws + L.U);
  float* VT = reinterpret_cast<float*>(ws + L.VT);
  float* Ur = reinterpret_cast<float*>(ws + L.Ur);
  float* Vr = reinterpret_cast<float*>(ws + L.Vr);
  float* rwork = reinterpret_cast<float*>(ws + L.rwork);
  int* info = reinterpret_cast<int*>(ws + L.info);
  float* work = reinterpret_cast<float*>(ws + L.work);
  const bool wide = K >= N;
  const int m = static_cast<int>(wide ? K : N), n = static_cast<int>(wide ? N : K);

  cusolverDnHandle_t h = device_handle();
  if (!h) return QLR_ERR_CUDA;
  rc = QLR_OK;
  for (int t = 0; t < iters && rc == QLR_OK; ++t) {
    // the residual to factor: W (t = 0), else W - dequant(Q_t)
    if (t == 0) {
      if (cudaMemcpyAsync(R, W, static_cast<size_t>(N) * K * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess) {
        rc = QLR_ERR_CUDA;
        break;
      }
    } else {
      count_launch();
      residual_kernel<<<grid_of(N * K), 256, 0, st>>>(W, N * K, nfk::view_of(out), R);
    }
    // column-major operand with at least as many rows as columns
    float* Acm = R;  // row-major N x K read as column-major K x N (ld K)
    if (!wide) {
      count_launch();
      transpose_kernel<<<dim3(static_cast<unsigned>((K + 31) / 32), static_cast<unsigned>((N + 31) / 32)), dim3(32, 8), 0,
                         st>>>(R, N, K, T);
      Acm = T;  // column-major N x K (ld N)
    }
    if (sv.set_stream(h, st) != CUSOLVER_STATUS_SUCCESS ||
        sv.gesvd(h, 'S', 'S', m, n, Acm, m, S, U, m, VT, n, work, lwork, rwork, info) != CUSOLVER_STATUS_SUCCESS) {
      rc = QLR_ERR_CUDA;
      break;
    }
    int hinfo = 0;
    if (cudaMemcpyAsync(&hinfo, info, 4, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess || hinfo != 0) {
      rc = QLR_ERR_CUDA;
      break;
    }
    count_launch(2);
    factors_kernel<<<grid_of(N * r + static_cast<int64_t>(r) * K), 256, 0, st>>>(U, VT, S, N, K, r, wide ? 1 : 0, Ur, Vr);
    lowrank_sub_kernel<<<dim3(static_cast<unsigned>((K + kLrTile - 1) / kLrTile),
                              static_cast<unsigned>((N + kLrTile - 1) / kLrTile)),
                         256, 0, st>>>(W, Ur, Vr, N, K, r, R);
    if (launch_quantize_nfk(R, N * K, bits, block, dq_block, out, stat, st) != cudaSuccess) rc = QLR_ERR_CUDA;
  }
  if (rc == QLR_OK) {
    count_launch();
    adapter_out_kernel<<<grid_of(static_cast<int64_t>(r) * K + N * r), 256, 0, st>>>(Ur, Vr, N, K, r, s, A, B);
    if (cudaGetLastError() != cudaSuccess || cudaStreamSynchronize(st) != cudaSuccess) rc = QLR_ERR_CUDA;
  }
  cudaStreamSynchronize(st);
  return rc;
}
