// LQ-LoRA initialisation (LQ-LoRA abstract: an iterative method splits each pretrained matrix into a
// low-rank part kept in high precision plus a quantised part that is cheap to store; the
// quantised part stays frozen and the low-rank part is the trainable adapter).  Read as the
// alternation
//     Q_0 = 0;  for t = 1..T:  L_t = rank-r truncated SVD of (W - dequant(Q_{t-1})),
//                              Q_t = NF-k quantisation of (W - L_t)
// with the adapter A = bf16(sqrt(S_r) V_r^T), B = bf16(U_r sqrt(S_r) / s), so s B A = L_T.
//
// The rank-r truncated SVD of the residual R [N, K] comes from the r largest eigenpairs of its Gram
// matrix on the smaller side: with n = min(N, K), G = R^T R (K <= N) or R R^T (N < K), G = V S^2 V^T,
// so the top-r right (or left) singular vectors are G's top-r eigenvectors and the other factor is
// R V_r / S_r (or R^T U_r / S_r).  Only r of the n eigenpairs are computed, instead of a full SVD of R.
// G and the projection are plain single-precision library GEMMs (cuBLAS), the eigenpairs a library
// eigensolver (cuSOLVER syevdx, index range n - r + 1 .. n); both are loaded with dlopen on first use, so
// the library itself has no link-time dependency on them.  Residuals, the rank-r subtraction, the factor
// split and the quantisation run in this library's kernels.  An offline, once-per-weight step.
#include <cuda_fp8.h>
#include <cublas_v2.h>
#include <cusolverDn.h>
#include <dlfcn.h>

#include <mutex>

#include "common.cuh"
#include "nfk.cuh"
#include "ptx.cuh"

namespace qlr {

namespace {

// ---- cuSOLVER and cuBLAS, resolved at run time --------------------------------------------------
struct Solver {
  decltype(&cusolverDnCreate) create = nullptr;
  decltype(&cusolverDnSetStream) set_stream = nullptr;
  decltype(&cusolverDnSsyevdx_bufferSize) evd_buffer = nullptr;
  decltype(&cusolverDnSsyevdx) evd = nullptr;
  decltype(&cublasCreate_v2) blas_create = nullptr;
  decltype(&cublasSetStream_v2) blas_set_stream = nullptr;
  decltype(&cublasSsyrk_v2) syrk = nullptr;
  decltype(&cublasSgemm_v2) gemm = nullptr;
  bool ok = false;
};

const Solver& solver() {
  static Solver s;
  static std::once_flag once;
  std::call_once(once, [] {
    void* h = dlopen("libcusolver.so.11", RTLD_NOW | RTLD_LOCAL);
    if (!h) h = dlopen("libcusolver.so", RTLD_NOW | RTLD_LOCAL);
    void* b = dlopen("libcublas.so.12", RTLD_NOW | RTLD_LOCAL);
    if (!b) b = dlopen("libcublas.so", RTLD_NOW | RTLD_LOCAL);
    if (!h || !b) return;
    s.create = reinterpret_cast<decltype(s.create)>(dlsym(h, "cusolverDnCreate"));
    s.set_stream = reinterpret_cast<decltype(s.set_stream)>(dlsym(h, "cusolverDnSetStream"));
    s.evd_buffer = reinterpret_cast<decltype(s.evd_buffer)>(dlsym(h, "cusolverDnSsyevdx_bufferSize"));
    s.evd = reinterpret_cast<decltype(s.evd)>(dlsym(h, "cusolverDnSsyevdx"));
    s.blas_create = reinterpret_cast<decltype(s.blas_create)>(dlsym(b, "cublasCreate_v2"));
    s.blas_set_stream = reinterpret_cast<decltype(s.blas_set_stream)>(dlsym(b, "cublasSetStream_v2"));
    s.syrk = reinterpret_cast<decltype(s.syrk)>(dlsym(b, "cublasSsyrk_v2"));
    s.gemm = reinterpret_cast<decltype(s.gemm)>(dlsym(b, "cublasSgemm_v2"));
    s.ok = s.create && s.set_stream && s.evd_buffer && s.evd && s.blas_create && s.blas_set_stream && s.syrk && s.gemm;
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

// The rank-r factors from the Gram matrix's top eigenpairs, split as Ur = U_r sqrt(S_r) [N, r] and
// Vr = sqrt(S_r) V_r^T [r, K], both row-major, components in descending order.  E holds the eigenvectors
// (column-major, leading dimension n, ascending eigenvalues lam[0 .. r-1]); P the projection of R onto
// them (column-major): tall (K <= N, n = K): E = V_r, P = R V_r = U_r S_r [N x r, ld N];
// wide (N < K, n = N): E = U_r, P = R^T U_r = V_r S_r [K x r, ld K].  s_c = sqrt(lam_c).
__global__ void gram_factors_kernel(const float* __restrict__ E, const float* __restrict__ lam,
                                    const float* __restrict__ P, int64_t N, int64_t K, int r, int tall,
                                    float* __restrict__ Ur, float* __restrict__ Vr) {
  const int64_t nu = N * r, total = nu + static_cast<int64_t>(r) * K;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    int c_out;
    int64_t pos;  // row i of Ur, or column k of Vr
    if (e < nu) {
      pos = e / r;
      c_out = static_cast<int>(e - pos * r);
    } else {
      const int64_t f = e - nu;
      c_out = static_cast<int>(f / K);
      pos = f - static_cast<int64_t>(c_out) * K;
    }
    const int c = r - 1 - c_out;                       // the eigensolver's ascending order
    const float sq = sqrtf(sqrtf(fmaxf(lam[c], 0.f)));  // sqrt(s_c)
    const float inv = sq > 0.f ? 1.0f / sq : 0.f;
    float v;
    if (e < nu)  // Ur[i][c_out]
      v = tall ? P[pos + static_cast<int64_t>(c) * N] * inv : E[pos + static_cast<int64_t>(c) * N] * sq;
    else         // Vr[c_out][k]
      v = tall ? E[pos + static_cast<int64_t>(c) * K] * sq : P[pos + static_cast<int64_t>(c) * K] * inv;
    (e < nu ? Ur : Vr)[e < nu ? e : e - nu] = v;
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
  size_t R, G, lam, P, Ur, Vr, info, work, total;
};

LqLayout lq_layout(int64_t N, int64_t K, int r, int lwork) {
  const int64_t n = N < K ? N : K, m = N < K ? K : N;
  LqLayout L;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += al256(bytes);
    return at;
  };
  L.R = take(static_cast<size_t>(N) * K * 4);
  L.G = take(static_cast<size_t>(n) * n * 4);
  L.lam = take(static_cast<size_t>(n) * 4);
  L.P = take(static_cast<size_t>(m) * r * 4);
  L.Ur = take(static_cast<size_t>(N) * r * 4);
  L.Vr = take(static_cast<size_t>(r) * K * 4);
  L.info = take(4);
  L.work = take(static_cast<size_t>(lwork) * 4);
  L.total = off;
  return L;
}

// One solver and one BLAS handle per device, created on the first call made while that device is current
// and kept for the life of the process (their own small device allocations happen once, not per call).
struct Handles {
  cusolverDnHandle_t sol = nullptr;
  cublasHandle_t blas = nullptr;
};

const Handles* device_handles() {
  static std::mutex mu;
  static Handles hs[64];
  const Solver& sv = solver();
  if (!sv.ok) return nullptr;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  Handles& h = hs[dev];
  if (!h.sol && sv.create(&h.sol) != CUSOLVER_STATUS_SUCCESS) h.sol = nullptr;
  if (!h.blas && sv.blas_create(&h.blas) != CUBLAS_STATUS_SUCCESS) h.blas = nullptr;
  return (h.sol && h.blas) ? &h : nullptr;
}

int evd_lwork(int64_t N, int64_t K, int r, int* lwork) {
  const Solver& sv = solver();
  if (!sv.ok) return QLR_ERR_UNSUPPORTED;
  const Handles* h = device_handles();
  if (!h) return QLR_ERR_CUDA;
  const int n = static_cast<int>(N < K ? N : K);
  int meig = 0;
  return sv.evd_buffer(h->sol, CUSOLVER_EIG_MODE_VECTOR, CUSOLVER_EIG_RANGE_I, CUBLAS_FILL_MODE_LOWER, n, nullptr, n, 0.f,
                       0.f, n - r + 1, n, &meig, nullptr, lwork) == CUSOLVER_STATUS_SUCCESS
             ? QLR_OK
             : QLR_ERR_CUDA;
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
  if (evd_lwork(N, K, r, &lwork) != QLR_OK) return 0;
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
  if ((rc = evd_lwork(N, K, r, &lwork))) return rc;
  const LqLayout L = lq_layout(N, K, r, lwork);
  if (!workspace || workspace_bytes < L.total) return QLR_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return QLR_ERR_ALIGN;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* R = reinterpret_cast<float*>(ws + L.R);
  float* G = reinterpret_cast<float*>(ws + L.G);
  float* lam = reinterpret_cast<float*>(ws + L.lam);
  float* P = reinterpret_cast<float*>(ws + L.P);
  float* Ur = reinterpret_cast<float*>(ws + L.Ur);
  float* Vr = reinterpret_cast<float*>(ws + L.Vr);
  int* info = reinterpret_cast<int*>(ws + L.info);
  float* work = reinterpret_cast<float*>(ws + L.work);
  // R row-major [N, K] is, column-major, Rc = R^T [K x N] with leading dimension K
  const bool tall = K <= N;
  const int n = static_cast<int>(tall ? K : N), Ni = static_cast<int>(N), Ki = static_cast<int>(K);
  const float one = 1.f, zero = 0.f;

  const Handles* h = device_handles();
  if (!h) return QLR_ERR_CUDA;
  if (sv.set_stream(h->sol, st) != CUSOLVER_STATUS_SUCCESS || sv.blas_set_stream(h->blas, st) != CUBLAS_STATUS_SUCCESS)
    return QLR_ERR_CUDA;
  rc = QLR_OK;
  for (int t = 0; t < iters && rc == QLR_OK; ++t) {
    // the residual to factor: W (t = 0), else W - dequant(Q_t)
    const float* Rt = W;
    if (t > 0) {
      count_launch();
      residual_kernel<<<grid_of(N * K), 256, 0, st>>>(W, N * K, nfk::view_of(out), R);
      Rt = R;
    }
    // Gram matrix on the smaller side (lower triangle): tall G = Rc Rc^T = R^T R [K x K];
    // wide G = Rc^T Rc = R R^T [N x N]
    if (sv.syrk(h->blas, CUBLAS_FILL_MODE_LOWER, tall ? CUBLAS_OP_N : CUBLAS_OP_T, n, tall ? Ni : Ki, &one, Rt, Ki,
                &zero, G, n) != CUBLAS_STATUS_SUCCESS) {
      rc = QLR_ERR_CUDA;
      break;
    }
    // its r largest eigenpairs (ascending; eigenvectors in G's first r columns)
    int meig = 0;
    if (sv.evd(h->sol, CUSOLVER_EIG_MODE_VECTOR, CUSOLVER_EIG_RANGE_I, CUBLAS_FILL_MODE_LOWER, n, G, n, 0.f, 0.f,
               n - r + 1, n, &meig, lam, work, lwork, info) != CUSOLVER_STATUS_SUCCESS ||
        meig != r) {
      rc = QLR_ERR_CUDA;
      break;
    }
    // the other side's factor: tall P = R V_r = Rc^T E [N x r]; wide P = R^T U_r = Rc E [K x r]
    if (sv.gemm(h->blas, tall ? CUBLAS_OP_T : CUBLAS_OP_N, CUBLAS_OP_N, tall ? Ni : Ki, r, n, &one, Rt, Ki, G, n, &zero,
                P, tall ? Ni : Ki) != CUBLAS_STATUS_SUCCESS) {
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
    gram_factors_kernel<<<grid_of(N * r + static_cast<int64_t>(r) * K), 256, 0, st>>>(G, lam, P, N, K, r, tall ? 1 : 0,
                                                                                         Ur, Vr);
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
