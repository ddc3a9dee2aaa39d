// Self-test of the bounded-wait path shared by the pipelined kernels (fused GEMM, adapter GEMM, decode).
//
// One CTA takes tensor memory as those kernels do, initialises an mbarrier that no thread and no copy will
// ever complete, and waits on it with the current wait bound.  The wait must run out, raise the abort flag,
// and the CTA must then release its tensor memory and report QLR_ERR_TIMEOUT through the status word, so
// the context stays usable: the next kernel that allocates tensor memory on the same SM gets it.
#include "common.cuh"
#include "ptx.cuh"

namespace qlr {

namespace {

struct alignas(8) SelfTestSmem {
  uint64_t never_completed;
  uint32_t tmem_base;
  int abort_flag;
};

__global__ void __launch_bounds__(64, 1) wait_selftest_kernel(long long limit, int32_t* status) {
  __shared__ SelfTestSmem s;
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(&s.never_completed, 1);  // one arrival expected; none is ever made
    s.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&s.tmem_base, 32);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    // every lane of the waiting warp gives up on its own bound (or on the flag another lane raised)
    mbar_wait(&s.never_completed, 0, &s.abort_flag, limit);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(s.tmem_base, 32);
  }
  if (threadIdx.x == 0) report(status, s.abort_flag ? QLR_ERR_TIMEOUT : QLR_OK);
}

}  // namespace

}  // namespace qlr

extern "C" int qlr_wait_selftest(int32_t* status, void* stream) {
  if (!status) return QLR_ERR_ARG;
  qlr::count_launch();
  qlr::wait_selftest_kernel<<<1, 64, 0, static_cast<cudaStream_t>(stream)>>>(qlr::wait_limit_cycles(), status);
  return cudaGetLastError() == cudaSuccess ? QLR_OK : QLR_ERR_CUDA;
}
