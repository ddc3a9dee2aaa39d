// SwiGLU of the MLP block (the LLaMA-7B-shaped workload): H = silu(G) * U, and its backward
//   dG = dH U sig(G) (1 + G (1 - sig(G))),   dU = dH silu(G).
// One definition serves the standalone kernels and the GEMM epilogues that fuse them, so both give the same
// bits: fp32 arithmetic with every multiplication and addition rounded on its own (no contraction into FMAs),
// and the sigmoid from the hardware exponential and a fast reciprocal, which keeps the epilogue's extra work
// per output small (the results are bf16; the approximations' few-ulp fp32 errors are far below that).
#pragma once
#include <cuda_runtime.h>

namespace qlr {

__device__ __forceinline__ float swiglu_sigmoid(float g) { return __fdividef(1.0f, __fadd_rn(1.0f, __expf(-g))); }

__device__ __forceinline__ float swiglu_h(float g, float u) {
  return __fmul_rn(__fmul_rn(g, swiglu_sigmoid(g)), u);
}

__device__ __forceinline__ void swiglu_grads(float dh, float g, float u, float& dg, float& du) {
  const float sg = swiglu_sigmoid(g);
  const float t = __fadd_rn(1.0f, __fmul_rn(g, __fsub_rn(1.0f, sg)));
  dg = __fmul_rn(__fmul_rn(__fmul_rn(dh, u), sg), t);
  du = __fmul_rn(__fmul_rn(dh, g), sg);
}

}  // namespace qlr
