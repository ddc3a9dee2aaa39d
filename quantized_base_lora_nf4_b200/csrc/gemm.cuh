// Host-side description of one tcgen05 GEMM launch (see gemm.cu).
#pragma once
#include <cuda.h>
#include <cuda_fp16.h>

#include "common.cuh"

namespace qlr {

// How the MMA "A" operand (the 128 TMEM-lane side) reaches shared memory.
enum ASrc : int {
  A_TMA_K = 0,   // TMA tile of a [Mm, Kred] row-major matrix (K-major)
  A_TMA_MN = 1,  // TMA tiles of a [Kred, Mm] row-major matrix (MN-major)
  A_DQ_K = 2,    // dequantised from packed codes of W [Mm = N, Kred = K] (forward)
  A_DQ_MN = 3    // dequantised from packed codes of W [Kred = N, Mm = K] (input gradient)
};
enum BSrc : int { B_TMA_K = 0, B_TMA_MN = 1 };
enum OutMode : int { OUT_BF16_T = 0, OUT_F32_D = 1 };
enum EpiMode : int { EPI_STORE = 0, EPI_SWIGLU_FWD = 1, EPI_SWIGLU_BWD = 2 };

struct DqParams {
  int fmt, bits, block, dq_block, group;
  int64_t N, K;
  // index arithmetic without division: blocks (NF) or groups (INT4) per row, and log2 of the
  // block, group and double-quantisation sizes (all powers of two)
  int64_t units_per_row;
  int unit_shift, dq_shift;
  const float* c1;
  const uint8_t* c1_fp8;
  const float* s2;
  const __half* scale;
  const __half* zero;
  Levels lv;
};

// The fused kernel's codes ring: kCodeRingBytes of shared memory that the host splits into a power-of-two
// number of slots of one TMA box each, at most kCodeRingSlots (the kernel initialises one full/empty
// barrier pair per possible slot).
constexpr int kCodeRingBytes = 32768;
constexpr int kCodeRingSlots = 8;
constexpr int kCodeRingSlotsLog2 = 3;
static_assert((1 << kCodeRingSlotsLog2) == kCodeRingSlots, "slot count is a power of two");

// D[Mm, Nn] = sum_k A[Mm, k] B[k, Nn]  (+ a tail segment of extra reduction columns)
struct GemmParams {
  int Mm, Nn;            // extents of D (MMA M side = TMEM lanes, MMA N side = TMEM columns)
  int n_main;            // 64-wide reduction steps of the main segment (all splits)
  int splits;            // split-K factor of the main segment (partials go to out[split])
  int n_tail;            // 64-wide reduction steps of the tail (only with splits == 1)
  int r_tail;            // reduction extent of the tail (its last step may be partial)
  int m_tiles, n_tiles;
  // fused kernels' work items: n_items in all; with token pairs, tiles from full_items on are split into
  // two items of one half each (n_items = full_items + 2 (m_tiles n_tiles - full_items))
  int n_items, full_items;
  int b_atom;            // MN-major B: elements per swizzle atom row (16, 32 or 64)
  void* out;             // OUT_BF16_T: bf16 [Nn, ldo] receiving D^T; OUT_F32_D: fp32 [splits][m_tiles*128][ldo]
  int64_t ldo;
  int accumulate;        // OUT_BF16_T: add the previous contents of out
  // epilogue: EPI_STORE writes D^T to out; EPI_SWIGLU_FWD writes it (U) to out and H = silu(G) U to aux_out
  // (G read from aux_g); EPI_SWIGLU_BWD treats it as dH (never stored) and writes dG to out, dU to aux_out
  // (G, U read from aux_g, aux_u).  Every auxiliary tensor has the layout of out.
  int epi;
  const uint16_t* aux_g;
  const uint16_t* aux_u;
  uint16_t* aux_out;
  DqParams dq;
  // codes ring of the fused kernel: one TMA box per slot covering code_steps main steps (2 for 3-bit
  // codes along K, whose 24-byte runs are not a legal box width), 2^code_slots_log2 slots of
  // code_box_bytes
  int code_bits, code_steps, code_slots_log2, code_box_bytes;
  // fused kernels: the tail's weight-side operand, copied into the A tile by the dequantiser warps
  // (forward: B [N, r], row-major; input gradient: A or its group expansion [r, K], row-major)
  const uint16_t* tail_a;
  int64_t tail_a_rows, tail_a_cols;
  int tail_pool_L;       // input gradient with the pooled adapter: tail row j is A[j, k / L] / L
  int32_t* status;
  long long wait_cycles; // bound of every pipeline wait (SM clock cycles)
};

struct GemmMaps {
  CUtensorMap a, b, a_tail, b_tail, codes;
};

// One adapter GEMM D[Mm, r] = sum_k A[Mm, k] B[k, r] (r <= 64).  The reduction may be split into
// `splits` parts for occupancy; each part's fp32 tile then goes to `part` and a reduction kernel
// sums the parts in split order.  The result is written as:
//   ADAPTER_ROWS_BF16   out[m, j] = bf16(scale * D[m, j])     (T_save, dT; ld_out = r)
//   ADAPTER_ROWS_F32    out[m, j] = D[m, j]                   (dB; ld_out = r)
//   ADAPTER_COLS_F32    out[j, m / L] = sum over m in a group of L of D[m, j] / L   (dA; ld_out = Ka)
enum AdapterOut : int { ADAPTER_ROWS_BF16 = 0, ADAPTER_ROWS_F32 = 1, ADAPTER_COLS_F32 = 2 };

struct AdapterParams {
  int Mm, r;
  int n_steps;   // 64-wide reduction steps
  int splits;
  int m_tiles;
  int b_atom;    // MN-major B: elements per swizzle atom row (32 or 64)
  int out_mode;
  float scale;
  int pool_L;    // ADAPTER_COLS_F32: group length (1 = none)
  void* out;
  int64_t ld_out;
  float* part;       // [splits][m_tiles * 128][BN] fp32 (splits > 1)
  int32_t* status;
  long long wait_cycles;  // bound of every pipeline wait (SM clock cycles)
};

cudaError_t launch_adapter(int a_src, int b_src, int bn, const AdapterParams& p, const GemmMaps& maps,
                           cudaStream_t st);
// Sums the split parts of an adapter GEMM in split order and applies its output transform.
cudaError_t launch_adapter_reduce(const AdapterParams& p, int bn, cudaStream_t st);

// Launches the fused dequant + tcgen05 kernel (a_src = A_DQ_K forward, A_DQ_MN input gradient).
cudaError_t launch_fused(int a_src, int bn, const GemmParams& p, const GemmMaps& maps, cudaStream_t st);

// Launches the engine variant for (a_src, b_src, BN, out, tail_a_mn).
cudaError_t launch_gemm(int a_src, int b_src, int bn, int out_mode, int tail_a_mn, const GemmParams& p,
                        const GemmMaps& maps, cudaStream_t st);

// Tensor-map helper: 2-D row-major [rows, cols] of elem_bytes elements, box [box_rows, box_cols].
int make_tmap(CUtensorMap* m, const void* base, int elem_bytes, uint64_t rows, uint64_t cols, uint32_t box_rows,
              uint32_t box_cols, int swizzle_bytes);

}  // namespace qlr
