// C-ABI entry points: argument validation (before any launch), workspace carving, tensor maps,
// and the launch sequence of each call.  See include/qlr.h for the contract of every function.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>

#include "common.cuh"
#include "gemm.cuh"

namespace qlr {

constexpr long long kDefaultWaitCycles = 4000000000LL;  // ~2 s at the B200 boost clock

__device__ int32_t g_status_sink;

static std::atomic<uint64_t> g_launches{0};
static std::atomic<long long> g_wait_cycles{kDefaultWaitCycles};
long long wait_limit_cycles() { return g_wait_cycles.load(std::memory_order_relaxed); }
void count_launch(int n) { g_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed); }

int32_t* status_or_sink(int32_t* status) {
  if (status) return status;
  static int32_t* sink = nullptr;
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  int dev = 0;
  cudaGetDevice(&dev);
  static int32_t* per_dev[64] = {nullptr};
  if (dev >= 0 && dev < 64 && !per_dev[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_sink) == cudaSuccess) per_dev[dev] = static_cast<int32_t*>(p);
  }
  sink = (dev >= 0 && dev < 64) ? per_dev[dev] : nullptr;
  return sink;
}

Levels levels_for(int bits) {
  Levels l;
  for (int i = 0; i < 16; ++i) l.v[i] = 0.f;
  if (bits >= 2 && bits <= 4) nf_levels_f32(bits, l.v);
  return l;
}

cudaError_t ensure_max_dynamic_smem_fn(const void* kern, int bytes) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int> done;  // (kernel, device) -> limit set
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  auto it = done.find({kern, dev});
  if (it != done.end() && it->second >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done[{kern, dev}] = bytes;
  return e;
}

int device_sm_count() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cache[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

}  // namespace qlr

using namespace qlr;

namespace {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }
inline int cuda_rc(cudaError_t e) { return e == cudaSuccess ? QLR_OK : QLR_ERR_CUDA; }
inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int check_qweight(const qlr_qweight* w) {
  if (!w || w->N <= 0 || w->K <= 0 || !w->codes) return QLR_ERR_ARG;
  if (!aligned16(w->codes)) return QLR_ERR_ALIGN;
  if (w->fmt == QLR_FMT_NFK) {
    if (w->bits < 2 || w->bits > 4) return QLR_ERR_ARG;
    if (w->block != 64 && w->block != 128) return QLR_ERR_ARG;
    if (w->dq_block != 0 && w->dq_block != 256) return QLR_ERR_ARG;
    if (w->dq_block ? (!w->c1_fp8 || !w->s2) : !w->c1) return QLR_ERR_ARG;
    if ((w->N * w->K) % 128) return QLR_ERR_SHAPE;
    return QLR_OK;
  }
  if (w->fmt == QLR_FMT_INT4G) {
    if (w->group != 32 && w->group != 64 && w->group != 128) return QLR_ERR_ARG;
    if (!w->scale || !w->zero) return QLR_ERR_ARG;
    if (w->K % w->group) return QLR_ERR_SHAPE;
    return QLR_OK;
  }
  return QLR_ERR_ARG;
}

// Shapes the fused tensor-core paths support.
int check_gemm_weight(const qlr_qweight* w) {
  int rc = check_qweight(w);
  if (rc) return rc;
  if (w->K % 64 || w->N % 8) return QLR_ERR_SHAPE;
  // 3-bit codes are loaded two 64-code steps per box along K (a 24-byte box width is not legal)
  if (w->fmt == QLR_FMT_NFK && w->bits == 3 && w->K % 128) return QLR_ERR_SHAPE;
  if (w->fmt == QLR_FMT_NFK && w->K % w->block) return QLR_ERR_SHAPE;
  if (w->N > (int64_t(1) << 30) || w->K > (int64_t(1) << 30)) return QLR_ERR_SHAPE;
  return QLR_OK;
}

// Width of the packed codes: NF-k codes are k bits, INT4 group codes 4.
int code_bits(const qlr_qweight* w) { return w->fmt == QLR_FMT_NFK ? w->bits : 4; }

// The fused kernel's codes ring (kCodeRingBytes) split into a power-of-two number, at most kCodeRingSlots,
// of slots of one TMA box each, so the kernel indexes it with masks and shifts.
void set_code_ring(GemmParams& p, int bits, int steps_per_box, int box_bytes) {
  p.code_bits = bits;
  p.code_steps = steps_per_box;
  p.code_box_bytes = box_bytes;
  int lg = kCodeRingSlotsLog2;
  while (lg > 0 && (box_bytes << lg) > kCodeRingBytes) --lg;
  p.code_slots_log2 = lg;
}

int check_rank(int r) { return (r == 8 || r == 16 || r == 32 || r == 64) ? QLR_OK : QLR_ERR_SHAPE; }

int adapter_bn(int r) { return r <= 32 ? 32 : 64; }

DqParams dq_params(const qlr_qweight* w) {
  DqParams d;
  d.fmt = w->fmt;
  d.bits = w->bits;
  d.block = w->block;
  d.dq_block = w->dq_block;
  d.group = w->group;
  d.N = w->N;
  d.K = w->K;
  d.c1 = w->c1;
  d.c1_fp8 = w->c1_fp8;
  d.s2 = w->s2;
  d.scale = reinterpret_cast<const __half*>(w->scale);
  d.zero = reinterpret_cast<const __half*>(w->zero);
  d.lv = levels_for(w->fmt == QLR_FMT_NFK ? w->bits : 4);
  const int unit = w->fmt == QLR_FMT_NFK ? w->block : w->group;
  d.units_per_row = w->K / unit;
  d.unit_shift = 0;
  while ((1 << d.unit_shift) < unit) ++d.unit_shift;
  d.dq_shift = 0;
  while (w->dq_block && (1 << d.dq_shift) < w->dq_block) ++d.dq_shift;
  return d;
}

// Work items of a fused launch.  With token pairs (512-token tiles) and more tiles than SMs, a last wave
// that fills at most half the SMs is split into half tiles (256 tokens each): twice as many items, each half
// as long, so the launch ends after about 2.5 instead of 3 tile times for 344 tiles on 148 SMs.
void set_items(GemmParams& p, int tok) {
  const int tiles = p.m_tiles * p.n_tiles;
  const int sms = device_sm_count();
  p.full_items = tiles;
  p.n_items = tiles;
  if (tok == 512 && tiles > sms) {
    const int rem = tiles % sms;
    if (rem > 0 && 2 * rem <= sms) {
      p.full_items = tiles - rem;
      p.n_items = p.full_items + 2 * rem;
    }
  }
}

// Split of a rank-r adapter GEMM's reduction: minimises waves x (steps per split + a fixed cost of
// two steps per work item) over the SMs.
int pick_splits(int64_t tiles, int64_t n_steps) {
  const int64_t sms = device_sm_count();
  int best = 1;
  double best_cost = 1e30;
  for (int s = 1; s <= 32; ++s) {
    if (s > 1 && n_steps / s < 2) break;
    const double waves = static_cast<double>(cdiv(tiles * s, sms));
    const double cost = waves * (static_cast<double>(n_steps) / s + 2.0);
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best = s;
    }
  }
  return best;
}

size_t adapter_ws_bytes(int64_t Mm, int64_t n_red, int r) {
  const int64_t m_tiles = cdiv(Mm, 128);
  const int S = pick_splits(m_tiles, cdiv(n_red, 64));
  if (S == 1) return 0;
  return align256(size_t(S) * m_tiles * 128 * adapter_bn(r) * 4);
}

// One adapter GEMM: D[Mm, r] over n_red reduction elements, A and B from row-major matrices.
struct AdapterGemm {
  int a_src, b_src, bn;
  int64_t Mm, n_red;
  const void* a_ptr;
  int64_t a_rows, a_cols;  // row-major extents of the A source matrix
  const void* b_ptr;
  int64_t b_rows, b_cols;
};

int run_adapter(const AdapterGemm& g, int r, int out_mode, float scale, int pool_L, void* out, int64_t ld_out,
                uint8_t* ws, int32_t* status, cudaStream_t st) {
  GemmMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  int rc;
  if (g.a_src == A_TMA_K)
    rc = make_tmap(&maps.a, g.a_ptr, 2, g.a_rows, g.a_cols, 128, 64, 128);
  else
    rc = make_tmap(&maps.a, g.a_ptr, 2, g.a_rows, g.a_cols, 64, 64, 128);
  if (rc) return rc;
  const int atom = g.bn >= 64 ? 64 : g.bn;
  if (g.b_src == B_TMA_K)
    rc = make_tmap(&maps.b, g.b_ptr, 2, g.b_rows, g.b_cols, g.bn, 64, 128);
  else
    rc = make_tmap(&maps.b, g.b_ptr, 2, g.b_rows, g.b_cols, 64, atom, atom * 2);
  if (rc) return rc;
  maps.a_tail = maps.a;
  maps.b_tail = maps.b;
  maps.codes = maps.a;
  AdapterParams p;
  std::memset(&p, 0, sizeof(p));
  p.Mm = static_cast<int>(g.Mm);
  p.r = r;
  p.n_steps = static_cast<int>(cdiv(g.n_red, 64));
  p.m_tiles = static_cast<int>(cdiv(g.Mm, 128));
  p.splits = pick_splits(p.m_tiles, p.n_steps);
  p.b_atom = atom;
  p.out_mode = out_mode;
  p.scale = scale;
  p.pool_L = pool_L;
  p.out = out;
  p.ld_out = ld_out;
  p.status = status;
  p.wait_cycles = wait_limit_cycles();
  if (p.splits > 1) p.part = reinterpret_cast<float*>(ws);
  if ((rc = cuda_rc(launch_adapter(g.a_src, g.b_src, g.bn, p, maps, st)))) return rc;
  if (p.splits > 1) return cuda_rc(launch_adapter_reduce(p, g.bn, st));
  return QLR_OK;
}

}  // namespace

extern "C" {

const char* qlr_error_string(int code) {
  switch (code) {
    case QLR_OK: return "ok";
    case QLR_ERR_ARG: return "invalid argument";
    case QLR_ERR_SHAPE: return "unsupported shape";
    case QLR_ERR_ALIGN: return "pointer not 16-byte aligned";
    case QLR_ERR_UNSUPPORTED: return "unsupported combination";
    case QLR_ERR_NONFINITE: return "non-finite input";
    case QLR_ERR_TIMEOUT: return "pipeline wait timed out";
    case QLR_ERR_CUDA: return "CUDA error";
    case QLR_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown error";
  }
}

int qlr_version(void) { return 100; }

uint64_t qlr_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

long long qlr_set_wait_limit(long long cycles) {
  return g_wait_cycles.exchange(cycles < 0 ? kDefaultWaitCycles : cycles, std::memory_order_relaxed);
}

int qlr_device_sm_count(void) { return device_sm_count(); }

int qlr_nf_levels(int bits, float* out) {
  if (!out || bits < 2 || bits > 4) return QLR_ERR_ARG;
  nf_levels_f32(bits, out);
  return QLR_OK;
}

int qlr_nf_decision_table(int bits, float* threshold, int32_t* base) {
  if (!threshold || !base || bits < 2 || bits > 4) return QLR_ERR_ARG;
  NfTable tab;
  if (!nf_decision_table(bits, &tab)) return QLR_ERR_UNSUPPORTED;
  for (int k = 0; k < 33; ++k) {
    threshold[k] = tab.t[k];
    base[k] = tab.base[k];
  }
  return QLR_OK;
}

int64_t qlr_qweight_part_bytes(int fmt, int64_t N, int64_t K, int bits, int block, int dq_block, int group,
                               int part) {
  if (N <= 0 || K <= 0) return QLR_ERR_ARG;
  const int64_t n = N * K;
  if (fmt == QLR_FMT_NFK) {
    if (bits < 2 || bits > 4 || (block != 64 && block != 128) || (dq_block != 0 && dq_block != 256))
      return QLR_ERR_ARG;
    const int64_t nb = cdiv(n, block);
    switch (part) {
      case QLR_PART_CODES: return nb * block * bits / 8;
      case QLR_PART_C1: return dq_block ? 0 : 4 * nb;
      case QLR_PART_C1_FP8: return dq_block ? nb : 0;
      case QLR_PART_S2: return dq_block ? 4 * cdiv(nb, dq_block) : 0;
      case QLR_PART_SCALE:
      case QLR_PART_ZERO: return 0;
      default: return QLR_ERR_ARG;
    }
  }
  if (fmt == QLR_FMT_INT4G) {
    if (group <= 0 || K % group) return QLR_ERR_ARG;
    switch (part) {
      case QLR_PART_CODES: return n / 2;
      case QLR_PART_SCALE:
      case QLR_PART_ZERO: return 2 * N * (K / group);
      case QLR_PART_C1:
      case QLR_PART_C1_FP8:
      case QLR_PART_S2: return 0;
      default: return QLR_ERR_ARG;
    }
  }
  return QLR_ERR_ARG;
}

int qlr_quantize_nf4(const float* W, int64_t N, int64_t K, int bits, int block, int dq_block,
                     const qlr_qweight* out, int32_t* status, void* stream) {
  if (!W || !out) return QLR_ERR_ARG;
  if (out->fmt != QLR_FMT_NFK || out->bits != bits || out->block != block || out->dq_block != dq_block ||
      out->N != N || out->K != K)
    return QLR_ERR_ARG;
  const int rc = check_qweight(out);
  if (rc) return rc;
  if (!aligned16(W)) return QLR_ERR_ALIGN;
  return cuda_rc(launch_quantize_nfk(W, N * K, bits, block, dq_block, out, status_or_sink(status), as_stream(stream)));
}

int qlr_quantize_int4_group(const float* W, int64_t N, int64_t K, int group, const qlr_qweight* out,
                            int32_t* status, void* stream) {
  if (!W || !out) return QLR_ERR_ARG;
  if (out->fmt != QLR_FMT_INT4G || out->group != group || out->N != N || out->K != K) return QLR_ERR_ARG;
  const int rc = check_qweight(out);
  if (rc) return rc;
  if (!aligned16(W)) return QLR_ERR_ALIGN;
  return cuda_rc(launch_quantize_int4g(W, N, K, group, out, status_or_sink(status), as_stream(stream)));
}

int qlr_dequant(const qlr_qweight* w, uint16_t* W_out, int32_t* status, void* stream) {
  (void)status;
  int rc = check_qweight(w);
  if (rc) return rc;
  if (!W_out) return QLR_ERR_ARG;
  if (!aligned16(W_out)) return QLR_ERR_ALIGN;
  if ((w->N * w->K) % 32) return QLR_ERR_SHAPE;
  return cuda_rc(launch_dequant(w, W_out, as_stream(stream)));
}

int qlr_qalora_merge(const qlr_qweight* w, const uint16_t* A, const uint16_t* B, int r, float s, int32_t* status,
                     void* stream) {
  (void)status;
  int rc = check_qweight(w);
  if (rc) return rc;
  if (w->fmt != QLR_FMT_INT4G) return QLR_ERR_ARG;
  if (!A || !B || r <= 0 || r > 1024) return QLR_ERR_ARG;
  return cuda_rc(launch_merge(w, A, B, r, s, as_stream(stream)));
}

// ---- forward -------------------------------------------------------------------------------------

size_t qlr_forward_workspace_bytes(const qlr_qweight* w, int64_t M, int r, int pooled) {
  if (check_qweight(w) || M <= 0 || check_rank(r)) return 0;
  if (!pooled && lora_down_small_supported(M)) return 0;  // the few-token kernel needs no scratch
  if (pooled && pooled_adapter_supported(w->K, w->group, r)) return 0;  // nor does the pooled-input kernel
  // the group expansion of A (pooled adapter), then the split partial sums
  return (pooled ? align256(size_t(r) * w->K * 2) : 0) + adapter_ws_bytes(M, w->K, r);
}

int qlr_lora_down(const qlr_qweight* w, const uint16_t* X, int64_t M, const uint16_t* A, int r, float s, int pooled,
                  uint16_t* T_save, void* workspace, size_t workspace_bytes, int32_t* status, void* stream) {
  int rc = check_gemm_weight(w);
  if (rc) return rc;
  if ((rc = check_rank(r))) return rc;
  if (M < 0) return QLR_ERR_ARG;
  if (M == 0) return QLR_OK;
  if (!X || !A || !T_save) return QLR_ERR_ARG;
  if (!aligned16(X) || !aligned16(A) || !aligned16(T_save)) return QLR_ERR_ALIGN;
  if (pooled && w->fmt != QLR_FMT_INT4G) return QLR_ERR_UNSUPPORTED;
  if (pooled && (w->K / w->group) % 8) return QLR_ERR_SHAPE;
  if (M > (int64_t(1) << 30)) return QLR_ERR_SHAPE;
  const size_t need = qlr_forward_workspace_bytes(w, M, r, pooled);
  if (need && (!workspace || workspace_bytes < need)) return QLR_ERR_WORKSPACE;
  if (need && (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return QLR_ERR_ALIGN;
  cudaStream_t st = as_stream(stream);
  int32_t* stat = status_or_sink(status);
  const int64_t K = w->K;
  if (!pooled && lora_down_small_supported(M)) return cuda_rc(launch_lora_down_small(X, M, K, A, r, s, T_save, st));
  if (!pooled && skinny_supported(M, K, r))
    return cuda_rc(launch_skinny(X, M, K, A, false, r, s, T_save, stat, wait_limit_cycles(), st));
  if (pooled && pooled_adapter_supported(K, w->group, r))
    return cuda_rc(launch_pooled_lora_down(X, M, K, w->group, A, r, s, T_save, st));
  // T_save = bf16(s * P(X) A^T) = bf16(s * X Aexp^T), Aexp[j, k] = A[j, k / L] / L for the pooled adapter
  const uint16_t* Ab = A;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (pooled) {
    uint16_t* Aexp = reinterpret_cast<uint16_t*>(ws);
    ws += align256(size_t(r) * K * 2);
    if ((rc = cuda_rc(launch_expand_adapter(A, r, K, w->group, Aexp, st)))) return rc;
    Ab = Aexp;
  }
  AdapterGemm g{A_TMA_K, B_TMA_K, adapter_bn(r), M, K, X, M, K, Ab, r, K};
  return run_adapter(g, r, ADAPTER_ROWS_BF16, s, 1, T_save, r, ws, stat, st);
}

namespace {

// Y = X dequant(W)^T + T_save B^T with the given epilogue (EPI_SWIGLU_FWD: Y is U and H = silu(G) U is
// written beside it; a decode-sized call runs the decode kernel and then the standalone SwiGLU kernel).
int forward_base_impl(const qlr_qweight* w, const uint16_t* X, int64_t M, const uint16_t* B, int r,
                      const uint16_t* T_save, uint16_t* Y, int epi, const uint16_t* G, uint16_t* H, int32_t* status,
                      void* stream) {
  int rc = check_gemm_weight(w);
  if (rc) return rc;
  if ((rc = check_rank(r))) return rc;
  if (M < 0) return QLR_ERR_ARG;
  if (M == 0) return QLR_OK;
  if (!X || !B || !Y || !T_save) return QLR_ERR_ARG;
  if (!aligned16(X) || !aligned16(B) || !aligned16(Y) || !aligned16(T_save)) return QLR_ERR_ALIGN;
  if (M > (int64_t(1) << 30)) return QLR_ERR_SHAPE;
  cudaStream_t st = as_stream(stream);
  int32_t* stat = status_or_sink(status);
  const int64_t N = w->N, K = w->K;
  // a few tokens of a 4-bit NF weight: the HBM-bound decode kernel
  if (decode_supported(w, M)) {
    if ((rc = cuda_rc(launch_decode(w, X, M, B, r, T_save, Y, stat, st)))) return rc;
    return epi == EPI_SWIGLU_FWD ? cuda_rc(launch_swiglu_fwd(G, Y, H, M * N, st)) : QLR_OK;
  }
  // Y = X dequant(W)^T + T_save B^T: fused dequant + tcgen05, computed as Y^T tiles (W rows on TMEM lanes)
  const int tok = M >= 512 ? 512 : (M >= 192 ? 256 : 64);  // tokens per tile
  const int bn_tok = tok == 512 ? 256 : tok;                // tokens per activation stage
  GemmMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  const int kb = code_bits(w);
  const int csteps = kb == 3 ? 2 : 1;  // 64-code steps per codes box
  if ((rc = make_tmap(&maps.codes, w->codes, 1, N, K * kb / 8, 128, 8 * kb * csteps, 0))) return rc;
  if ((rc = make_tmap(&maps.b, X, 2, M, K, bn_tok, 64, 128))) return rc;
  if ((rc = make_tmap(&maps.b_tail, T_save, 2, M, r, bn_tok, 64, 128))) return rc;
  maps.a = maps.b;
  maps.a_tail = maps.b;
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  p.Mm = static_cast<int>(N);
  p.Nn = static_cast<int>(M);
  p.n_main = static_cast<int>(K / 64);
  p.splits = 1;
  p.n_tail = static_cast<int>(cdiv(r, 64));
  p.r_tail = r;
  p.m_tiles = static_cast<int>(cdiv(N, 128));
  p.n_tiles = static_cast<int>(cdiv(M, tok));
  set_items(p, tok);
  p.b_atom = 64;
  set_code_ring(p, kb, csteps, 128 * 8 * kb * csteps);
  p.out = Y;
  p.ldo = N;
  p.accumulate = 0;
  p.epi = epi;
  p.aux_g = G;
  p.aux_out = H;
  p.dq = dq_params(w);
  p.tail_a = B;
  p.tail_a_rows = N;
  p.tail_a_cols = r;
  p.status = stat;
  p.wait_cycles = wait_limit_cycles();
  return cuda_rc(launch_gemm(A_DQ_K, B_TMA_K, tok, OUT_BF16_T, 0, p, maps, st));
}

}  // namespace

int qlr_forward_base(const qlr_qweight* w, const uint16_t* X, int64_t M, const uint16_t* B, int r,
                     const uint16_t* T_save, uint16_t* Y, int32_t* status, void* stream) {
  return forward_base_impl(w, X, M, B, r, T_save, Y, EPI_STORE, nullptr, nullptr, status, stream);
}

int qlr_forward_swiglu(const qlr_qweight* w_up, const uint16_t* X, int64_t M, const uint16_t* B_up, int r,
                       const uint16_t* T_up, const uint16_t* G, uint16_t* U, uint16_t* H, int32_t* status,
                       void* stream) {
  if (M > 0 && (!G || !H)) return QLR_ERR_ARG;
  if (!aligned16(G) || !aligned16(H)) return QLR_ERR_ALIGN;
  if (w_up && w_up->N % 8) return QLR_ERR_SHAPE;
  return forward_base_impl(w_up, X, M, B_up, r, T_up, U, EPI_SWIGLU_FWD, G, H, status, stream);
}

int qlr_forward(const qlr_qweight* w, const uint16_t* X, int64_t M, const uint16_t* A, const uint16_t* B, int r,
                float s, int pooled, uint16_t* Y, uint16_t* T_save, void* workspace, size_t workspace_bytes,
                int32_t* status, void* stream) {
  int rc = check_gemm_weight(w);
  if (rc) return rc;
  if ((rc = check_rank(r))) return rc;
  if (M < 0) return QLR_ERR_ARG;
  if (M == 0) return QLR_OK;
  if (!X || !A || !B || !Y || !T_save) return QLR_ERR_ARG;
  if ((rc = qlr_lora_down(w, X, M, A, r, s, pooled, T_save, workspace, workspace_bytes, status, stream))) return rc;
  return qlr_forward_base(w, X, M, B, r, T_save, Y, status, stream);
}

// ---- backward: adapter gradients -------------------------------------------------------------------

size_t qlr_backward_lora_workspace_bytes(const qlr_qweight* w, int64_t M, int r, int pooled) {
  if (check_qweight(w) || M <= 0 || check_rank(r)) return 0;
  // split partial sums of the three GEMMs, which run one after another (the pooled adapter's dA: the
  // partial sums of its token blocks)
  const size_t a = adapter_ws_bytes(M, w->N, r);
  const size_t b = adapter_ws_bytes(w->N, M, r);
  const size_t c = (pooled && pooled_adapter_supported(w->K, w->group, r)) ? pooled_dA_workspace_bytes(M, w->K, w->group, r)
                                                                          : adapter_ws_bytes(w->K, M, r);
  return a > b ? (a > c ? a : c) : (b > c ? b : c);
}

namespace {

// Shared validation of the adapter-gradient calls; fills *need with the workspace size.
int check_backward_lora(const qlr_qweight* w, int64_t M, int r, int pooled, const void* workspace,
                        size_t workspace_bytes) {
  int rc = check_gemm_weight(w);
  if (rc) return rc;
  if ((rc = check_rank(r))) return rc;
  if (M < 0) return QLR_ERR_ARG;
  if (pooled && w->fmt != QLR_FMT_INT4G) return QLR_ERR_UNSUPPORTED;
  if (pooled && (w->K / w->group) % 8) return QLR_ERR_SHAPE;
  if (M > (int64_t(1) << 30)) return QLR_ERR_SHAPE;
  if (M == 0) return QLR_OK;
  const size_t need = qlr_backward_lora_workspace_bytes(w, M, r, pooled);
  if (need && (!workspace || workspace_bytes < need)) return QLR_ERR_WORKSPACE;
  if (need && (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return QLR_ERR_ALIGN;
  return QLR_OK;
}

int run_dT(const qlr_qweight* w, const uint16_t* dY, int64_t M, const uint16_t* B, int r, float s, uint16_t* dT_out,
           void* workspace, int32_t* status, cudaStream_t st) {
  // dT = bf16(s dY B)
  if (skinny_supported(M, w->N, r))
    return cuda_rc(launch_skinny(dY, M, w->N, B, true, r, s, dT_out, status_or_sink(status), wait_limit_cycles(), st));
  AdapterGemm g{A_TMA_K, B_TMA_MN, adapter_bn(r), M, w->N, dY, M, w->N, B, w->N, r};
  return run_adapter(g, r, ADAPTER_ROWS_BF16, s, 1, dT_out, r, static_cast<uint8_t*>(workspace),
                     status_or_sink(status), st);
}

int run_dAdB(const qlr_qweight* w, const uint16_t* X, const uint16_t* dY, const uint16_t* T_save, const uint16_t* dT,
             int64_t M, int r, int pooled, float* dA, float* dB, void* workspace, int32_t* status, cudaStream_t st) {
  const int64_t N = w->N, K = w->K;
  const int64_t Ka = pooled ? K / w->group : K;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* stat = status_or_sink(status);
  const int bn = adapter_bn(r);
  int rc;
  // dB = dY^T T_save  (rows of D are output features, reduction over tokens)
  {
    AdapterGemm g{A_TMA_MN, B_TMA_MN, bn, N, M, dY, M, N, T_save, M, r};
    if ((rc = run_adapter(g, r, ADAPTER_ROWS_F32, 1.0f, 1, dB, r, ws, stat, st))) return rc;
  }
  // pooled adapter: dA = dT^T P(X) from the group means of X
  if (pooled && pooled_adapter_supported(K, w->group, r))
    return cuda_rc(launch_pooled_dA(X, M, K, w->group, dT, r, dA, reinterpret_cast<float*>(ws), st));
  // dA^T = X^T dT over all K inputs; the pooled adapter sums each group of L inputs and divides by L
  AdapterGemm g{A_TMA_MN, B_TMA_MN, bn, K, M, X, M, K, dT, M, r};
  return run_adapter(g, r, ADAPTER_COLS_F32, 1.0f, pooled ? w->group : 1, dA, Ka, ws, stat, st);
}

int zero_grads(const qlr_qweight* w, int r, int pooled, float* dA, float* dB, cudaStream_t st) {
  const int64_t Ka = pooled ? w->K / w->group : w->K;
  if (cudaMemsetAsync(dA, 0, size_t(r) * Ka * 4, st) != cudaSuccess) return QLR_ERR_CUDA;
  return cuda_rc(cudaMemsetAsync(dB, 0, size_t(w->N) * r * 4, st));
}

}  // namespace

int qlr_backward_lora(const qlr_qweight* w, const uint16_t* X, const uint16_t* dY, const uint16_t* T_save,
                      const uint16_t* B, int64_t M, int r, float s, int pooled, float* dA, float* dB,
                      uint16_t* dT_out, void* workspace, size_t workspace_bytes, int32_t* status, void* stream) {
  int rc = check_backward_lora(w, M, r, pooled, workspace, workspace_bytes);
  if (rc) return rc;
  if (!dA || !dB) return QLR_ERR_ARG;
  if (M > 0 && (!X || !dY || !T_save || !B || !dT_out)) return QLR_ERR_ARG;
  if (!aligned16(X) || !aligned16(dY) || !aligned16(T_save) || !aligned16(B) || !aligned16(dA) || !aligned16(dB) ||
      !aligned16(dT_out))
    return QLR_ERR_ALIGN;
  cudaStream_t st = as_stream(stream);
  if (M == 0) return zero_grads(w, r, pooled, dA, dB, st);  // no tokens: the gradients are zero
  if ((rc = run_dT(w, dY, M, B, r, s, dT_out, workspace, status, st))) return rc;
  return run_dAdB(w, X, dY, T_save, dT_out, M, r, pooled, dA, dB, workspace, status, st);
}

int qlr_backward_lora_dT(const qlr_qweight* w, const uint16_t* dY, int64_t M, const uint16_t* B, int r, float s,
                         uint16_t* dT_out, void* workspace, size_t workspace_bytes, int32_t* status, void* stream) {
  int rc = check_backward_lora(w, M, r, 0, workspace, workspace_bytes);
  if (rc) return rc;
  if (M == 0) return QLR_OK;
  if (!dY || !B || !dT_out) return QLR_ERR_ARG;
  if (!aligned16(dY) || !aligned16(B) || !aligned16(dT_out)) return QLR_ERR_ALIGN;
  return run_dT(w, dY, M, B, r, s, dT_out, workspace, status, as_stream(stream));
}

int qlr_backward_lora_dAdB(const qlr_qweight* w, const uint16_t* X, const uint16_t* dY, const uint16_t* T_save,
                           const uint16_t* dT, int64_t M, int r, int pooled, float* dA, float* dB, void* workspace,
                           size_t workspace_bytes, int32_t* status, void* stream) {
  int rc = check_backward_lora(w, M, r, pooled, workspace, workspace_bytes);
  if (rc) return rc;
  if (!dA || !dB) return QLR_ERR_ARG;
  if (M > 0 && (!X || !dY || !T_save || !dT)) return QLR_ERR_ARG;
  if (!aligned16(X) || !aligned16(dY) || !aligned16(T_save) || !aligned16(dT) || !aligned16(dA) || !aligned16(dB))
    return QLR_ERR_ALIGN;
  cudaStream_t st = as_stream(stream);
  if (M == 0) return zero_grads(w, r, pooled, dA, dB, st);
  return run_dAdB(w, X, dY, T_save, dT, M, r, pooled, dA, dB, workspace, status, st);
}

// ---- backward: input gradient --------------------------------------------------------------------

size_t qlr_backward_dx_workspace_bytes(const qlr_qweight* w, int64_t M, int r, int pooled) {
  (void)w;
  (void)M;
  (void)r;
  (void)pooled;
  return 0;  // the pooled adapter's group expansion is formed while the tail rows are copied
}

namespace {

// dX = dY dequant(W) + P^T(dT A) with the given epilogue (EPI_SWIGLU_BWD: dX is dH, never stored; dG and dU
// are written from G and U).
int backward_dx_impl(const qlr_qweight* w, const uint16_t* dY, int64_t M, const uint16_t* A, const uint16_t* dT,
                     int r, int pooled, int accumulate, uint16_t* dX, int epi, const uint16_t* G, const uint16_t* U,
                     uint16_t* dU, int32_t* status, void* stream) {
  int rc = check_gemm_weight(w);
  if (rc) return rc;
  if ((rc = check_rank(r))) return rc;
  if (M < 0) return QLR_ERR_ARG;
  if (M == 0) return QLR_OK;
  if (!dY || !A || !dT || !dX) return QLR_ERR_ARG;
  if (!aligned16(dY) || !aligned16(A) || !aligned16(dT) || !aligned16(dX)) return QLR_ERR_ALIGN;
  if (pooled && w->fmt != QLR_FMT_INT4G) return QLR_ERR_UNSUPPORTED;
  if (M == 0) return QLR_OK;
  if (M > (int64_t(1) << 30)) return QLR_ERR_SHAPE;
  cudaStream_t st = as_stream(stream);
  int32_t* stat = status_or_sink(status);
  const int64_t N = w->N, K = w->K;
  const uint16_t* At = A;
  const int tok = M >= 512 ? 512 : (M >= 192 ? 256 : 64);  // tokens per tile
  const int bn_tok = tok == 512 ? 256 : tok;                // tokens per activation stage
  GemmMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  const int kb = code_bits(w);
  if ((rc = make_tmap(&maps.codes, w->codes, 1, N, K * kb / 8, 64, 16 * kb, 0))) return rc;
  if ((rc = make_tmap(&maps.b, dY, 2, M, N, bn_tok, 64, 128))) return rc;
  if ((rc = make_tmap(&maps.b_tail, dT, 2, M, r, bn_tok, 64, 128))) return rc;
  maps.a = maps.b;
  maps.a_tail = maps.b;
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  p.Mm = static_cast<int>(K);
  p.Nn = static_cast<int>(M);
  p.n_main = static_cast<int>(cdiv(N, 64));
  p.splits = 1;
  p.n_tail = static_cast<int>(cdiv(r, 64));
  p.r_tail = r;
  p.m_tiles = static_cast<int>(cdiv(K, 128));
  p.n_tiles = static_cast<int>(cdiv(M, tok));
  set_items(p, tok);
  p.b_atom = 64;
  set_code_ring(p, kb, 1, 64 * 16 * kb);
  p.out = dX;
  p.ldo = K;
  p.accumulate = accumulate ? 1 : 0;
  p.epi = epi;
  p.aux_g = G;
  p.aux_u = U;
  p.aux_out = dU;
  p.dq = dq_params(w);
  p.tail_a = At;
  p.tail_a_rows = r;
  p.tail_a_cols = pooled ? K / w->group : K;
  p.tail_pool_L = pooled ? w->group : 0;
  p.status = stat;
  p.wait_cycles = wait_limit_cycles();
  return cuda_rc(launch_gemm(A_DQ_MN, B_TMA_K, tok, OUT_BF16_T, 1, p, maps, st));
}

}  // namespace

int qlr_backward_dx(const qlr_qweight* w, const uint16_t* dY, int64_t M, const uint16_t* A, const uint16_t* dT,
                    int r, int pooled, int accumulate, uint16_t* dX, void* workspace, size_t workspace_bytes,
                    int32_t* status, void* stream) {
  (void)workspace;
  (void)workspace_bytes;
  return backward_dx_impl(w, dY, M, A, dT, r, pooled, accumulate, dX, EPI_STORE, nullptr, nullptr, nullptr, status,
                          stream);
}

int qlr_backward_dx_swiglu(const qlr_qweight* w_down, const uint16_t* dY, int64_t M, const uint16_t* A,
                           const uint16_t* dT, int r, const uint16_t* G, const uint16_t* U, uint16_t* dG, uint16_t* dU,
                           int32_t* status, void* stream) {
  if (M > 0 && (!G || !U || !dU)) return QLR_ERR_ARG;
  if (!aligned16(G) || !aligned16(U) || !aligned16(dU)) return QLR_ERR_ALIGN;
  if (w_down && w_down->K % 8) return QLR_ERR_SHAPE;
  return backward_dx_impl(w_down, dY, M, A, dT, r, 0, 0, dG, EPI_SWIGLU_BWD, G, U, dU, status, stream);
}

// ---- SwiGLU ---------------------------------------------------------------------------------------

int qlr_swiglu_forward(const uint16_t* G, const uint16_t* U, uint16_t* H, int64_t n, void* stream) {
  if (n < 0 || (n && (!G || !U || !H))) return QLR_ERR_ARG;
  if (n % 8) return QLR_ERR_SHAPE;
  if (!aligned16(G) || !aligned16(U) || !aligned16(H)) return QLR_ERR_ALIGN;
  return cuda_rc(launch_swiglu_fwd(G, U, H, n, as_stream(stream)));
}

int qlr_swiglu_backward(const uint16_t* dH, const uint16_t* G, const uint16_t* U, uint16_t* dG, uint16_t* dU,
                        int64_t n, void* stream) {
  if (n < 0 || (n && (!dH || !G || !U || !dG || !dU))) return QLR_ERR_ARG;
  if (n % 8) return QLR_ERR_SHAPE;
  if (!aligned16(dH) || !aligned16(G) || !aligned16(U) || !aligned16(dG) || !aligned16(dU)) return QLR_ERR_ALIGN;
  return cuda_rc(launch_swiglu_bwd(dH, G, U, dG, dU, n, as_stream(stream)));
}

}  // extern "C"
