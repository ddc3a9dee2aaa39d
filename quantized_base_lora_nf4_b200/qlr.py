"""Python binding of the C ABI in include/qlr.h (argument marshalling only).

Every computation runs in libqlr.so's CUDA kernels; this module allocates the caller-owned
device buffers with PyTorch, passes raw pointers and the current stream, and raises
``QLRError`` on a negative return code.  It never computes anything on the CPU and has no
fallback: without the built library (or without a GPU) the calls fail.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqlr.so")

FMT_NFK = 1
FMT_INT4G = 2
PART_CODES, PART_C1, PART_C1_FP8, PART_S2, PART_SCALE, PART_ZERO = range(6)

ERRORS = {0: "OK", -1: "ERR_ARG", -2: "ERR_SHAPE", -3: "ERR_ALIGN", -4: "ERR_UNSUPPORTED",
          -5: "ERR_NONFINITE", -6: "ERR_TIMEOUT", -7: "ERR_CUDA", -8: "ERR_WORKSPACE"}

EXPORTED = (
    "qlr_error_string", "qlr_version", "qlr_qweight_part_bytes", "qlr_nf_levels", "qlr_nf_decision_table",
    "qlr_quantize_nf4",
    "qlr_quantize_int4_group", "qlr_dequant", "qlr_qalora_merge", "qlr_forward_workspace_bytes", "qlr_forward",
    "qlr_backward_lora_workspace_bytes", "qlr_backward_lora", "qlr_backward_dx_workspace_bytes",
    "qlr_backward_dx", "qlr_swiglu_forward", "qlr_swiglu_backward", "qlr_device_sm_count", "qlr_lora_down",
    "qlr_forward_base", "qlr_launch_count", "qlr_backward_lora_noalloc", "qlr_lqlora_init_workspace_bytes",
    "qlr_lqlora_init", "qlr_nf_quant_error_workspace_bytes", "qlr_nf_quant_error", "qlr_lqlora_allocate",
    "qlr_set_wait_limit", "qlr_wait_selftest", "qlr_loqa_grad", "qlr_forward_swiglu", "qlr_backward_dx_swiglu",
    "qlr_backward_lora_dT", "qlr_backward_lora_dAdB",
)


class QLRError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {ERRORS.get(code, code)} ({code})")


class CQWeight(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("bits", ctypes.c_int32), ("block", ctypes.c_int32),
                ("dq_block", ctypes.c_int32), ("group", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("N", ctypes.c_int64), ("K", ctypes.c_int64),
                ("codes", ctypes.c_void_p), ("c1", ctypes.c_void_p), ("c1_fp8", ctypes.c_void_p),
                ("s2", ctypes.c_void_p), ("scale", ctypes.c_void_p), ("zero", ctypes.c_void_p)]


_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libqlr.so is not built ({LIB_PATH}); run `python -m quantized_base_lora_nf4_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I, I64, F, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    QP = ctypes.POINTER(CQWeight)
    sig = {
        "qlr_error_string": (ctypes.c_char_p, [I]),
        "qlr_version": (I, []),
        "qlr_device_sm_count": (I, []),
        "qlr_qweight_part_bytes": (I64, [I, I64, I64, I, I, I, I, I]),
        "qlr_nf_levels": (I, [I, P]),
        "qlr_quantize_nf4": (I, [P, I64, I64, I, I, I, QP, P, P]),
        "qlr_quantize_int4_group": (I, [P, I64, I64, I, QP, P, P]),
        "qlr_dequant": (I, [QP, P, P, P]),
        "qlr_qalora_merge": (I, [QP, P, P, I, F, P, P]),
        "qlr_forward_workspace_bytes": (SZ, [QP, I64, I, I]),
        "qlr_forward": (I, [QP, P, I64, P, P, I, F, I, P, P, P, SZ, P, P]),
        "qlr_backward_lora_workspace_bytes": (SZ, [QP, I64, I, I]),
        "qlr_backward_lora": (I, [QP, P, P, P, P, I64, I, F, I, P, P, P, P, SZ, P, P]),
        "qlr_backward_dx_workspace_bytes": (SZ, [QP, I64, I, I]),
        "qlr_backward_dx": (I, [QP, P, I64, P, P, I, I, I, P, P, SZ, P, P]),
        "qlr_swiglu_forward": (I, [P, P, P, I64, P]),
        "qlr_swiglu_backward": (I, [P, P, P, P, P, I64, P]),
        "qlr_lora_down": (I, [QP, P, I64, P, I, F, I, P, P, SZ, P, P]),
        "qlr_forward_base": (I, [QP, P, I64, P, I, P, P, P, P]),
        "qlr_launch_count": (ctypes.c_uint64, []),
        "qlr_backward_lora_noalloc": (I, [QP, P, P, P, P, I64, I, F, I, P, P, P, P, P]),
        "qlr_lqlora_init_workspace_bytes": (SZ, [I64, I64, I]),
        "qlr_lqlora_init": (I, [P, I64, I64, I, I, I, I, F, I, QP, P, P, P, SZ, P, P]),
        "qlr_nf_quant_error_workspace_bytes": (SZ, [I64, I64, I, I, I]),
        "qlr_nf_quant_error": (I, [P, I64, I64, I, I, I, P, P, SZ, P, P]),
        "qlr_lqlora_allocate": (I, [P, P, I, I, I64, I64, P, P]),
        "qlr_set_wait_limit": (ctypes.c_longlong, [ctypes.c_longlong]),
        "qlr_wait_selftest": (I, [P, P]),
        "qlr_loqa_grad": (I, [QP, P, P, I64, P, P, P, P]),
        "qlr_forward_swiglu": (I, [QP, P, I64, P, I, P, P, P, P, P, P]),
        "qlr_backward_dx_swiglu": (I, [QP, P, I64, P, P, I, P, P, P, P, P, P]),
        "qlr_backward_lora_dT": (I, [QP, P, I64, P, I, F, P, P, SZ, P, P]),
        "qlr_backward_lora_dAdB": (I, [QP, P, P, P, P, I64, I, I, P, P, P, SZ, P, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def _check(rc: int, where: str) -> None:
    if rc != 0:
        raise QLRError(rc, where)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _empty(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device=device)


@dataclass
class QWeight:
    """A quantised weight: metadata plus the caller-owned device buffers of include/qlr.h's qlr_qweight."""

    fmt: int
    N: int
    K: int
    bits: int = 4
    block: int = 64
    dq_block: int = 256
    group: int = 32
    codes: Optional[torch.Tensor] = None
    c1: Optional[torch.Tensor] = None
    c1_fp8: Optional[torch.Tensor] = None
    s2: Optional[torch.Tensor] = None
    scale: Optional[torch.Tensor] = None
    zero: Optional[torch.Tensor] = None
    _c: CQWeight = field(default=None, repr=False)

    def struct(self) -> CQWeight:
        c = CQWeight()
        c.fmt, c.bits, c.block, c.dq_block, c.group, c.reserved = (self.fmt, self.bits, self.block, self.dq_block,
                                                                    self.group, 0)
        c.N, c.K = self.N, self.K
        for name in ("codes", "c1", "c1_fp8", "s2", "scale", "zero"):
            t = getattr(self, name)
            setattr(c, name, None if t is None else t.data_ptr())
        self._c = c
        return c

    def ref(self):
        return ctypes.byref(self.struct())

    @property
    def pooled_inputs(self) -> int:
        return self.K // self.group


def part_bytes(fmt, N, K, bits=4, block=64, dq_block=256, group=32, part=PART_CODES) -> int:
    n = lib().qlr_qweight_part_bytes(fmt, N, K, bits, block, dq_block, group, part)
    if n < 0:
        raise QLRError(int(n), "qlr_qweight_part_bytes")
    return int(n)


def alloc_qweight(fmt: int, N: int, K: int, device, bits=4, block=64, dq_block=256, group=32) -> QWeight:
    q = QWeight(fmt, N, K, bits, block, dq_block, group)
    nb = lambda part: part_bytes(fmt, N, K, bits, block, dq_block, group, part)  # noqa: E731
    q.codes = _empty(nb(PART_CODES), device)
    if fmt == FMT_NFK:
        if dq_block:
            q.c1_fp8 = _empty(nb(PART_C1_FP8), device)
            q.s2 = torch.empty(max(nb(PART_S2) // 4, 4), dtype=torch.float32, device=device)
        else:
            q.c1 = torch.empty(max(nb(PART_C1) // 4, 4), dtype=torch.float32, device=device)
    else:
        q.scale = torch.empty((N, K // group), dtype=torch.float16, device=device)
        q.zero = torch.empty((N, K // group), dtype=torch.float16, device=device)
    return q


def nf_levels(bits: int) -> torch.Tensor:
    out = (ctypes.c_float * (1 << bits))()
    _check(lib().qlr_nf_levels(bits, ctypes.cast(out, ctypes.c_void_p)), "qlr_nf_levels")
    return torch.tensor(list(out), dtype=torch.float32)


def nf_decision_table(bits: int):
    """(threshold[33], base[33]) of the NF-k quantiser's nearest-level decision (host arrays)."""
    t = (ctypes.c_float * 33)()
    b = (ctypes.c_int32 * 33)()
    _check(lib().qlr_nf_decision_table(bits, ctypes.cast(t, ctypes.c_void_p), ctypes.cast(b, ctypes.c_void_p)),
           "qlr_nf_decision_table")
    return list(t), list(b)


def new_status(device) -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=device)


def quantize_nf4(W: torch.Tensor, bits: int = 4, block: int = 64, dq_block: int = 256,
                 status: Optional[torch.Tensor] = None, stream=None) -> QWeight:
    N, K = W.shape
    q = alloc_qweight(FMT_NFK, N, K, W.device, bits, block, dq_block)
    _check(lib().qlr_quantize_nf4(_ptr(W), N, K, bits, block, dq_block, q.ref(), _ptr(status), _stream(stream)),
           "qlr_quantize_nf4")
    return q


def quantize_int4_group(W: torch.Tensor, group: int = 32, status: Optional[torch.Tensor] = None,
                        stream=None) -> QWeight:
    N, K = W.shape
    q = alloc_qweight(FMT_INT4G, N, K, W.device, group=group)
    _check(lib().qlr_quantize_int4_group(_ptr(W), N, K, group, q.ref(), _ptr(status), _stream(stream)),
           "qlr_quantize_int4_group")
    return q


def dequant(q: QWeight, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty((q.N, q.K), dtype=torch.bfloat16, device=q.codes.device)
    _check(lib().qlr_dequant(q.ref(), _ptr(out), None, _stream(stream)), "qlr_dequant")
    return out


def qalora_merge(q: QWeight, A: torch.Tensor, B: torch.Tensor, s: float, stream=None) -> None:
    _check(lib().qlr_qalora_merge(q.ref(), _ptr(A), _ptr(B), A.shape[0], float(s), None, _stream(stream)),
           "qlr_qalora_merge")


def lqlora_init(W: torch.Tensor, bits: int, block: int, dq_block: int, r: int, s: float, iters: int,
                status: Optional[torch.Tensor] = None, stream=None) -> Tuple[QWeight, torch.Tensor, torch.Tensor]:
    """LQ-LoRA initialisation of an fp32 weight: the quantised part and the adapter (A [r, K], B [N, r])."""
    N, K = W.shape
    q = alloc_qweight(FMT_NFK, N, K, W.device, bits, block, dq_block)
    A = torch.empty((r, K), dtype=torch.bfloat16, device=W.device)
    B = torch.empty((N, r), dtype=torch.bfloat16, device=W.device)
    nbytes = int(lib().qlr_lqlora_init_workspace_bytes(N, K, r)) if iters > 0 else 0
    ws = _empty(max(nbytes, 256), W.device)
    _check(lib().qlr_lqlora_init(_ptr(W), N, K, bits, block, dq_block, r, float(s), iters, q.ref(), _ptr(A), _ptr(B),
                                 _ptr(ws), nbytes, _ptr(status), _stream(stream)), "qlr_lqlora_init")
    return q, A, B


def nf_quant_error(W: torch.Tensor, bits: int, block: int, dq_block: int, out: Optional[torch.Tensor] = None,
                   ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Squared reconstruction error of NF-k quantising W, as a one-element float64 device tensor."""
    N, K = W.shape
    nbytes = int(lib().qlr_nf_quant_error_workspace_bytes(N, K, bits, block, dq_block))
    if ws is None or ws.numel() < nbytes:
        ws = _empty(max(nbytes, 256), W.device)
    if out is None:
        out = torch.empty(1, dtype=torch.float64, device=W.device)
    _check(lib().qlr_nf_quant_error(_ptr(W), N, K, bits, block, dq_block, _ptr(out), _ptr(ws), nbytes, None,
                                    _stream(stream)), "qlr_nf_quant_error")
    return out


def lqlora_allocate(err, cost_bits, budget_bits: int, unit_bits: int):
    """Budgeted option per matrix (host arrays [n_mat, n_opt]): returns (choices, total error)."""
    import numpy as np
    e = np.ascontiguousarray(err, dtype=np.float64)
    c = np.ascontiguousarray(cost_bits, dtype=np.int64)
    n_mat, n_opt = e.shape
    choice = np.zeros(n_mat, dtype=np.int32)
    total = ctypes.c_double(0.0)
    _check(lib().qlr_lqlora_allocate(e.ctypes.data, c.ctypes.data, n_mat, n_opt, int(budget_bits), int(unit_bits),
                                     choice.ctypes.data, ctypes.byref(total)), "qlr_lqlora_allocate")
    return [int(x) for x in choice], float(total.value)


class Workspace:
    """A growable device scratch buffer handed to the library (256-byte aligned by PyTorch)."""

    def __init__(self, device):
        self.device = device
        self.buf = _empty(256, device)

    def get(self, nbytes: int) -> torch.Tensor:
        if self.buf.numel() < nbytes:
            self.buf = _empty(nbytes, self.device)
        return self.buf


def forward(q: QWeight, X: torch.Tensor, A: torch.Tensor, B: torch.Tensor, s: float, pooled: bool = False,
            Y: Optional[torch.Tensor] = None, T_save: Optional[torch.Tensor] = None,
            ws: Optional[Workspace] = None, status: Optional[torch.Tensor] = None,
            stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    M = X.shape[0]
    r = A.shape[0]
    dev = X.device
    if Y is None:
        Y = torch.empty((M, q.N), dtype=torch.bfloat16, device=dev)
    if T_save is None:
        T_save = torch.empty((M, r), dtype=torch.bfloat16, device=dev)
    qs = q.struct()
    need = lib().qlr_forward_workspace_bytes(ctypes.byref(qs), M, r, int(pooled))
    w = (ws or Workspace(dev)).get(need)
    _check(lib().qlr_forward(ctypes.byref(qs), _ptr(X), M, _ptr(A), _ptr(B), r, float(s), int(pooled), _ptr(Y),
                             _ptr(T_save), _ptr(w), w.numel(), _ptr(status), _stream(stream)), "qlr_forward")
    return Y, T_save


def lora_down(q: QWeight, X: torch.Tensor, A: torch.Tensor, s: float, pooled: bool = False,
              T_save: Optional[torch.Tensor] = None, ws: Optional[Workspace] = None,
              status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    M = X.shape[0]
    r = A.shape[0]
    if T_save is None:
        T_save = torch.empty((M, r), dtype=torch.bfloat16, device=X.device)
    qs = q.struct()
    need = lib().qlr_forward_workspace_bytes(ctypes.byref(qs), M, r, int(pooled))
    w = (ws or Workspace(X.device)).get(need)
    _check(lib().qlr_lora_down(ctypes.byref(qs), _ptr(X), M, _ptr(A), r, float(s), int(pooled), _ptr(T_save),
                               _ptr(w), w.numel(), _ptr(status), _stream(stream)), "qlr_lora_down")
    return T_save


def forward_base(q: QWeight, X: torch.Tensor, B: torch.Tensor, T_save: torch.Tensor, Y: Optional[torch.Tensor] = None,
                 status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    M = X.shape[0]
    if Y is None:
        Y = torch.empty((M, q.N), dtype=torch.bfloat16, device=X.device)
    _check(lib().qlr_forward_base(q.ref(), _ptr(X), M, _ptr(B), B.shape[1], _ptr(T_save), _ptr(Y), _ptr(status),
                                  _stream(stream)), "qlr_forward_base")
    return Y


def forward_swiglu(q_up: QWeight, X: torch.Tensor, B_up: torch.Tensor, T_up: torch.Tensor, G: torch.Tensor,
                   U: Optional[torch.Tensor] = None, H: Optional[torch.Tensor] = None,
                   status: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Up projection U and the SwiGLU H = silu(G) * U in one launch (G: the gate projection's output)."""
    M = X.shape[0]
    if U is None:
        U = torch.empty((M, q_up.N), dtype=torch.bfloat16, device=X.device)
    if H is None:
        H = torch.empty_like(U)
    _check(lib().qlr_forward_swiglu(q_up.ref(), _ptr(X), M, _ptr(B_up), B_up.shape[1], _ptr(T_up), _ptr(G), _ptr(U),
                                    _ptr(H), _ptr(status), _stream(stream)), "qlr_forward_swiglu")
    return U, H


def backward_dx_swiglu(q_down: QWeight, dY: torch.Tensor, A: torch.Tensor, dT: torch.Tensor, G: torch.Tensor,
                       U: torch.Tensor, dG: Optional[torch.Tensor] = None, dU: Optional[torch.Tensor] = None,
                       status: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """The down projection's input gradient dH turned into (dG, dU) in its epilogue (dH never stored)."""
    M = dY.shape[0]
    if dG is None:
        dG = torch.empty((M, q_down.K), dtype=torch.bfloat16, device=dY.device)
    if dU is None:
        dU = torch.empty_like(dG)
    _check(lib().qlr_backward_dx_swiglu(q_down.ref(), _ptr(dY), M, _ptr(A), _ptr(dT), A.shape[0], _ptr(G), _ptr(U),
                                        _ptr(dG), _ptr(dU), _ptr(status), _stream(stream)), "qlr_backward_dx_swiglu")
    return dG, dU


def launch_count() -> int:
    return int(lib().qlr_launch_count())


def set_wait_limit(cycles: int) -> int:
    """Bound (SM clock cycles) of the pipeline waits of the kernels launched next; < 0 restores the
    default.  Returns the previous bound."""
    return int(lib().qlr_set_wait_limit(int(cycles)))


def wait_selftest(status: torch.Tensor, stream=None) -> None:
    """A kernel whose wait can only run out: it must set *status to the timeout code and free its tensor memory."""
    _check(lib().qlr_wait_selftest(_ptr(status), _stream(stream)), "qlr_wait_selftest")


def backward_lora(q: QWeight, X: torch.Tensor, dY: torch.Tensor, T_save: torch.Tensor, B: torch.Tensor, s: float,
                  pooled: bool = False, dA: Optional[torch.Tensor] = None, dB: Optional[torch.Tensor] = None,
                  dT: Optional[torch.Tensor] = None, ws: Optional[Workspace] = None,
                  status: Optional[torch.Tensor] = None, stream=None):
    M = X.shape[0]
    r = B.shape[1]
    dev = X.device
    Ka = q.K // q.group if pooled else q.K
    if dA is None:
        dA = torch.empty((r, Ka), dtype=torch.float32, device=dev)
    if dB is None:
        dB = torch.empty((q.N, r), dtype=torch.float32, device=dev)
    if dT is None:
        dT = torch.empty((M, r), dtype=torch.bfloat16, device=dev)
    qs = q.struct()
    need = lib().qlr_backward_lora_workspace_bytes(ctypes.byref(qs), M, r, int(pooled))
    w = (ws or Workspace(dev)).get(need)
    _check(lib().qlr_backward_lora(ctypes.byref(qs), _ptr(X), _ptr(dY), _ptr(T_save), _ptr(B), M, r, float(s),
                                   int(pooled), _ptr(dA), _ptr(dB), _ptr(dT), _ptr(w), w.numel(), _ptr(status),
                                   _stream(stream)), "qlr_backward_lora")
    return dA, dB, dT


def loqa_grad(q: QWeight, X: torch.Tensor, dY: torch.Tensor, dscale: Optional[torch.Tensor] = None,
              dzero: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None, stream=None):
    """LoQA: gradients of the loss with respect to the INT4 weight's scale and zero point, fp32 [N, K/group]."""
    G = q.K // q.group
    dev = X.device
    if dscale is None:
        dscale = torch.empty((q.N, G), dtype=torch.float32, device=dev)
    if dzero is None:
        dzero = torch.empty((q.N, G), dtype=torch.float32, device=dev)
    _check(lib().qlr_loqa_grad(q.ref(), _ptr(X), _ptr(dY), X.shape[0], _ptr(dscale), _ptr(dzero), _ptr(status),
                               _stream(stream)), "qlr_loqa_grad")
    return dscale, dzero


def backward_lora_dT(q: QWeight, dY: torch.Tensor, B: torch.Tensor, s: float, dT: Optional[torch.Tensor] = None,
                     ws: Optional[Workspace] = None, status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """First half of backward_lora: dT = bf16(s dY B)."""
    M, r = dY.shape[0], B.shape[1]
    if dT is None:
        dT = torch.empty((M, r), dtype=torch.bfloat16, device=dY.device)
    qs = q.struct()
    need = lib().qlr_backward_lora_workspace_bytes(ctypes.byref(qs), M, r, 0)
    w = (ws or Workspace(dY.device)).get(need)
    _check(lib().qlr_backward_lora_dT(ctypes.byref(qs), _ptr(dY), M, _ptr(B), r, float(s), _ptr(dT), _ptr(w), w.numel(),
                                      _ptr(status), _stream(stream)), "qlr_backward_lora_dT")
    return dT


def backward_lora_dAdB(q: QWeight, X: torch.Tensor, dY: torch.Tensor, T_save: torch.Tensor, dT: torch.Tensor,
                       pooled: bool = False, dA: Optional[torch.Tensor] = None, dB: Optional[torch.Tensor] = None,
                       ws: Optional[Workspace] = None, status: Optional[torch.Tensor] = None, stream=None):
    """Second half of backward_lora: dB = dY^T T_save and dA = dT^T P(X)."""
    M, r = X.shape[0], dT.shape[1]
    dev = X.device
    Ka = q.K // q.group if pooled else q.K
    if dA is None:
        dA = torch.empty((r, Ka), dtype=torch.float32, device=dev)
    if dB is None:
        dB = torch.empty((q.N, r), dtype=torch.float32, device=dev)
    qs = q.struct()
    need = lib().qlr_backward_lora_workspace_bytes(ctypes.byref(qs), M, r, int(pooled))
    w = (ws or Workspace(dev)).get(need)
    _check(lib().qlr_backward_lora_dAdB(ctypes.byref(qs), _ptr(X), _ptr(dY), _ptr(T_save), _ptr(dT), M, r, int(pooled),
                                        _ptr(dA), _ptr(dB), _ptr(w), w.numel(), _ptr(status), _stream(stream)),
           "qlr_backward_lora_dAdB")
    return dA, dB


def backward_dx(q: QWeight, dY: torch.Tensor, A: torch.Tensor, dT: torch.Tensor, pooled: bool = False,
                dX: Optional[torch.Tensor] = None, accumulate: bool = False, ws: Optional[Workspace] = None,
                status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    M = dY.shape[0]
    r = A.shape[0]
    dev = dY.device
    if dX is None:
        dX = torch.empty((M, q.K), dtype=torch.bfloat16, device=dev)
    qs = q.struct()
    need = lib().qlr_backward_dx_workspace_bytes(ctypes.byref(qs), M, r, int(pooled))
    w = (ws or Workspace(dev)).get(need)
    _check(lib().qlr_backward_dx(ctypes.byref(qs), _ptr(dY), M, _ptr(A), _ptr(dT), r, int(pooled), int(accumulate),
                                 _ptr(dX), _ptr(w), w.numel(), _ptr(status), _stream(stream)), "qlr_backward_dx")
    return dX


def swiglu_forward(G: torch.Tensor, U: torch.Tensor, H: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    if H is None:
        H = torch.empty_like(G)
    _check(lib().qlr_swiglu_forward(_ptr(G), _ptr(U), _ptr(H), G.numel(), _stream(stream)), "qlr_swiglu_forward")
    return H


def swiglu_backward(dH: torch.Tensor, G: torch.Tensor, U: torch.Tensor, dG=None, dU=None, stream=None):
    if dG is None:
        dG = torch.empty_like(G)
    if dU is None:
        dU = torch.empty_like(U)
    _check(lib().qlr_swiglu_backward(_ptr(dH), _ptr(G), _ptr(U), _ptr(dG), _ptr(dU), G.numel(), _stream(stream)),
           "qlr_swiglu_backward")
    return dG, dU
