"""Seeded synthetic inputs shared by the oracle, the tests, the smoke run and the bench.

This module draws random numbers and rounds bf16 inputs to bf16; it holds no
arithmetic of the method itself (no quantiser, no codebook, no GEMM). The
workloads follow the five layer shapes the quantised-base + LoRA pages and
their benchmark table describe:

* ``tiny``      one 256x256 layer, NF4 block 64 with double quantisation, r=8, s=2, 16 tokens
* ``qalora``    one 4096x4096 layer, INT4 group 32, pooled adapter r=16, s=1, 2048 tokens
* ``mlp7b``     LLaMA-7B MLP block (gate/up 11008x4096, down 4096x11008), NF4+DQ, r=64, s=0.25, 4096 tokens
* ``decode70b`` one 28672x8192 projection, NF4+DQ, r=64, s=0.25, 1/4/16 tokens, forward only
* ``lqlora``    32 layers x 7 linears of a 7B model, per-matrix NF-k (k in {2,3,4}) and block (64/128)
                drawn from the seed, r=64, s=0.25, 2048 tokens

Value distributions: W ~ N(0, sigma_W^2) in fp32; A, B ~ N(0, 0.01^2); X and dY ~ N(0, 1);
A, B, X, dY are rounded to bf16 (round-to-nearest-even) because the layer consumes
them in bf16.  Every tensor has its own numpy ``SeedSequence`` sub-stream
``[seed, matrix_index, tensor_id]`` with tensor ids W=0, A=1, B=2, X=3, dY=4, so any
single tensor can be regenerated without drawing the others.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Tuple

import numpy as np

TENSOR_ID = {"W": 0, "A": 1, "B": 2, "X": 3, "dY": 4, "kb": 5}


def rng_for(seed: int, matrix_index: int, tensor: str) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([seed, matrix_index, TENSOR_ID[tensor]]))


def to_bf16_values(a: np.ndarray) -> np.ndarray:
    """Round an fp32 array to the nearest bf16 value (ties to even); returns fp32."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def normal(seed: int, matrix_index: int, tensor: str, shape: Tuple[int, ...], sigma: float,
           bf16: bool) -> np.ndarray:
    g = rng_for(seed, matrix_index, tensor)
    a = g.standard_normal(size=shape, dtype=np.float32)
    if sigma != 1.0:
        a *= np.float32(sigma)
    return to_bf16_values(a) if bf16 else a


@dataclasses.dataclass(frozen=True)
class LinearSpec:
    """One quantised linear: W is [N, K] (out x in), A is [r, K_a], B is [N, r]."""

    name: str
    N: int
    K: int
    fmt: str                 # "nfk" or "int4g"
    bits: int = 4            # NF-k bit width
    block: int = 64          # NF-k first-level block (consecutive weights, row-major)
    dq_block: int = 256      # double-quantisation group of first-level constants (0: off)
    group: int = 32          # INT4 group length along K (QA-LoRA)
    r: int = 8
    s: float = 1.0
    sigma_w: float = 0.02
    pooled: bool = False     # QA-LoRA: adapter sees the group mean of the input

    @property
    def k_adapter(self) -> int:
        return self.K // self.group if self.pooled else self.K


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    M: int                          # tokens per step
    linears: Tuple[LinearSpec, ...]
    kind: str                       # "single", "mlp", "decode", "stack"
    token_counts: Tuple[int, ...] = ()
    description: str = ""


def _tiny() -> Workload:
    return Workload("tiny", 16, (LinearSpec("w", 256, 256, "nfk", 4, 64, 256, r=8, s=2.0),),
                    "single", description="NF4 256x256, block 64, DQ 256, r=8, s=2, 16 tokens")


def _qalora() -> Workload:
    return Workload("qalora", 2048,
                    (LinearSpec("w", 4096, 4096, "int4g", group=32, r=16, s=1.0, pooled=True),),
                    "single", description="INT4 group 32 4096x4096, pooled adapter r=16, s=1, 2048 tokens")


def _mlp7b() -> Workload:
    s = 16.0 / 64.0
    return Workload("mlp7b", 4096, (
        LinearSpec("gate", 11008, 4096, "nfk", 4, 64, 256, r=64, s=s),
        LinearSpec("up", 11008, 4096, "nfk", 4, 64, 256, r=64, s=s),
        LinearSpec("down", 4096, 11008, "nfk", 4, 64, 256, r=64, s=s),
    ), "mlp", description="LLaMA-7B MLP, NF4+DQ, r=64, s=16/64, SwiGLU, 4096 tokens")


def _decode70b() -> Workload:
    return Workload("decode70b", 16, (LinearSpec("w", 28672, 8192, "nfk", 4, 64, 256, r=64, s=0.25,
                                                 sigma_w=0.015),),
                    "decode", token_counts=(1, 4, 16),
                    description="NF4+DQ 28672x8192 projection, r=64, s=0.25, forward at 1/4/16 tokens")


LQ_SHAPES = (("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
             ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008))


def lqlora_choices(seed: int, layers: int = 32) -> List[Tuple[int, int]]:
    """Per-matrix (bits, block) for the mixed stack, drawn uniformly from the seed, layer-major."""
    g = rng_for(seed, 0, "kb")
    n = layers * len(LQ_SHAPES)
    bits = g.choice(np.array([2, 3, 4]), size=n)
    blocks = g.choice(np.array([64, 128]), size=n)
    return [(int(b), int(k)) for b, k in zip(bits, blocks)]


def _lqlora(seed: int = 0, layers: int = 32) -> Workload:
    ch = lqlora_choices(seed, layers)
    lins = []
    for layer in range(layers):
        for j, (nm, n, k) in enumerate(LQ_SHAPES):
            bits, block = ch[layer * len(LQ_SHAPES) + j]
            lins.append(LinearSpec(f"L{layer}.{nm}", n, k, "nfk", bits, block, 256, r=64, s=0.25))
    return Workload("lqlora", 2048, tuple(lins), "stack",
                    description="32-layer 7B stack, per-matrix NF-k (k in 2,3,4) and block (64/128), r=64, 2048 tokens")


def workload(name: str, seed: int = 0) -> Workload:
    if name == "tiny":
        return _tiny()
    if name == "qalora":
        return _qalora()
    if name == "mlp7b":
        return _mlp7b()
    if name == "decode70b":
        return _decode70b()
    if name == "lqlora":
        return _lqlora(seed)
    raise KeyError(name)


WORKLOADS = ("tiny", "qalora", "mlp7b", "decode70b", "lqlora")


def linear_tensors(spec: LinearSpec, M: int, seed: int = 0, matrix_index: int = 0,
                   with_x: bool = True, with_dy: bool = True, M_x: Optional[int] = None) -> Dict[str, np.ndarray]:
    """W (fp32), A, B (bf16 values), X [M, K] and dY [M, N] (bf16 values) for one linear."""
    out = {
        "W": normal(seed, matrix_index, "W", (spec.N, spec.K), spec.sigma_w, bf16=False),
        "A": normal(seed, matrix_index, "A", (spec.r, spec.k_adapter), 0.01, bf16=True),
        "B": normal(seed, matrix_index, "B", (spec.N, spec.r), 0.01, bf16=True),
    }
    if with_x:
        out["X"] = normal(seed, matrix_index, "X", (M if M_x is None else M_x, spec.K), 1.0, bf16=True)
    if with_dy:
        out["dY"] = normal(seed, matrix_index, "dY", (M, spec.N), 1.0, bf16=True)
    return out


def random_matrix(seed: int, matrix_index: int, tensor: str, shape, sigma: float = 1.0,
                  bf16: bool = False) -> np.ndarray:
    """A free-form seeded draw for tests (edge shapes, ragged tails)."""
    return normal(seed, matrix_index, tensor, tuple(shape), sigma, bf16)
