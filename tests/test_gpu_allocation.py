"""LQ-LoRA's budgeted allocation on the GPU: the quantisation error of each option against the
oracle's, and a whole plan (GPU errors, the library's allocator) against the oracle's plan."""
import numpy as np
import pytest
import torch

from oracle import allocation as AL
from oracle import quantize as Q
from synth import random_matrix

from gpu_helpers import DEV, f32_dev

pytestmark = pytest.mark.gpu

OPTIONS = [(k, b) for k in (2, 3, 4) for b in (64, 128)]


@pytest.mark.parametrize("bits,block,dq", [(4, 64, 256), (3, 128, 256), (2, 64, 0), (4, 128, 0)])
def test_quantisation_error_matches_the_oracle(cuda_lib, bits, block, dq):
    W = random_matrix(21, bits, "W", (200, 384), 0.02)
    got = float(cuda_lib.nf_quant_error(f32_dev(W), bits, block, dq).item())
    ref = AL.squared_error(W, Q.dequant_nfk(Q.quantize_nfk(W, bits, block, dq)))
    assert abs(got - ref) <= 1e-9 * ref


def test_plan_for_a_small_stack_matches_the_oracle(cuda_lib):
    shapes = [(256, 512), (512, 256), (128, 1024), (384, 384), (256, 768), (640, 128)]
    sigmas = [0.02, 0.05, 0.01, 0.03, 0.02, 0.04]
    mats = [random_matrix(31, i, "W", s, sg) for i, (s, sg) in enumerate(zip(shapes, sigmas))]
    err_gpu = np.zeros((len(mats), len(OPTIONS)))
    err_ref = np.zeros_like(err_gpu)
    cost = np.zeros(err_gpu.shape, dtype=np.int64)
    for i, W in enumerate(mats):
        Wd = f32_dev(W)
        for o, (k, b) in enumerate(OPTIONS):
            err_gpu[i, o] = float(cuda_lib.nf_quant_error(Wd, k, b, 256).item())
            err_ref[i, o] = AL.squared_error(W, Q.dequant_nfk(Q.quantize_nfk(W, k, b, 256)))
            cost[i, o] = AL.nf_cost_bits(W.shape[0], W.shape[1], k, b, 256)
    torch.cuda.synchronize()
    assert np.all(np.abs(err_gpu - err_ref) <= 1e-9 * err_ref)
    params = sum(W.size for W in mats)
    budget = int(3.0 * params)  # 3 bits per parameter on average, constants included
    choice, total = cuda_lib.lqlora_allocate(err_gpu, cost, budget, 64)
    ref_choice, ref_total = AL.allocate(err_ref, cost, budget, 64)
    assert choice == ref_choice
    assert abs(total - ref_total) <= 1e-9 * ref_total
    # the plan spends the budget where it buys the most: no worse than the best single option that fits
    uniform = [o for o in range(len(OPTIONS)) if cost[:, o].sum() <= budget]
    assert total <= min(err_ref[:, o].sum() for o in uniform) + 1e-12
