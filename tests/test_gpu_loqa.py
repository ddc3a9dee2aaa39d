"""GPU parity of the LoQA scale and zero-point gradients (LoQA abstract, read on the group-wise INT4 format)
against the fp64 oracle: relative Frobenius error and per-row bounds, on ragged shapes (rows, inputs and
tokens that do not fill a tile), every group length, merged (non-integer) zero points, no tokens, and the
full QA-LoRA layer."""
import numpy as np
import pytest
import torch

from oracle import loqa as LQ
from oracle import quantize as Q
from synth import LinearSpec, linear_tensors, workload
from tests.gpu_helpers import DEV, bf16_dev, f32_dev, host
from tests.test_gpu_layer import check_close

pytestmark = [pytest.mark.gpu, pytest.mark.filterwarnings("ignore::RuntimeWarning")]


def _run(qlr, spec, M, seed, merge=False):
    t = linear_tensors(spec, M, seed=seed)
    ref = Q.quantize_int4_group(t["W"], spec.group)
    q = qlr.quantize_int4_group(f32_dev(t["W"]), spec.group)
    zero = ref["zero"]
    if merge:  # zero points after a QA-LoRA merge are fp16 values off the integer grid
        A = t["A"]
        qlr.qalora_merge(q, bf16_dev(A), bf16_dev(t["B"]), 4.0)
        zero = Q.qalora_merge(ref, A, t["B"], 4.0)
    st = qlr.new_status(DEV)
    dS, dZ = qlr.loqa_grad(q, bf16_dev(t["X"]), bf16_dev(t["dY"]), status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    np.testing.assert_array_equal(q.zero.cpu().numpy().view(np.uint16), zero.view(np.uint16))
    g = LQ.scale_zero_grads(t["X"], t["dY"], ref["codes"].reshape(spec.N, spec.K), ref["scale"], zero, spec.group)
    check_close(host(dS), g["dscale"], "dscale")
    check_close(host(dZ), g["dzero"], "dzero")


@pytest.mark.parametrize("group", [32, 64, 128])
@pytest.mark.parametrize("M", [1, 64, 300])
def test_loqa_grad_ragged(cuda_lib, group, M):
    spec = LinearSpec("w", 264, 384, "int4g", group=group, r=16, s=1.0, pooled=True)
    _run(cuda_lib, spec, M, seed=group + M)


def test_loqa_grad_merged_zero_points(cuda_lib):
    spec = LinearSpec("w", 520, 640, "int4g", group=32, r=16, s=1.0, pooled=True)
    _run(cuda_lib, spec, 200, seed=3, merge=True)


def test_loqa_grad_several_tiles_per_cta(cuda_lib):
    # 48 row tiles x 12 input tiles = 576 tiles on at most 148 persistent CTAs: both accumulators in turn
    spec = LinearSpec("w", 6144, 3072, "int4g", group=64, r=16, s=1.0, pooled=True)
    _run(cuda_lib, spec, 256, seed=9)


def test_loqa_grad_no_tokens(cuda_lib):
    qlr = cuda_lib
    spec = LinearSpec("w", 128, 256, "int4g", group=32, r=16, s=1.0, pooled=True)
    t = linear_tensors(spec, 4, seed=1)
    q = qlr.quantize_int4_group(f32_dev(t["W"]), 32)
    X = torch.empty((0, 256), dtype=torch.bfloat16, device=DEV)
    dY = torch.empty((0, 128), dtype=torch.bfloat16, device=DEV)
    dS = torch.full((128, 8), float("nan"), device=DEV)
    dZ = torch.full((128, 8), float("nan"), device=DEV)
    qlr.loqa_grad(q, X, dY, dscale=dS, dzero=dZ)
    torch.cuda.synchronize()
    assert float(dS.abs().sum()) == 0 and float(dZ.abs().sum()) == 0


def test_loqa_grad_qalora_full_size(cuda_lib):
    wl = workload("qalora")
    _run(cuda_lib, wl.linears[0], wl.M, seed=0)
