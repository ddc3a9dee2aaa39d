"""GPU parity of the rank-r products at many tokens (QLoRA explainer, "Background: how LoRA works"):
T_save = bf16(s X A^T) through qlr_lora_down and dT = bf16(s dY B) through qlr_backward_lora_dT, which
at 1024 or more tokens with r = 16, 32 or 64 run as one launch of 4-CTA clusters that split the reduction and sum
their partial tiles in shared memory.  Checked against the fp64 oracle on ragged token counts (not a
multiple of the 64-token tile), a reduction whose split leaves the last CTA of a cluster nothing to do,
and the layer shapes; and run twice for bit-identical results (the partials are summed in a fixed order)."""
import numpy as np
import pytest
import torch

from oracle import layer as OL
from synth import LinearSpec, linear_tensors
from tests.gpu_helpers import DEV, bf16_dev, f32_dev, host
from tests.test_gpu_layer import check_close

pytestmark = [pytest.mark.gpu, pytest.mark.filterwarnings("ignore::RuntimeWarning")]


@pytest.mark.parametrize("r", [16, 32, 64])
@pytest.mark.parametrize("M,N,K", [(1100, 192, 320), (1024, 64, 11008), (2048, 4096, 4096), (1077, 11008, 576)])
def test_rank_r_products_match_the_oracle(cuda_lib, M, N, K, r):
    qlr = cuda_lib
    spec = LinearSpec("w", N, K, "nfk", 4, 64, 256, r=r, s=0.5)
    t = linear_tensors(spec, M, seed=M + N)
    q = qlr.quantize_nf4(f32_dev(t["W"]), 4, 64, 256)
    X, dY, A, B = bf16_dev(t["X"]), bf16_dev(t["dY"]), bf16_dev(t["A"]), bf16_dev(t["B"])
    st = qlr.new_status(DEV)
    T1 = qlr.lora_down(q, X, A, spec.s, status=st)
    dT1 = qlr.backward_lora_dT(q, dY, B, spec.s, status=st)
    T2 = qlr.lora_down(q, X, A, spec.s, status=st)
    dT2 = qlr.backward_lora_dT(q, dY, B, spec.s, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.equal(T1, T2) and torch.equal(dT1, dT2)
    zeros = np.zeros((1, K))
    ref_T = spec.s * OL.forward(t["X"], zeros, t["A"], t["B"][:1], spec.s)["T"]
    ref_dT = OL.backward(t["dY"], t["X"], np.zeros((N, K)), t["A"], t["B"], spec.s)["dT"]
    check_close(host(T1), ref_T, "T")
    check_close(host(dT1), ref_dT, "dT")
