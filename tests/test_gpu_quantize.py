"""GPU parity of the quantisers, dequantiser and merge: bit-exact against the oracle."""
import numpy as np
import pytest
import torch

from oracle import quantize as Q
from oracle.numerics import bf16_bits
from synth import random_matrix, linear_tensors, workload
from tests.gpu_helpers import DEV, bf16_dev, f32_dev, host, host_bytes

pytestmark = [pytest.mark.gpu, pytest.mark.filterwarnings("ignore::RuntimeWarning")]


def _compare_nf(q_gpu, q_ref, rows=None):
    n_codes_bytes = q_ref["packed"].size
    np.testing.assert_array_equal(host_bytes(q_gpu.codes)[:n_codes_bytes], q_ref["packed"])
    if q_ref["dq_block"]:
        nb = q_ref["c1_fp8"].size
        np.testing.assert_array_equal(host_bytes(q_gpu.c1_fp8)[:nb], q_ref["c1_fp8"])
        np.testing.assert_array_equal(host(q_gpu.s2)[: q_ref["s2"].size].view(np.uint32), q_ref["s2"].view(np.uint32))
    else:
        np.testing.assert_array_equal(host(q_gpu.c1)[: q_ref["c1"].size].view(np.uint32), q_ref["c1"].view(np.uint32))


@pytest.mark.parametrize("bits,block,dq", [(4, 64, 256), (4, 128, 256), (4, 64, 0), (3, 64, 256), (3, 128, 0),
                                           (2, 64, 256), (2, 128, 256)])
@pytest.mark.parametrize("shape", [(256, 256), (96, 640), (40, 128 * 70)])
def test_nf_quantize_bit_exact(cuda_lib, bits, block, dq, shape):
    qlr = cuda_lib
    W = random_matrix(21, bits * 1000 + block + dq, "W", shape, 0.02)
    W[3, :block] = 0.0                      # a zero block
    W[5, 7] = 0.5                           # an outlier
    ref = Q.quantize_nfk(W, bits, block, dq)
    q = qlr.quantize_nf4(f32_dev(W), bits, block, dq)
    torch.cuda.synchronize()
    _compare_nf(q, ref)
    Wd = qlr.dequant(q)
    np.testing.assert_array_equal(bf16_bits(host(Wd)), bf16_bits(Q.dequant_nfk(ref)))


def test_nf_quantize_full_size_decode_projection(cuda_lib):
    """28672 x 8192 (the 70B-like decode projection): codes, constants and dequant checked on
    whole double-quantisation groups of sampled rows (2 rows per group at K = 8192)."""
    qlr = cuda_lib
    spec = workload("decode70b").linears[0]
    W = random_matrix(0, 0, "W", (spec.N, spec.K), spec.sigma_w)
    q = qlr.quantize_nf4(f32_dev(W), 4, 64, 256)
    Wd = qlr.dequant(q)
    torch.cuda.synchronize()
    codes = host_bytes(q.codes)
    c8 = host_bytes(q.c1_fp8)
    s2 = host(q.s2)
    wd = Wd.view(torch.int16)
    rng = np.random.default_rng(5)
    for r0 in sorted(rng.choice(spec.N // 2, 24, replace=False) * 2):
        sub = W[r0:r0 + 2]
        ref = Q.quantize_nfk(sub, 4, 64, 256)
        b0 = r0 * spec.K // 2
        np.testing.assert_array_equal(codes[b0:b0 + ref["packed"].size], ref["packed"])
        blk0 = r0 * spec.K // 64
        np.testing.assert_array_equal(c8[blk0:blk0 + ref["c1_fp8"].size], ref["c1_fp8"])
        assert s2[blk0 // 256] == ref["s2"][0]
        got = wd[r0:r0 + 2].cpu().numpy().view(np.uint16)
        np.testing.assert_array_equal(got, bf16_bits(Q.dequant_nfk(ref)))


def test_nf_quantize_reports_nonfinite(cuda_lib):
    qlr = cuda_lib
    W = random_matrix(22, 0, "W", (64, 256), 0.02)
    W[10, 10] = np.inf
    st = qlr.new_status(DEV)
    qlr.quantize_nf4(f32_dev(W), 4, 64, 256, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == -5


@pytest.mark.parametrize("group", [32, 64, 128])
@pytest.mark.parametrize("shape", [(64, 256), (40, 384), (4096, 4096)])
def test_int4_group_quantize_bit_exact(cuda_lib, group, shape):
    qlr = cuda_lib
    W = random_matrix(23, group, "W", shape, 0.02)
    W[0, :group] = 0.0
    W[1, group:2 * group] = np.abs(W[1, group:2 * group])
    ref = Q.quantize_int4_group(W, group)
    q = qlr.quantize_int4_group(f32_dev(W), group)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_bytes(q.codes), ref["packed"])
    np.testing.assert_array_equal(q.scale.cpu().numpy().view(np.uint16), ref["scale"].view(np.uint16))
    np.testing.assert_array_equal(q.zero.cpu().numpy().view(np.uint16), ref["zero"].view(np.uint16))
    Wd = qlr.dequant(q)
    np.testing.assert_array_equal(bf16_bits(host(Wd)), bf16_bits(Q.dequant_int4_group(ref)))


def test_int4_group_quantize_ties_bit_exact(cuda_lib):
    # values at exact k + 1/2 steps of a 0.0625 scale: both sides round code and zero point half to even
    qlr = cuda_lib
    s = 0.0625
    W = random_matrix(24, 0, "W", (8, 128), 0.02)
    W[0, :32] = 0.0
    W[0, :5] = [15 * s, 0.5 * s, 1.5 * s, 2.5 * s, 3.5 * s]
    W[1, :32] = 0.0
    W[1, :4] = [-2.5 * s, 12.5 * s, 0.5 * s, 1.5 * s]
    ref = Q.quantize_int4_group(W, 32)
    q = qlr.quantize_int4_group(f32_dev(W), 32)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_bytes(q.codes), ref["packed"])
    np.testing.assert_array_equal(q.scale.cpu().numpy().view(np.uint16), ref["scale"].view(np.uint16))
    np.testing.assert_array_equal(q.zero.cpu().numpy().view(np.uint16), ref["zero"].view(np.uint16))


def test_qalora_merge_bit_exact_and_lossless(cuda_lib):
    qlr = cuda_lib
    wl = workload("qalora")
    spec = wl.linears[0]
    t = linear_tensors(spec, 64, seed=0)
    ref = Q.quantize_int4_group(t["W"], spec.group)
    q = qlr.quantize_int4_group(f32_dev(t["W"]), spec.group)
    qlr.qalora_merge(q, bf16_dev(t["A"]), bf16_dev(t["B"]), spec.s)
    torch.cuda.synchronize()
    zp = Q.qalora_merge(ref, t["A"], t["B"], spec.s)
    np.testing.assert_array_equal(q.zero.cpu().numpy().view(np.uint16), zp.view(np.uint16))
    Wd = qlr.dequant(q)
    np.testing.assert_array_equal(bf16_bits(host(Wd)), bf16_bits(Q.dequant_int4_group(ref, zero=zp)))


def _nf_tie_inputs(bits: int, per_pair: int = 6) -> np.ndarray:
    """fp32 values u between each pair of adjacent levels a < b at the switch from the lower to the upper
    level: every u whose fp32 distances to a and b are equal (the oracle keeps the lower index), and the
    last u nearer a and the first u nearer b, found by scanning the fp32 neighbours of the midpoint."""
    from oracle.codebook import nf_codebook_f32
    lev = nf_codebook_f32(bits)
    out = []
    for a, b in zip(lev[:-1], lev[1:]):
        mid = np.float32((np.float64(a) + np.float64(b)) / 2)
        base = int(np.array([mid]).view(np.int32)[0])
        u = np.arange(base - 512, base + 513, dtype=np.int64).astype(np.int32).view(np.float32)
        u = np.unique(u[(u > a) & (u < b)])
        da = np.abs((u - a).astype(np.float32))
        db = np.abs((u - b).astype(np.float32))
        out.extend(u[da == db][:per_pair].tolist())
        below, above = u[da < db], u[da > db]
        out.extend([below.max(), above.min()])
    return np.array(out, np.float32)


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("block,dq", [(64, 256), (128, 0)])
def test_nf_quantize_ties_bit_exact(cuda_lib, bits, block, dq):
    """Inputs exactly between two levels in fp32 distance: the GPU's level search must keep the lower index,
    as the oracle's first-index argmin does.  Blocks with absmax 1 (u = w exactly) and blocks scaled by
    0.8125 and 3.0 (the division decides which side the quotient falls)."""
    qlr = cuda_lib
    ties = _nf_tie_inputs(bits)
    assert ties.size >= 2 * (2 ** bits - 1)
    rows = []
    for c1 in (1.0, 0.8125, 3.0):
        for start in range(0, ties.size, block - 1):
            blk = np.zeros(block, np.float32)
            seg = (ties[start:start + block - 1] * np.float32(c1)).astype(np.float32)
            blk[0] = np.float32(c1)              # the block's absmax
            blk[1:1 + seg.size] = seg
            rows.append(blk)
    W = np.concatenate(rows)
    W = np.concatenate([W, np.zeros((-W.size) % 256, np.float32)]).reshape(-1, 256)
    ref = Q.quantize_nfk(W, bits, block, dq)
    q = qlr.quantize_nf4(f32_dev(W), bits, block, dq)
    torch.cuda.synchronize()
    _compare_nf(q, ref)


def _ulp_neighbours(x: np.ndarray, width: int) -> np.ndarray:
    """x and its fp32 neighbours up to `width` ulps either side (same sign)."""
    b = np.asarray(x, np.float32).view(np.int32).astype(np.int64)
    out = np.concatenate([(b + d) for d in range(-width, width + 1)])
    out = out[(out >= -2 ** 31) & (out < 2 ** 31)].astype(np.int32).view(np.float32)
    return out[np.isfinite(out)]


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("block", [64, 128])
def test_nf_quantize_random_divisors_at_switch_points(cuda_lib, bits, block):
    """Quotients fp32(w / absmax) within two ulps of every switch of the oracle's code, for absmax drawn
    log-uniformly over [1e-4, 10] and at both ends of the quantiser's one-reciprocal-per-block division
    (2^-64, 2^64) and past them (2^-70, 2^70, plain division): every quotient that decides a code must be
    the correctly rounded fp32 one, as in the oracle."""
    qlr = cuda_lib
    sw = _nf_tie_inputs(bits)
    rng = np.random.default_rng(100 + bits)
    ms = list((10.0 ** rng.uniform(-4, 1, 24)).astype(np.float32))
    ms += [np.float32(v) for v in (2.0 ** -64, 2.0 ** -64 * (1 + 2.0 ** -23), 2.0 ** 64, 2.0 ** 64 * (1 - 2.0 ** -24),
                                   2.0 ** -70, 2.0 ** 70, 1.9999999 * 2.0 ** -64)]
    rows = []
    for m in ms:
        x = _ulp_neighbours((sw.astype(np.float64) * np.float64(m)).astype(np.float32), 2)
        x = x[np.abs(x) <= m]
        for start in range(0, x.size, block - 1):
            blk = np.zeros(block, np.float32)
            seg = x[start:start + block - 1]
            blk[0] = m
            blk[1:1 + seg.size] = seg
            rows.append(blk)
    W = np.concatenate(rows)
    W = np.concatenate([W, np.zeros((-W.size) % 256, np.float32)]).reshape(-1, 256)
    ref = Q.quantize_nfk(W, bits, block, 256)
    q = qlr.quantize_nf4(f32_dev(W), bits, block, 256)
    torch.cuda.synchronize()
    _compare_nf(q, ref)


def test_int4_group_quantize_random_scales_at_half_steps(cuda_lib):
    """Inputs whose fp32 quotient x / scale plus the zero point lands within an ulp of k + 1/2, for groups
    with random ranges (log-uniform over [1e-3, 10] either side of zero, or one-sided), and a group whose
    fp16 scale overflows: the quantiser's one-reciprocal-per-group division must give the oracle's codes."""
    qlr = cuda_lib
    rng = np.random.default_rng(7)
    groups = []
    for gi in range(96):
        a, b = (10.0 ** rng.uniform(-3, 1, 2)).astype(np.float32)
        lo, hi = (np.float32(-a), np.float32(b)) if gi % 3 else ((np.float32(0.0), np.float32(b)) if gi % 2
                                                                  else (np.float32(-a), np.float32(0.0)))
        probe = np.zeros((1, 32), np.float32)
        probe[0, 0], probe[0, 1] = lo, hi
        pr = Q.quantize_int4_group(probe, 32)
        sc = np.float64(pr["scale"].reshape(-1)[0].astype(np.float32))
        z = np.float64(pr["zero"].reshape(-1)[0].astype(np.float32))
        if sc == 0:
            continue
        ks = np.arange(0, 15, dtype=np.float64)
        x = _ulp_neighbours(((ks + 0.5 - z) * sc).astype(np.float32), 1)
        x = x[(x >= lo) & (x <= hi)]
        for start in range(0, x.size, 30):
            g = np.zeros(32, np.float32)
            g[0], g[1] = lo, hi
            seg = x[start:start + 30]
            g[2:2 + seg.size] = seg
            groups.append(g)
    big = np.zeros(32, np.float32)
    big[0], big[1], big[2], big[3] = -2.0 ** 66, 2.0 ** 65, 3.0, -1e20
    groups.append(big)
    W = np.stack(groups)
    W = np.concatenate([W, np.zeros(((-W.shape[0]) % 4, 32), np.float32)]).reshape(-1, 128)
    ref = Q.quantize_int4_group(W, 32)
    q = qlr.quantize_int4_group(f32_dev(W), 32)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_bytes(q.codes), ref["packed"])
    np.testing.assert_array_equal(q.scale.cpu().numpy().view(np.uint16), ref["scale"].view(np.uint16))
    np.testing.assert_array_equal(q.zero.cpu().numpy().view(np.uint16), ref["zero"].view(np.uint16))
