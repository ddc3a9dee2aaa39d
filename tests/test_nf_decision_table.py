"""Host pin of the NF-k quantiser's nearest-level decision table (qlr_nf_decision_table) against the
oracle's rule (QLoRA explainer, "Background: what is quantization?": first index of the smallest fp32
|u - level|).  The table is host arithmetic, so this runs without a GPU: every u in the fp32
neighbourhoods of the level midpoints, of the table's thresholds and of the cell boundaries, plus random
draws and the special values, must get the oracle's code from code = base[k] + (u >= threshold[k]) with
k = round-half-even(16 u) + 16."""
import numpy as np
import pytest

from oracle import quantize as Q
from oracle.codebook import nf_codebook_f32


def _neighbours(v: float, width: int) -> np.ndarray:
    b = int(np.array([np.float32(v)]).view(np.int32)[0])
    if b < 0:  # negative floats: walk the magnitude bits
        mag = b & 0x7FFFFFFF
        bits = np.arange(max(mag - width, 0), mag + width + 1, dtype=np.int64) | 0x80000000
        return bits.astype(np.uint32).view(np.float32)
    return np.arange(max(b - width, 0), b + width + 1, dtype=np.int64).astype(np.uint32).view(np.float32)


def _table_codes(u: np.ndarray, t, base) -> np.ndarray:
    k = (np.rint(u.astype(np.float64) * 16.0) + 16).astype(np.int64)  # exact: 16 u is exact in fp64
    assert k.min() >= 0 and k.max() <= 32
    thr = np.asarray(t, np.float32)[k]
    return np.asarray(base, np.int64)[k] + (u >= thr)


def _oracle_codes(u: np.ndarray, bits: int) -> np.ndarray:
    # the oracle's blockwise rule with an absmax of 1: fp32(u / 1) = u
    return Q.nf_codes(u.reshape(-1, 1), np.ones(u.size, np.float32), bits).reshape(-1).astype(np.int64)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_decision_table_matches_the_rule(bits):
    from quantized_base_lora_nf4_b200 import qlr
    t, base = qlr.nf_decision_table(bits)
    lev = nf_codebook_f32(bits)
    pts = []
    for a, b in zip(lev[:-1], lev[1:]):
        pts.append(_neighbours((float(a) + float(b)) / 2, 2048))
    for x in t:
        if np.isfinite(x):
            pts.append(_neighbours(x, 256))
    for k in range(34):
        pts.append(_neighbours((k - 16.5) / 16.0, 256))
    rng = np.random.default_rng(bits)
    pts.append(rng.uniform(-1, 1, 200_000).astype(np.float32))
    pts.append(np.array([-1.0, 1.0, 0.0, -0.0, *lev.tolist()], np.float32))
    u = np.concatenate(pts).astype(np.float32)
    u = u[(u >= -1) & (u <= 1)]
    np.testing.assert_array_equal(_table_codes(u, t, base), _oracle_codes(u, bits))
    # one threshold per code change, in increasing order
    finite = [x for x in t if np.isfinite(x)]
    assert len(finite) == 2 ** bits - 1 and finite == sorted(finite)


def test_decision_table_rejects_bad_bits():
    from quantized_base_lora_nf4_b200 import qlr
    with pytest.raises(qlr.QLRError):
        qlr.nf_decision_table(5)
