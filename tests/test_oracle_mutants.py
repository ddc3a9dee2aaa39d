"""The oracle's pins catch plausible mistakes: each case plants one mistake in a copy of oracle/ (on
the CPU; the library is not involved) and runs the pin tests of that module against the copy, which
must fail.  A curated subset of a larger check: scale factors dropped, operands transposed, signs
and offsets wrong, rounding rules changed, the wrong matrix factorised, a plan read back in the wrong
order."""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTANTS = [
    ("layer.py", "dB = s * (dY.T @ T)", "dB = (dY.T @ T)", "test_oracle_layer.py"),
    ("layer.py", "dX = dY @ Wdq + (unpool(dTA, L).astype(dtype) if L else dTA)",
     "dX = dY @ Wdq.T + (unpool(dTA, L).astype(dtype) if L else dTA)", "test_oracle_layer.py"),
    ("layer.py", "dG = dH * U * sig * (1.0 + G * (1.0 - sig))", "dG = dH * U * sig * (1.0 - G * (1.0 - sig))",
     "test_oracle_layer.py"),
    ("layer.py", "return X.reshape(M, K // L, L).mean(axis=-1)", "return X.reshape(M, L, K // L).mean(axis=1)",
     "test_oracle_layer.py"),
    ("quantize.py", "idx[c == 0] = zero_index(bits)", "idx[c == 0] = 0", "test_oracle_quantize.py"),
    ("quantize.py", 'return (e4m3_decode(q["c1_fp8"]).astype(np.float32) * s2b).astype(np.float32)',
     'return (e4m3_decode(q["c1_fp8"]).astype(np.float32)).astype(np.float32)', "test_oracle_quantize.py"),
    ("quantize.py", "code = np.where(ok[..., None], np.clip(np.rint(t), 0, 15), 0).astype(np.uint8)",
     "code = np.where(ok[..., None], np.clip(np.floor(t + 0.5), 0, 15), 0).astype(np.uint8)", "test_oracle_quantize.py"),
    ("quantize.py", "return qalora_merged_zero_fp64(q, A, B, s).astype(np.float16)",
     "return qalora_merged_zero_fp64(q, A, B, s).astype(np.float32).astype(np.float16)", "test_oracle_quantize.py"),
    ("codebook.py", "return 1.0 - 0.5 * (1.0 / (2.0 * (n - 1)) + 1.0 / (2.0 * n))",
     "return 1.0 - 0.5 * (1.0 / (2.0 * (n + 1)) + 1.0 / (2.0 * n))", "test_oracle_codebook.py"),
    ("numerics.py", "pick = np.where(tie, np.where(lo % 2 == 0, lo, hi), pick)", "pick = np.where(tie, hi, pick)",
     "test_oracle_numerics.py"),
    ("lqlora.py", "U, S, Vt = np.linalg.svd(W64 - deq, full_matrices=False)",
     "U, S, Vt = np.linalg.svd(W64, full_matrices=False)", "test_oracle_lqlora.py"),
    ("allocation.py", "for i in range(m - 1, -1, -1):", "for i in range(m):", "test_oracle_allocation.py"),
    # the dequantised value's rounding (pinned by literal bf16 ties in test_oracle_dequant_rounding.py)
    ("quantize.py", "return bf16_rn(vals.reshape(-1)[: N * K]).reshape(N, K)", "return vals.reshape(-1)[: N * K].reshape(N, K)",
     "test_oracle_dequant_rounding.py"),
    ("quantize.py", 'vals = levels[q["codes"]].reshape(-1, block) * scales[:, None]   # fp32 * fp32 -> fp32',
     'vals = (levels[q["codes"]].reshape(-1, block) * e4m3_decode(q["c1_fp8"]).astype(np.float32)[:, None])'
     '.astype(np.float32) * np.repeat(q["s2"], q["dq_block"])[: q["c1_fp8"].size][:, None]',
     "test_oracle_dequant_rounding.py"),
    ("quantize.py", "return bf16_rn(v.reshape(-1)).reshape(N, K)", "return v.reshape(N, K)", "test_oracle_dequant_rounding.py"),
    ("quantize.py", "v = (d * sc[..., None]).astype(np.float32)",
     'v = (d.astype(np.float16) * q["scale"][..., None]).astype(np.float32)', "test_oracle_dequant_rounding.py"),
    ("numerics.py", "r = ((u + np.uint64(0x7FFF) + lsb) & np.uint64(0xFFFF0000)).astype(np.uint32)",
     "r = (u & np.uint64(0xFFFF0000)).astype(np.uint32)", "test_oracle_dequant_rounding.py"),
    # LoQA's scale and zero-point gradients (pinned by finite differences and brute force)
    ("loqa.py", "dzero = -np.asarray(scale, np.float64) * Gg.sum(axis=-1)", "dzero = np.asarray(scale, np.float64) * Gg.sum(axis=-1)",
     "test_oracle_loqa.py"),
    ("loqa.py", "dscale = (Gg * (cg - z[..., None])).sum(axis=-1)", "dscale = (Gg * cg).sum(axis=-1)", "test_oracle_loqa.py"),
    ("loqa.py", "Gg = G.reshape(N, K // L, L)", "Gg = G.reshape(N, L, K // L).transpose(0, 2, 1)", "test_oracle_loqa.py"),
]


@pytest.mark.parametrize("module,old,new,tests", MUTANTS, ids=[f"{m[0]}:{i}" for i, m in enumerate(MUTANTS)])
def test_planted_mistake_is_caught(tmp_path, module, old, new, tests):
    for d in ("oracle", "synth", "tests"):
        shutil.copytree(os.path.join(ROOT, d), tmp_path / d, ignore=shutil.ignore_patterns("__pycache__"))
    path = tmp_path / "oracle" / module
    src = path.read_text()
    assert src.count(old) == 1, "the mutated line is no longer in the oracle"
    path.write_text(src.replace(old, new))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider", f"tests/{tests}"],
                       cwd=tmp_path, capture_output=True, text=True, timeout=600)
    assert r.returncode == 1, f"planted mistake not caught:\n{r.stdout[-2000:]}"
