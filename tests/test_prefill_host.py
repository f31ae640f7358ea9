"""Host-side checks of the prefill kernel's constants (no GPU)."""

import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _poly():
    src = open(os.path.join(ROOT, "mla_latent_kv_35_b200", "csrc", "common.cuh")).read()
    m = re.search(r"kExp2Poly\[4\]\s*=\s*\{([^}]*)\}", src)
    assert m, "kExp2Poly not found"
    return [np.float32(float(x.strip().rstrip("f"))) for x in m.group(1).split(",")]


def test_exp2_polynomial_relative_error():
    """The cubic that stands in for 2^f on [-1/2, 1/2], evaluated in fp32
    Horner form as the kernel does, is within 1e-4 of 2^f in relative terms
    (bf16 rounding of P is 2^-9)."""
    c = _poly()
    f = np.linspace(-0.5, 0.5, 100001).astype(np.float32)
    p = np.float32(c[3])
    for i in (2, 1, 0):
        p = (p * f + c[i]).astype(np.float32)
    rel = np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)
    assert rel.max() < 1e-4


def test_exp2_range_reduction():
    """x = n + f with n from the low mantissa bits of x + 1.5 * 2^23, exactly,
    over the clamped range [-125, 9]; the reassembled 2^x stays normal."""
    c = _poly()
    x = np.linspace(-125.0, 9.0, 200001).astype(np.float32)
    t = (x + np.float32(12582912.0)).astype(np.float32)
    n = (t - np.float32(12582912.0)).astype(np.float32)
    assert np.array_equal(n, np.rint(x))
    f = (x - n).astype(np.float32)
    assert np.abs(f).max() <= 0.5
    j = t.view(np.int32) - 0x4B400000
    assert np.array_equal(j, np.rint(x).astype(np.int32))
    p = np.float32(c[3])
    for i in (2, 1, 0):
        p = (p * f + c[i]).astype(np.float32)
    out = ((p.view(np.uint32) + (j.astype(np.uint32) << np.uint32(23))).astype(np.uint32)
           ).view(np.float32)
    rel = np.abs(out.astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 1e-4
    assert np.all(out > 0) and np.all(np.isfinite(out))
