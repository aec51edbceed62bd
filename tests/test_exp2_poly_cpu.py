"""The scoring epilogue's FMA-pipe 2^x against exp2 in fp64 (CPU emulation of the kernel's fp32 steps).

The score kernel computes a share of its exponentials as 2^n * p(f) (n = round(x), f = x - n, p a degree-5
minimax polynomial) instead of on the MUFU unit.  Both kinds must agree with 2^x to well within the 1e-4
relative ranking band of the kept sets, so the polynomial's constants are read from the kernel source and its
arithmetic replayed here in fp32 (fused multiply-adds emulated in fp64 and rounded once): the relative error must
stay below 3e-7 over the whole argument range the kernel can see.
"""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "agent_kv_cache_lse_b200", "csrc", "score_tc.cu")


def _coefficients():
    with open(SRC) as f:
        text = f.read()
    body = text[text.index("float2 exp2_fma2(float2 x)"):]
    body = body[:body.index("\n}\n")]
    found = dict(re.findall(r"kC(\d) = ([0-9.eE+-]+)f", body))
    return [np.float32(float(found[str(i)])) for i in range(len(found))]


def _fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_poly32(x):
    c = _coefficients()
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    k_round = np.float32(12582912.0)
    t = (x + k_round).astype(np.float32)
    n = (t - k_round).astype(np.float32)
    f = _fma32(n, np.float32(-1.0) * np.ones_like(n), x)
    p = np.full_like(f, c[-1])
    for ci in c[-2::-1]:
        p = _fma32(p, f, np.full_like(f, ci))
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.astype(np.int32).view(np.float32)


def test_polynomial_degree_and_error_bound():
    c = _coefficients()
    assert len(c) == 6
    x = np.concatenate([np.linspace(-126.0, 30.0, 2_000_001, dtype=np.float32),
                        np.linspace(-1.0, 1.0, 200_001, dtype=np.float32)])
    got = exp2_poly32(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 3e-7, rel.max()


def test_absent_column_contributes_a_negligible_amount():
    """-inf (an absent column's -lse) clamps to 2^-126, far below any score tolerance."""
    v = exp2_poly32(np.array([-np.inf, -500.0], dtype=np.float32)).astype(np.float64)
    assert np.all(v > 0) and np.all(v < 1.2e-38 * 1.01)
