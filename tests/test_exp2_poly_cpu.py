"""The FMA-pipe 2^x of the selection kernel (`exp2_fma2` in csrc/sm100.cuh), emulated step for step
in fp32 on the CPU: its largest relative error over the arguments the selection feeds it must stay
inside the 2^-22 that the certified selection band budgets for an exponential.

The coefficients are read from the header, so the check is of the constants that ship.  The fused
multiply-adds are emulated as an exact fp64 product plus the addend, rounded once to fp32 (exact
for these operand sizes but for a rare double rounding, which the bound's margin covers).
"""

import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "free_sparse_attention_reuse_b200", "csrc", "sm100.cuh")


def _coefficients():
    src = open(HEADER).read()
    body = src[src.index("float2 exp2_fma2(float2 x)"):]
    body = body[:body.index("return make_float2")]
    vals = dict(re.findall(r"\b(c[0-5]) = ([0-9.eE+-]+)f", body))
    return [np.float32(float(vals[f"c{i}"])) for i in range(6)]


def _fma32(a, b, c):
    return np.float32(np.float64(a) * np.float64(b) + np.float64(c))


def _round_down32(v64):
    r = np.float32(v64)
    if np.float64(r) > v64:
        r = np.nextafter(r, np.float32(-np.inf))
    return r


def exp2_fma2_emulated(xs, c):
    out = np.empty(len(xs), dtype=np.float64)
    magic = np.float32(12582912.0)
    for i, x in enumerate(np.asarray(xs, dtype=np.float32)):
        x = np.float32(min(max(x, np.float32(-126.0)), np.float32(126.0)))
        t = _round_down32(np.float64(x) + np.float64(magic))   # floor(x) + 1.5 * 2^23
        n = np.float32(np.float64(t) - np.float64(magic))
        f = np.float32(np.float64(x) - np.float64(n))
        q = _fma32(c[5], f, c[4])
        for k in (3, 2, 1, 0):
            q = _fma32(q, f, c[k])
        ti = np.array([t], dtype=np.float32).view(np.int32)[0].astype(np.int64)
        qi = np.array([q], dtype=np.float32).view(np.int32)[0].astype(np.int64)
        bits = (qi + ((ti << 23) & 0xFFFFFFFF)) & 0xFFFFFFFF
        out[i] = np.array([bits], dtype=np.uint32).view(np.float32)[0]
    return out


def test_exp2_fma2_within_the_exponential_budget():
    c = _coefficients()
    rng = np.random.default_rng(3)
    xs = np.concatenate([np.linspace(-126.0, 0.0, 40001), -30.0 * rng.random(20000), [0.0, -1.0, -0.5, -125.75]])
    got = exp2_fma2_emulated(xs, c)
    ref = np.exp2(np.asarray(xs, dtype=np.float32).astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 2.0 ** -22, rel.max()


def test_exp2_fma2_exact_at_integers_and_clamped():
    c = _coefficients()
    got = exp2_fma2_emulated([-3.0, -10.0, -126.0, -200.0, 0.0], c)
    # p(0) = c0 is within 2^-23 of 1; integers scale it exactly; below -126 the clamp holds
    assert np.allclose(got, [2.0 ** -3, 2.0 ** -10, 2.0 ** -126, 2.0 ** -126, 1.0], rtol=2.0 ** -22, atol=0)
