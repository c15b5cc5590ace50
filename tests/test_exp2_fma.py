"""CPU check of the FMA-pipe exp2 that computes half of the prefill
softmax's exponentials (exp2_fma in csrc/ptx.cuh).  The coefficients are read
from the header itself, and the kernel's steps (round x to the nearest
integer with the 1.5 * 2^23 trick, Horner in fp32 fused multiply-adds,
exponent-field add, 0 below -125) are replayed in fp32 against the exact
2^x.  The bound, 5e-6 relative, is far below the 2^-9 rounding that the
softmax weights get next (they are packed to bf16 for the P V product)."""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "block_sparse_long_08_b200", "csrc", "ptx.cuh")


def _coefficients():
    src = open(HDR).read()
    body = src[src.index("float exp2_fma(float x)"):]
    body = body[:body.index("}")]
    c4, c3 = map(float, re.search(r"fmaf\(([-0-9.e]+)f, f, ([-0-9.e]+)f\)", body).groups())
    rest = [float(v) for v in re.findall(r"fmaf\(p, f, ([-0-9.e]+)f\)", body)]
    return [np.float32(v) for v in (c4, c3, *rest)]   # highest degree first


def _fma32(a, b, c):
    # a*b of two fp32 values is exact in fp64; one rounding to fp32 after the add
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _exp2_fma(x):
    x = np.asarray(x, dtype=np.float32)
    with np.errstate(invalid="ignore", over="ignore"):
        t = (x + np.float32(12582912.0)).astype(np.float32)
        i = t.view(np.int32).astype(np.int64) - 0x4B400000
        f = (x - (t - np.float32(12582912.0)).astype(np.float32)).astype(np.float32)
        c = _coefficients()
        p = _fma32(np.full_like(f, c[0]), f, np.full_like(f, c[1]))
        for ck in c[2:]:
            p = _fma32(p, f, np.full_like(f, ck))
        bits = (p.view(np.int32).astype(np.int64) + (i << 23)).astype(np.int64)
        r = (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)
    return np.where(x < -125.0, np.float32(0.0), r)


def test_coefficients_are_a_degree_four_polynomial():
    c = _coefficients()
    assert len(c) == 5
    # 2^f = sum (f ln 2)^n / n!: the fit stays close to the Taylor terms
    taylor = [np.log(2) ** n / float(np.prod(range(1, n + 1))) for n in range(5)]
    for got, want in zip(reversed(c), taylor):
        assert abs(float(got) - want) <= 0.01 * want + 1e-3


def test_relative_error_over_the_softmax_range():
    x = np.concatenate([np.linspace(-125.0, 0.0, 2_000_001),
                        -np.arange(0, 126, dtype=np.float64),          # integers
                        -np.arange(0, 126, dtype=np.float64) - 0.5])   # rounding ties
    x = x.astype(np.float32)
    x = x[x >= -125.0]
    got = _exp2_fma(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got - want) / want
    assert rel.max() <= 5e-6, rel.max()
    assert abs(float(_exp2_fma(np.float32(0.0))) - 1.0) <= 5e-6


def test_masked_scores_give_zero():
    x = np.array([-np.inf, -1e30, -125.5, -126.0, -200.0], dtype=np.float32)
    assert np.all(_exp2_fma(x) == 0.0)
