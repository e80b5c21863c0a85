"""The FMA-pipe 2^x of the attention kernels, checked on the host.

The kernels can evaluate part of their exponentials as 2^x = 2^n * p(f) with
n = round(x), f = x - n in [-1/2, 1/2] and p a minimax polynomial.  This test
reads the coefficients from the kernel sources, repeats the kernels' float32
arithmetic in numpy (the 1.5 * 2^23 rounding trick, Horner with fused steps
rounded to float32, the exponent added into the bit pattern) and checks the
relative error against 2^x in float64 over the whole range the kernels use.
"""
import os
import re

import numpy as np
import pytest

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "dynamic_block_sparse_indicator_b200", "csrc")


def coefficients(fname, func):
    src = open(os.path.join(CSRC, fname)).read()
    body = src[src.index(func):]
    body = body[:body.index("}")]
    return [np.float32(float(v)) for v in re.findall(r"c\d = ([0-9.e+-]+)f", body)]


def emulate(x, c):
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    r = np.float32(12582912.0)
    t = (x + r).astype(np.float32)
    n = (t - r).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = np.full_like(f, c[-1])
    for ck in c[-2::-1]:
        p = (p.astype(np.float64) * f + ck).astype(np.float32)   # one fused multiply-add
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


@pytest.mark.parametrize("fname,func,deg,bound", [
    ("prism_av_norm.cu", "exp2_poly(", 3, 8e-5),
    ("prism_attn_fwd.cu", "exp2_poly4(", 4, 3e-6),
])
def test_polynomial_exp2_error(fname, func, deg, bound):
    c = coefficients(fname, func)
    assert len(c) == deg + 1
    x = np.concatenate([np.linspace(-120.0, 15.9, 2_000_001), np.linspace(-0.5, 0.5, 100_001)])
    y = emulate(x, c).astype(np.float64)
    want = np.exp2(x.astype(np.float32).astype(np.float64))
    rel = np.abs(y / want - 1.0)
    assert rel.max() < bound, rel.max()
    # clamped below -126: a tiny non-negative number, never a wrapped exponent
    z = emulate(np.array([-130.0, -500.0, -1e6], dtype=np.float32), c)
    assert np.all(z >= 0) and np.all(z < 2.0 ** -125)
