"""The FMA-pipe 2^x of csrc/exp2_poly.cuh (an off-by-default option of the
attention softmax), checked on the host: its four coefficients are read
from the header as text and the same float32 steps are replayed with
numpy (floor, Horner cubic on [0, 1), exponent added to the bit pattern).
Pins the header's stated accuracy (max relative error 7.6e-5 on normal
results, far below the bf16 rounding of P) and its exact 0 below -126.
Just above -126 a result can fall in the denormal range, where the bit
pattern carries the cubic's fraction without its leading one (relative
error up to about 1.5e-4, on values below 2^-125 that add nothing)."""
import os
import re

import numpy as np

HEADER = os.path.join(os.path.dirname(__file__), "..", "block_sparse_attention_36_b200", "csrc", "exp2_poly.cuh")


def _coeffs():
    text = open(HEADER).read()
    c = {int(k): np.float32(v) for k, v in re.findall(r"kExp2C(\d)\s*=\s*([-0-9.eE+]+)f", text)}
    assert sorted(c) == [0, 1, 2, 3]
    return c


def _exp2_poly(x):
    c = _coeffs()
    x = np.asarray(x, dtype=np.float32)
    xc = np.maximum(x, np.float32(-126.0))
    n = np.floor(xc).astype(np.float32)
    f = (xc - n).astype(np.float32)
    p = c[3]
    for k in (2, 1, 0):
        p = (p * f + c[k]).astype(np.float32)
    bits = (p.view(np.int32).astype(np.int64) + (n.astype(np.int64) << 23)) & 0xFFFFFFFF
    r = bits.astype(np.uint32).view(np.float32)
    return np.where(x < np.float32(-126.0), np.float32(0.0), r)


def test_relative_error_matches_the_header():
    x = np.concatenate([np.linspace(-125.0, 8.0, 400001), -np.arange(0, 126, dtype=np.float64)]).astype(np.float32)
    x = x[x >= -125.0]
    got = _exp2_poly(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 8e-5, rel.max()


def test_integers_and_masked_inputs():
    # at integer x the cubic is evaluated at f = 0: 2^x times kExp2C0
    c0 = float(_coeffs()[0])
    for k in (-125, -20, -1, 0, 3):
        assert abs(float(_exp2_poly(np.float32(k))) / 2.0 ** k - c0) < 1e-7
    assert float(_exp2_poly(np.float32(-np.inf))) == 0.0
    assert float(_exp2_poly(np.float32(-126.5))) == 0.0
    assert not np.isnan(_exp2_poly(np.linspace(-200, 8, 1001, dtype=np.float32))).any()
