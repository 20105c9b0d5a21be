"""The FMA-pipe 2^x used for part of the prefill softmax (csrc/exp2_poly.cuh),
replayed step by step in float32 on the CPU from the header's constants, and
checked against 2^x in float64: relative error below 1e-4 over the range the
softmax feeds it, exact zero-ish underflow at the clamp, NaN propagation."""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "scaled_dot_product_15_b200", "csrc", "exp2_poly.cuh")


def _consts():
    src = open(HDR).read()
    get = lambda n: np.float32(float(re.search(rf"{n} = ([-0-9.e]+)f;", src).group(1)))
    return [get(f"kC{i}") for i in range(4)], get("kMagic"), get("kMinX")


def _emulate(x):
    (c0, c1, c2, c3), magic, minx = _consts()
    x = np.asarray(x, dtype=np.float32)
    x = np.where(np.isnan(x), x, np.maximum(x, minx)).astype(np.float32)
    # add rounded toward -inf: floor of the exact sum (|x| small, magic large)
    t = (np.floor(x.astype(np.float64) + np.float64(magic))).astype(np.float32)
    t = np.where(np.isnan(x), np.float32(np.nan), t)
    j = (t - magic).astype(np.float32)
    f = (x - j).astype(np.float32)  # exact: fma(j, -1, x)
    p = (np.float32(c3) * f + c2).astype(np.float32)
    p = (p * f + c1).astype(np.float32)
    p = (p * f + c0).astype(np.float32)
    pb = p.view(np.uint32).astype(np.uint64)
    tb = t.view(np.uint32).astype(np.uint64)
    r = ((pb + ((tb << np.uint64(23)) & np.uint64(0xFFFFFFFF))) & np.uint64(0xFFFFFFFF)).astype(np.uint32)
    return r.view(np.float32)


def test_relative_error_over_softmax_range():
    x = np.linspace(-40.0, 8.0, 2_000_001, dtype=np.float32)
    y = _emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() < 1e-4, rel.max()
    assert np.all(y > 0)


def test_integers_and_clamp():
    x = np.arange(-125, 9, dtype=np.float32)
    y = _emulate(x).astype(np.float64)
    assert np.all(np.abs(y / np.exp2(x.astype(np.float64)) - 1.0) < 1e-4)
    low = _emulate(np.array([-126.0, -127.5, -1000.0, -np.inf], dtype=np.float32))
    assert np.all(low >= 0) and np.all(low < 1.2e-38)  # no wrap into the sign bit


def test_nan_propagates():
    assert np.isnan(_emulate(np.array([np.nan], dtype=np.float32))).all()
