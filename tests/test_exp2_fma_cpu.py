"""The FMA-pipe exp2 of the attention softmax (tp_device.cuh exp2_fma),
re-executed step by step in float32 numpy with the coefficients read from the
header, against numpy's exp2: the relative error stays below 1e-4 over the
softmax's input range, far below the bf16 rounding the probabilities get
(2^-8), and the magic-number rounding and exponent add behave as stated
(exact powers of two at integers, monotone, clamped below -125)."""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "megatron_tensor_transformer_gemm_b200", "csrc", "tp_device.cuh")


def _coeffs():
    src = open(HDR).read()
    return [np.float32(float(re.search(rf"kExp2C{k} = ([0-9.e+-]+)f", src).group(1))) for k in range(4)]


def exp2_fma(x):
    c0, c1, c2, c3 = _coeffs()
    f32 = np.float32
    x = np.maximum(x.astype(np.float32), f32(-125.0))
    t = (x + f32(12582912.0)).astype(np.float32)
    n = (t - f32(12582912.0)).astype(np.float32)
    f = (x - n).astype(np.float32)
    # fmaf(fmaf(fmaf(c3, f, c2), f, c1), f, c0), each fma rounded once
    q = ((c3.astype(np.float64) * f + c2).astype(np.float32))
    q = ((q.astype(np.float64) * f + c1).astype(np.float32))
    q = ((q.astype(np.float64) * f + c0).astype(np.float32))
    bits = q.view(np.int32).astype(np.int64) + ((t.view(np.int32).astype(np.int64) << 23) & 0xFFFFFFFF)
    bits = ((bits + 2 ** 31) % 2 ** 32 - 2 ** 31).astype(np.int32)
    return bits.view(np.float32)


def test_exp2_fma_relative_error():
    x = np.linspace(-124.0, 8.0, 2_000_001, dtype=np.float64).astype(np.float32)
    got = exp2_fma(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(got / ref - 1.0)) < 1e-4


def test_exp2_fma_integers_monotone_and_clamp():
    ints = np.arange(-120, 9, dtype=np.float32)
    got = exp2_fma(ints)
    assert np.all(np.abs(got / np.exp2(ints.astype(np.float64)) - 1) < 1e-4)
    x = np.linspace(-20, 8, 100001, dtype=np.float32)
    y = exp2_fma(x)
    assert np.all(np.diff(y.astype(np.float64)) >= -1e-7 * y[1:])  # monotone up to the fit error
    tiny = exp2_fma(np.array([-200.0, -1e30], dtype=np.float32))
    assert np.all(tiny > 0) and np.all(tiny < 1e-37)
