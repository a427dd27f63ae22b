"""The FMA-pipe 2^x the attention kernels use for part of their exponentials
(ex2_fma in csrc/attention_tc.cuh): x = n + f with n the nearest integer
(found by adding 1.5 * 2^23), 2^f from a cubic on [-0.5, 0.5], n shifted into
the exponent bits.  Its coefficients are read from
the source and evaluated in float32 the way the kernel does it; the relative
error against 2^x (fp64) must stay below 1e-4 over the range the softmax uses
(x <= 8 after the lazy rescale, down to the flush-to-zero point), which is
well under the 2^-9 rounding of the bf16 probabilities it feeds.  No GPU."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "decoder_only_transformer_02_b200",
                   "csrc", "attention_tc.cuh")


def _coeffs():
    text = open(SRC).read()
    body = text[text.index("float ex2_fma(float x)"):]
    body = body[:body.index("}")]
    line = [ln for ln in body.splitlines() if "const float p = " in ln][0]
    c = [float(v) for v in re.findall(r"([0-9]+\.[0-9]+)f", line)]
    assert len(c) == 4
    c3, c2, c1, c0 = c
    return np.float32(c0), np.float32(c1), np.float32(c2), np.float32(c3)


def _ex2_fma(x):
    c0, c1, c2, c3 = _coeffs()
    f32 = np.float32
    x = np.asarray(x, dtype=f32)
    xc = np.maximum(x, f32(-127.0))
    t = (xc + f32(12582912.0)).astype(f32)
    f = (xc - (t - f32(12582912.0)).astype(f32)).astype(f32)
    p = ((c3 * f + c2).astype(f32) * f + c1).astype(f32)
    p = (p * f + c0).astype(f32)
    bits = (p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)) & 0xFFFFFFFF
    y = bits.astype(np.uint32).view(np.float32)
    return np.where(x < -125.0, f32(0.0), y)


def test_relative_error_bound():
    x = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001), -np.linspace(0.0, 1.0, 100_001)]).astype(np.float32)
    got = _ex2_fma(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 1e-4, rel.max()


def test_flush_and_integers():
    x = np.array([-np.inf, -200.0, -125.5, 0.0, 1.0, 3.0, -5.0], dtype=np.float32)
    y = _ex2_fma(x)
    assert y[0] == 0 and y[1] == 0 and y[2] == 0
    # integer arguments are exact up to the cubic's error at f = 0
    np.testing.assert_allclose(y[3:], [1.0, 2.0, 8.0, 1 / 32], rtol=1e-4)
