"""The prefill softmax's FMA-pipe 2^x (ex2_fma in csrc/pa_prefill.cu), emulated on the CPU.

The kernel computes part of its exponentials as 2^round(x) (exponent field) times
a cubic in f = x - round(x). This emulates that fp32 arithmetic step by step
(coefficients read from the kernel source) and checks it against numpy's exp2
over the range the kernel feeds it, [-125, 8] (stale max: p <= 2^8), and
below -125 (exactly 0, like the MUFU instruction's flush of tiny results).
"""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "paged_kv_cache_475_b200", "csrc", "pa_prefill.cu")


def _coeffs():
    text = open(SRC).read()
    return [np.float32(float(re.search(rf"kExp2C{i} = ([0-9.e+-]+)f;", text).group(1))) for i in range(4)]


def _fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def ex2_fma_emulated(x):
    c0, c1, c2, c3 = _coeffs()
    x_in = x.astype(np.float32)
    x = np.clip(x_in, np.float32(-125), np.float32(125))
    magic = np.float32(12582912.0)
    y = (x + magic).astype(np.float32)
    j = (y - magic).astype(np.float32)
    f = (x - j).astype(np.float32)
    p = _fma32(_fma32(_fma32(np.full_like(f, c3), f, np.full_like(f, c2)), f, np.full_like(f, c1)), f,
               np.full_like(f, c0))
    bits = p.view(np.int32) + (y.view(np.int32) << np.int32(23))
    return np.where(~(x_in >= np.float32(-125)), np.float32(0), bits.view(np.float32))


def test_relative_error_over_the_softmax_range():
    x = np.concatenate([np.linspace(-125, 8, 2_000_001, dtype=np.float32),
                        np.array([0.0, -0.5, 0.5, -1.0, 1.0, 7.999, -124.5], dtype=np.float32)])
    got = ex2_fma_emulated(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 1e-4, rel.max()
    assert np.all(np.isfinite(got)) and np.all(got > 0)


def test_exact_powers_and_clamp():
    ints = np.arange(-120, 9, dtype=np.float32)
    got = ex2_fma_emulated(ints).astype(np.float64)
    assert np.abs(got / np.exp2(ints.astype(np.float64)) - 1).max() < 1e-4
    low = ex2_fma_emulated(np.array([-np.inf, -1e30, -200.0, -126.0], dtype=np.float32))
    assert np.all(low == 0)
    edge = ex2_fma_emulated(np.array([-125.0], dtype=np.float32)).astype(np.float64)
    assert abs(edge[0] / 2.0 ** -125 - 1) < 1e-4
