"""Error bound of ex2_fma, the FMA-pipe 2^x used for part of the attention
softmax: the coefficients are read from the CUDA header and the float32
arithmetic of the routine is emulated step by step in numpy, then compared with
exact 2^x (float64) over the input range the kernel feeds it."""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "dynamic_block_sparse_last_b200", "csrc", "ptx.cuh")


def coefficients(prefix="kEx2C", count=4):
    src = open(HDR).read()
    vals = dict(re.findall(prefix + r"(\d)\s*=\s*([0-9.eE+-]+)f", src))
    return [np.float32(vals[str(i)]) for i in range(count)]


def fma32(a, b, c):
    return (a.astype(np.float64) * b + c).astype(np.float32)   # single rounding, as fmaf


def ex2_fma_emulated(x, prefix="kEx2C", count=4):
    c = coefficients(prefix, count)
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    j = (x + magic).astype(np.float32)
    n = (j - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = fma32(np.full_like(f, c[-1]), f, c[-2])
    for k in range(count - 3, -1, -1):
        p = fma32(p, f, c[k])
    bits = p.view(np.int32) + ((j.view(np.int32) - np.int32(0x4B400000)) << 23)
    return bits.view(np.float32)


def test_relative_error_below_1e4_over_kernel_range():
    x = np.concatenate([np.linspace(-125.0, 8.5, 1_000_001), np.arange(-125, 9, 0.5)]).astype(np.float32)
    got = ex2_fma_emulated(x).astype(np.float64)
    rel = np.abs(got / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 1e-4, rel.max()


def test_reduction_is_exact_at_integers_and_halves():
    x = np.arange(-20, 9, dtype=np.float32)
    got = ex2_fma_emulated(x).astype(np.float64)
    assert np.allclose(got, np.exp2(x.astype(np.float64)), rtol=1e-4)
    assert np.all(np.diff(got) > 0)

