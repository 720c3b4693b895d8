"""The error bound of the integer block dot product, checked on the CPU.

The CUDA GEMV meets x (fp16) with the 4-bit codes of a q4_0 block through integer
arithmetic: the block's 32 values become 16-bit fixed point relative to the block's
largest exponent, split into a low unsigned and a high signed byte, and the block sum
`sum (c - 8) X` is formed from two byte-digit dot products. `test_gpu_kernels` bounds the
GEMV error by a term for that rounding. This file restates the arithmetic in numpy
(exact integers) and checks that:
  * the two digit sums reconstruct `sum (c - 8) X` exactly and stay within 2^23 (exact in
    fp32);
  * the block result is within 2^-15 * max|x| * sum|c - 8| (times the scale) of the exact
    fp64 product, the term the GPU bound carries;
on random blocks and on blocks built to stress it: wide exponent ranges, values at
rounding ties, extreme codes, zeros and subnormals. Nothing here imports the CUDA path.
"""
from __future__ import annotations

import numpy as np
import pytest


def _half_exp(h16: np.ndarray) -> np.ndarray:
    e = (h16.view(np.uint16) >> 10) & 31
    return np.where(e == 0, 1, e).astype(np.int64)


def _block(x16: np.ndarray, codes: np.ndarray):
    """(integer block sum, its value, exact value) for one 32-column block."""
    xf = x16.astype(np.float64)
    em = int(_half_exp(x16).max())
    X = np.rint(xf * 2.0 ** (29 - em)).astype(np.int64)  # round half to even, like the kernel
    assert np.all(np.abs(X) < 2 ** 15)
    d0 = X & 255                                          # low byte, unsigned
    d1 = X >> 8                                           # high byte, signed (arithmetic shift)
    assert np.all((d1 >= -128) & (d1 <= 127))
    s0 = int((codes * d0).sum() - 8 * d0.sum())
    s1 = int((codes * d1).sum() - 8 * d1.sum())
    s = s1 * 256 + s0
    assert s == int(((codes - 8) * X).sum())
    assert abs(s) <= 2 ** 23
    value = float(np.float32(s)) * 2.0 ** (em - 29)        # exact: |s| <= 2^23
    return value, float(((codes - 8) * xf).sum())


def _bound(x16, codes):
    return 2.0 ** -15 * float(np.abs(x16.astype(np.float64)).max()) * float(np.abs(codes - 8).sum())


@pytest.mark.parametrize("seed", range(6))
def test_random_blocks_within_bound(seed):
    rng = np.random.default_rng(seed)
    for _ in range(2000):
        scale = 10.0 ** rng.uniform(-6, 3)
        x16 = (rng.standard_normal(32) * scale).astype(np.float16)
        codes = rng.integers(0, 16, 32)
        v, exact = _block(x16, codes)
        assert abs(v - exact) <= _bound(x16, codes) + 1e-300


def test_adversarial_blocks_within_bound():
    rng = np.random.default_rng(42)
    cases = []
    # one large value, the rest tiny: most of the block is rounded
    x = np.full(32, 1e-3, dtype=np.float16); x[7] = np.float16(60000.0); cases.append(x)
    # values that land exactly halfway between fixed-point steps
    big = np.float16(1024.0)
    x = np.concatenate([[big], (np.arange(31) + 0.5).astype(np.float16) * np.float16(2.0 ** -4)]).astype(np.float16)
    cases.append(x)
    # subnormals only, and mixed signs of equal magnitude
    cases.append((rng.standard_normal(32) * 1e-6).astype(np.float16))
    cases.append(np.array([1.0, -1.0] * 16, dtype=np.float16))
    cases.append(np.zeros(32, dtype=np.float16))
    # full fp16 range inside one block
    cases.append(np.array([2.0 ** e for e in range(-14, 16)] + [65504.0, -65504.0], dtype=np.float16))
    for x16 in cases:
        for codes in (np.zeros(32, np.int64), np.full(32, 15, np.int64), rng.integers(0, 16, 32),
                      np.where(np.arange(32) % 2 == 0, 0, 15)):
            v, exact = _block(x16, codes)
            assert abs(v - exact) <= _bound(x16, codes) + 1e-300, (x16, codes)


def test_exact_when_block_exponents_are_close():
    """Every value within 2^4 of the block's largest exponent is represented exactly."""
    rng = np.random.default_rng(7)
    for _ in range(500):
        e = rng.integers(-10, 12)
        mant = rng.integers(1024, 2048, 32) / 1024.0
        x16 = (mant * 2.0 ** (e - rng.integers(0, 5, 32)) * rng.choice([-1, 1], 32)).astype(np.float16)
        codes = rng.integers(0, 16, 32)
        v, exact = _block(x16, codes)
        assert v == exact
