"""Pins of the oracle's fp16 GEMV (the fp16 tied head) and of its fp16 table.

The fp16 head computes y[r] = sum_c W[r][c] x[c] with W and x stored as IEEE
binary16 ("Gemma-4-12B-CoreAI", tiered-v3/ section: the vocabulary path kept at
fp16). numpy's own float16 decoding and a float64 matmul are the independent
reference; the inputs include the encodings a hand-written decoder gets wrong
(subnormals, signed zeros, the largest finite value).
"""
from __future__ import annotations

import numpy as np
import pytest

import datagen as DG
from datagen import workloads as WL
from oracle import oracle as O


def _special_bits() -> np.ndarray:
    vals = np.array([0.0, -0.0, 65504.0, -65504.0, 6.1035156e-05, 5.9604645e-08, -5.9604645e-08,
                     1.0, -1.0, 0.5, 3.0e-06, 1024.0, 0.099975586], dtype=np.float16)
    return vals.view(np.uint16)


@pytest.mark.parametrize("n,k,nrhs", [(37, 256, 1), (64, 512, 3), (5, 2048, 8)])
def test_gemv_f16_matches_numpy(n, k, nrhs):
    rng = np.random.default_rng(n * 1000 + k + nrhs)
    w = rng.standard_normal((n, k)).astype(np.float16)
    x = (rng.standard_normal((nrhs, k)) * 0.5).astype(np.float16)
    sb = _special_bits()
    w.view(np.uint16)[0, : sb.size] = sb          # special encodings in the weights
    x.view(np.uint16)[0, -sb.size:] = sb          # ... and in x
    w[1] = 0.0                                    # a zero row
    want = w.astype(np.float64) @ x.astype(np.float64).T
    got = O.gemv_f16(w.view(np.uint16), x.view(np.uint16))
    np.testing.assert_allclose(got, want.T, rtol=1e-12, atol=1e-9)
    assert np.all(got[:, 1] == 0.0)


def test_gemv_f16_single_vector_shape():
    w = np.eye(256, dtype=np.float16)[:7]
    x = np.arange(256).astype(np.float16)
    got = O.gemv_f16(w.view(np.uint16), x.view(np.uint16))
    assert got.shape == (7,)
    assert np.array_equal(got, np.arange(7, dtype=np.float64))


def test_fp16_table_is_the_rounded_draws():
    """The oracle's fp16 tied table: the embedding's N(0, 0.02) draws rounded to
    nearest-even fp16 (numpy's rounding as the reference), element by element."""
    cfg = dict(WL.MICRO, head_fp16=1)
    seed = 7
    om = O.Model(cfg, seed=seed, variant=0)
    got = om.embed_f16()
    V, H = cfg["vocab"], cfg["hidden"]
    want = DG.normal(seed, DG.STREAM_EMBED, V * H, 0.02).astype(np.float16).view(np.uint16).reshape(V, H)
    assert got.shape == (V, H)
    assert np.array_equal(got, want)
