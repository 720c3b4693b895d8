"""Pins of the oracle's int8 KV cache ("Gemma-4-12B-CoreAI", per-tier cost section:
K/V rows stored as int8 would halve the cache).

The row format: codes int8 with one fp32 scale per row (value = code x scale),
scale = amax / 127 and code = clamp(rint(x / scale), -127, 127), both fp32
divisions. Checked against a hand-worked row (tests/golden/kv_int8_row.txt),
against the properties any such quantizer must have, and, for the attention over
int8 rows, against the already-pinned fp16 attention on rows whose values
code x scale are exact fp16 numbers (the int8 path must then agree bit for bit).
The whole decoder with int8 KV is pinned in test_oracle_decoder_pin.py.
"""
from __future__ import annotations

import os

import numpy as np
import pytest

from datagen import workloads as WL
from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "kv_int8_row.txt")


def _golden():
    d = {}
    for line in open(GOLDEN):
        if line.startswith("#") or not line.strip():
            continue
        k, *v = line.split()
        d[k] = v
    x = np.array([int(t, 16) for t in d["values"]], dtype=np.uint16)
    codes = np.array([int(t) for t in d["codes"]], dtype=np.int8)
    scale = np.array([int(d["scale"][0], 16)], dtype=np.uint32).view(np.float32)[0]
    return x, codes, scale


def test_hand_worked_row():
    x, codes, scale = _golden()
    got_c, got_s = O.kv_quantize_row(x)
    assert np.array_equal(got_c, codes)
    assert got_s.view(np.uint32) == scale.view(np.uint32)


def _rows():
    rng = np.random.default_rng(5)
    rows = [rng.standard_normal(256).astype(np.float16) for _ in range(20)]
    rows += [(rng.standard_normal(512) * 1e-6).astype(np.float16)]        # subnormal range
    rows += [np.full(64, 3.0, dtype=np.float16), np.full(64, -0.125, dtype=np.float16)]
    spike = np.zeros(256, dtype=np.float16)
    spike[17] = -65504.0
    spike[3] = 1.0
    rows += [spike, np.zeros(32, dtype=np.float16)]
    return rows


@pytest.mark.parametrize("i", range(len(_rows())))
def test_quantizer_properties(i):
    x = _rows()[i]
    c, s = O.kv_quantize_row(x.view(np.uint16))
    xf = x.astype(np.float64)
    amax = np.max(np.abs(xf))
    assert np.all(np.abs(c.astype(np.int64)) <= 127)
    if amax == 0:
        assert s == 0 and np.all(c == 0)
        return
    assert abs(float(s) - amax / 127) <= 2 ** -23 * amax / 127      # fp32 rounding of amax / 127
    k = int(np.argmax(np.abs(xf)))
    assert abs(int(c[k])) == 127 and np.sign(c[k]) == np.sign(xf[k])  # the extreme maps to +-127
    err = np.abs(xf - c.astype(np.float64) * float(s))
    assert np.all(err <= float(s) * (0.5 + 1e-5))                     # rounding to the nearest code
    cn, sn = O.kv_quantize_row((-x).view(np.uint16))                  # odd symmetry
    assert sn == s and np.array_equal(cn, -c)


def _exact_rows(rng, shape):
    """int8 rows whose values code * 2^-6 are exact fp16 numbers."""
    codes = rng.integers(-127, 128, size=shape).astype(np.int8)
    scales = np.full(shape[:-1], 2.0 ** -6, dtype=np.float32)
    vals = (codes.astype(np.float64) * 2.0 ** -6).astype(np.float16)
    assert np.array_equal(vals.astype(np.float64), codes * 2.0 ** -6)
    return codes, scales, vals.view(np.uint16)


def test_attention_over_int8_rows_reduces_to_fp16():
    rng = np.random.default_rng(11)
    n_q, n_kv, hd, R, W = 8, 2, 64, 48, 20
    q16 = rng.standard_normal((n_q, hd)).astype(np.float16).view(np.uint16)
    k8, ks, k16 = _exact_rows(rng, (n_kv, R, hd))
    v8, vs, v16 = _exact_rows(rng, (n_kv, R, hd))
    for q in (5, 47, 130):
        a = O.attn_ring_i8(q16, k8, ks, v8, vs, R, W, q)
        b = O.attn_ring(q16, k16, v16, R, W, q)
        assert np.array_equal(a, b)
    L = 37
    k8, ks, k16 = _exact_rows(rng, (L, 1, hd))
    v8, vs, v16 = _exact_rows(rng, (L, 1, hd))
    a = O.attn_linear_i8(q16, k8, ks, v8, vs, L)
    b = O.attn_linear(q16, k16, v16, L)
    assert np.array_equal(a, b)


def test_int8_scales_enter_the_scores_and_values():
    """Scaling every row's scale by 2 (and halving the codes' meaning nowhere else)
    doubles every key and value: the output doubles (V) and the softmax sharpens
    exactly as for keys doubled in fp64."""
    rng = np.random.default_rng(12)
    n_q, hd, L = 4, 32, 9
    q16 = rng.standard_normal((n_q, hd)).astype(np.float16).view(np.uint16)
    k8 = rng.integers(-127, 128, size=(L, 1, hd)).astype(np.int8)
    v8 = rng.integers(-127, 128, size=(L, 1, hd)).astype(np.int8)
    ks = (rng.random((L, 1)) * 0.01 + 0.001).astype(np.float32)
    vs = (rng.random((L, 1)) * 0.01 + 0.001).astype(np.float32)
    out = O.attn_linear_i8(q16, k8, ks, v8, vs, L)
    qd = q16.view(np.float16).astype(np.float64)
    K = k8[:, 0].astype(np.float64) * ks.astype(np.float64)
    V = v8[:, 0].astype(np.float64) * vs.astype(np.float64)
    s = qd @ K.T
    p = np.exp(s - s.max(axis=1, keepdims=True))
    ref = (p / p.sum(axis=1, keepdims=True)) @ V
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-15)


def _verify_logits(cfg, single_pass):
    from tests.test_oracle_pins import _run_verify
    return _run_verify(cfg, ring=2 * cfg["window"], single_pass=single_pass)


def test_int8_single_pass_R2W_equals_two_pass_bitwise():
    cfg = dict(WL.MICRO, kv_int8=1)
    a = _verify_logits(cfg, True)
    b = _verify_logits(cfg, False)
    assert np.array_equal(a, b)


def test_int8_cache_holds_quantized_rows():
    """After a decode step the int8 cache row of its position equals the quantizer
    applied to the step's fp16 K/V rows (KV head 0, every layer)."""
    cfg = dict(WL.MICRO, kv_int8=1)
    m = O.Model(cfg, seed=2, variant=1)
    c = O.Cache(m, 32)
    pos = 19
    for p in range(pos):
        O.decode_step(m, c, p, token=p + 3, want_logits=False)
    r = O.decode_step(m, c, pos, token=7, want_dump=True)
    sl = gl = 0
    for l in range(cfg["n_layers"]):
        full = WL.layer_is_full(cfg, l)
        hd = cfg["gl_head_dim"] if full else cfg["sl_head_dim"]
        for kv in (0, 1):
            codes, scales = c.global_i8(gl, kv) if full else c.ring_i8(sl, kv)
            row = pos if full else pos % c.R
            want_c, want_s = O.kv_quantize_row(r["kv"][l, 0, kv, :hd])
            assert np.array_equal(codes[0, row], want_c) and scales[0, row] == want_s
        gl, sl = (gl + 1, sl) if full else (gl, sl + 1)


def test_code8_numpy_twin_matches_c_header():
    """The synthetic int8 history's generator: numpy twin and C header agree code for
    code (ties to even included), the codes have standard deviation ~36 and span the
    clamped range."""
    import datagen as DG
    n = 200_000
    want = np.empty(n, dtype=np.int8)
    O.fill_code8(want, 5, 0x123, start=17)
    got = DG.code8(5, 0x123, n, start=17)
    assert np.array_equal(got, want)
    assert abs(got.astype(np.float64).std() / 36 - 1) < 0.01
    assert got.min() == -127 and got.max() == 127
    z = DG.unit_normal(5, 0x123, n, start=17).astype(np.float64) * 36
    ties = np.abs(z - np.floor(z) - 0.5) < 1e-12
    assert np.array_equal(got[ties], np.clip(2 * np.round(z[ties] / 2), -127, 127).astype(np.int8))
    inner = (np.abs(z) < 126.5) & ~ties
    assert np.array_equal(got[inner], np.rint(z[inner]).astype(np.int8))
