"""Pins of the CPU oracle to things other than itself (no GPU).

Each test checks one oracle function against a library routine, a hand-worked
example, a closed form, an invariant or brute force, chosen so that a plausible
mistake (a dropped term, a wrong sign or index, a transposed operand) fails.
"""
from __future__ import annotations

import math
import os

import numpy as np
import pytest
import torch

import datagen as DG
from datagen import workloads as WL
from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------ datagen --

def test_datagen_numpy_twin_matches_c_header_through_packing():
    """numpy twin and C header give the same fp32 normals: packing the numpy
    values with the oracle reproduces the bytes of the oracle model's tensor,
    which the oracle generated with the C header."""
    m = O.Model(WL.MICRO, seed=7)
    qs_ref, sc_ref = m.tensor(1, DG.T_WO)
    rows, k = qs_ref.shape[0], qs_ref.shape[1] * 2
    w = DG.normal(7, DG.stream_layer(1, DG.T_WO), rows * k, 0.02).reshape(rows, k)
    qs, sc = O.q4_0_pack(w)
    assert np.array_equal(qs, qs_ref) and np.array_equal(sc, sc_ref)


def test_datagen_normal_moments_and_support():
    z = DG.unit_normal(3, 11, 400_000).astype(np.float64)
    assert abs(z.mean()) < 0.01 and abs(z.var() - 1.0) < 0.01
    assert np.abs(z).max() < 6.0
    # fourth moment of Irwin-Hall(12) is 3 - 1.2/12 = 2.9
    assert abs((z ** 4).mean() - 2.9) < 0.05


def test_datagen_ids_uniform():
    ids = DG.uniform_int(0, DG.STREAM_PREFIX_IDS, 200_000, 4096)
    counts = np.bincount(ids, minlength=4096)
    assert ids.min() >= 0 and ids.max() < 4096
    # multinomial counts: std close to sqrt(mean) (Poisson), no empty bins
    assert abs(counts.std() / math.sqrt(counts.mean()) - 1.0) < 0.1 and counts.min() > 0


# --------------------------------------------------------------------- fp16 --

def test_f16_to_double_exhaustive_vs_numpy():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = O.f16_value(bits)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_f16_from_double_vs_numpy_rounding():
    rng = np.random.default_rng(1)
    vals = np.concatenate([
        rng.standard_normal(200_000) * np.exp(rng.uniform(-20, 12, 200_000)),
        # exact ties between neighbouring halves, normal and subnormal
        (np.arange(1024, 2048, dtype=np.float64) + 0.5) * 2.0 ** -10,
        (np.arange(0, 1024, dtype=np.float64) + 0.5) * 2.0 ** -24,
        np.array([65504.0, 65519.99, 65520.0, 1e6, -1e6, 0.0, -0.0, 2.0 ** -25, 2.0 ** -26,
                  3 * 2.0 ** -26, np.inf, -np.inf]),
    ])
    ref = vals.astype(np.float16).view(np.uint16)
    got = O.f16_bits(vals)
    assert np.array_equal(got, ref)


# --------------------------------------------------------------------- q4_0 --

def _read_golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            if line.startswith("#") or ":" not in line:
                continue
            k, v = line.split(":", 1)
            out[k.strip()] = v.split()
    return out


def test_q4_0_hand_worked_block():
    g = _read_golden("q4_0_block.txt")
    x = np.array([float(v) for v in g["x"]], dtype=np.float32)[None, :]
    qs, sc = O.q4_0_pack(x)
    assert [int(v, 16) for v in g["bytes"]] == list(qs[0])
    assert sc[0, 0] == int(g["scale_bits"][0], 16)
    codes = np.array([int(c) for c in g["codes"]])
    assert np.array_equal(O.q4_0_unpack(qs, sc)[0], (codes - 8) * 0.5)


def test_q4_0_scale_rounding_and_sign():
    # m = +1.0 -> d = -0.125 (negative scale); the extreme element gets code 0.
    x = np.zeros((1, 32), dtype=np.float32)
    x[0, 0], x[0, 1], x[0, 2] = 1.0, 0.9, -0.9375
    qs, sc = O.q4_0_pack(x)
    assert sc[0, 0] == 0xB000  # -0.125
    w = O.q4_0_unpack(qs, sc)[0]
    assert w[0] == 1.0                  # -8 * d
    assert w[1] == -7 * -0.125          # 0.9 / -0.125 = -7.2 -> -7
    assert w[2] == 7 * -0.125           # 7.5 -> 8 clipped to 7 (the +8 side)
    # m = 0.3 -> d = fp16(-0.0375) = -0.037506103515625 (fp16 0xA8CD)
    y = np.zeros((1, 32), dtype=np.float32)
    y[0, 5] = 0.3
    qs, sc = O.q4_0_pack(y)
    assert sc[0, 0] == 0xA8CD
    assert O.q4_0_unpack(qs, sc)[0, 5] == -8 * -0.037506103515625


def _q4_blocks(rows=64, k=256, seed=0):
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal((rows, k)) * 0.02).astype(np.float32)
    w[0] = 0.0                                   # zero row
    w[1, :32] = 1e-30                            # scale underflows to 0
    w[2, :32] = np.linspace(-1, 1, 32)           # ties in |x|: first wins (-1)
    w[3, :] = rng.choice([-3.0, 3.0], size=k)    # every element is extreme
    w[4, :] *= 1e4
    return w


def test_q4_0_invariants():
    w = _q4_blocks()
    qs, sc = O.q4_0_pack(w)
    deq = O.q4_0_unpack(qs, sc)
    d = np.repeat(O.f16_value(sc), 32, axis=1)
    err = np.abs(w.astype(np.float64) - deq)
    # codes on [0, 15] by construction of nibbles; check the reconstruction bounds
    xq = w.astype(np.float64) / np.where(d == 0, 1, d)
    clipped = xq > 7.5
    assert np.all(err[~clipped & (d != 0)] <= np.abs(d[~clipped & (d != 0)]) / 2 * (1 + 1e-6))
    assert np.all(err[clipped] <= np.abs(d[clipped]) * (1 + 1e-6))
    assert np.all(deq[0] == 0) and np.all(deq[1, :32] == 0)
    # the extreme element of every block reconstructs to -8 d (code 0)
    for r in range(w.shape[0]):
        for t in range(w.shape[1] // 32):
            blk = w[r, 32 * t:32 * t + 32]
            i = int(np.argmax(np.abs(blk)))
            if d[r, 32 * t] != 0:
                assert deq[r, 32 * t + i] == -8 * d[r, 32 * t]
    assert deq[2, 0] == -8 * d[2, 0] and d[2, 0] > 0  # first of the tied extremes is -1


def test_q4_0_idempotent_and_rejects():
    w = _q4_blocks(seed=3)
    qs, sc = O.q4_0_pack(w)
    qs2, sc2 = O.q4_0_pack(O.q4_0_unpack(qs, sc).astype(np.float32))
    assert np.array_equal(qs, qs2) and np.array_equal(sc, sc2)
    bad = w.copy()
    bad[5, 7] = np.nan
    with pytest.raises(ValueError):
        O.q4_0_pack(bad)
    bad[5, 7] = np.inf
    with pytest.raises(ValueError):
        O.q4_0_pack(bad)
    with pytest.raises(ValueError):
        O.q4_0_pack(np.zeros((2, 48), dtype=np.float32))


# --------------------------------------------------------------------- GEMV --

@pytest.mark.parametrize("n,k", [(7, 32), (64, 1024), (33, 96)])
def test_gemv_vs_numpy_matmul(n, k):
    rng = np.random.default_rng(n * k)
    w = (rng.standard_normal((n, k)) * 0.02).astype(np.float32)
    qs, sc = O.q4_0_pack(w)
    x16 = rng.standard_normal((3, k)).astype(np.float16)
    y = O.gemv(qs, sc, x16.view(np.uint16))
    ref = x16.astype(np.float64) @ O.q4_0_unpack(qs, sc).T
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-14)


# -------------------------------------------------------------- elementwise --

def test_rmsnorm_vs_torch_and_closed_form():
    rng = np.random.default_rng(5)
    x = rng.standard_normal(257)
    w = 1 + 0.1 * rng.standard_normal(257)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (257,), torch.from_numpy(w), eps=1e-6)
    np.testing.assert_allclose(O.rmsnorm(x, w, 1e-6), ref.numpy(), rtol=1e-13)
    # constant vector c*1: y = c / sqrt(c^2 + eps) * w
    y = O.rmsnorm(np.full(16, -3.0), None, 1e-6)
    np.testing.assert_allclose(y, np.full(16, -3.0 / math.sqrt(9.0 + 1e-6)), rtol=1e-15)


def test_rope_invariants_and_values():
    rng = np.random.default_rng(9)
    x = rng.standard_normal(512)
    # position 0 is the identity
    assert np.array_equal(O.rope(x, 256, 1e6, 0), x)
    # norm preserved, pairs >= rot untouched (full layers: 64 of 256 rotate)
    y = O.rope(x, 64, 1e6, 777)
    assert abs(np.linalg.norm(y) - np.linalg.norm(x)) < 1e-12
    untouched = np.r_[64:256, 256 + 64:512]
    assert np.array_equal(y[untouched], x[untouched])
    assert not np.allclose(y[:64], x[:64])
    # rotate-half pairing (i, i + hd/2): pair 0 with frequency 1 turns by pos radians
    e = np.zeros(8)
    e[0] = 1.0
    z = O.rope(e, 4, 10000.0, 1)
    np.testing.assert_allclose([z[0], z[4]], [0.5403023058681398, 0.8414709848078965], rtol=1e-15)
    # relative position: <rope(q,p), rope(k,s)> depends only on p - s
    q, k = rng.standard_normal(256), rng.standard_normal(256)
    d1 = O.rope(q, 128, 1e4, 1000) @ O.rope(k, 128, 1e4, 990)
    d2 = O.rope(q, 128, 1e4, 50010) @ O.rope(k, 128, 1e4, 50000)
    assert abs(d1 - d2) < 1e-9
    # rotating by p then by -p is the identity
    back = O.rope(O.rope(x[:256], 128, 1e4, 4321), 128, 1e4, -4321)
    np.testing.assert_allclose(back, x[:256], atol=1e-12)


def test_rope_far_position_against_mpmath():
    mpmath = pytest.importorskip("mpmath")
    mpmath.mp.dps = 40
    pos, hd = 131071, 512
    x = np.random.default_rng(2).standard_normal(hd)
    y = O.rope(x, 64, 1e6, pos)
    for i in (0, 1, 17, 63):
        ang = mpmath.mpf(pos) * mpmath.power(mpmath.mpf(10) ** 6, -mpmath.mpf(2 * i) / hd)
        c, s = mpmath.cos(ang), mpmath.sin(ang)
        a, b = mpmath.mpf(x[i]), mpmath.mpf(x[i + hd // 2])
        assert abs(float(a * c - b * s) - y[i]) < 1e-9
        assert abs(float(b * c + a * s) - y[i + hd // 2]) < 1e-9


def test_gelu_tanh_and_softcap():
    g = np.linspace(-8, 8, 1001)
    ref = torch.nn.functional.gelu(torch.from_numpy(g), approximate="tanh").numpy()
    got = np.array([O.gelu_tanh(v) for v in g])
    np.testing.assert_allclose(got, ref, rtol=1e-14, atol=1e-15)
    # gelu(x) - gelu(-x) = x
    assert all(abs(O.gelu_tanh(v) - O.gelu_tanh(-v) - v) < 1e-14 for v in g)
    # softcap: odd, bounded by the cap, slope 1 at 0, hits cap/2 at cap*atanh(1/2)
    assert O.softcap(0.0, 30.0) == 0.0
    assert O.softcap(-5.0, 30.0) == -O.softcap(5.0, 30.0)
    assert abs(O.softcap(1e-6, 30.0) - 1e-6) < 1e-17
    assert abs(O.softcap(30.0 * math.atanh(0.5), 30.0) - 15.0) < 1e-12
    assert O.softcap(1e4, 30.0) <= 30.0


# ----------------------------------------------------------------- attention --

def _sdpa(q, k, v, mask):
    """torch scaled_dot_product_attention (scale 1.0) over explicit keys."""
    qt = torch.from_numpy(q)[None, :, None, :]          # [1, H, 1, D]
    kt = torch.from_numpy(k)[None]                      # [1, H, L, D]
    vt = torch.from_numpy(v)[None]
    mt = torch.from_numpy(mask)[None, :, None, :]
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mt, scale=1.0)[0, :, 0]


@pytest.mark.parametrize("W,R,G", [(4, 8, 2), (8, 16, 1), (6, 12, 4), (5, 5, 2)])
def test_ring_attention_vs_brute_force_linear(W, R, G):
    """Ring with the implied-position window test == linear history with the
    window mask, at positions spanning >= 10 wraps of the ring."""
    rng = np.random.default_rng(W * 100 + R)
    n_kv, hd = 2, 16
    n_q = n_kv * G
    npos = 12 * R
    hist_k = rng.standard_normal((npos, n_kv, hd)).astype(np.float16)
    hist_v = rng.standard_normal((npos, n_kv, hd)).astype(np.float16)
    ring_k = np.zeros((n_kv, R, hd), dtype=np.float16)
    ring_v = np.zeros((n_kv, R, hd), dtype=np.float16)
    for q in range(npos):
        ring_k[:, q % R] = hist_k[q]        # slot = pos mod R
        ring_v[:, q % R] = hist_v[q]
        if q % 7 and q > 2 * R:
            continue
        qv = rng.standard_normal((n_q, hd)).astype(np.float16)
        got = O.attn_ring(qv.view(np.uint16), ring_k.view(np.uint16), ring_v.view(np.uint16), R, W, q)
        # implied positions: exactly the window [max(0, q-W+1), q]
        ip = O.ring_implied_positions(R, W, q)
        assert sorted(ip[ip >= 0].tolist()) == list(range(max(0, q - W + 1), q + 1))
        lo = max(0, q - W + 1)
        kk = np.repeat(hist_k[:q + 1].transpose(1, 0, 2), G, axis=0).astype(np.float64)
        vv = np.repeat(hist_v[:q + 1].transpose(1, 0, 2), G, axis=0).astype(np.float64)
        mask = np.zeros((n_q, q + 1), dtype=bool)
        mask[:, lo:] = True
        ref = _sdpa(qv.astype(np.float64), kk, vv, mask).numpy()
        np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)


def test_linear_attention_vs_sdpa():
    rng = np.random.default_rng(4)
    L, n_kv, G, hd = 300, 1, 16, 64
    k = rng.standard_normal((L, n_kv, hd)).astype(np.float16)
    v = rng.standard_normal((L, n_kv, hd)).astype(np.float16)
    q = rng.standard_normal((G, hd)).astype(np.float16)
    got = O.attn_linear(q.view(np.uint16), k.view(np.uint16), v.view(np.uint16), 211)
    kk = np.repeat(k[:211].transpose(1, 0, 2), G, axis=0).astype(np.float64)
    vv = np.repeat(v[:211].transpose(1, 0, 2), G, axis=0).astype(np.float64)
    ref = _sdpa(q.astype(np.float64), kk, vv, np.ones((G, 211), dtype=bool)).numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)


# ------------------------------------------------------------ decoder-level --

def _drafts(blocks, K, V, seed=0):
    ids = DG.uniform_int(seed, DG.STREAM_DRAFT_IDS, blocks * K, V).reshape(blocks, K)
    acc = DG.uniform_int(seed, DG.STREAM_ACCEPTED, blocks, K + 1)
    return ids, acc


def _run_verify(cfg, ring, single_pass, blocks=12, K=4, prefix=20, seed=0):
    m = O.Model(cfg, seed=seed, variant=1)
    cache = O.Cache(m, capacity=prefix + blocks * K + 8, ring=ring)
    V = cfg["vocab"]
    pre = DG.uniform_int(seed, DG.STREAM_PREFIX_IDS, prefix, V)
    for p in range(prefix):
        O.decode_step(m, cache, p, token=int(pre[p]), want_logits=False)
    ids, acc = _drafts(blocks, K, V, seed)
    pos, out = prefix, []
    for b in range(blocks):
        n = int(acc[b])
        if single_pass:
            r = O.verify_block(m, cache, pos, ids=ids[b], accepted=K, mode=1)
        else:
            r = O.verify_block(m, cache, pos, ids=ids[b], accepted=0, mode=0)
            O.verify_block(m, cache, pos, ids=ids[b], accepted=n, mode=0, want_logits=False)
        out.append(r["logits"])
        pos += n
    return np.stack(out)


def test_single_pass_R2W_equals_two_pass_bitwise():
    """With R = 2W a single pass (accepted_count = K each call, continue from
    p + n) gives the same logits, bit for bit, as the two-pass protocol."""
    cfg = dict(WL.MICRO)
    a = _run_verify(cfg, ring=2 * cfg["window"], single_pass=True)
    b = _run_verify(cfg, ring=2 * cfg["window"], single_pass=False)
    assert np.array_equal(a, b)


def test_single_pass_RW_differs_from_two_pass():
    """Negative control: with R = W a rejected row left in the ring is admitted
    by a later query, so the single pass no longer matches the two-pass result."""
    cfg = dict(WL.MICRO)
    a = _run_verify(cfg, ring=cfg["window"], single_pass=True)
    b = _run_verify(cfg, ring=cfg["window"], single_pass=False)
    assert not np.array_equal(a, b)


def test_k_eq_v_structure():
    cfg = WL.MICRO
    m = O.Model(cfg, seed=1, variant=1)
    c = O.Cache(m, 16)
    r = O.decode_step(m, c, 3, token=17, want_dump=True)
    full = [l for l in range(cfg["n_layers"]) if WL.layer_is_full(cfg, l)]
    assert full
    hd = cfg["gl_head_dim"]
    for l in full:
        kraw = r["vraw"][l, 0, :hd]
        v16 = r["kv"][l, 0, 1, :hd]
        k16 = r["kv"][l, 0, 0, :hd]
        ref = torch.nn.functional.rms_norm(torch.from_numpy(kraw), (hd,), None, eps=cfg["rms_eps"])
        assert np.array_equal(v16, ref.numpy().astype(np.float16).view(np.uint16))
        assert not np.array_equal(k16, v16)


def test_capacity_invariance_bitwise():
    cfg = WL.MICRO
    m = O.Model(cfg, seed=2)
    ids = DG.uniform_int(2, DG.STREAM_PREFIX_IDS, 60, cfg["vocab"])
    outs = []
    for cap in (64, 4096):
        c = O.Cache(m, cap)
        for p in range(60):
            r = O.decode_step(m, c, p, token=int(ids[p]), want_logits=(p % 10 == 9))
            if p % 10 == 9:
                outs.append(r["logits"])
    half = len(outs) // 2
    for a, b in zip(outs[:half], outs[half:]):
        assert np.array_equal(a, b)
