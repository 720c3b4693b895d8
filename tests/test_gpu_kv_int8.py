"""The int8 KV cache ("Gemma-4-12B-CoreAI", per-tier cost section: K/V rows as int8
halve the cache) against the oracle.

* Flash-decode over int8 rows (ring and linear entry points) against the oracle's
  attention over the same codes and scales: |o - o_ref| <= 2e-3 (1 + |o_ref|).
* The tiny decoder with kv_int8, from a GPU-written history handed to the oracle
  before each compared step: decode steps and a verify block against the oracle
  (the decode tolerance), and the rows a step writes: placement exact; layer 0's
  codes within one step and scales within fp16 rounding of the oracle's (both
  sides quantize their own fp16 rows, which agree within an fp16 ulp in layer 0).
* One period of the 12B shapes at 32K decode and at 128K verify (K = 4) over the
  same seeded int8 history on both sides.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import datagen as DG
from datagen import synth as S
from datagen import workloads as WL
from int4_q4_gemv_b200 import build as B
from int4_q4_gemv_b200 import q4g as Q
from oracle import oracle as O

pytestmark = pytest.mark.gpu

TOL, TIE = 2e-2, 1e-3


@pytest.fixture(scope="module", autouse=True)
def _built():
    B.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def sp():
    return S.stream_ptr()


def _ws(n_q, hd):
    nb = Q.q4g_flash_decode_workspace_bytes(n_q, hd)
    return torch.empty(nb, dtype=torch.uint8, device="cuda"), nb


def _codes_scales(rng, shape, scale_lo, scale_hi):
    codes = rng.integers(-127, 128, size=shape).astype(np.int8)
    scales = (scale_lo + (scale_hi - scale_lo) * rng.random(shape[:-1])).astype(np.float32)
    return codes, scales


@pytest.mark.parametrize("n_q,n_kv,W,R,pos", [(16, 8, 1024, 2048, 5000), (16, 8, 1024, 2048, 700),
                                              (8, 2, 256, 512, 1531), (8, 8, 100, 160, 333)])
def test_flash_decode_ring_i8_vs_oracle(n_q, n_kv, W, R, pos):
    hd = 256
    rng = np.random.default_rng(pos + W + 1)
    q = rng.standard_normal((n_q, hd)).astype(np.float16)
    k8, ks = _codes_scales(rng, (n_kv, R, hd), 0.002, 0.01)
    v8, vs = _codes_scales(rng, (n_kv, R, hd), 0.005, 0.02)
    ws, nb = _ws(n_q, hd)
    out = torch.empty((n_q, hd), dtype=torch.float16, device="cuda")
    t = [torch.from_numpy(a).cuda() for a in (q, k8, ks, v8, vs)]
    Q.q4g_flash_decode_ring_i8(t[0].data_ptr(), n_q, n_kv, hd, t[1].data_ptr(), t[2].data_ptr(), t[3].data_ptr(),
                               t[4].data_ptr(), R, W, pos, out.data_ptr(), ws.data_ptr(), nb, sp())
    ref = O.attn_ring_i8(q.view(np.uint16), k8, ks, v8, vs, R, W, pos)
    got = out.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - ref) <= 2e-3 * (1 + np.abs(ref)))


@pytest.mark.parametrize("n_q,length", [(16, 1), (16, 4096), (16, 20001), (8, 3000)])
def test_flash_decode_linear_i8_vs_oracle(n_q, length):
    hd = 512
    rng = np.random.default_rng(length + 2)
    q = rng.standard_normal((n_q, hd)).astype(np.float16)
    cap = length + 17
    k8, ks = _codes_scales(rng, (cap, 1, hd), 0.002, 0.01)
    v8, vs = _codes_scales(rng, (cap, 1, hd), 0.005, 0.02)
    ws, nb = _ws(n_q, hd)
    out = torch.empty((n_q, hd), dtype=torch.float16, device="cuda")
    t = [torch.from_numpy(a).cuda() for a in (q, k8, ks, v8, vs)]
    Q.q4g_flash_decode_linear_i8(t[0].data_ptr(), n_q, 1, hd, t[1].data_ptr(), t[2].data_ptr(), t[3].data_ptr(),
                                 t[4].data_ptr(), length, out.data_ptr(), ws.data_ptr(), nb, sp())
    ref = O.attn_linear_i8(q.view(np.uint16), k8, ks, v8, vs, length)
    got = out.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - ref) <= 2e-3 * (1 + np.abs(ref)))


def _check(got, ref, where):
    rms = float(np.sqrt(np.mean(ref ** 2)))
    err = float(np.max(np.abs(got - ref)))
    assert err <= TOL * rms, f"{where}: max err {err} > {TOL} * rms {rms}"
    a_ref, a_got = int(np.argmax(ref.astype(np.float32))), int(np.argmax(got))
    if a_ref != a_got:
        assert float(ref[a_ref] - ref[a_got]) <= TIE * rms, f"{where}: argmax {a_got} != {a_ref}"


def _handoff_i8(gc, oc):
    v = gc.view
    for i in range(v.n_sliding):
        for kv in (0, 1):
            c, s = oc.ring_i8(i, kv)
            gcodes, gscales = gc.ring_i8(i, kv)
            c[...] = gcodes.cpu().numpy()
            s[...] = gscales.cpu().numpy()
    for i in range(v.n_full):
        for kv in (0, 1):
            c, s = oc.global_i8(i, kv)
            gcodes, gscales = gc.global_i8(i, kv)
            c[...] = gcodes.cpu().numpy()
            s[...] = gscales.cpu().numpy()


def test_tiny_int8_decode_verify_and_cache_rows():
    """The GPU runs a 300-token prefix alone; its int8 cache is handed to the oracle
    before every compared step, so both sides read the same history and differ only
    by the step's own rows. (Compared over a free-running history instead, the two
    sides' fp16 K/V rows, equal within an fp16 ulp, round to int8 codes that differ
    by one where a value sits at a code boundary; such a flip moves the value by
    scale = amax / 127, far more than the fp16 ulp, and the flips accumulate in the
    history.)"""
    cfg = dict(WL.TINY, kv_int8=1)
    seed, V = 6, cfg["vocab"]
    g = S.SynthDecoder(cfg, seed=seed, variant=1)
    om = O.Model(cfg, seed=seed, variant=1)
    gc, oc = g.new_cache(512), O.Cache(om, 512)
    assert gc.view.kv_int8 == 1
    lg = torch.empty((8, V), dtype=torch.float32, device="cuda")
    am = torch.empty(8, dtype=torch.int32, device="cuda")
    ids = DG.uniform_int(seed, DG.STREAM_PREFIX_IDS, 330, V)
    for pos in range(300):                  # the window (256) slides
        Q.q4g_decode_step(g.handle, gc.handle, int(ids[pos]), pos, 0, 0, sp())
    torch.cuda.synchronize()
    R = gc.view.ring
    for pos in range(300, 304):
        _handoff_i8(gc, oc)
        before = {i: [t.clone() for t in gc.ring_i8(i, 0)] for i in range(gc.view.n_sliding)}
        Q.q4g_decode_step(g.handle, gc.handle, int(ids[pos]), pos, lg.data_ptr(), am.data_ptr(), sp())
        r = O.decode_step(om, oc, pos, token=int(ids[pos]))
        torch.cuda.synchronize()
        _check(lg[0].cpu().numpy().astype(np.float64), r["logits"][0], f"pos {pos}")
        for i in range(gc.view.n_sliding):   # placement: only slot pos mod R changed
            codes, scales = gc.ring_i8(i, 0)
            changed = (codes != before[i][0]).any(dim=-1) | (scales != before[i][1])
            changed[:, pos % R] = False
            assert not bool(changed.any()), f"ring {i}: rows other than {pos % R} changed"
        c0, s0 = gc.ring_i8(0, 0)             # layer 0's new row against the oracle's
        oc0, os0 = oc.ring_i8(0, 0)
        gcode = c0[:, pos % R].cpu().numpy().astype(np.int64)
        ocode = oc0[:, pos % R].astype(np.int64)
        assert np.max(np.abs(gcode - ocode)) <= 1, "layer 0 codes"
        np.testing.assert_allclose(s0[:, pos % R].cpu().numpy(), os0[:, pos % R], rtol=2e-3)
    # a verify block of 4 rows against the oracle's two-pass protocol, same history
    _handoff_i8(gc, oc)
    K, pos = 4, 304
    blk = DG.uniform_int(seed, DG.STREAM_DRAFT_IDS, K, V).astype(np.int32)
    ids_d = torch.from_numpy(blk).cuda()
    Q.q4g_verify_block(g.handle, gc.handle, ids_d.data_ptr(), K, pos, K, lg.data_ptr(), am.data_ptr(), sp())
    r = O.verify_block(om, oc, pos, ids=blk, accepted=0, mode=0)
    torch.cuda.synchronize()
    for i in range(K):
        _check(lg[i].cpu().numpy().astype(np.float64), r["logits"][i], f"verify row {i}")
    Q.q4g_model_check(g.handle, sp())


def test_12b_period_int8_32k_decode_and_128k_verify():
    cfg = dict(WL.B12, n_layers=WL.B12["full_every"], kv_int8=1)
    seed, V = 4, cfg["vocab"]
    g = S.SynthDecoder(cfg, seed=seed, variant=1)
    om = O.Model(cfg, seed=seed, variant=1)
    lg = torch.empty((4, V), dtype=torch.float32, device="cuda")
    am = torch.empty(4, dtype=torch.int32, device="cuda")
    C = 32768
    gc, oc = g.new_cache(C), O.Cache(om, C)
    S.fill_history(gc)
    O.fill_history(oc)
    ids = DG.uniform_int(seed, DG.STREAM_PREFIX_IDS, 2, V)
    for i, pos in enumerate((C - 2, C - 1)):
        Q.q4g_decode_step(g.handle, gc.handle, int(ids[i]), pos, lg.data_ptr(), am.data_ptr(), sp())
        r = O.decode_step(om, oc, pos, token=int(ids[i]))
        torch.cuda.synchronize()
        _check(lg[0].cpu().numpy().astype(np.float64), r["logits"][0], f"32K pos {pos}")
    gc.close()
    oc.close()
    C, K = 131072, 4
    gc, oc = g.new_cache(C), O.Cache(om, C)
    S.fill_history(gc, seed=98)
    O.fill_history(oc, seed=98)
    acc = DG.uniform_int(seed, DG.STREAM_ACCEPTED, 2, K + 1)
    pos = C - 2 * K
    for b in range(2):
        blk = DG.uniform_int(seed, DG.STREAM_DRAFT_IDS, (b + 1) * K, V)[b * K:].astype(np.int32)
        ids_d = torch.from_numpy(blk).cuda()
        Q.q4g_verify_block(g.handle, gc.handle, ids_d.data_ptr(), K, pos, K, lg.data_ptr(), am.data_ptr(), sp())
        r = O.verify_block(om, oc, pos, ids=blk, accepted=0, mode=0)
        O.verify_block(om, oc, pos, ids=blk, accepted=int(acc[b]), mode=0, want_logits=False)
        torch.cuda.synchronize()
        for i in range(K):
            _check(lg[i].cpu().numpy().astype(np.float64), r["logits"][i], f"128K block {b} row {i}")
        pos += int(acc[b])
    Q.q4g_model_check(g.handle, sp())


def test_tiny_int8_verify_eight_rows_after_handoff():
    """A verify block of K = 8 rows (32 query rows per KV head on the tensor-core
    ring path) over a handed-off int8 history, against the oracle's two-pass protocol,
    and the argmax output of every row."""
    cfg = dict(WL.TINY, kv_int8=1)
    seed, V, K = 9, cfg["vocab"], 8
    g = S.SynthDecoder(cfg, seed=seed, variant=1)
    om = O.Model(cfg, seed=seed, variant=1)
    gc, oc = g.new_cache(512), O.Cache(om, 512)
    ids = DG.uniform_int(seed, DG.STREAM_PREFIX_IDS, 280, V)
    for pos in range(270):
        Q.q4g_decode_step(g.handle, gc.handle, int(ids[pos]), pos, 0, 0, sp())
    torch.cuda.synchronize()
    _handoff_i8(gc, oc)
    blk = DG.uniform_int(seed, DG.STREAM_DRAFT_IDS, K, V).astype(np.int32)
    ids_d = torch.from_numpy(blk).cuda()
    lg = torch.empty((K, V), dtype=torch.float32, device="cuda")
    am = torch.empty(K, dtype=torch.int32, device="cuda")
    Q.q4g_verify_block(g.handle, gc.handle, ids_d.data_ptr(), K, 270, K, lg.data_ptr(), am.data_ptr(), sp())
    r = O.verify_block(om, oc, 270, ids=blk, accepted=0, mode=0)
    torch.cuda.synchronize()
    got32 = lg.cpu().numpy()
    for i in range(K):
        _check(got32[i].astype(np.float64), r["logits"][i], f"row {i}")
        assert int(am[i]) == int(np.argmax(got32[i]))
    Q.q4g_model_check(g.handle, sp())


def test_int8_capacity_and_graph_invariance_bitwise():
    """With int8 rows the logits do not depend on the cache capacity (512 or 1536),
    nor on graph replay against eager launches."""
    cfg = dict(WL.TINY, kv_int8=1)
    V = cfg["vocab"]
    g = S.SynthDecoder(cfg, seed=2, variant=1)
    caches = [g.new_cache(512), g.new_cache(1536), g.new_cache(512)]
    ids = DG.uniform_int(2, DG.STREAM_PREFIX_IDS, 300, V)
    lg = torch.empty((3, V), dtype=torch.float32, device="cuda")
    for pos in range(300):
        want = pos % 50 == 49
        for j, c in enumerate(caches):
            eager = j == 2
            if eager:
                Q.q4g_model_set_option(g.handle, Q.Q4G_OPT_CUDA_GRAPH, 0)
            Q.q4g_decode_step(g.handle, c.handle, int(ids[pos]), pos, lg[j].data_ptr() if want else 0, 0, sp())
            if eager:
                Q.q4g_model_set_option(g.handle, Q.Q4G_OPT_CUDA_GRAPH, 1)
        if want:
            torch.cuda.synchronize()
            assert torch.equal(lg[0], lg[1]), f"capacity, pos {pos}"
            assert torch.equal(lg[0], lg[2]), f"graph vs eager, pos {pos}"
    Q.q4g_model_check(g.handle, sp())
