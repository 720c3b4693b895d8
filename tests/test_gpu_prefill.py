"""Chunked prefill (q4g_prefill_chunk) against the oracle's decode-only prefill.

A chunk of S <= 64 tokens must leave the cache and produce the last row's logits
exactly as S decode steps in order would ("Gemma-4-12B-CoreAI", tiered-v3/
section: the last-row-only prefill entry point at S = 64), up to the rounding
of the multi-row GEMVs. The oracle runs the same tokens one decode step at a
time; logits are compared within the decode tolerance (max |err| <= 2e-2 RMS,
the same argmax unless the oracle's own top-2 gap is below 1e-3 RMS), on the
chunk's last row and on the decode steps that follow, which read every row the
chunks wrote.
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


def _check(got, ref, where):
    rms = float(np.sqrt(np.mean(ref ** 2)))
    err = float(np.max(np.abs(got - ref)))
    assert err <= TOL * rms, f"{where}: max err {err} > {TOL} * rms {rms}"
    a_ref, a_got = int(np.argmax(ref.astype(np.float32))), int(np.argmax(got))
    if a_ref != a_got:
        assert float(ref[a_ref] - ref[a_got]) <= TIE * rms, f"{where}: argmax {a_got} != {a_ref}"


def _run(cfg, seed, variant, capacity, chunks, n_decode):
    """chunks: list of (pos0, S); tokens are seeded ids. Returns nothing; asserts."""
    sp = S.stream_ptr()
    g = S.SynthDecoder(cfg, seed=seed, variant=variant)
    gc = g.new_cache(capacity)
    om = O.Model(cfg, seed=seed, variant=variant)
    oc = O.Cache(om, capacity)
    V = cfg["vocab"]
    end = max(p + n for p, n in chunks)
    ids = DG.uniform_int(seed, DG.STREAM_PREFIX_IDS, end + n_decode, V).astype(np.int32)
    ids_d = torch.from_numpy(ids).cuda()
    lg = torch.empty(V, dtype=torch.float32, device="cuda")
    am = torch.zeros(1, dtype=torch.int32, device="cuda")
    pos = 0
    for p0, n in chunks:
        assert p0 == pos
        lg.fill_(float("nan"))
        Q.q4g_prefill_chunk(g.handle, gc.handle, ids_d[p0:].data_ptr(), n, p0, lg.data_ptr(), am.data_ptr(), sp)
        r = None
        for q in range(p0, p0 + n):
            r = O.decode_step(om, oc, q, token=int(ids[q]), want_logits=q == p0 + n - 1)
        torch.cuda.synchronize()
        got = lg.cpu().numpy()
        _check(got.astype(np.float64), r["logits"][0], f"chunk at {p0} (S = {n}), last row")
        assert int(am) == int(np.argmax(got)), "argmax of the last row"
        pos = p0 + n
    dl = torch.empty(V, dtype=torch.float32, device="cuda")
    for q in range(pos, pos + n_decode):
        Q.q4g_decode_step(g.handle, gc.handle, int(ids[q]), q, dl.data_ptr(), 0, sp)
        r = O.decode_step(om, oc, q, token=int(ids[q]))
        torch.cuda.synchronize()
        _check(dl.cpu().numpy().astype(np.float64), r["logits"][0], f"decode at {q} after the chunks")
    Q.q4g_model_check(g.handle, sp)
    gc.close()
    g.close()
    om.close()


def test_tiny_chunks_then_decode():
    """64 + ragged 37 + 64 + 64 + 64 rows, then decode: the last chunks reach past the
    window of 256, so the window slides inside a chunk."""
    _run(WL.TINY, seed=8, variant=1, capacity=512,
         chunks=[(0, 64), (64, 37), (101, 64), (165, 64), (229, 64)], n_decode=3)


def test_tiny_chunks_across_the_ring_wrap():
    """Chunks that straddle the ring's wrap (R = 512): rows land in slots pos mod R."""
    _run(WL.TINY, seed=9, variant=0, capacity=1024,
         chunks=[(0, 64)] + [(64 * i, 64) for i in range(1, 8)] + [(512, 40), (552, 64)], n_decode=2)


def test_12b_period_chunk_then_decode():
    """One period of the 12B shapes (5 sliding + 1 full layer, the 262,144-row head):
    a 64-row chunk at position 0, a ragged 19-row chunk, then two decode steps."""
    cfg = dict(WL.B12, n_layers=WL.B12["full_every"])
    _run(cfg, seed=10, variant=1, capacity=4096, chunks=[(0, 64), (64, 19)], n_decode=2)


def test_prefill_range_errors():
    cfg = WL.TINY
    sp = S.stream_ptr()
    g = S.SynthDecoder(cfg, seed=1, variant=0)
    gc = g.new_cache(128)
    ids = torch.zeros(80, dtype=torch.int32, device="cuda")
    for n, p0 in ((0, 0), (65, 0), (10, 120), (1, -1)):
        with pytest.raises(Q.Q4GError) as e:
            Q.q4g_prefill_chunk(g.handle, gc.handle, ids.data_ptr(), n, p0, 0, 0, sp)
        assert e.value.status == Q.Q4G_ERANGE
    with pytest.raises(Q.Q4GError) as e:
        Q.q4g_prefill_chunk(g.handle, gc.handle, 0, 4, 0, 0, 0, sp)
    assert e.value.status == Q.Q4G_EINVAL
