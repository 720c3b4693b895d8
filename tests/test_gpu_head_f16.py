"""The fp16 tied embedding / head ("Gemma-4-12B-CoreAI", tiered-v3/ section: the
vocabulary path kept at fp16) against the oracle.

* q4g_gemv_f16 element by element against the oracle's fp16 GEMV, within the
  worst-case bound of fp32 accumulation of exact fp16 products: k * 2^-24 * sum|w x|.
* The tiny decoder with head_fp16 = 1: its fp16 table bitwise, decode steps and a
  verify block within the decode tolerance (max |err| <= 2e-2 RMS, same argmax).
* The 12B-class head shape (262144 x 3840) on sampled rows.
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

TOL = 2e-2


@pytest.fixture(scope="module", autouse=True)
def _built():
    B.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _bound(w16: np.ndarray, x16: np.ndarray) -> np.ndarray:
    k = w16.shape[1]
    a = np.abs(w16.view(np.float16).astype(np.float64)) @ np.abs(x16.view(np.float16).astype(np.float64)).T
    return a.T * k * 2.0 ** -24 + 1e-30


def _run(w: torch.Tensor, x: torch.Tensor) -> np.ndarray:
    n, k = w.shape
    nrhs = x.shape[0]
    y = torch.empty((nrhs, n), dtype=torch.float32, device="cuda")
    Q.q4g_gemv_f16(w.data_ptr(), n, k, x.data_ptr(), nrhs, y.data_ptr(), S.stream_ptr())
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("n,k,nrhs", [(37, 256, 1), (2500, 3840, 1), (777, 1024, 3), (300, 3840, 8),
                                      (129, 8192, 5)])
def test_gemv_f16_vs_oracle(n, k, nrhs):
    seed = n + k + nrhs
    w = torch.empty((n, k), dtype=torch.float16, device="cuda")
    S.fill_normal_f16(w, seed, DG.STREAM_EMBED, 0.02)
    x = torch.empty((nrhs, k), dtype=torch.float16, device="cuda")
    S.fill_normal_f16(x, seed, DG.stream_hidden(0), 1.0)
    got = _run(w, x)
    w16 = w.cpu().numpy().view(np.uint16)
    x16 = x.cpu().numpy().view(np.uint16)
    ref = O.gemv_f16(w16, x16).reshape(nrhs, n)
    err = np.abs(got - ref)
    assert np.all(err <= _bound(w16, x16)), f"max err {err.max()}"


def test_gemv_f16_rejects_bad_shapes():
    w = torch.zeros((4, 256), dtype=torch.float16, device="cuda")
    x = torch.zeros((1, 256), dtype=torch.float16, device="cuda")
    y = torch.zeros((1, 4), dtype=torch.float32, device="cuda")
    for n, k, nrhs in [(4, 128, 1), (4, 256, 0), (4, 256, 9), (4, 16384, 1)]:
        with pytest.raises(Q.Q4GError):
            Q.q4g_gemv_f16(w.data_ptr(), n, k, x.data_ptr(), nrhs, y.data_ptr(), S.stream_ptr())
    Q.q4g_gemv_f16(w.data_ptr(), 0, 256, x.data_ptr(), 1, y.data_ptr(), S.stream_ptr())  # empty: no-op


def test_head_shape_sampled_rows():
    """The 12B-class fp16 head, 262144 x 3840, one activation row: 4096 sampled rows
    (a seeded spread plus the first and last) against the oracle."""
    n, k = 262144, 3840
    w = torch.empty((n, k), dtype=torch.float16, device="cuda")
    S.fill_normal_f16(w, 0, DG.STREAM_EMBED, 0.02)
    x = torch.empty((1, k), dtype=torch.float16, device="cuda")
    S.fill_normal_f16(x, 0, DG.stream_hidden(1), 1.0)
    got = _run(w, x)[0]
    rows = np.unique(np.concatenate([[0, n - 1], DG.uniform_int(5, DG.STREAM_DRAFT_IDS, 4094, n)]))
    w16 = w[torch.from_numpy(rows).cuda()].cpu().numpy().view(np.uint16)
    x16 = x.cpu().numpy().view(np.uint16)
    ref = O.gemv_f16(w16, x16).reshape(1, -1)
    err = np.abs(got[rows] - ref[0])
    assert np.all(err <= _bound(w16, x16)[0]), f"max err {err.max()}"


def _check(got, ref, where):
    rms = float(np.sqrt(np.mean(ref ** 2)))
    err = float(np.max(np.abs(got - ref)))
    assert err <= TOL * rms, f"{where}: max err {err} > {TOL} * rms {rms}"
    a_ref, a_got = int(np.argmax(ref.astype(np.float32))), int(np.argmax(got))
    if a_ref != a_got:
        assert float(ref[a_ref] - ref[a_got]) <= 1e-3 * rms, f"{where}: argmax {a_got} != {a_ref}"


def test_tiny_fp16_head_decode_and_verify():
    cfg = WL.TINY_F16
    seed, V = 2, cfg["vocab"]
    g = S.SynthDecoder(cfg, seed=seed, variant=1)
    om = O.Model(cfg, seed=seed, variant=1)
    assert np.array_equal(g.embed_f16.cpu().numpy().view(np.uint16), om.embed_f16())
    gc, oc = g.new_cache(512), O.Cache(om, 512)
    lg = torch.empty((8, V), dtype=torch.float32, device="cuda")
    am = torch.empty(8, dtype=torch.int32, device="cuda")
    ids = DG.uniform_int(seed, DG.STREAM_PREFIX_IDS, 300, V)
    for pos in range(300):                  # beyond W = 256: the window slides
        want = pos % 50 == 49
        Q.q4g_decode_step(g.handle, gc.handle, int(ids[pos]), pos, lg.data_ptr() if want else 0,
                          am.data_ptr(), S.stream_ptr())
        r = O.decode_step(om, oc, pos, token=int(ids[pos]), want_logits=want)
        if want:
            torch.cuda.synchronize()
            _check(lg[0].cpu().numpy().astype(np.float64), r["logits"][0], f"pos {pos}")
    K, pos = 4, 300
    blk = DG.uniform_int(seed, DG.STREAM_DRAFT_IDS, K, V).astype(np.int32)
    ids_d = torch.from_numpy(blk).cuda()
    Q.q4g_verify_block(g.handle, gc.handle, ids_d.data_ptr(), K, pos, K, lg.data_ptr(), am.data_ptr(),
                       S.stream_ptr())
    r = O.verify_block(om, oc, pos, ids=blk, accepted=0, mode=0)
    torch.cuda.synchronize()
    got = lg[:K].cpu().numpy().astype(np.float64)
    for i in range(K):
        _check(got[i], r["logits"][i], f"verify row {i}")
        assert int(am[i]) == int(np.argmax(lg[i].cpu().numpy()))  # lowest index of the largest logit
    Q.q4g_model_check(g.handle, S.stream_ptr())
