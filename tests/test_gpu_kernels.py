"""Kernel-level parity of the CUDA path against the oracle (through the C-ABI).

Tolerances:
  * q4_0 pack: bit-exact (integer codes and fp16 scales).
  * GEMV: |y - y_ref| <= 2e-4 * sum_b |d_b| sum_b |x| + 2^-15 * sum_b |d_b| max_b |x| sum_b |c - 8|
    + 1e-6 (sums over the 32 columns of block b). First term, the fp32 arithmetic: per
    block the fp16 path accumulates 32 products (64 + c) x (each <= 79 |x|) in fp32, a
    rounding error below 32 * 2^-24 * 79 * sum|x| ~ 1.5e-4 sum|x| before the scale d.
    Second term, the integer path: x enters it as 16-bit fixed point relative to the
    block's largest exponent, each value off by at most 2^-15 of the block maximum and
    weighted by |c - 8|; the block sums themselves are exact integers. The reference is
    fp64 on the same fp16 x and dequantised weights.
  * attention: fp16 output, |o - o_ref| <= 2e-3 * (1 + |o_ref|): half an fp16 ulp
    (2^-11 relative) plus the fp16 hi/lo probability split (~2^-22).
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


@pytest.fixture(scope="module", autouse=True)
def _built():
    B.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.init()


def sp():
    return S.stream_ptr()


def _adversarial(rows, k, seed):
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal((rows, k)) * 0.02).astype(np.float32)
    if rows > 6 and k >= 64:
        w[0] = 0.0
        w[1, :32] = -0.0
        w[1, 32:64] = 1e-30
        w[2, :32] = np.linspace(-1, 1, 32)
        w[3, :] = rng.choice([-3.0, 3.0], size=k)
        w[4, :] *= 1e4
        w[5, :32] = np.array([0.25, 1.25, -1.25, 0.75] * 8, dtype=np.float32)  # exact halfway codes
        w[6, :] = (rng.integers(-8, 8, size=k) * 0.125).astype(np.float32)
    return w


@pytest.mark.parametrize("rows,k", [(1, 32), (37, 96), (64, 1024), (300, 3840)])
def test_pack_bitexact_vs_oracle(rows, k):
    w = _adversarial(rows, k, rows + k)
    qs_ref, sc_ref = O.q4_0_pack(w)
    wd = torch.from_numpy(w).cuda()
    qs = torch.empty((rows, k // 2), dtype=torch.uint8, device="cuda")
    sc = torch.empty((rows, k // 32), dtype=torch.int16, device="cuda")
    Q.q4g_q4_0_pack(wd.data_ptr(), rows, k, qs.data_ptr(), sc.data_ptr(), 1, sp())
    assert np.array_equal(qs.cpu().numpy(), qs_ref)
    assert np.array_equal(sc.cpu().numpy().view(np.uint16), sc_ref)
    # host-pointer path, and unpack (exact: (c - 8) * d fits fp32)
    qh = np.zeros_like(qs_ref)
    sh = np.zeros_like(sc_ref)
    Q.q4g_q4_0_pack(w.ctypes.data, rows, k, qh.ctypes.data, sh.ctypes.data, 0, sp())
    assert np.array_equal(qh, qs_ref) and np.array_equal(sh, sc_ref)
    out = torch.empty((rows, k), dtype=torch.float32, device="cuda")
    Q.q4g_q4_0_unpack(qs.data_ptr(), sc.data_ptr(), rows, k, out.data_ptr(), 1, sp())
    assert np.array_equal(out.cpu().numpy().astype(np.float64), O.q4_0_unpack(qs_ref, sc_ref))


def test_pack_rejects_non_finite():
    w = torch.zeros((4, 64), dtype=torch.float32, device="cuda")
    w[2, 5] = float("nan")
    qs = torch.empty((4, 32), dtype=torch.uint8, device="cuda")
    sc = torch.empty((4, 2), dtype=torch.int16, device="cuda")
    with pytest.raises(Q.Q4GError) as e:
        Q.q4g_q4_0_pack(w.data_ptr(), 4, 64, qs.data_ptr(), sc.data_ptr(), 1, sp())
    assert e.value.status == Q.Q4G_EINVAL
    w[2, 5] = float("inf")
    with pytest.raises(Q.Q4GError):
        Q.q4g_q4_0_pack(w.data_ptr(), 4, 64, qs.data_ptr(), sc.data_ptr(), 1, sp())


def _gemv_bound(qs, sc, x16):
    d = np.abs(O.f16_value(sc))                                  # [n][nb]
    xa = np.abs(x16.view(np.float16).astype(np.float64))         # [r][k]
    n, nb = sc.shape
    xb = xa.reshape(xa.shape[0], nb, 32).sum(axis=2)             # [r][nb]
    xm = xa.reshape(xa.shape[0], nb, 32).max(axis=2)             # [r][nb]
    q = qs.reshape(n, nb, 16).astype(np.int64)                   # byte b: column b (low), b + 16 (high)
    cabs = np.abs((q & 15) - 8).sum(axis=2) + np.abs((q >> 4) - 8).sum(axis=2)  # [n][nb]
    return 2e-4 * (xb @ d.T) + 2.0 ** -15 * (xm @ (d * cabs).T) + 1e-6   # [r][n]


def _run_gemv(qs_t, sc_t, n, k, x16):
    r = x16.shape[0]
    xd = torch.from_numpy(x16.view(np.int16).copy()).cuda()
    y = torch.empty((r, n), dtype=torch.float32, device="cuda")
    Q.q4g_gemv(qs_t.data_ptr(), sc_t.data_ptr(), n, k, xd.data_ptr(), r, y.data_ptr(), sp())
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("n,k,nrhs", [(16, 32, 1), (40, 96, 1), (1000, 1024, 1), (2048, 4096, 2),
                                      (333, 3840, 3), (512, 15360, 4), (96, 8192, 8), (4096, 1024, 5)])
def test_gemv_vs_oracle(n, k, nrhs):
    rng = np.random.default_rng(n + k)
    w = _adversarial(n, k, n * 7 + k)
    qs, sc = O.q4_0_pack(w)
    x16 = rng.standard_normal((nrhs, k)).astype(np.float16).view(np.uint16)
    y = _run_gemv(torch.from_numpy(qs).cuda(), torch.from_numpy(sc.view(np.int16)).cuda(), n, k, x16)
    ref = O.gemv(qs, sc, x16)
    assert np.all(np.abs(y - ref) <= _gemv_bound(qs, sc, x16))


@pytest.mark.parametrize("name,n,k,seed", WL.GEMV_SHAPES)
def test_gemv_full_size_sampled_rows(name, n, k, seed):
    """The four microbench shapes at full size (weights from the seeded recipe,
    packed on the device), checked against the oracle on sampled rows."""
    qs_t, sc_t = S.packed_tensor(n, k, seed, DG.stream_bench_w(seed))
    x = torch.empty(k, dtype=torch.float16, device="cuda")
    S.fill_normal_f16(x, seed, DG.stream_bench_x(seed), 1.0)
    y = torch.empty(n, dtype=torch.float32, device="cuda")
    Q.q4g_gemv(qs_t.data_ptr(), sc_t.data_ptr(), n, k, x.data_ptr(), 1, y.data_ptr(), sp())
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([np.arange(16), np.arange(n - 16, n),
                                     np.random.default_rng(seed).integers(0, n, 512)]))
    qs = qs_t[rows].cpu().numpy()
    sc = sc_t[rows].cpu().numpy().view(np.uint16)
    # the oracle packs the same seeded weights itself for the sampled rows
    w_rows = np.stack([DG.normal(seed, DG.stream_bench_w(seed), k, 0.02, start=int(r) * k) for r in rows])
    qs_o, sc_o = O.q4_0_pack(w_rows)
    assert np.array_equal(qs, qs_o) and np.array_equal(sc, sc_o)
    x16 = x.cpu().numpy().view(np.uint16)[None, :]
    assert np.array_equal(x16[0], DG.normal(seed, DG.stream_bench_x(seed), k, 1.0).astype(np.float16).view(np.uint16))
    ref = O.gemv(qs_o, sc_o, x16)[0]
    got = y.cpu().numpy().astype(np.float64)[rows]
    assert np.all(np.abs(got - ref) <= _gemv_bound(qs_o, sc_o, x16)[0])


def _attn_ws(n_q, hd):
    nbytes = Q.q4g_flash_decode_workspace_bytes(n_q, hd)
    return torch.empty(nbytes, dtype=torch.uint8, device="cuda"), nbytes


@pytest.mark.parametrize("n_q,n_kv,W,R,pos", [
    (16, 8, 1024, 2048, 5000),     # 12B-class sliding shape, wrapped ring
    (16, 8, 1024, 2048, 700),      # young ring (q < W): unwritten slots masked
    (8, 2, 256, 512, 1531),        # tiny-config shape
    (4, 1, 64, 128, 0),            # a single live key
    (16, 8, 100, 160, 333),        # window not a multiple of the tile
    (8, 8, 1024, 2048, 3001),      # one query row per KV head
    (2, 2, 256, 512, 700),         # one row per head, few heads
])
def test_flash_decode_ring_vs_oracle(n_q, n_kv, W, R, pos):
    hd = 256
    rng = np.random.default_rng(pos + W)
    q = rng.standard_normal((n_q, hd)).astype(np.float16)
    kc = rng.standard_normal((n_kv, R, hd)).astype(np.float16)
    vc = rng.standard_normal((n_kv, R, hd)).astype(np.float16)
    ws, nb = _attn_ws(n_q, hd)
    out = torch.empty((n_q, hd), dtype=torch.float16, device="cuda")
    qd, kd, vd = (torch.from_numpy(a).cuda() for a in (q, kc, vc))
    Q.q4g_flash_decode_ring(qd.data_ptr(), n_q, n_kv, hd, kd.data_ptr(), vd.data_ptr(), R, W, pos,
                            out.data_ptr(), ws.data_ptr(), nb, sp())
    ref = O.attn_ring(q.view(np.uint16), kc.view(np.uint16), vc.view(np.uint16), R, W, pos)
    got = out.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - ref) <= 2e-3 * (1 + np.abs(ref)))


@pytest.mark.parametrize("n_q,length", [(16, 1), (16, 63), (16, 4096), (16, 20001), (8, 3000), (16, 131072)])
def test_flash_decode_linear_vs_oracle(n_q, length):
    hd = 512
    rng = np.random.default_rng(length)
    q = rng.standard_normal((n_q, hd)).astype(np.float16)
    cap = length + 17
    kc = rng.standard_normal((cap, 1, hd)).astype(np.float16)
    vc = rng.standard_normal((cap, 1, hd)).astype(np.float16)
    ws, nb = _attn_ws(n_q, hd)
    out = torch.empty((n_q, hd), dtype=torch.float16, device="cuda")
    qd, kd, vd = (torch.from_numpy(a).cuda() for a in (q, kc, vc))
    Q.q4g_flash_decode_linear(qd.data_ptr(), n_q, 1, hd, kd.data_ptr(), vd.data_ptr(), length,
                              out.data_ptr(), ws.data_ptr(), nb, sp())
    ref = O.attn_linear(q.view(np.uint16), kc.view(np.uint16), vc.view(np.uint16), length)
    got = out.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - ref) <= 2e-3 * (1 + np.abs(ref)))


@pytest.mark.parametrize("kind", [Q.Q4G_GEMV_WARP_STREAM, Q.Q4G_GEMV_REGISTER, Q.Q4G_GEMV_STAGE])
@pytest.mark.parametrize("n,k,nrhs", [(3840, 15360, 1), (8192, 3840, 1), (1000, 1024, 2), (3840, 4096, 4),
                                      (260, 3840, 2), (77, 256, 1), (3840, 15360, 4), (1000, 8192, 8),
                                      (531, 3840, 3), (40, 256, 7)])
def test_gemv_every_kernel_meets_the_oracle_bound(kind, n, k, nrhs):
    """Each GEMV kernel (forced for the whole process, falling back where it
    cannot take the call) meets the oracle bound on the same inputs, including
    ragged row counts and the largest k."""
    rng = np.random.default_rng(n + 3 * k)
    w = _adversarial(n, k, n + k + 1)
    qs, sc = O.q4_0_pack(w)
    x16 = rng.standard_normal((nrhs, k)).astype(np.float16).view(np.uint16)
    qs_t, sc_t = torch.from_numpy(qs).cuda(), torch.from_numpy(sc.view(np.int16)).cuda()
    ref = O.gemv(qs, sc, x16)
    Q.q4g_set_gemv_kernel(kind)
    try:
        y = _run_gemv(qs_t, sc_t, n, k, x16)
    finally:
        Q.q4g_set_gemv_kernel(Q.Q4G_GEMV_AUTO)
    assert np.all(np.abs(y - ref) <= _gemv_bound(qs, sc, x16))
