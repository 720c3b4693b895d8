"""Seeded synthetic-input generators (numpy twin of ``datagen/q4g_datagen.h``).

Shared by the CPU oracle's tests and by the GPU harness. Nothing here computes
any step of the decode method: these functions only map (seed, stream, index)
to numbers, with the same definitions as the C header, so that host, device
and numpy fills of the same tensor are bit-identical.

Large tensors (the 12B-class weights) are filled on the device by
``libq4g_datagen.so`` (built from ``datagen/q4g_datagen_fill.cu``) or on the
host by the oracle, which includes the header directly.
"""
from __future__ import annotations

import numpy as np

M64 = np.uint64(0xFFFFFFFFFFFFFFFF)
_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_C1 = np.uint64(0xBF58476D1CE4E5B9)
_C2 = np.uint64(0x94D049BB133111EB)
_SKEY = np.uint64(0xD1B54A32D192ED03)

# Stream ids (same values as the C header).
STREAM_EMBED = 0x100
STREAM_FINAL_NORM = 0x101
T_WQ, T_WK, T_WV, T_WO, T_WGATE, T_WUP, T_WDOWN = range(7)
(T_NORM_IN, T_NORM_POST_ATTN, T_NORM_PRE_FFN, T_NORM_POST_FFN,
 T_NORM_Q, T_NORM_K, T_LAYER_SCALAR) = range(7, 14)
STREAM_PREFIX_IDS = 0x300000
STREAM_DRAFT_IDS = 0x400000
STREAM_ACCEPTED = 0x500000


def stream_layer(layer: int, tensor: int) -> int:
    return 0x1000 + layer * 0x20 + tensor


def stream_hidden(pos: int) -> int:
    return 0x200000 + pos


def stream_bench_x(s: int) -> int:
    return 0x600000 + s


def stream_bench_w(s: int) -> int:
    return 0x700000 + s


def stream_attn(s: int) -> int:
    return 0x800000 + s


def _mix64(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _C1
    z = (z ^ (z >> np.uint64(27))) * _C2
    return z ^ (z >> np.uint64(31))


def _splitmix64(x):
    with np.errstate(over="ignore"):
        return _mix64(np.asarray(x, dtype=np.uint64) + _GOLDEN)


def key(seed: int, stream: int) -> np.uint64:
    with np.errstate(over="ignore"):
        s = _splitmix64(np.uint64(seed))
        return np.uint64(_splitmix64(s ^ (np.uint64(stream) * _SKEY)))


def _word(k: np.uint64, idx: np.ndarray, j: int) -> np.ndarray:
    with np.errstate(over="ignore"):
        return _splitmix64(k + np.uint64(4) * idx + np.uint64(j))


def _indices(start: int, n: int) -> np.ndarray:
    return np.arange(start, start + n, dtype=np.uint64)


def unit_normal(seed: int, stream: int, n: int, start: int = 0) -> np.ndarray:
    """Irwin-Hall(12) unit normals, fp32, exact."""
    k = key(seed, stream)
    idx = _indices(start, n)
    s = np.zeros(n, dtype=np.int64)
    mask = np.uint64(0xFFFF)
    for j in range(3):
        w = _word(k, idx, j)
        for t in range(4):
            s += ((w >> np.uint64(16 * t)) & mask).astype(np.int64)
    return ((s - 393210).astype(np.float32) * np.float32(1.0 / 65536.0)).astype(np.float32)


def code8(seed: int, stream: int, n: int, start: int = 0) -> np.ndarray:
    """Seeded int8 codes: 36 x the unit normal, rounded half to even in exact integer
    arithmetic, clamped to [-127, 127] (the C header's dg_code8)."""
    k = key(seed, stream)
    idx = _indices(start, n)
    s = np.zeros(n, dtype=np.int64)
    mask = np.uint64(0xFFFF)
    for j in range(3):
        w = _word(k, idx, j)
        for t in range(4):
            s += ((w >> np.uint64(16 * t)) & mask).astype(np.int64)
    t = 9 * (s - 393210)
    q = t >> 14
    r = t - q * 16384
    q = q + ((r > 8192) | ((r == 8192) & ((q & 1) == 1))).astype(np.int64)
    return np.clip(q, -127, 127).astype(np.int8)


def normal(seed: int, stream: int, n: int, sigma: float, start: int = 0) -> np.ndarray:
    z = unit_normal(seed, stream, n, start)
    return (z * np.float32(sigma)).astype(np.float32)


def uniform_int(seed: int, stream: int, n: int, hi: int, start: int = 0) -> np.ndarray:
    k = key(seed, stream)
    w = _word(k, _indices(start, n), 3)
    return (w % np.uint64(hi)).astype(np.int64)


def uniform_float(seed: int, stream: int, n: int, lo: float, hi: float, start: int = 0) -> np.ndarray:
    k = key(seed, stream)
    w = _word(k, _indices(start, n), 3)
    u = (w >> np.uint64(40)).astype(np.float32) * np.float32(1.0 / 16777216.0)
    span = np.float32(np.float32(hi) - np.float32(lo))
    return (np.float32(lo) + (span * u).astype(np.float32)).astype(np.float32)


def gain(seed: int, stream: int, n: int, start: int = 0) -> np.ndarray:
    """Norm gain of the seeded variant: fp32(1 + N(0, 0.1))."""
    return (np.float32(1.0) + normal(seed, stream, n, 0.1, start)).astype(np.float32)


def history_stream(kind: str, ordinal: int, kv: int) -> int:
    """Stream id of the synthetic K/V history of one cache tensor
    (kind "ring": sliding-layer ordinal; "global": full-layer ordinal)."""
    return stream_attn((0x1000 if kind == "ring" else 0x2000) + 2 * ordinal + kv)


def history_sigma(kv: int, hd: int) -> float:
    """Standard deviation of the synthetic K/V history: the per-element scale the
    decoder itself writes. K rows are RoPE(rmsnorm(k) * gain) with gains of
    hd^(-1/4) (variants 0 and 1), whose elements have RMS hd^(-1/4); V rows are a
    scale-free RMSNorm, RMS 1."""
    return float(qk_gain_base(hd)) if kv == 0 else 1.0


def history_scale8(kv: int, hd: int) -> np.float32:
    """Row scale of the synthetic int8 K/V history: codes carry 36 per standard
    deviation, so code x scale has the standard deviation history_sigma."""
    return np.float32(np.float32(history_sigma(kv, hd)) / np.float32(36.0))


def qk_gain_base(hd: int) -> np.float32:
    """hd^(-1/4) as the fp32 constant of the C header (unit-variance q.k scores)."""
    return np.float32({256: 0.25, 512: 0.21022410381342863, 64: 0.35355339059327373,
                       32: 0.42044820762685725}.get(hd, 1.0))


def qk_gain(seed: int, stream: int, hd: int, variant: int) -> np.ndarray:
    """q_norm / k_norm gains: variant 0 the base, 1 the base times the seeded
    gain, 2 unit gains."""
    if variant == 2:
        return np.ones(hd, dtype=np.float32)
    b = qk_gain_base(hd)
    if variant != 1:
        return np.full(hd, b, dtype=np.float32)
    return (b * gain(seed, stream, hd)).astype(np.float32)
