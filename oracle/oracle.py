"""ctypes wrapper of the CPU oracle (oracle/liboracle.so): TEST INFRASTRUCTURE ONLY.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may import
this module. It never touches the CUDA library.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

import datagen as DG

from . import build as _build

_LIB = None


class OrConfig(C.Structure):
    _fields_ = [(n, C.c_int32) for n in (
        "n_layers", "hidden", "n_q_heads", "ffn", "vocab",
        "sl_kv_heads", "sl_head_dim", "window", "ring",
        "gl_kv_heads", "gl_head_dim", "full_every", "full_offset", "rope_pairs_full")] + \
        [(n, C.c_double) for n in ("rope_theta_sl", "rope_theta_gl", "rms_eps", "softcap",
                                   "embed_scale")] + [("v_norm_sliding", C.c_int32), ("head_fp16", C.c_int32),
                                                       ("kv_int8", C.c_int32)]


def _p(a):
    return a.ctypes.data_as(C.c_void_p) if a is not None else None


def lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = C.CDLL(path)
        vp, i64, i32, dbl, u64 = C.c_void_p, C.c_int64, C.c_int32, C.c_double, C.c_uint64
        sig = {
            "or_f16_from_double_array": (None, [vp, i64, vp]),
            "or_f16_to_double_array": (None, [vp, i64, vp]),
            "or_num_threads": (C.c_int, []),
            "or_set_num_threads": (None, [C.c_int]),
            "or_q4_0_pack": (C.c_int, [vp, i64, i64, vp, vp]),
            "or_q4_0_unpack": (None, [vp, vp, i64, i64, vp]),
            "or_gemv": (None, [vp, vp, i64, i64, C.c_int, vp, vp]),
            "or_gemv_f16": (None, [vp, i64, i64, C.c_int, vp, vp]),
            "or_model_embed_f16": (vp, [vp]),
            "or_rmsnorm": (None, [vp, vp, i64, dbl, vp]),
            "or_rope": (None, [vp, i64, i64, dbl, i64]),
            "or_gelu_tanh": (dbl, [dbl]),
            "or_softcap": (dbl, [dbl, dbl]),
            "or_attn_ring": (None, [vp, C.c_int, C.c_int, C.c_int, vp, vp, i64, i64, i64, vp]),
            "or_attn_linear": (None, [vp, C.c_int, C.c_int, C.c_int, vp, vp, i64, vp]),
            "or_ring_implied_positions": (None, [i64, i64, i64, vp]),
            "or_attn_ring_i8": (None, [vp, C.c_int, C.c_int, C.c_int, vp, vp, vp, vp, i64, i64, i64, vp]),
            "or_attn_linear_i8": (None, [vp, C.c_int, C.c_int, C.c_int, vp, vp, vp, vp, i64, vp]),
            "or_kv_quantize_row": (None, [vp, C.c_int, vp, vp]),
            "or_fill_code8": (None, [vp, i64, u64, u64, i64]),
            "or_cache_ring_i8": (vp, [vp, C.c_int, C.c_int, C.POINTER(vp)]),
            "or_cache_global_i8": (vp, [vp, C.c_int, C.c_int, C.POINTER(vp)]),
            "or_model_create": (vp, [C.POINTER(OrConfig), u64, C.c_int, C.c_int]),
            "or_model_destroy": (None, [vp]),
            "or_model_tensor": (i64, [vp, C.c_int, C.c_int, C.POINTER(vp), C.POINTER(vp),
                                      C.POINTER(i64)]),
            "or_cache_create": (vp, [vp, i64, i64]),
            "or_cache_destroy": (None, [vp]),
            "or_cache_clone": (vp, [vp]),
            "or_cache_ring": (vp, [vp, C.c_int, C.c_int]),
            "or_cache_global": (vp, [vp, C.c_int, C.c_int]),
            "or_fill_normal_f16": (None, [vp, i64, u64, u64, C.c_float, i64]),
            "or_verify_block": (C.c_int, [vp, vp, vp, vp, C.c_int, i64, C.c_int, C.c_int,
                                          vp, vp, vp, vp, vp]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


# ---------------------------------------------------------------- fp16 ----

def f16_bits(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.empty(x.shape, dtype=np.uint16)
    lib().or_f16_from_double_array(_p(x), x.size, _p(y))
    return y


def f16_value(bits) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    y = np.empty(b.shape, dtype=np.float64)
    lib().or_f16_to_double_array(_p(b), b.size, _p(y))
    return y


def set_threads(n: int) -> None:
    lib().or_set_num_threads(int(n))


def num_threads() -> int:
    return int(lib().or_num_threads())


# ---------------------------------------------------------------- q4_0 ----

def q4_0_pack(w):
    w = np.ascontiguousarray(w, dtype=np.float32)
    rows, k = w.shape
    qs = np.zeros((rows, k // 2), dtype=np.uint8)
    sc = np.zeros((rows, max(k // 32, 0)), dtype=np.uint16)
    rc = lib().or_q4_0_pack(_p(w), rows, k, _p(qs), _p(sc))
    if rc != 0:
        raise ValueError("q4_0 pack rejected the input (k % 32 != 0 or a non-finite value)")
    return qs, sc


def q4_0_unpack(qs, sc, k=None):
    qs = np.ascontiguousarray(qs, dtype=np.uint8)
    sc = np.ascontiguousarray(sc, dtype=np.uint16)
    rows = qs.shape[0]
    k = qs.shape[1] * 2 if k is None else k
    w = np.empty((rows, k), dtype=np.float64)
    lib().or_q4_0_unpack(_p(qs), _p(sc), rows, k, _p(w))
    return w


def gemv(qs, sc, x16):
    """y = dequant(W) @ x for x given as fp16 bits, shape [k] or [nrhs, k]."""
    qs = np.ascontiguousarray(qs, dtype=np.uint8)
    sc = np.ascontiguousarray(sc, dtype=np.uint16)
    x16 = np.ascontiguousarray(x16, dtype=np.uint16)
    n, k = qs.shape[0], qs.shape[1] * 2
    nrhs = 1 if x16.ndim == 1 else x16.shape[0]
    y = np.empty((nrhs, n), dtype=np.float64)
    lib().or_gemv(_p(qs), _p(sc), n, k, nrhs, _p(x16), _p(y))
    return y[0] if x16.ndim == 1 else y


def gemv_f16(w16, x16):
    """y = W @ x for fp16 weights W [n][k] and x as fp16 bits, shape [k] or [nrhs, k]."""
    w16 = np.ascontiguousarray(w16, dtype=np.uint16)
    x16 = np.ascontiguousarray(x16, dtype=np.uint16)
    n, k = w16.shape
    nrhs = 1 if x16.ndim == 1 else x16.shape[0]
    y = np.empty((nrhs, n), dtype=np.float64)
    lib().or_gemv_f16(_p(w16), n, k, nrhs, _p(x16), _p(y))
    return y[0] if x16.ndim == 1 else y


# ------------------------------------------------------------ elementwise --

def rmsnorm(x, w=None, eps=1e-6):
    x = np.ascontiguousarray(x, dtype=np.float64)
    wv = None if w is None else np.ascontiguousarray(w, dtype=np.float64)
    y = np.empty_like(x)
    lib().or_rmsnorm(_p(x), _p(wv), x.size, float(eps), _p(y))
    return y


def rope(x, rot_pairs, theta, pos):
    y = np.array(x, dtype=np.float64, copy=True)
    lib().or_rope(_p(y), y.size, int(rot_pairs), float(theta), int(pos))
    return y


def gelu_tanh(g: float) -> float:
    return lib().or_gelu_tanh(float(g))


def softcap(z: float, cap: float) -> float:
    return lib().or_softcap(float(z), float(cap))


# -------------------------------------------------------------- attention --

def attn_ring(q16, kc, vc, R, W, q):
    """q16 [n_q][hd]; kc/vc [n_kv][R][hd] fp16 bits; returns [n_q][hd] double."""
    q16 = np.ascontiguousarray(q16, dtype=np.uint16)
    kc = np.ascontiguousarray(kc, dtype=np.uint16)
    vc = np.ascontiguousarray(vc, dtype=np.uint16)
    n_q, hd = q16.shape
    n_kv = kc.shape[0]
    out = np.empty((n_q, hd), dtype=np.float64)
    lib().or_attn_ring(_p(q16), n_q, n_kv, hd, _p(kc), _p(vc), int(R), int(W), int(q), _p(out))
    return out


def attn_linear(q16, kc, vc, length):
    """q16 [n_q][hd]; kc/vc [L][n_kv][hd] fp16 bits; keys 0..length-1."""
    q16 = np.ascontiguousarray(q16, dtype=np.uint16)
    kc = np.ascontiguousarray(kc, dtype=np.uint16)
    vc = np.ascontiguousarray(vc, dtype=np.uint16)
    n_q, hd = q16.shape
    n_kv = kc.shape[1]
    out = np.empty((n_q, hd), dtype=np.float64)
    lib().or_attn_linear(_p(q16), n_q, n_kv, hd, _p(kc), _p(vc), int(length), _p(out))
    return out


def attn_ring_i8(q16, k8, ks, v8, vs, R, W, q):
    """int8 rows: k8/v8 [n_kv][R][hd] codes, ks/vs [n_kv][R] fp32 scales."""
    q16 = np.ascontiguousarray(q16, dtype=np.uint16)
    k8, v8 = (np.ascontiguousarray(a, dtype=np.int8) for a in (k8, v8))
    ks, vs = (np.ascontiguousarray(a, dtype=np.float32) for a in (ks, vs))
    n_q, hd = q16.shape
    out = np.empty((n_q, hd), dtype=np.float64)
    lib().or_attn_ring_i8(_p(q16), n_q, k8.shape[0], hd, _p(k8), _p(ks), _p(v8), _p(vs), int(R), int(W),
                          int(q), _p(out))
    return out


def attn_linear_i8(q16, k8, ks, v8, vs, length):
    """int8 rows: k8/v8 [L][n_kv][hd] codes, ks/vs [L][n_kv] fp32 scales; keys 0..length-1."""
    q16 = np.ascontiguousarray(q16, dtype=np.uint16)
    k8, v8 = (np.ascontiguousarray(a, dtype=np.int8) for a in (k8, v8))
    ks, vs = (np.ascontiguousarray(a, dtype=np.float32) for a in (ks, vs))
    n_q, hd = q16.shape
    out = np.empty((n_q, hd), dtype=np.float64)
    lib().or_attn_linear_i8(_p(q16), n_q, k8.shape[1], hd, _p(k8), _p(ks), _p(v8), _p(vs), int(length),
                            _p(out))
    return out


def kv_quantize_row(x16):
    """int8 KV row of fp16 bits x16 [hd]: (codes int8 [hd], scale float32)."""
    x16 = np.ascontiguousarray(x16, dtype=np.uint16)
    codes = np.empty(x16.size, dtype=np.int8)
    sc = np.zeros(1, dtype=np.float32)
    lib().or_kv_quantize_row(_p(x16), x16.size, _p(codes), _p(sc))
    return codes, sc[0]


def ring_implied_positions(R, W, q):
    out = np.empty(int(R), dtype=np.int64)
    lib().or_ring_implied_positions(int(R), int(W), int(q), _p(out))
    return out


# ------------------------------------------------------------------ model --

def make_config(d: dict) -> OrConfig:
    c = OrConfig()
    for name, _ in OrConfig._fields_:
        setattr(c, name, d[name])
    return c


class Model:
    """Oracle decoder with weights from the seeded recipe (datagen)."""

    def __init__(self, cfg: dict, seed: int = 0, variant: int = 0, nthreads: int = 0):
        self.cfg = dict(cfg)
        self._c = make_config(cfg)
        self.h = lib().or_model_create(C.byref(self._c), seed, variant, nthreads)
        if not self.h:
            raise RuntimeError("oracle model creation failed")

    def tensor(self, layer: int, t: int):
        qs, sc, cols = C.c_void_p(), C.c_void_p(), C.c_int64()
        rows = lib().or_model_tensor(self.h, layer, t, C.byref(qs), C.byref(sc), C.byref(cols))
        if rows == 0:
            return None
        k = cols.value
        q = np.ctypeslib.as_array(C.cast(qs, C.POINTER(C.c_uint8)), shape=(rows, k // 2)).copy()
        s = np.ctypeslib.as_array(C.cast(sc, C.POINTER(C.c_uint16)), shape=(rows, k // 32)).copy()
        return q, s

    def embed_f16(self):
        """The fp16 tied table (copy) when cfg["head_fp16"], else None."""
        ptr = lib().or_model_embed_f16(self.h)
        if not ptr:
            return None
        V, H = self.cfg["vocab"], self.cfg["hidden"]
        return np.ctypeslib.as_array(C.cast(ptr, C.POINTER(C.c_uint16)), shape=(V, H)).copy()

    def close(self):
        if self.h:
            lib().or_model_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class Cache:
    def __init__(self, model: Model, capacity: int, ring: int = 0, _handle=None):
        self.model = model
        self.capacity = capacity
        self.R = ring if ring else model.cfg["ring"]
        self.h = _handle if _handle is not None else lib().or_cache_create(model.h, capacity, ring)

    def clone(self) -> "Cache":
        return Cache(self.model, self.capacity, self.R, _handle=lib().or_cache_clone(self.h))

    def ring(self, sl_index: int, kv: int) -> np.ndarray:
        cfg = self.model.cfg
        ptr = lib().or_cache_ring(self.h, sl_index, kv)
        shape = (cfg["sl_kv_heads"], self.R, cfg["sl_head_dim"])
        return np.ctypeslib.as_array(C.cast(ptr, C.POINTER(C.c_uint16)), shape=shape)

    def global_(self, gl_index: int, kv: int) -> np.ndarray:
        cfg = self.model.cfg
        ptr = lib().or_cache_global(self.h, gl_index, kv)
        shape = (cfg["gl_kv_heads"], self.capacity, cfg["gl_head_dim"])
        return np.ctypeslib.as_array(C.cast(ptr, C.POINTER(C.c_uint16)), shape=shape)

    def _i8(self, fn, index, kv, rows, nkv, hd):
        sp = C.c_void_p()
        ptr = fn(self.h, index, kv, C.byref(sp))
        codes = np.ctypeslib.as_array(C.cast(ptr, C.POINTER(C.c_int8)), shape=(nkv, rows, hd))
        scales = np.ctypeslib.as_array(C.cast(sp, C.POINTER(C.c_float)), shape=(nkv, rows))
        return codes, scales

    def ring_i8(self, sl_index: int, kv: int):
        """int8 cache: (codes [n_kv][R][hd] int8, scales [n_kv][R] fp32), views."""
        cfg = self.model.cfg
        return self._i8(lib().or_cache_ring_i8, sl_index, kv, self.R, cfg["sl_kv_heads"], cfg["sl_head_dim"])

    def global_i8(self, gl_index: int, kv: int):
        cfg = self.model.cfg
        return self._i8(lib().or_cache_global_i8, gl_index, kv, self.capacity, cfg["gl_kv_heads"],
                        cfg["gl_head_dim"])

    def close(self):
        if self.h:
            lib().or_cache_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def fill_code8(out: np.ndarray, seed: int, stream: int, start: int = 0):
    """Seeded int8 codes from the C header (datagen's dg_code8)."""
    assert out.dtype == np.int8 and out.flags["C_CONTIGUOUS"]
    lib().or_fill_code8(_p(out), out.size, seed, stream, start)


def fill_normal_f16(out: np.ndarray, seed: int, stream: int, sigma: float = 1.0, start: int = 0):
    assert out.dtype == np.uint16 and out.flags["C_CONTIGUOUS"]
    lib().or_fill_normal_f16(_p(out), out.size, seed, stream, sigma, start)


def fill_history(cache: Cache, seed: int = 99):
    """Seeded fp16 K/V in every ring slot and every global row at the scale the
    decoder writes (datagen.history_sigma), from the same streams as the GPU
    harness (datagen.history_stream)."""
    cfg = cache.model.cfg
    n_sl = sum(1 for l in range(cfg["n_layers"]) if not _is_full(cfg, l))
    n_gl = cfg["n_layers"] - n_sl
    if cfg.get("kv_int8"):  # seeded codes and the constant row scale (datagen.code8)
        for kind, n, hd, get in (("ring", n_sl, cfg["sl_head_dim"], cache.ring_i8),
                                 ("global", n_gl, cfg["gl_head_dim"], cache.global_i8)):
            for i in range(n):
                for kv in (0, 1):
                    codes, scales = get(i, kv)
                    codes[...] = DG.code8(seed, DG.history_stream(kind, i, kv), codes.size).reshape(codes.shape)
                    scales[...] = DG.history_scale8(kv, hd)
        return
    for i in range(n_sl):
        for kv in (0, 1):
            fill_normal_f16(cache.ring(i, kv), seed, DG.history_stream("ring", i, kv),
                            DG.history_sigma(kv, cfg["sl_head_dim"]))
    for i in range(n_gl):
        for kv in (0, 1):
            fill_normal_f16(cache.global_(i, kv), seed, DG.history_stream("global", i, kv),
                            DG.history_sigma(kv, cfg["gl_head_dim"]))


def _is_full(cfg, l):
    return cfg["full_every"] > 0 and l % cfg["full_every"] == cfg["full_offset"]


def verify_block(model: Model, cache: Cache, pos0: int, ids=None, hidden=None, accepted=None,
                 mode: int = 0, want_logits: bool = True, want_dump: bool = False):
    """Run K rows at positions pos0.. (decode: K = 1). See or_verify_block."""
    cfg = model.cfg
    if ids is not None:
        ids_a = np.ascontiguousarray(np.atleast_1d(ids), dtype=np.int32)
        K = ids_a.size
        hid = None
    else:
        hid = np.ascontiguousarray(np.atleast_2d(hidden), dtype=np.float32)
        K = hid.shape[0]
        ids_a = None
    acc = K if accepted is None else int(accepted)
    V, H, L = cfg["vocab"], cfg["hidden"], cfg["n_layers"]
    hdmax = max(cfg["gl_head_dim"], cfg["sl_head_dim"])
    logits = np.empty((K, V), dtype=np.float64) if want_logits else None
    am = np.empty(K, dtype=np.int32)
    dump = np.empty((K, L + 1, H), dtype=np.float64) if want_dump else None
    kvd = np.empty((L, K, 2, hdmax), dtype=np.uint16) if want_dump else None
    vraw = np.empty((L, K, hdmax), dtype=np.float64) if want_dump else None
    rc = lib().or_verify_block(model.h, cache.h, _p(ids_a), _p(hid), K, int(pos0), acc, int(mode),
                               _p(logits), _p(am), _p(dump), _p(kvd), _p(vraw))
    if rc != 0:
        raise ValueError("oracle verify_block rejected its arguments")
    out = dict(argmax=am, logits=logits)
    if want_dump:
        out.update(dump=dump, kv=kvd, vraw=vraw)
    return out


def decode_step(model, cache, pos, token=None, hidden=None, **kw):
    if token is not None:
        return verify_block(model, cache, pos, ids=[token], **kw)
    return verify_block(model, cache, pos, hidden=np.atleast_2d(hidden), **kw)
