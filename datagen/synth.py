"""Synthetic decoder on the GPU from the seeded recipe (test and bench harness).

Weights are generated on the device by libq4g_datagen.so (the same
(seed, stream, index) definitions as the oracle's C generator and the numpy
twin) and quantised with the library's own q4g_q4_0_pack. torch provides the
device memory and the stream; nothing here computes a step of the decode.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np
import torch

import datagen as DG
from datagen import workloads as WL
from int4_q4_gemv_b200 import q4g as Q

_HERE = os.path.dirname(os.path.abspath(__file__))
_DG = None


def dglib():
    global _DG
    if _DG is None:
        path = os.path.join(_HERE, "libq4g_datagen.so")
        if not os.path.exists(path):
            raise RuntimeError(f"{path} missing; run `python -m int4_q4_gemv_b200.build`")
        L = C.CDLL(path)
        vp, ll, ull, f = C.c_void_p, C.c_longlong, C.c_ulonglong, C.c_float
        for name, args in {
            "dg_fill_normal_f32": [vp, ll, ull, ull, f, ll, vp],
            "dg_fill_normal_f16": [vp, ll, ull, ull, f, ll, vp],
            "dg_fill_gain_f32": [vp, ll, ull, ull, vp],
            "dg_fill_uniform_int": [vp, ll, ull, ull, ll, ll, vp],
            "dg_fill_code8": [vp, ll, ull, ull, ll, vp],
            "dg_fill_const_f32": [vp, ll, f, vp],
        }.items():
            fn = getattr(L, name)
            fn.restype = C.c_int
            fn.argtypes = args
        _DG = L
    return _DG


def stream_ptr(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ok(rc):
    if rc != 0:
        raise RuntimeError(f"datagen fill failed: cuda error {rc}")


def fill_normal_f32(t: torch.Tensor, seed, stream_id, sigma, start=0):
    _ok(dglib().dg_fill_normal_f32(t.data_ptr(), t.numel(), seed, stream_id, sigma, start, stream_ptr()))


def fill_normal_f16(t: torch.Tensor, seed, stream_id, sigma, start=0):
    _ok(dglib().dg_fill_normal_f16(t.data_ptr(), t.numel(), seed, stream_id, sigma, start, stream_ptr()))


def fill_code8(t: torch.Tensor, seed, stream_id, start=0):
    assert t.dtype == torch.int8 and t.is_contiguous()
    _ok(dglib().dg_fill_code8(t.data_ptr(), t.numel(), seed, stream_id, start, stream_ptr()))


def fill_const(t: torch.Tensor, v: float):
    assert t.dtype == torch.float32 and t.is_contiguous()
    _ok(dglib().dg_fill_const_f32(t.data_ptr(), t.numel(), float(v), stream_ptr()))


def fill_gain(t: torch.Tensor, seed, stream_id):
    _ok(dglib().dg_fill_gain_f32(t.data_ptr(), t.numel(), seed, stream_id, stream_ptr()))


def fill_uniform_int(t: torch.Tensor, seed, stream_id, hi, start=0):
    _ok(dglib().dg_fill_uniform_int(t.data_ptr(), t.numel(), seed, stream_id, hi, start, stream_ptr()))


def packed_tensor(rows: int, cols: int, seed: int, stream_id: int, device="cuda", sigma=0.02,
                  chunk_rows: int = 16384):
    """N(0, sigma) [rows][cols] from the seeded recipe, q4_0-packed by the library."""
    qs = torch.empty((rows, cols // 2), dtype=torch.uint8, device=device)
    sc = torch.empty((rows, cols // 32), dtype=torch.int16, device=device)
    tmp = torch.empty((min(rows, chunk_rows), cols), dtype=torch.float32, device=device)
    for r0 in range(0, rows, chunk_rows):
        nr = min(chunk_rows, rows - r0)
        w = tmp[:nr]
        fill_normal_f32(w, seed, stream_id, sigma, start=r0 * cols)
        Q.q4g_q4_0_pack(w.data_ptr(), nr, cols, qs[r0].data_ptr(), sc[r0].data_ptr(), 1, stream_ptr())
    return qs, sc


def config_struct(cfg: dict) -> Q.q4g_config:
    c = Q.q4g_config()
    for name, _ in Q.q4g_config._fields_:
        setattr(c, name, cfg[name])
    return c


class SynthDecoder:
    """The seeded synthetic decoder as a libq4g model (weights borrowed from torch)."""

    def __init__(self, cfg: dict, seed: int = 0, variant: int = 0, device: str = "cuda"):
        self.cfg = dict(cfg)
        self.seed, self.variant, self.device = seed, variant, device
        c = self.cfg
        H, Hq = c["hidden"], c["n_q_heads"]
        self._keep = []
        layers = (Q.q4g_layer_weights * c["n_layers"])()
        for l in range(c["n_layers"]):
            full = WL.layer_is_full(c, l)
            hd = c["gl_head_dim"] if full else c["sl_head_dim"]
            nkv = c["gl_kv_heads"] if full else c["sl_kv_heads"]
            s = lambda t: DG.stream_layer(l, t)
            Lw = layers[l]
            shapes = [("wq", Hq * hd, H, DG.T_WQ), ("wk", nkv * hd, H, DG.T_WK),
                      ("wo", H, Hq * hd, DG.T_WO), ("wgate", c["ffn"], H, DG.T_WGATE),
                      ("wup", c["ffn"], H, DG.T_WUP), ("wdown", H, c["ffn"], DG.T_WDOWN)]
            if not full:
                shapes.append(("wv", nkv * hd, H, DG.T_WV))
            for name, rows, cols, t in shapes:
                qs, sc = packed_tensor(rows, cols, seed, s(t), device)
                self._keep += [qs, sc]
                setattr(Lw, name, Q.q4g_qtensor(qs.data_ptr(), sc.data_ptr()))
            for name, n, t in [("norm_in", H, DG.T_NORM_IN), ("norm_post_attn", H, DG.T_NORM_POST_ATTN),
                               ("norm_pre_ffn", H, DG.T_NORM_PRE_FFN),
                               ("norm_post_ffn", H, DG.T_NORM_POST_FFN)]:
                g = torch.ones(n, dtype=torch.float32, device=device)
                if variant == 1:
                    fill_gain(g, seed, s(t))
                self._keep.append(g)
                setattr(Lw, name, g.data_ptr())
            for name, t in [("norm_q", DG.T_NORM_Q), ("norm_k", DG.T_NORM_K)]:
                base = 1.0 if variant == 2 else float(DG.qk_gain_base(hd))  # variant 2: unit gains
                g = torch.full((hd,), base, dtype=torch.float32, device=device)
                if variant == 1:
                    gv = torch.empty(hd, dtype=torch.float32, device=device)
                    fill_gain(gv, seed, s(t))
                    g = g * gv                    # one fp32 multiply, as the recipe defines
                self._keep.append(g)
                setattr(Lw, name, g.data_ptr())
            Lw.layer_scalar = 1.0 if variant != 1 else float(
                DG.uniform_float(seed, s(DG.T_LAYER_SCALAR), 1, 0.5, 1.5)[0])
        nf = torch.ones(H, dtype=torch.float32, device=device)
        if variant == 1:
            fill_gain(nf, seed, DG.STREAM_FINAL_NORM)
        self.embed_f16 = None
        if c.get("head_fp16"):  # the same N(0, 0.02) draws, kept at fp16
            e16 = torch.empty((c["vocab"], H), dtype=torch.float16, device=device)
            fill_normal_f16(e16, seed, DG.STREAM_EMBED, 0.02)
            eq = es = None
            self.embed_f16 = e16
            self._keep += [e16, nf]
            emb = Q.q4g_qtensor(0, 0)
        else:
            eq, es = packed_tensor(c["vocab"], H, seed, DG.STREAM_EMBED, device)
            self._keep += [eq, es, nf]
            emb = Q.q4g_qtensor(eq.data_ptr(), es.data_ptr())
        self.embed_qs, self.embed_sc = eq, es
        self._layers = layers
        self._w = Q.q4g_weights(layers, emb, nf.data_ptr(),
                                self.embed_f16.data_ptr() if self.embed_f16 is not None else 0)
        self._cfg_struct = config_struct(c)
        torch.cuda.synchronize()
        self.handle = Q.q4g_model_create(self._cfg_struct, self._w)

    def tensor(self, layer: int, name: str):
        """(qs, scales) torch tensors of one weight tensor (for byte comparisons)."""
        if name == "embed":
            return self.embed_qs, self.embed_sc
        lw = self._layers[layer]
        t = getattr(lw, name)
        for i in range(0, len(self._keep) - 1):
            a, b = self._keep[i], self._keep[i + 1]
            if a.dtype == torch.uint8 and a.data_ptr() == t.qs:
                return a, b
        return None

    def new_cache(self, capacity: int) -> "SynthCache":
        return SynthCache(self, capacity)

    def sibling(self, **overrides) -> "SynthSibling":
        """A second model handle over the same weights with some configuration
        fields changed (for example kv_int8=1)."""
        return SynthSibling(self, overrides)

    def close(self):
        if getattr(self, "handle", None):
            Q.q4g_model_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class SynthSibling:
    """A model handle that borrows a SynthDecoder's weights (which must outlive it)."""

    def __init__(self, parent: SynthDecoder, overrides: dict):
        self.parent = parent
        self.cfg = dict(parent.cfg, **overrides)
        self.device = parent.device
        self._cfg_struct = config_struct(self.cfg)
        self.handle = Q.q4g_model_create(self._cfg_struct, parent._w)

    def new_cache(self, capacity: int) -> "SynthCache":
        return SynthCache(self, capacity)

    def close(self):
        if getattr(self, "handle", None):
            Q.q4g_model_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class SynthCache:
    def __init__(self, model: SynthDecoder, capacity: int):
        self.model = model
        self.capacity = capacity
        n = Q.q4g_cache_bytes(model.handle, capacity)
        self.buf = torch.zeros(n, dtype=torch.uint8, device=model.device)
        self.handle = Q.q4g_cache_init(model.handle, capacity, self.buf.data_ptr(), n)
        self.view = Q.q4g_cache_layout(self.handle)

    def ring(self, i: int, kv: int) -> torch.Tensor:
        v = self.view
        off = (v.ring_v_offset if kv else v.ring_k_offset) + i * v.ring_layer_bytes
        n = v.sl_kv_heads * v.ring * v.sl_head_dim
        return self.buf[off:off + 2 * n].view(torch.float16).view(v.sl_kv_heads, v.ring, v.sl_head_dim)

    def global_(self, i: int, kv: int) -> torch.Tensor:
        v = self.view
        off = (v.global_v_offset if kv else v.global_k_offset) + i * v.global_layer_bytes
        n = v.gl_kv_heads * v.capacity * v.gl_head_dim
        return self.buf[off:off + 2 * n].view(torch.float16).view(v.gl_kv_heads, v.capacity, v.gl_head_dim)

    def _i8(self, off, so, nkv, rows, hd):
        codes = self.buf[off:off + nkv * rows * hd].view(torch.int8).view(nkv, rows, hd)
        scales = self.buf[off + so:off + so + 4 * nkv * rows].view(torch.float32).view(nkv, rows)
        return codes, scales

    def ring_i8(self, i: int, kv: int):
        """int8 cache: (codes [n_kv][R][hd] int8, scales [n_kv][R] fp32), views of the buffer."""
        v = self.view
        off = (v.ring_v_offset if kv else v.ring_k_offset) + i * v.ring_layer_bytes
        return self._i8(off, v.ring_scale_offset, v.sl_kv_heads, v.ring, v.sl_head_dim)

    def global_i8(self, i: int, kv: int):
        v = self.view
        off = (v.global_v_offset if kv else v.global_k_offset) + i * v.global_layer_bytes
        return self._i8(off, v.global_scale_offset, v.gl_kv_heads, v.capacity, v.gl_head_dim)

    def close(self):
        if getattr(self, "handle", None):
            Q.q4g_cache_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def fill_history(cache: SynthCache, seed: int = 99):
    """Seeded fp16 K/V history in every ring slot and every global row, at the scale
    the decoder writes (datagen.history_sigma: K ~ N(0, hd^(-1/2)), V ~ N(0, 1)); for
    an int8 cache, seeded codes (datagen.code8) with the row scale
    datagen.history_scale8, the same standard deviations."""
    v = cache.view
    if v.kv_int8:
        for i in range(v.n_sliding):
            for kv in (0, 1):
                c, sc = cache.ring_i8(i, kv)
                fill_code8(c, seed, DG.history_stream("ring", i, kv))
                fill_const(sc, DG.history_scale8(kv, v.sl_head_dim))
        for i in range(v.n_full):
            for kv in (0, 1):
                c, sc = cache.global_i8(i, kv)
                fill_code8(c, seed, DG.history_stream("global", i, kv))
                fill_const(sc, DG.history_scale8(kv, v.gl_head_dim))
        return
    for i in range(v.n_sliding):
        for kv in (0, 1):
            fill_normal_f16(cache.ring(i, kv), seed, DG.history_stream("ring", i, kv),
                            DG.history_sigma(kv, v.sl_head_dim))
    for i in range(v.n_full):
        for kv in (0, 1):
            fill_normal_f16(cache.global_(i, kv), seed, DG.history_stream("global", i, kv),
                            DG.history_sigma(kv, v.gl_head_dim))
