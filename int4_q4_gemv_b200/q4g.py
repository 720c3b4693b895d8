"""Python binding of libq4g (include/q4g.h): argument marshalling only.

Every function keeps the C name and takes raw device pointers (ints), sizes and a
CUDA stream handle. All computation runs in the library's CUDA kernels; if the
library is missing this module raises instead of falling back to anything else.
"""
from __future__ import annotations

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libq4g.so")

Q4G_OK, Q4G_EINVAL, Q4G_ERANGE, Q4G_ENOMEM, Q4G_ECUDA, Q4G_ETIMEOUT = range(6)
Q4G_OPT_CUDA_GRAPH, Q4G_OPT_PDL, Q4G_OPT_DUMP, Q4G_OPT_PROFILE, Q4G_OPT_TEST_STALL = 1, 2, 3, 4, 5
Q4G_OPT_ATTN_CLUSTER = 6
Q4G_OPT_TRACE = 8
KIND_NAMES = ["step_init", "qkv_gemv", "attn_sliding", "attn_full", "attn_combine", "o_gemv",
              "gate_up_gemv", "down_gemv", "head_gemv"]

EXPORTS = [
    "q4g_last_error", "q4g_status_string", "q4g_abi_version",
    "q4g_q4_0_pack", "q4g_q4_0_unpack", "q4g_gemv", "q4g_gemv_f16",
    "q4g_flash_decode_workspace_bytes", "q4g_flash_decode_ring", "q4g_flash_decode_linear",
    "q4g_flash_decode_ring_i8", "q4g_flash_decode_linear_i8",
    "q4g_model_create", "q4g_model_destroy", "q4g_model_check", "q4g_model_set_option",
    "q4g_cache_bytes", "q4g_cache_init", "q4g_cache_reset", "q4g_cache_destroy", "q4g_cache_layout",
    "q4g_decode_step", "q4g_decode_step_device_token", "q4g_decode_step_hidden",
    "q4g_decode_step_host", "q4g_verify_block", "q4g_prefill_chunk", "q4g_model_profile_read",
    "q4g_flash_decode_ring_noalloc", "q4g_set_gemv_kernel",
]
Q4G_NOALLOC_SCRATCH_BYTES = 1 << 20


class Q4GError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(msg)
        self.status = status


class q4g_config(C.Structure):
    _fields_ = [(n, C.c_int32) for n in (
        "n_layers", "hidden", "n_q_heads", "ffn", "vocab", "sl_kv_heads", "sl_head_dim", "window",
        "ring", "gl_kv_heads", "gl_head_dim", "full_every", "full_offset", "rope_pairs_full")] + \
        [(n, C.c_float) for n in ("rope_theta_sl", "rope_theta_gl", "rms_eps", "softcap",
                                  "embed_scale")] + [("v_norm_sliding", C.c_int32), ("head_fp16", C.c_int32),
                                                     ("kv_int8", C.c_int32)]


class q4g_qtensor(C.Structure):
    _fields_ = [("qs", C.c_void_p), ("scales", C.c_void_p)]


class q4g_layer_weights(C.Structure):
    _fields_ = [(n, q4g_qtensor) for n in ("wq", "wk", "wv", "wo", "wgate", "wup", "wdown")] + \
        [(n, C.c_void_p) for n in ("norm_in", "norm_post_attn", "norm_pre_ffn", "norm_post_ffn",
                                   "norm_q", "norm_k")] + [("layer_scalar", C.c_float)]


class q4g_weights(C.Structure):
    _fields_ = [("layers", C.POINTER(q4g_layer_weights)), ("embed", q4g_qtensor),
                ("norm_final", C.c_void_p), ("embed_f16", C.c_void_p)]


class q4g_launch_record(C.Structure):
    _fields_ = [("kind", C.c_int32), ("layer", C.c_int32), ("ms", C.c_float), ("bytes", C.c_double)]


class q4g_cache_view(C.Structure):
    _fields_ = [("capacity", C.c_int64), ("ring", C.c_int64)] + \
        [(n, C.c_int32) for n in ("n_sliding", "n_full", "sl_kv_heads", "sl_head_dim",
                                  "gl_kv_heads", "gl_head_dim")] + \
        [(n, C.c_size_t) for n in ("ring_k_offset", "ring_v_offset", "ring_layer_bytes",
                                   "global_k_offset", "global_v_offset", "global_layer_bytes",
                                   "total_bytes")] + \
        [("kv_int8", C.c_int32), ("ring_scale_offset", C.c_size_t), ("global_scale_offset", C.c_size_t)]


_lib = None


def lib() -> C.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"libq4g.so not found at {LIB_PATH}; build it with `python -m int4_q4_gemv_b200.build`")
        L = C.CDLL(LIB_PATH)
        vp, i32, i64, sz, f32 = C.c_void_p, C.c_int32, C.c_int64, C.c_size_t, C.c_float
        sig = {
            "q4g_last_error": (C.c_char_p, []),
            "q4g_status_string": (C.c_char_p, [C.c_int]),
            "q4g_abi_version": (C.c_int, []),
            "q4g_q4_0_pack": (C.c_int, [vp, i64, i64, vp, vp, C.c_int, vp]),
            "q4g_q4_0_unpack": (C.c_int, [vp, vp, i64, i64, vp, C.c_int, vp]),
            "q4g_gemv": (C.c_int, [vp, vp, i64, i64, vp, i32, vp, vp]),
            "q4g_gemv_f16": (C.c_int, [vp, i64, i64, vp, i32, vp, vp]),
            "q4g_flash_decode_workspace_bytes": (sz, [i32, i32]),
            "q4g_flash_decode_ring": (C.c_int, [vp, i32, i32, i32, vp, vp, i64, i64, i64, vp, vp, sz, vp]),
            "q4g_flash_decode_linear": (C.c_int, [vp, i32, i32, i32, vp, vp, i64, vp, vp, sz, vp]),
            "q4g_flash_decode_ring_i8": (C.c_int, [vp, i32, i32, i32, vp, vp, vp, vp, i64, i64, i64, vp, vp, sz,
                                                   vp]),
            "q4g_flash_decode_linear_i8": (C.c_int, [vp, i32, i32, i32, vp, vp, vp, vp, i64, vp, vp, sz, vp]),
            "q4g_model_create": (C.c_int, [C.POINTER(q4g_config), C.POINTER(q4g_weights), C.POINTER(vp)]),
            "q4g_model_destroy": (None, [vp]),
            "q4g_model_check": (C.c_int, [vp, vp]),
            "q4g_model_set_option": (C.c_int, [vp, C.c_int, C.c_ssize_t]),
            "q4g_cache_bytes": (C.c_int, [vp, i64, C.POINTER(sz)]),
            "q4g_cache_init": (C.c_int, [vp, i64, vp, sz, C.POINTER(vp)]),
            "q4g_cache_reset": (C.c_int, [vp, vp]),
            "q4g_cache_destroy": (None, [vp]),
            "q4g_cache_layout": (C.c_int, [vp, C.POINTER(q4g_cache_view)]),
            "q4g_decode_step": (C.c_int, [vp, vp, i32, i64, vp, vp, vp]),
            "q4g_decode_step_device_token": (C.c_int, [vp, vp, vp, i64, vp, vp, vp]),
            "q4g_decode_step_hidden": (C.c_int, [vp, vp, vp, i64, vp, vp, vp]),
            "q4g_decode_step_host": (C.c_int, [vp, vp, i32, i64, vp, vp, vp]),
            "q4g_verify_block": (C.c_int, [vp, vp, vp, i32, i64, i32, vp, vp, vp]),
            "q4g_prefill_chunk": (C.c_int, [vp, vp, vp, i32, i64, vp, vp, vp]),
            "q4g_model_profile_read": (i32, [vp, C.POINTER(q4g_launch_record), i32, vp]),
            "q4g_flash_decode_ring_noalloc": (C.c_int, [vp, i32, i32, i32, vp, vp, i64, i64, i64, vp, vp]),
            "q4g_set_gemv_kernel": (C.c_int, [i32]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def check(status: int) -> None:
    if status != Q4G_OK:
        L = lib()
        raise Q4GError(status, f"{L.q4g_status_string(status).decode()}: {L.q4g_last_error().decode()}")


def _call(name, *args):
    st = getattr(lib(), name)(*args)
    check(st)


# ---- the C entry points, same names --------------------------------------

def q4g_abi_version() -> int:
    return lib().q4g_abi_version()


def q4g_q4_0_pack(w, rows, k, qs, scales, on_device, stream):
    _call("q4g_q4_0_pack", w, rows, k, qs, scales, on_device, stream)


def q4g_q4_0_unpack(qs, scales, rows, k, w, on_device, stream):
    _call("q4g_q4_0_unpack", qs, scales, rows, k, w, on_device, stream)


def q4g_gemv(qs, scales, n, k, x_f16, nrhs, y, stream):
    _call("q4g_gemv", qs, scales, n, k, x_f16, nrhs, y, stream)


def q4g_gemv_f16(w16, n, k, x_f16, nrhs, y, stream):
    _call("q4g_gemv_f16", w16, n, k, x_f16, nrhs, y, stream)


Q4G_GEMV_AUTO, Q4G_GEMV_WARP_STREAM, Q4G_GEMV_REGISTER, Q4G_GEMV_STAGE = 0, 2, 3, 4


def q4g_set_gemv_kernel(kind):
    _call("q4g_set_gemv_kernel", kind)


def q4g_flash_decode_workspace_bytes(n_q_heads, head_dim) -> int:
    return int(lib().q4g_flash_decode_workspace_bytes(n_q_heads, head_dim))


def q4g_flash_decode_ring(q, n_q, n_kv, head_dim, k_ring, v_ring, ring, window, pos, out, ws, ws_bytes, stream):
    _call("q4g_flash_decode_ring", q, n_q, n_kv, head_dim, k_ring, v_ring, ring, window, pos, out, ws,
          ws_bytes, stream)


def q4g_flash_decode_linear(q, n_q, n_kv, head_dim, k, v, length, out, ws, ws_bytes, stream):
    _call("q4g_flash_decode_linear", q, n_q, n_kv, head_dim, k, v, length, out, ws, ws_bytes, stream)


def q4g_flash_decode_ring_i8(q, n_q, n_kv, head_dim, k_codes, k_scales, v_codes, v_scales, ring, window, pos,
                             out, ws, ws_bytes, stream):
    _call("q4g_flash_decode_ring_i8", q, n_q, n_kv, head_dim, k_codes, k_scales, v_codes, v_scales, ring, window,
          pos, out, ws, ws_bytes, stream)


def q4g_flash_decode_linear_i8(q, n_q, n_kv, head_dim, k_codes, k_scales, v_codes, v_scales, length, out, ws,
                               ws_bytes, stream):
    _call("q4g_flash_decode_linear_i8", q, n_q, n_kv, head_dim, k_codes, k_scales, v_codes, v_scales, length, out,
          ws, ws_bytes, stream)


def q4g_flash_decode_ring_noalloc(q, n_q, n_kv, head_dim, k_ring, v_ring, ring, window, pos, out, stream):
    _call("q4g_flash_decode_ring_noalloc", q, n_q, n_kv, head_dim, k_ring, v_ring, ring, window, pos, out,
          stream)


def q4g_model_create(cfg: q4g_config, weights: q4g_weights) -> int:
    h = C.c_void_p()
    _call("q4g_model_create", C.byref(cfg), C.byref(weights), C.byref(h))
    return h.value


def q4g_model_destroy(model) -> None:
    lib().q4g_model_destroy(model)


def q4g_model_check(model, stream) -> None:
    _call("q4g_model_check", model, stream)


def q4g_model_set_option(model, opt, value) -> None:
    _call("q4g_model_set_option", model, opt, value)


def q4g_cache_bytes(model, capacity) -> int:
    n = C.c_size_t()
    _call("q4g_cache_bytes", model, capacity, C.byref(n))
    return n.value


def q4g_cache_init(model, capacity, buf, nbytes) -> int:
    h = C.c_void_p()
    _call("q4g_cache_init", model, capacity, buf, nbytes, C.byref(h))
    return h.value


def q4g_cache_reset(cache, stream) -> None:
    _call("q4g_cache_reset", cache, stream)


def q4g_cache_destroy(cache) -> None:
    lib().q4g_cache_destroy(cache)


def q4g_cache_layout(cache) -> q4g_cache_view:
    v = q4g_cache_view()
    _call("q4g_cache_layout", cache, C.byref(v))
    return v


def q4g_decode_step(model, cache, token, pos, logits, argmax, stream):
    _call("q4g_decode_step", model, cache, token, pos, logits, argmax, stream)


def q4g_decode_step_device_token(model, cache, token_dev, pos, logits, argmax, stream):
    _call("q4g_decode_step_device_token", model, cache, token_dev, pos, logits, argmax, stream)


def q4g_decode_step_hidden(model, cache, hidden, pos, logits, argmax, stream):
    _call("q4g_decode_step_hidden", model, cache, hidden, pos, logits, argmax, stream)


def q4g_decode_step_host(model, cache, token, pos, logits_host, argmax_host, stream):
    _call("q4g_decode_step_host", model, cache, token, pos, logits_host, argmax_host, stream)


def q4g_verify_block(model, cache, ids, K, pos0, accepted_count, logits, argmax, stream):
    _call("q4g_verify_block", model, cache, ids, K, pos0, accepted_count, logits, argmax, stream)


def q4g_prefill_chunk(model, cache, ids, S, pos0, logits, argmax, stream):
    _call("q4g_prefill_chunk", model, cache, ids, S, pos0, logits, argmax, stream)


def q4g_model_profile_read(model, stream, max_records: int = 1 << 16):
    """Launch records since the last read: list of (kind, layer, ms, bytes)."""
    buf = (q4g_launch_record * max_records)()
    n = lib().q4g_model_profile_read(model, buf, max_records, stream)
    if n < 0:
        check(Q4G_ECUDA)
    return [(buf[i].kind, buf[i].layer, buf[i].ms, buf[i].bytes) for i in range(min(n, max_records))]
