"""Workload definitions (shapes, seeds, lengths) of the synthetic inputs.

Sizes only: nothing here computes any step of the decode method. The tests fill
the oracle's configuration struct and the library's configuration struct from
these dictionaries separately.
"""
from __future__ import annotations

import math

import numpy as np


def _f32(x: float) -> float:
    return float(np.float32(x))


def decoder(n_layers, hidden, n_q_heads, ffn, vocab, sl_kv_heads, window, ring,
            sl_head_dim=256, gl_kv_heads=1, gl_head_dim=512, full_every=6, full_offset=5,
            rope_pairs_full=64):
    return dict(
        n_layers=n_layers, hidden=hidden, n_q_heads=n_q_heads, ffn=ffn, vocab=vocab,
        sl_kv_heads=sl_kv_heads, sl_head_dim=sl_head_dim, window=window, ring=ring,
        gl_kv_heads=gl_kv_heads, gl_head_dim=gl_head_dim, full_every=full_every,
        full_offset=full_offset, rope_pairs_full=rope_pairs_full,
        rope_theta_sl=1.0e4, rope_theta_gl=1.0e6, rms_eps=_f32(1e-6), softcap=30.0,
        embed_scale=_f32(math.sqrt(hidden)), v_norm_sliding=1, head_fp16=0, kv_int8=0)


# Tiny 6-layer decoder (layers 0-4 sliding, layer 5 full): parity config.
TINY = decoder(n_layers=6, hidden=1024, n_q_heads=8, ffn=4096, vocab=4096,
               sl_kv_heads=2, window=256, ring=512)

# TINY with the fp16 tied embedding / head.
TINY_F16 = dict(TINY, head_fp16=1)

# 12B-class decoder: 48 layers, full attention at 5, 11, ..., 47.
B12 = decoder(n_layers=48, hidden=3840, n_q_heads=16, ffn=15360, vocab=262144,
              sl_kv_heads=8, window=1024, ring=2048)

# Very small shapes for CPU-only oracle self-tests (not a workload of the pages).
MICRO = decoder(n_layers=3, hidden=128, n_q_heads=4, ffn=256, vocab=512,
                sl_kv_heads=2, window=8, ring=16, sl_head_dim=32, gl_head_dim=64,
                full_every=3, full_offset=2, rope_pairs_full=8)

# GEMV microbench shapes (rows N, columns K), seeds 1-4.
GEMV_SHAPES = [
    ("ffn_up_3840x15360", 15360, 3840, 1),
    ("ffn_down_15360x3840", 3840, 15360, 2),
    ("qkv_3840x8192", 8192, 3840, 3),
    ("vocab_head_3840x262144", 262144, 3840, 4),
]
# the fp16 tied head's GEMV (2 bytes per weight)
GEMV_F16_SHAPES = [("vocab_head_f16_3840x262144", 262144, 3840, 5)]

# Flash-decode microbench: hd512 single-KV-head cache lengths.
ATTN_GLOBAL_LENGTHS = [4096, 8192, 16384, 32768, 65536, 131072]

# Decode configs on the 12B-class decoder.
CONFIG_TINY = dict(model=TINY, seed=0, prefill_hidden=384, greedy_steps=16)
CONFIG_B12_4K = dict(model=B12, seed=0, context=4096, greedy_steps=128)
CONFIG_B12_32K = dict(model=B12, seed=0, context=32768, greedy_steps=128)
CONFIG_B12_128K_VERIFY = dict(model=B12, seed=0, context=131072, verify_k=4, blocks=64)


def layer_is_full(cfg: dict, layer: int) -> bool:
    return cfg["full_every"] > 0 and layer % cfg["full_every"] == cfg["full_offset"]
