"""Capacity ladder at scale: a cache's capacity is an allocation size, not part of the
computation.

The 12B-class decoder (48 layers) decodes 2,000 seeded tokens into a 32K-capacity
cache and, in lockstep, into a 128K-capacity cache: the logits of every step are
bitwise equal. Then the 32K cache is promoted: its live contents (every ring layer,
and rows 0..1999 of every global layer, located through q4g_cache_layout) move
into a fresh 128K cache, and decoding continues there and in the cache that was
128K from the start: bitwise equal again, with the same greedy tokens.
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

pytestmark = pytest.mark.gpu


def promote(src: S.SynthCache, dst: S.SynthCache, live: int):
    """Copy the live contents of src into dst (a cache of a larger capacity)."""
    vs, vd = src.view, dst.view
    assert vs.ring == vd.ring and vs.n_sliding == vd.n_sliding and vs.n_full == vd.n_full
    for i in range(vs.n_sliding):
        for kv in (0, 1):
            dst.ring(i, kv).copy_(src.ring(i, kv))
    for i in range(vs.n_full):
        for kv in (0, 1):
            dst.global_(i, kv)[:, :live].copy_(src.global_(i, kv)[:, :live])


def test_capacity_ladder_32k_to_128k_bitwise():
    B.build()
    cfg = WL.B12
    sp = S.stream_ptr()
    g = S.SynthDecoder(cfg, seed=0, variant=0)
    small, big = g.new_cache(32768), g.new_cache(131072)
    V, fed, more = cfg["vocab"], 2000, 48
    ids = DG.uniform_int(11, DG.STREAM_PREFIX_IDS, fed, V)
    lg = torch.empty((2, V), dtype=torch.float32, device="cuda")
    am = torch.empty(2, dtype=torch.int32, device="cuda")
    for pos in range(fed):
        check = pos % 100 == 99
        for j, c in enumerate((small, big)):
            Q.q4g_decode_step(g.handle, c.handle, int(ids[pos]), pos, lg[j].data_ptr() if check else 0,
                              am[j:].data_ptr(), sp)
        if check:
            torch.cuda.synchronize()
            assert torch.equal(lg[0], lg[1]), f"capacities differ at position {pos}"
            assert int(am[0]) == int(am[1])
    torch.cuda.synchronize()
    Q.q4g_model_check(g.handle, sp)
    promoted = g.new_cache(131072)
    promote(small, promoted, fed)
    small.close()
    torch.cuda.synchronize()
    tok = [int(am[1])] * 2
    for pos in range(fed, fed + more):
        for j, c in enumerate((promoted, big)):
            Q.q4g_decode_step(g.handle, c.handle, tok[j], pos, lg[j].data_ptr(), am[j:].data_ptr(), sp)
        torch.cuda.synchronize()
        assert torch.equal(lg[0], lg[1]), f"promoted cache differs at position {pos}"
        tok = [int(am[0]), int(am[1])]
        assert tok[0] == tok[1]
    Q.q4g_model_check(g.handle, sp)
