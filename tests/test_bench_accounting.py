"""The benchmark's byte accounting (the HBM fraction and the roofline divide by it),
checked against the counts the 12B-class shapes fix:
  * weights: QKV (q 16 x 256 rows, k and v 8 x 256 on sliding layers; q 16 x 512 and
    k 512 on full layers, v taken from k), O, gate|up, down per layer, and the tied
    262,144 x 3840 head, at 0.5625 B per weight (16 B codes + 2 B scale per 32);
  * K/V read at query position q: per sliding layer 8 heads x 256 x 2 (K, V) x 2 B per
    live position (min(q + 1, 1024)), per full layer 512 x 2 x 2 B per position (q + 1);
  * launches: step init + head, 5 per sliding and 6 per full layer."""
from __future__ import annotations

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from datagen import workloads as WL  # noqa: E402


def test_weight_bytes_12b():
    H, F, V = 3840, 15360, 262144
    sl = (16 * 256 + 2 * 8 * 256) * H + H * 16 * 256 + 2 * F * H + H * F
    gl = (16 * 512 + 512) * H + H * 16 * 512 + 2 * F * H + H * F
    weights = 40 * sl + 8 * gl + V * H
    assert bench.weight_bytes(WL.B12) == weights * 0.5625
    assert abs(bench.weight_bytes(WL.B12) - 6.697e9) < 1e6


def test_kv_bytes_12b():
    for q in (0, 100, 1023, 1024, 4095, 32767, 131071):
        sl = 40 * min(q + 1, 1024) * 8 * 256 * 2 * 2
        gl = 8 * (q + 1) * 512 * 2 * 2
        assert bench.kv_bytes(WL.B12, q) == float(sl + gl)
    # at a full window: 335.5 MB of ring reads plus 16,384 B per token of context
    assert bench.kv_bytes(WL.B12, 4095) == 40 * 1024 * 8192 + 16384 * 4096


def test_launches_per_step_12b():
    assert bench.launches_per_step(WL.B12) == 2 + 40 * 5 + 8 * 6 == 250
