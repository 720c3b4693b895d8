"""Timeline of one decode layer of the per-kernel path (one launch per GEMV and
attention kernel) on the device clock (observability harness).

Runs a few decode steps of the synthetic 12B-class decoder (fewer layers by
default) with the library's trace option and prints, for layer 1 on a common
time base (ns of %globaltimer from the QKV launch's entry), when CTA 0 of each
launch entered, when its dependency wait ended, when the fused norm's inputs had arrived and
both norms were reduced (fused-norm launches), when its x prologue finished,
when its first stage was ready and when its last stage was reduced; for the
sliding-window attention launch the phases of its first CTA, and the spread of
the times at which gate|up's CTAs finished.

    python -m int4_q4_gemv_b200.timeline [--layers 6] [--context 4096] [--steps 3]
"""
from __future__ import annotations

import argparse
import json

import numpy as np
import torch

from datagen import synth as S
from datagen import workloads as WL
from int4_q4_gemv_b200 import q4g as Q

GEMV_SLOTS = 256  # entries per GEMV launch in the trace buffer (the C header's layout)


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--layers", type=int, default=6)
    ap.add_argument("--context", type=int, default=4096)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--json", action="store_true", help="one JSON object per step instead of text")
    a = ap.parse_args()
    cfg = dict(WL.B12, n_layers=a.layers)
    g = S.SynthDecoder(cfg, seed=0)
    c = g.new_cache(a.context)
    S.fill_history(c)
    sp = S.stream_ptr()
    tr = torch.zeros(6 * GEMV_SLOTS, dtype=torch.int64, device="cuda")
    am = torch.zeros(a.steps + 8, dtype=torch.int32, device="cuda")
    pos0 = a.context - a.steps - 8
    for i in range(6):  # warm-up: graphs captured, caches in steady state
        Q.q4g_decode_step(g.handle, c.handle, 5 + i, pos0 + i, 0, am[i:].data_ptr(), sp)
    torch.cuda.synchronize()
    Q.q4g_model_set_option(g.handle, Q.Q4G_OPT_TRACE, tr.data_ptr())
    for step in range(a.steps):
        tr.zero_()
        Q.q4g_decode_step(g.handle, c.handle, 11 + step, pos0 + 6 + step, 0, am[6 + step:].data_ptr(), sp)
        torch.cuda.synchronize()
        t = tr.cpu().numpy().astype(np.int64)
        t0 = t[GEMV_SLOTS]  # QKV entry

        def us(v):
            return round((int(v) - int(t0)) / 1e3, 2) if v else None

        out = {"step": step}
        names = ["entry", "dependency_wait", "queries", "scan", "warp_merge", "cluster_sync", "output", "exit"]
        out["attention"] = {n: us(v) for n, v in zip(names, t[4 * GEMV_SLOTS:4 * GEMV_SLOTS + 8])}
        for name, base in (("qkv", 1), ("o", 2), ("gate_up", 0), ("down", 3)):
            r = t[base * GEMV_SLOTS:(base + 1) * GEMV_SLOTS]
            out[name] = {"entry": us(r[0]), "dependency_wait": us(r[1]), "norm_inputs": us(r[3]),
                         "norms": us(r[4]), "x_digits": us(r[2]), "first_stage_ready": us(r[72]),
                         "last_stage_reduced": us(r[5])}
        ends = t[5 * GEMV_SLOTS:6 * GEMV_SLOTS]
        ends = ends[ends > 0]
        if len(ends):
            e = np.sort((ends - t0) / 1e3)
            out["gate_up_cta_ends"] = {"ctas": int(len(e)), "first": round(float(e[0]), 2),
                                        "median": round(float(np.median(e)), 2), "p90": round(float(e[int(0.9 * (len(e) - 1))]), 2),
                                        "last": round(float(e[-1]), 2)}
        if a.json:
            print(json.dumps(out))
            continue
        print(f"step {step} (us from the QKV launch's entry, CTA 0)")
        att = out["attention"]
        print("  attention " + " ".join(f"{k} {v}" for k, v in att.items()))
        for name in ("qkv", "o", "gate_up", "down"):
            print(f"  {name:9s} " + " ".join(f"{k} {v}" for k, v in out[name].items()))
        if "gate_up_cta_ends" in out:
            print("  gate_up CTA ends " + " ".join(f"{k} {v}" for k, v in out["gate_up_cta_ends"].items()))
    Q.q4g_model_set_option(g.handle, Q.Q4G_OPT_TRACE, 0)


if __name__ == "__main__":
    main()
