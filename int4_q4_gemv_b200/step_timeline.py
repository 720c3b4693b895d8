"""Phase timeline of the persistent decode-step kernel on the device clock
(observability harness for the library's trace option).

Runs decode steps of the synthetic 12B-class decoder over seeded synthetic history
with Q4G_OPT_TRACE set and reports, per phase kind (QKV, attention, attention merge,
O, gate|up, down, head), the mean over layers of CTA 0's intervals (ns of
%globaltimer): from the previous phase's start to this phase's start (the phase
length as the grid sees it), from the phase start to its inputs being ready (the
norm prologue, the queries, the x digits), and from the inputs to CTA 0's last
stage being computed.

    python -m int4_q4_gemv_b200.step_timeline [--layers 48] [--context 4096] [--steps 3]
"""
from __future__ import annotations

import argparse
import json

import numpy as np
import torch

from datagen import synth as S
from datagen import workloads as WL
from int4_q4_gemv_b200 import q4g as Q

KINDS = ["qkv", "attention", "merge", "o", "gate_up", "down"]


def phase_table(t: np.ndarray, n_layers: int) -> dict:
    """Per phase kind: mean [phase length, start -> inputs ready, inputs -> compute done] in us."""
    NP = 6 * n_layers + 1
    st = t[: 4 * NP].reshape(NP, 4).astype(np.float64)
    out = {}
    for k, name in enumerate(KINDS + ["head"]):
        idx = [6 * l + k for l in range(n_layers)] if k < 6 else [NP - 1]
        lens, pro, comp = [], [], []
        for p in idx:
            if st[p, 0] == 0:  # a phase this kernel folds into another (sliding-layer merge)
                continue
            q = p + 1
            while q < NP and st[q, 0] == 0:
                q += 1
            nxt = st[q, 0] if q < NP else t[4 * NP + 1]
            lens.append((nxt - st[p, 0]) / 1e3)
            if st[p, 1] > 0:
                pro.append((st[p, 1] - st[p, 0]) / 1e3)
            if st[p, 2] > 0 and st[p, 1] > 0:
                comp.append((st[p, 2] - st[p, 1]) / 1e3)
        out[name] = {"phase_us": float(np.mean(lens)) if lens else None,
                     "inputs_us": float(np.mean(pro)) if pro else None,
                     "compute_us": float(np.mean(comp)) if comp else None}
    out["step_us"] = float((t[4 * NP + 1] - t[4 * NP]) / 1e3)
    return out


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--layers", type=int, default=48)
    ap.add_argument("--context", type=int, default=4096)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--json", action="store_true")
    ap.add_argument("--poll-ns", type=int, default=None, help="Q4G_OPT_STEP_POLL_NS (default: the library's)")
    ap.add_argument("--grid-sync", type=int, choices=[0, 1], default=None,
                    help="Q4G_OPT_STEP_GRID_SYNC (default: the library's)")
    a = ap.parse_args()
    cfg = dict(WL.B12, n_layers=a.layers)
    g = S.SynthDecoder(cfg, seed=0, step_kernel=1)
    if a.grid_sync is not None:
        Q.q4g_model_set_option(g.handle, Q.Q4G_OPT_STEP_GRID_SYNC, a.grid_sync)
    if a.poll_ns is not None:
        Q.q4g_model_set_option(g.handle, Q.Q4G_OPT_STEP_POLL_NS, a.poll_ns)
    c = g.new_cache(a.context)
    S.fill_history(c)
    sp = S.stream_ptr()
    NP = 6 * a.layers + 1
    tr = torch.zeros(4 * NP + 2, dtype=torch.int64, device="cuda")
    Q.q4g_model_set_option(g.handle, Q.Q4G_OPT_TRACE, tr.data_ptr())
    tables = []
    for s in range(a.steps):
        pos = a.context - a.steps + s
        Q.q4g_decode_step(g.handle, c.handle, 11 + s, pos, 0, 0, sp)
        torch.cuda.synchronize()
        tables.append(phase_table(tr.cpu().numpy(), a.layers))
    Q.q4g_model_set_option(g.handle, Q.Q4G_OPT_TRACE, 0)
    Q.q4g_model_check(g.handle, sp)
    last = tables[-1]
    if a.json:
        print(json.dumps(last))
        return
    print(f"step on CTA 0: {last['step_us']:.1f} us ({a.layers} layers, context {a.context})")
    print(f"{'phase':10s} {'length':>8s} {'inputs':>8s} {'compute':>8s}   (us, mean over layers)")
    for name in KINDS + ["head"]:
        r = last[name]
        f = lambda v: f"{v:8.2f}" if v is not None else "       -"
        print(f"{name:10s} {f(r['phase_us'])} {f(r['inputs_us'])} {f(r['compute_us'])}")


if __name__ == "__main__":
    main()
