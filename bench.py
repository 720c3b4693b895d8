#!/usr/bin/env python
"""Decode throughput of the 12B-class q4_0 decoder at batch 1 on B200.

Workload: the 12B-class synthetic decoder (48 layers, full attention at 5, 11, ...,
47; sliding W=1024 in a ring of R=2048, 8 KV heads x hd 256; full layers 1 KV head x
hd 512 with k_eq_v; hidden 3840, 16 query heads, FFN 15360 GeGLU, vocab 262,144
tied; q4_0 weights from the seeded recipe), context C (default 4096): a seeded
random-id prefix of C - (W + K) tokens is run through the model, then W warm-up and
K timed greedy decode steps end at position C - 1. A step is one full decode step
(embedding, 48 layers, head, softcap, argmax). The weights (6.7 GB) exceed L2, so no
flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--context C] [--impl reference]

Prints one JSON line. Under torchrun each rank decodes its own sequence on its own
GPU (replicas: the step has no cross-GPU exchange), value = all ranks' tokens / max
rank time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode tokens/s at batch 1 and achieved HBM GB/s as % of B200 peak, per context"


def max_over_ranks(v: float, world: int, device) -> float:
    """The maximum of v over all ranks (one all-reduce that every rank takes)."""
    if world <= 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_rate(units_per_rank: int, world: int, seconds: float) -> float:
    """Whole-job throughput of `world` independent replicas that each process
    units_per_rank units, timed by the slowest rank's seconds (weak scaling)."""
    return world * units_per_rank / seconds


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--context", type=int, default=4096)
    ap.add_argument("--impl", choices=["q4g", "reference"], default="q4g")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--prefix", choices=["model", "synthetic"], default="model",
                    help="model: run the random-id prefix through the decoder; synthetic: "
                         "seeded N(0,1) K/V history (same bytes read per step)")
    ap.add_argument("--profile-steps", type=int, default=4)
    ap.add_argument("--e2e-steps", type=int, default=32)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=None,
                    help="fewer layers of the same shapes (profiling captures of a small case)")
    ap.add_argument("--gemv-chain", type=int, choices=[0, 1], default=None,
                    help="run O, gate|up, down and the next QKV of a layer as one persistent launch "
                         "(default: the library's default)")
    return ap.parse_args()


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ---------------------------------------------------------------- bytes ----

def weight_bytes(cfg) -> float:
    from datagen import workloads as WL
    H, Hq, F = cfg["hidden"], cfg["n_q_heads"], cfg["ffn"]
    total = 0
    for l in range(cfg["n_layers"]):
        full = WL.layer_is_full(cfg, l)
        hd = cfg["gl_head_dim"] if full else cfg["sl_head_dim"]
        nkv = cfg["gl_kv_heads"] if full else cfg["sl_kv_heads"]
        rows_qkv = Hq * hd + nkv * hd + (0 if full else nkv * hd)
        total += rows_qkv * H + H * Hq * hd + 2 * F * H + H * F
    total += cfg["vocab"] * H
    return total * 0.5625  # 16 bytes of codes + 2 bytes of scale per 32 weights


def kv_bytes(cfg, q) -> float:
    """Live K/V bytes read at query position q: per sliding layer K and V of
    min(q + 1, W) positions, per full layer K and V of q + 1 positions (fp16)."""
    from datagen import workloads as WL
    n_sl = sum(1 for l in range(cfg["n_layers"]) if not WL.layer_is_full(cfg, l))
    n_gl = cfg["n_layers"] - n_sl
    sl = n_sl * min(q + 1, cfg["window"]) * cfg["sl_kv_heads"] * cfg["sl_head_dim"] * 2 * 2
    gl = n_gl * (q + 1) * cfg["gl_kv_heads"] * cfg["gl_head_dim"] * 2 * 2
    return float(sl + gl)


def launches_per_step(cfg) -> int:
    from datagen import workloads as WL
    n = 2  # step init + head
    for l in range(cfg["n_layers"]):
        n += 6 if WL.layer_is_full(cfg, l) else 5
    return n


# --------------------------------------------------------------- clocks ----

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        out = {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        rows = [l.split(", ") for l in self.lines if l.count(",") >= 8]
        if not rows:
            return out
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        out["samples"] = len(rows)
        out["sm_mhz"] = statistics.median(sm) if sm else None
        out["sm_max_mhz"] = float(rows[0][2]) if rows[0][2].replace(".", "").isdigit() else None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in rows:
            for name, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(name)
        out["reasons"] = sorted(reasons)
        return out


# ------------------------------------------------------------ reference ----

def oracle_sample(cfg, seed, max_seconds=120.0, min_steps=1, max_steps=4, context=4096, warmup=0):
    """The oracle on a bounded sample of the decode step: a 12B-shaped model with one
    period of the layer pattern (5 sliding + 1 full layer) and the full tied head, one
    decode step at `context` - 1 over seeded synthetic history (after `warmup` untimed
    steps of the same kind); the per-token time of the 48-layer step is
    8 x (sample step - head) + head."""
    import numpy as np
    from oracle import oracle as O
    sample_cfg = dict(cfg, n_layers=cfg["full_every"])
    t0 = time.perf_counter()
    m = O.Model(sample_cfg, seed=seed)
    build_s = time.perf_counter() - t0
    c = O.Cache(m, context)
    O.fill_history(c, seed=99)
    qs, sc = m.tensor(-1, 100)
    x16 = np.random.default_rng(0).standard_normal(cfg["hidden"]).astype(np.float16).view(np.uint16)
    th = time.perf_counter()
    O.gemv(qs, sc, x16)
    t_head = time.perf_counter() - th
    for i in range(warmup):
        O.decode_step(m, c, context - 1, token=3 + i, want_logits=False)
    times = []
    budget_t = time.perf_counter()
    for i in range(max_steps):
        ts = time.perf_counter()
        O.decode_step(m, c, context - 1, token=7 + i, want_logits=False)
        times.append(time.perf_counter() - ts)
        if i + 1 >= min_steps and time.perf_counter() - budget_t > max_seconds:
            break
    t_step = statistics.median(times)
    per_token = (cfg["n_layers"] // cfg["full_every"]) * (t_step - t_head) + t_head
    return dict(tok_s=1.0 / per_token, per_token_s=per_token, steps=len(times), t_head=t_head,
                t_sample=t_step, cores=O.num_threads(), build_s=build_s, warmup=warmup)


def run_reference(args, cfg):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    t0 = time.perf_counter()
    # warm-up steps of the same sample (at most 3: one oracle step takes ~20 s)
    r = oracle_sample(cfg, args.seed, max_seconds=120.0, min_steps=1, max_steps=max(1, min(args.steps, 4)),
                      context=args.context, warmup=min(max(args.warmup, 0), 3))
    sample = (f"{r['steps']} oracle decode step(s), after {r['warmup']} untimed, of a 12B-shaped "
              f"{cfg['full_every']}-layer sample "
              f"(5 sliding + 1 full + 262144-row head) at position {args.context - 1} over seeded "
              f"history, scaled to 48 layers")
    line = {
        "impl": "reference", "metric": METRIC, "value": r["tok_s"], "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": r["steps"], "warmup": r["warmup"], "ms_per_step": r["per_token_s"] * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": f"12B-class q4_0 decoder, context {args.context}, batch 1",
                   "context": args.context},
        "cpu_baseline": {"value": r["tok_s"], "unit": "tokens/s", "cores": r["cores"], "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": r["tok_s"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s": time.perf_counter() - t0,
    }
    return line


# ----------------------------------------------------------------- main ----

def main():
    args = parse_args()
    from datagen import workloads as WL
    cfg = dict(WL.B12)
    if args.layers:
        cfg["n_layers"] = args.layers
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        line = run_reference(args, cfg)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local))

    from int4_q4_gemv_b200 import build as B
    if rank == 0 or world == 1:
        B.build()
    if world > 1:
        dist.barrier()
    import datagen as DG
    from datagen import synth as S
    from int4_q4_gemv_b200 import q4g as Q

    C, K, W = args.context, args.steps, args.warmup
    assert K >= 1 and W >= 3 and K + W < C, "need steps >= 1, warmup >= 3 and steps + warmup < context"
    t_setup = time.perf_counter()
    model = S.SynthDecoder(cfg, seed=args.seed)
    if args.gemv_chain is not None:
        Q.q4g_model_set_option(model.handle, Q.Q4G_OPT_GEMV_CHAIN, args.gemv_chain)
    cache = model.new_cache(C)
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream
    V = cfg["vocab"]
    prefix = C - (W + K)
    am = torch.zeros(C + 1, dtype=torch.int32, device="cuda")
    if args.prefix == "model":
        ids = DG.uniform_int(args.seed + rank, DG.STREAM_PREFIX_IDS, prefix, V)
        for p in range(prefix):
            Q.q4g_decode_step(model.handle, cache.handle, int(ids[p]), p, 0, am[p:].data_ptr(), sp)
    else:
        S.fill_history(cache, seed=99 + rank)
        am[prefix - 1] = 11
    torch.cuda.synchronize()
    setup_s = time.perf_counter() - t_setup

    def steps(p0, n):
        for p in range(p0, p0 + n):
            Q.q4g_decode_step_device_token(model.handle, cache.handle, am[p - 1:].data_ptr(), p, 0,
                                           am[p:].data_ptr(), sp)

    steps(prefix, W)
    torch.cuda.synchronize()
    props = torch.cuda.get_device_properties(local)
    gpu_id = str(getattr(props, "uuid", local))
    if gpu_id and not gpu_id.startswith("GPU-") and "-" in gpu_id:
        gpu_id = "GPU-" + gpu_id
    clocks = ClockSampler(gpu_id)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    steps(prefix + W, K)
    ev1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = max_over_ranks(ev0.elapsed_time(ev1), world, "cuda")
    if world > 1:
        dist.barrier()
    ms_per_step = ms / K
    tok_s = replica_rate(K, world, ms / 1e3)
    positions = range(prefix + W, C)
    bytes_per_tok = weight_bytes(cfg) + statistics.mean(kv_bytes(cfg, q) for q in positions)
    peak, peak_kind = measured_peaks()
    gbs = bytes_per_tok / (ms_per_step / 1e3) / 1e9

    # ---- per-kernel breakdown (profile mode: eager launches bracketed by events) ----
    Q.q4g_model_set_option(model.handle, Q.Q4G_OPT_PROFILE, 1)
    P = args.profile_steps
    steps(C - P, P)
    recs = Q.q4g_model_profile_read(model.handle, sp)
    Q.q4g_model_set_option(model.handle, Q.Q4G_OPT_PROFILE, 0)
    kinds = {}
    for kind, layer, kms, kbytes in recs:
        k = kinds.setdefault(Q.KIND_NAMES[kind], {"launches": 0, "ms": 0.0, "bytes": 0.0})
        k["launches"] += 1
        k["ms"] += kms
        k["bytes"] += kbytes
    gemv = [v for n, v in kinds.items() if n.endswith("_gemv")]
    g_ms = sum(v["ms"] for v in gemv)
    g_bytes = sum(v["bytes"] for v in gemv)
    g_launch = sum(v["launches"] for v in gemv)
    prof_step_ms = sum(v["ms"] for v in kinds.values()) / max(P, 1)
    launches_step = sum(v["launches"] for v in kinds.values()) / max(P, 1)
    breakdown = {n: {"launches_per_step": v["launches"] / P, "ms_per_step": v["ms"] / P,
                     "gbs": v["bytes"] / (v["ms"] / 1e3) / 1e9 if v["ms"] else None}
                 for n, v in sorted(kinds.items())}
    achieved = g_bytes / (g_ms / 1e3) / 1e9 if g_ms else None
    traffic = None
    tp = os.path.join(ROOT, "profiles", "gemv_q4_traffic.json")
    if os.path.exists(tp):
        with open(tp) as f:
            tr = json.load(f)
        src = open(os.path.join(ROOT, "int4_q4_gemv_b200", "csrc", "q4g_gemv.cu"), "rb").read()
        if tr.get("source_sha256") == hashlib.sha256(src).hexdigest():
            traffic = tr.get("bytes_per_launch")

    # ---- end to end: host token in, host argmax out, per step ----
    E = min(args.e2e_steps, C)
    am_host = torch.zeros(1, dtype=torch.int32).pin_memory()
    tok = int(am[C - 1].item())
    if world > 1:
        dist.barrier()
    t0 = time.perf_counter()
    for p in range(C - E, C):
        Q.q4g_decode_step_host(model.handle, cache.handle, tok, p, 0, am_host.data_ptr(), sp)
        tok = int(am_host[0])
    e2e_s = max_over_ranks(time.perf_counter() - t0, world, "cuda")
    e2e_tok_s = replica_rate(E, world, e2e_s)

    cpu = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        r = oracle_sample(cfg, args.seed, max_seconds=20.0, min_steps=1, max_steps=2, context=C)
        cpu = {"value": r["tok_s"], "unit": "tokens/s", "cores": r["cores"], "kind": "oracle",
               "sample": f"{r['steps']} oracle decode step(s) of a 12B-shaped 6-layer sample "
                         f"(5 sliding + 1 full + the 262144-row head) at position {C - 1} over seeded "
                         f"history, scaled to 48 layers"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": tok_s, "unit": "tokens/s", "n_gpus": world, "steps": K,
            "warmup": W, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "q4_0 x f16 -> f32", "data": "synthetic",
            "config": {"workload": f"12B-class q4_0 decoder ({cfg['n_layers']} layers, h 3840, vocab 262144), "
                                   f"context {C}, batch 1, greedy decode",
                       "context": C, "global_batch": world, "seq_len": C,
                       "parallelism": f"replicas{world}", "prefix": args.prefix,
                       "l2": "inputs larger than L2 (6.7 GB of weights read per step)"},
            "hbm": {"bytes_per_token": bytes_per_tok, "gbs_per_gpu": gbs, "peak_gbs": peak,
                    "frac": gbs / peak, "peak_kind": peak_kind},
            "roofline": {"bound": "hbm", "kernel": "q4_0 GEMV (every GEMV launch of a step, chains included)",
                         "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": (achieved / peak) if achieved else None, "traffic": traffic,
                         "launches_per_step": g_launch / max(P, 1),
                         "peak_kind": f"{peak_kind} (burst copy)"},
            "kernels": breakdown, "profiled_step_ms": prof_step_ms,
            "e2e": {"value": e2e_tok_s, "unit": "tokens/s", "h2d_bytes_per_step": 4,
                    "d2h_bytes_per_step": 4, "api": "q4g_decode_step_host"},
            "cpu_baseline": cpu, "gpu_launches": int(round(launches_step * K)),
            "clocks": {"sm_mhz": clk["sm_mhz"], "sm_max_mhz": clk["sm_max_mhz"], "reasons": clk["reasons"],
                       "samples": clk["samples"]},
            "setup_s": setup_s,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
