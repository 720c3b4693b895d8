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

Besides the headline context the line carries:
  * per_context: 32K decode over seeded synthetic history and the 128K verify config
    (K = 4 draft rows, seeded accepted counts) in blocks/s, each with its HBM fraction,
    the same two with the int8 KV cache, and 1,024 tokens of chunked prefill;
  * roofline: the dominant kernel (the q4_0 GEMV), its time inside the timed graph
    step taken as its share of a profile pass with CUDA events around every launch;
  * microbench: the four q4_0 GEMV shapes (seeds 1-4) and flash-decode alone (hd 256
    ring, hd 512 linear at 4K..128K), each rotated over copies larger than L2;
  * cpu_baseline: the oracle on the host cores, all threads and one thread.

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
    ap.add_argument("--kv-int8", action="store_true",
                    help="the headline run with the int8 KV cache (kv_int8 = 1)")
    ap.add_argument("--quick", action="store_true",
                    help="the headline context only (no other contexts, no microbenchmarks)")
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
    min(q + 1, W) positions, per full layer K and V of q + 1 positions (fp16 rows of
    2 * hd bytes; int8 rows of hd bytes plus a 4-byte scale)."""
    from datagen import workloads as WL
    n_sl = sum(1 for l in range(cfg["n_layers"]) if not WL.layer_is_full(cfg, l))
    n_gl = cfg["n_layers"] - n_sl
    row = (lambda hd: hd + 4) if cfg.get("kv_int8") else (lambda hd: 2 * hd)
    sl = n_sl * min(q + 1, cfg["window"]) * cfg["sl_kv_heads"] * row(cfg["sl_head_dim"]) * 2
    gl = n_gl * (q + 1) * cfg["gl_kv_heads"] * row(cfg["gl_head_dim"]) * 2
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

def cpu_model_name() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def oracle_sample(cfg, seed, max_seconds=120.0, min_steps=1, max_steps=4, context=4096, warmup=0,
                  threads=0, model=None):
    """The oracle on a bounded sample of the decode step: a 12B-shaped model with one
    period of the layer pattern (5 sliding + 1 full layer) and the full tied head, one
    decode step at `context` - 1 over seeded synthetic history (after `warmup` untimed
    steps of the same kind); the per-token time of the 48-layer step is extrapolated as
    8 x (sample step - head) + head. threads = 0: every host core."""
    import numpy as np
    from oracle import oracle as O
    sample_cfg = dict(cfg, n_layers=cfg["full_every"])
    t0 = time.perf_counter()
    m = model if model is not None else O.Model(sample_cfg, seed=seed)
    build_s = time.perf_counter() - t0
    all_threads = O.num_threads()
    if threads:
        O.set_threads(threads)
    try:
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
        cores = O.num_threads()
    finally:
        O.set_threads(all_threads)
    t_step = statistics.median(times)
    per_token = (cfg["n_layers"] // cfg["full_every"]) * (t_step - t_head) + t_head
    return dict(tok_s=1.0 / per_token, per_token_s=per_token, steps=len(times), t_head=t_head,
                t_sample=t_step, cores=cores, build_s=build_s, warmup=warmup, model=m)


def sample_text(r, cfg, context):
    return (f"{r['steps']} oracle decode step(s) (after {r['warmup']} untimed) of a 12B-shaped "
            f"{cfg['full_every']}-layer sample (5 sliding + 1 full + the 262144-row head) at position "
            f"{context - 1} over seeded history, {r['t_sample']:.2f} s each on {r['cores']} thread(s); "
            f"tokens/s extrapolated to the 48-layer step as 8 x (sample - head) + head; "
            f"CPU: {cpu_model_name()}")


def run_reference(args, cfg):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    t0 = time.perf_counter()
    # each step is one bounded sample step (about 3-20 s): at most 4 of them, so the run
    # ends within a few minutes whatever --steps says
    r = oracle_sample(cfg, args.seed, max_seconds=120.0, min_steps=1, max_steps=max(1, min(args.steps, 4)),
                      context=args.context, warmup=min(max(args.warmup, 0), 3))
    sample = sample_text(r, cfg, args.context)
    line = {
        "impl": "reference", "metric": METRIC, "value": r["tok_s"], "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": r["steps"], "warmup": r["warmup"],
        "ms_per_step": r["t_sample"] * 1e3, "ms_per_token_extrapolated": r["per_token_s"] * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": f"12B-class q4_0 decoder, context {args.context}, batch 1",
                   "context": args.context},
        "cpu_baseline": {"value": r["tok_s"], "unit": "tokens/s", "cores": r["cores"], "kind": "oracle",
                         "sample": sample, "extrapolated": True, "cpu": cpu_model_name()},
        "e2e": {"value": r["tok_s"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s": time.perf_counter() - t0,
    }
    return line


# ------------------------------------------------------------ GPU parts ----

def decode_loop(Q, model, cache, am, p0, n, sp):
    """n greedy steps from p0: each step's token is the previous step's argmax on the device."""
    for p in range(p0, p0 + n):
        Q.q4g_decode_step_device_token(model.handle, cache.handle, am[p - 1:].data_ptr(), p, 0,
                                       am[p:].data_ptr(), sp)


def measure_context(Q, S, model, cfg, C, K, W, sp, stream):
    """K timed decode steps ending at position C - 1 over seeded synthetic history."""
    import torch
    cache = model.new_cache(C)
    S.fill_history(cache, seed=99)
    am = torch.zeros(C + 1, dtype=torch.int32, device="cuda")
    p0 = C - (W + K)
    am[p0 - 1] = 11
    decode_loop(Q, model, cache, am, p0, W, sp)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    decode_loop(Q, model, cache, am, p0 + W, K, sp)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / K
    bpt = weight_bytes(cfg) + statistics.mean(kv_bytes(cfg, q) for q in range(p0 + W, C))
    Q.q4g_model_check(model.handle, sp)
    cache.close()
    del cache
    return ms, bpt


def measure_verify(Q, S, DG, model, cfg, C, Kv, blocks, warm, seed, sp, stream):
    """Verify blocks of Kv draft rows (seeded ids, seeded accepted counts n ~ U{0..Kv},
    the next block at pos0 + n) over seeded synthetic history at context C."""
    import numpy as np
    import torch
    V = cfg["vocab"]
    nb = blocks + warm
    ids = torch.from_numpy(DG.uniform_int(seed, DG.STREAM_DRAFT_IDS, nb * Kv, V).astype(np.int32)).cuda()
    acc = DG.uniform_int(seed, DG.STREAM_ACCEPTED, nb, Kv + 1)
    cache = model.new_cache(C)
    S.fill_history(cache, seed=98)
    am = torch.zeros(nb * Kv, dtype=torch.int32, device="cuda")
    pos = C - Kv * nb
    starts = []
    for b in range(nb):
        starts.append(pos)
        pos += int(acc[b])
    for b in range(warm):
        Q.q4g_verify_block(model.handle, cache.handle, ids[b * Kv:].data_ptr(), Kv, starts[b], Kv, 0,
                           am[b * Kv:].data_ptr(), sp)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for b in range(warm, nb):
        Q.q4g_verify_block(model.handle, cache.handle, ids[b * Kv:].data_ptr(), Kv, starts[b], Kv, 0,
                           am[b * Kv:].data_ptr(), sp)
    e1.record(stream)
    torch.cuda.synchronize()
    Q.q4g_model_check(model.handle, sp)
    ms = e0.elapsed_time(e1) / blocks
    bpb = weight_bytes(cfg) + statistics.mean(kv_bytes(cfg, starts[b] + Kv - 1) for b in range(warm, nb))
    accepted = int(sum(int(acc[b]) for b in range(warm, nb)))
    cache.close()
    del cache
    return ms, bpb, accepted


def measure_prefill(Q, DG, model, cfg, n_tokens, seed, sp, stream):
    """Chunked prefill of n_tokens seeded ids from position 0 into a fresh cache, in
    64-token chunks (q4g_prefill_chunk, last row's logits of the last chunk); one
    untimed pass first (graph capture), then the timed one on another cache."""
    import numpy as np
    import torch
    V = cfg["vocab"]
    ids = torch.from_numpy(DG.uniform_int(seed, DG.STREAM_PREFIX_IDS, n_tokens, V).astype(np.int32)).cuda()
    lg = torch.empty(V, dtype=torch.float32, device="cuda")
    am = torch.zeros(1, dtype=torch.int32, device="cuda")
    ms = None
    for rep in range(2):
        cache = model.new_cache(n_tokens)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for p0 in range(0, n_tokens, 64):
            n = min(64, n_tokens - p0)
            last = p0 + n == n_tokens
            Q.q4g_prefill_chunk(model.handle, cache.handle, ids[p0:].data_ptr(), n, p0,
                                lg.data_ptr() if last else 0, am.data_ptr() if last else 0, sp)
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
        Q.q4g_model_check(model.handle, sp)
        cache.close()
        del cache
    return ms


def time_rotating(fn, n_items, reps, stream):
    """Mean time of fn(i) over reps passes of i = 0..n_items-1 (CUDA events)."""
    import torch
    for i in range(min(n_items, 3)):
        fn(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        for i in range(n_items):
            fn(i)
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / (reps * n_items)


def microbench(Q, S, DG, WL, peak, sp, stream):
    """The kernel microbenchmarks of the decode step's pieces, through the standalone
    C-ABI entry points, each rotated over copies larger than L2 (126 MB)."""
    import math
    import torch
    l2 = 126e6
    out = {"gemv": [], "flash_decode": []}
    for name, n, k, seed0 in WL.GEMV_SHAPES:
        wbytes = n * k * 0.5625
        per_seed = max(1, math.ceil(4 * l2 / wbytes / 4))
        mats = []
        for sd in (1, 2, 3, 4):
            qs, sc = S.packed_tensor(n, k, sd, DG.stream_bench_w(sd))
            mats.append((qs, sc))
            for _ in range(per_seed - 1):
                mats.append((qs.clone(), sc.clone()))
        x = torch.empty(k, dtype=torch.float16, device="cuda")
        S.fill_normal_f16(x, seed0, DG.stream_bench_x(seed0), 1.0)
        y = torch.empty(n, dtype=torch.float32, device="cuda")
        ms = time_rotating(lambda i: Q.q4g_gemv(mats[i][0].data_ptr(), mats[i][1].data_ptr(), n, k, x.data_ptr(), 1,
                                                y.data_ptr(), sp), len(mats), 4, stream)
        b = wbytes + k * 2 + n * 4
        out["gemv"].append({"shape": name, "rows": n, "cols": k, "seeds": [1, 2, 3, 4], "copies": len(mats),
                            "us": ms * 1e3, "gbs": b / (ms / 1e3) / 1e9, "frac": b / (ms / 1e3) / 1e9 / peak})
        # the same matrices against 4 activation rows (a verify block of K = 4): weights read once
        try:
            x4 = torch.empty(4 * k, dtype=torch.float16, device="cuda")
            S.fill_normal_f16(x4, seed0, DG.stream_bench_x(seed0), 1.0)
            y4 = torch.empty(4 * n, dtype=torch.float32, device="cuda")
            ms4 = time_rotating(lambda i: Q.q4g_gemv(mats[i][0].data_ptr(), mats[i][1].data_ptr(), n, k,
                                                     x4.data_ptr(), 4, y4.data_ptr(), sp), len(mats), 4, stream)
            b4 = wbytes + 4 * k * 2 + 4 * n * 4
            out.setdefault("gemv_rows4", []).append(
                {"shape": name, "activation_rows": 4, "us": ms4 * 1e3, "gbs": b4 / (ms4 / 1e3) / 1e9,
                 "frac": b4 / (ms4 / 1e3) / 1e9 / peak, "vs_rows1": ms / ms4})
        except Exception as e:  # a microbenchmark never costs the bench line
            out.setdefault("gemv_rows4", []).append({"shape": name, "error": str(e)[:200]})
        del mats
        torch.cuda.empty_cache()
    # flash-decode alone: 16 query heads over an hd 256 ring (8 KV heads, W 1024, R 2048, full window)
    nq, hd, nkv, W, R = 16, 256, 8, 1024, 2048
    kvb = nkv * R * hd * 2
    copies = max(2, math.ceil(4 * l2 / (2 * kvb)))
    ks = [torch.empty(nkv * R * hd, dtype=torch.float16, device="cuda") for _ in range(copies)]
    vs = [torch.empty_like(ks[0]) for _ in range(copies)]
    for i in range(copies):
        S.fill_normal_f16(ks[i], 1, DG.stream_attn(10 + 2 * i), 0.25)
        S.fill_normal_f16(vs[i], 1, DG.stream_attn(11 + 2 * i), 1.0)
    q = torch.empty(nq * hd, dtype=torch.float16, device="cuda")
    S.fill_normal_f16(q, 1, DG.stream_attn(1), 1.0)
    o = torch.empty(nq * hd, dtype=torch.float16, device="cuda")
    wsb = Q.q4g_flash_decode_workspace_bytes(nq, hd)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    ms = time_rotating(lambda i: Q.q4g_flash_decode_ring(q.data_ptr(), nq, nkv, hd, ks[i].data_ptr(), vs[i].data_ptr(),
                                                         R, W, 5000, o.data_ptr(), ws.data_ptr(), wsb, sp),
                       copies, 4, stream)
    b = nkv * W * hd * 2 * 2
    out["flash_decode"].append({"kind": "ring hd256", "n_q": nq, "n_kv": nkv, "window": W, "ring": R,
                                "copies": copies, "us": ms * 1e3, "gbs": b / (ms / 1e3) / 1e9,
                                "frac": b / (ms / 1e3) / 1e9 / peak})
    del ks, vs
    torch.cuda.empty_cache()
    # hd 512, one KV head, linear cache of length L
    hd = 512
    wsb = Q.q4g_flash_decode_workspace_bytes(nq, hd)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    q = torch.empty(nq * hd, dtype=torch.float16, device="cuda")
    S.fill_normal_f16(q, 2, DG.stream_attn(2), 1.0)
    o = torch.empty(nq * hd, dtype=torch.float16, device="cuda")
    for L in WL.ATTN_GLOBAL_LENGTHS:
        per = L * hd * 2
        copies = max(2, math.ceil(4 * l2 / (2 * per)))
        ks = [torch.empty(L * hd, dtype=torch.float16, device="cuda") for _ in range(copies)]
        vs = [torch.empty_like(ks[0]) for _ in range(copies)]
        for i in range(copies):
            S.fill_normal_f16(ks[i], 2, DG.stream_attn(100 + 2 * i), 0.21)
            S.fill_normal_f16(vs[i], 2, DG.stream_attn(101 + 2 * i), 1.0)
        ms = time_rotating(lambda i: Q.q4g_flash_decode_linear(q.data_ptr(), nq, 1, hd, ks[i].data_ptr(),
                                                               vs[i].data_ptr(), L, o.data_ptr(), ws.data_ptr(),
                                                               wsb, sp), copies, 4, stream)
        b = 2 * per
        out["flash_decode"].append({"kind": "linear hd512", "n_q": nq, "n_kv": 1, "length": L, "copies": copies,
                                    "us": ms * 1e3, "gbs": b / (ms / 1e3) / 1e9,
                                    "frac": b / (ms / 1e3) / 1e9 / peak})
        del ks, vs
        torch.cuda.empty_cache()
    return out


# ----------------------------------------------------------------- main ----

def main():
    args = parse_args()
    from datagen import workloads as WL
    cfg = dict(WL.B12)
    if args.layers:
        cfg["n_layers"] = args.layers
    if args.kv_int8:
        cfg["kv_int8"] = 1
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

    decode_loop(Q, model, cache, am, prefix, W, sp)
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
    decode_loop(Q, model, cache, am, prefix + W, K, sp)
    ev1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    Q.q4g_model_check(model.handle, sp)
    ms = max_over_ranks(ev0.elapsed_time(ev1), world, "cuda")
    if world > 1:
        dist.barrier()
    ms_per_step = ms / K
    tok_s = replica_rate(K, world, ms / 1e3)
    positions = range(prefix + W, C)
    bytes_per_tok = weight_bytes(cfg) + statistics.mean(kv_bytes(cfg, q) for q in positions)
    peak, peak_kind = measured_peaks()
    gbs = bytes_per_tok / (ms_per_step / 1e3) / 1e9

    # ---- per-kernel breakdown (profile mode: the launches of a step bracketed by events) ----
    Q.q4g_model_set_option(model.handle, Q.Q4G_OPT_PROFILE, 1)
    P = args.profile_steps
    decode_loop(Q, model, cache, am, C - P, P, sp)
    recs = Q.q4g_model_profile_read(model.handle, sp)
    Q.q4g_model_set_option(model.handle, Q.Q4G_OPT_PROFILE, 0)
    kinds = {}
    for kind, layer, kms, kbytes in recs:
        k = kinds.setdefault(Q.KIND_NAMES[kind], {"launches": 0, "ms": 0.0, "bytes": 0.0})
        k["launches"] += 1
        k["ms"] += kms
        k["bytes"] += kbytes
    prof_step_ms = sum(v["ms"] for v in kinds.values()) / max(P, 1)
    launches_step = sum(v["launches"] for v in kinds.values()) / max(P, 1)
    breakdown = {n: {"launches_per_step": v["launches"] / P, "ms_per_step": v["ms"] / P,
                     "gbs": v["bytes"] / (v["ms"] / 1e3) / 1e9 if v["ms"] else None}
                 for n, v in sorted(kinds.items())}
    # the dominant kernel: the q4_0 GEMV. Its time inside the timed (graph-replayed)
    # step is its share of the eager profile pass applied to the timed step, so it
    # never exceeds ms_per_step; the eager per-launch time is reported beside it.
    gemv = [v for n, v in kinds.items() if n.endswith("_gemv")]
    gemv_launches = sum(v["launches"] for v in gemv) / max(P, 1)
    gemv_ms_eager = sum(v["ms"] for v in gemv) / max(P, 1)
    k_bytes = sum(v["bytes"] for v in gemv) / max(P, 1) / max(gemv_launches, 1)   # per launch
    share = gemv_ms_eager / prof_step_ms if prof_step_ms else None
    k_ms = share * ms_per_step / max(gemv_launches, 1) if share else None            # per launch, in the graph
    k_ms_eager = gemv_ms_eager / max(gemv_launches, 1)
    kernel_name = "q4_0 GEMV (every GEMV launch of a step)"
    achieved = k_bytes / (k_ms / 1e3) / 1e9 if k_ms else None
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
    cache.close()
    del cache
    torch.cuda.empty_cache()

    # ---- the other contexts and the microbenchmarks (rank 0 of a single-GPU run) ----
    per_context = {str(C): {"kind": "decode", "tokens_per_s": tok_s / world, "ms_per_step": ms_per_step,
                            "bytes_per_token": bytes_per_tok, "gbs": gbs, "frac": gbs / peak,
                            "history": args.prefix}}
    micro = None
    if world == 1 and not args.quick:
        for C2 in (32768,):
            if C2 == C:
                continue
            K2 = min(K, 50)
            ms2, bpt2 = measure_context(Q, S, model, cfg, C2, K2, max(W, 3), sp, stream)
            per_context[str(C2)] = {"kind": "decode", "tokens_per_s": 1e3 / ms2, "ms_per_step": ms2,
                                    "bytes_per_token": bpt2, "gbs": bpt2 / (ms2 / 1e3) / 1e9,
                                    "frac": bpt2 / (ms2 / 1e3) / 1e9 / peak, "steps": K2,
                                    "history": "synthetic"}
        Kv, nb = 4, 16
        msv, bpb, accepted = measure_verify(Q, S, DG, model, cfg, 131072, Kv, nb, 2, args.seed, sp, stream)
        per_context["131072_verify_k4"] = {
            "kind": "verify", "k": Kv, "blocks": nb, "blocks_per_s": 1e3 / msv, "ms_per_block": msv,
            "accepted_tokens_per_s": accepted / (nb * msv / 1e3), "rows_per_s": Kv * 1e3 / msv,
            "bytes_per_block": bpb, "gbs": bpb / (msv / 1e3) / 1e9, "frac": bpb / (msv / 1e3) / 1e9 / peak,
            "accepted_count": "seeded U{0..4}", "history": "synthetic"}
        # the int8 KV cache (kv_int8): the same weights under a second model handle
        m8 = model.sibling(kv_int8=1)
        ms8, bpt8 = measure_context(Q, S, m8, m8.cfg, 32768, 50, 4, sp, stream)
        per_context["32768_kv_int8"] = {"kind": "decode", "kv": "int8", "tokens_per_s": 1e3 / ms8,
                                        "ms_per_step": ms8, "bytes_per_token": bpt8,
                                        "gbs": bpt8 / (ms8 / 1e3) / 1e9, "frac": bpt8 / (ms8 / 1e3) / 1e9 / peak,
                                        "steps": 50, "history": "synthetic"}
        msv8, bpb8, acc8 = measure_verify(Q, S, DG, m8, m8.cfg, 131072, Kv, nb, 2, args.seed, sp, stream)
        per_context["131072_verify_k4_kv_int8"] = {
            "kind": "verify", "kv": "int8", "k": Kv, "blocks": nb, "blocks_per_s": 1e3 / msv8,
            "ms_per_block": msv8, "accepted_tokens_per_s": acc8 / (nb * msv8 / 1e3), "rows_per_s": Kv * 1e3 / msv8,
            "bytes_per_block": bpb8, "gbs": bpb8 / (msv8 / 1e3) / 1e9, "frac": bpb8 / (msv8 / 1e3) / 1e9 / peak,
            "accepted_count": "seeded U{0..4}", "history": "synthetic"}
        m8.close()
        npf = 1024
        mspf = measure_prefill(Q, DG, model, cfg, npf, args.seed, sp, stream)
        per_context["prefill_1024_c64"] = {
            "kind": "prefill", "tokens": npf, "chunk": 64, "rows_per_pass": 4, "ms": mspf,
            "tokens_per_s": npf / (mspf / 1e3),
            "note": "64-token chunks from position 0 into a fresh cache, each as passes of 4 rows; "
                    "the head only for the last chunk's last pass"}
        micro = microbench(Q, S, DG, WL, peak, sp, stream)

    cpu = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        r = oracle_sample(cfg, args.seed, max_seconds=20.0, min_steps=1, max_steps=2, context=C)
        cpu = {"value": r["tok_s"], "unit": "tokens/s", "cores": r["cores"], "kind": "oracle",
               "sample": sample_text(r, cfg, C), "extrapolated": True, "cpu": cpu_model_name()}
        r1 = oracle_sample(cfg, args.seed, max_seconds=1.0, min_steps=1, max_steps=1, context=C, threads=1,
                           model=r["model"])
        cpu["single_thread"] = {"value": r1["tok_s"], "unit": "tokens/s", "cores": 1,
                                "sample": sample_text(r1, cfg, C)}

    if rank == 0:
        line = {
            "metric": METRIC, "value": tok_s, "unit": "tokens/s", "n_gpus": world, "steps": K,
            "warmup": W, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "q4_0 x f16 -> f32", "data": "synthetic",
            "config": {"workload": f"12B-class q4_0 decoder ({cfg['n_layers']} layers, h 3840, vocab 262144), "
                                   f"context {C}, batch 1, greedy decode",
                       "context": C, "global_batch": world, "seq_len": C,
                       "parallelism": f"replicas{world}", "prefix": args.prefix,
                       "kv_cache": "int8" if args.kv_int8 else "fp16",
                       "l2": "inputs larger than L2 (6.7 GB of weights read per step)"},
            "hbm": {"bytes_per_token": bytes_per_tok, "gbs_per_gpu": gbs, "peak_gbs": peak,
                    "frac": gbs / peak, "peak_kind": peak_kind},
            "per_context": per_context,
            "roofline": {"bound": "hbm", "kernel": kernel_name,
                         "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": (achieved / peak) if achieved else None, "traffic": traffic,
                         "bytes_per_launch": k_bytes, "ms_per_launch": k_ms,
                         "ms_per_launch_eager": k_ms_eager, "launches_per_step": gemv_launches,
                         "timing": "the GEMV launches' share of an eager profile pass (CUDA events around "
                                   "every launch) times the timed graph step, per launch",
                         "peak_kind": f"{peak_kind} (burst copy)"},
            "kernels": breakdown, "profiled_step_ms": prof_step_ms,
            "microbench": micro,
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
