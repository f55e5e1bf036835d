#!/usr/bin/env python
"""Benchmark of one SVG2 attention layer on B200.

One step = the whole hot path over one synthetic layer: k-means on Q and on K (k-means++ seeding
plus Lloyd iterations), centroid scoring and top-p selection, permutation of Q, K, V, and the
variable-block-size sparse attention with the inverse permutation fused into its epilogue, all
through the C ABI of libsvg2.  Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config wan720p] [--top-p 0.9]
  python bench.py --impl reference ...     # the CPU oracle, timed on a bounded sample

With N > 1 (torchrun), every rank runs its own layer (replicas, weak scaling: the layer's heads
are independent and there is no exchange on the path); the time is the max over ranks.  With
--shard heads the ranks instead split the heads of one layer (strong scaling, still no exchange).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_attention_video_head_b200 import inputs as I  # noqa: E402

METRIC = "per-layer SVG2 attention ms and sparse-attn TFLOP/s vs BF16 peak"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="svg2", choices=["svg2", "reference"])
    ap.add_argument("--config", default="wan720p", choices=sorted(I.CONFIGS))
    ap.add_argument("--top-p", type=float, default=0.9)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-heads-per-group", type=int, default=12,
                    help="heads per transfer group in the end-to-end call (copies overlap the other groups' compute)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-sweep", action="store_true", help="skip the top-p sweep (selection + attention per p)")
    ap.add_argument("--heads", type=int, default=0, help="run only this many heads of the layer (profiling cases)")
    ap.add_argument("--no-denoise", action="store_true", help="skip the denoising-loop driver measurement")
    ap.add_argument("--shard", default="replicas", choices=["replicas", "heads"],
                    help="N > 1: every rank runs its own layer (replicas, weak scaling) or the ranks split the "
                         "heads of one layer (strong scaling)")
    ap.add_argument("--no-warm", action="store_true", help="skip the warm-start denoising-sequence measurement")
    ap.add_argument("--warm-steps", type=int, default=10)
    ap.add_argument("--no-layer-call", action="store_true", help="skip the single svg2_layer call at top-p 0.5")
    ap.add_argument("--no-fp8", action="store_true", help="skip the FP8 attention variant's record")
    ap.add_argument("--second", default="hunyuan720p", choices=["none"] + sorted(I.CONFIGS),
                    help="a second configuration measured after the first (stages, top-p sweep, dense attention)")
    ap.add_argument("--seed-tokens", type=int, default=16384,
                    help="k-means++ candidates per (b,h): every ceil(N/seed_tokens)-th token (0 = all tokens)")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": j["hbm_gbs"], "bf16": j["bf16_tflops"], "bf16_sustained": j["bf16_tflops_sustained"],
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


def gen_inputs(cfg, step=0, heads=None):
    """The layer's synthetic inputs for `heads` (default: all of them), stacked as [1, len(heads), ...]."""
    import multiprocessing as mp
    heads = list(range(cfg.H)) if heads is None else list(heads)
    procs = max(1, min(len(heads), len(os.sched_getaffinity(0))))
    if procs == 1:
        parts = [I.head_inputs(cfg, 0, h, step) for h in heads]
    else:
        with mp.get_context("spawn").Pool(procs) as pool:
            parts = pool.starmap(I.head_inputs, [(cfg, 0, h, step) for h in heads])
    return {k: np.stack([p[k] for p in parts])[None] for k in parts[0]}


# DRAM traffic of one sparse-attention launch from an ncu capture of a 4-head cut of the Wan-720p
# layer (dram__bytes_read.sum + dram__bytes_write.sum = 242.6 MB + 62.9 MB), scaled by heads; valid
# only for the kernel source it was taken on (sha256 of svg2_attn.cu), else reported as null.
ATTN_TRAFFIC = {"sha256": "5d676feb5bb9696a0912839103b85c5bd59af583faf74c082eb38fb0c5d484f9",
                "workload": "wan720p", "heads_captured": 4, "bytes_captured": 242.608128e6 + 62.930688e6,
                "summary": "profiles/sparse_attn_kernel_wan720p_4heads.md"}


def attn_traffic(cfg):
    import hashlib
    src = os.path.join(ROOT, "sparse_attention_video_head_b200", "csrc", "svg2_attn.cu")
    with open(src, "rb") as f:
        if hashlib.sha256(f.read()).hexdigest() != ATTN_TRAFFIC["sha256"] or cfg.name != ATTN_TRAFFIC["workload"]:
            return None
    return ATTN_TRAFFIC["bytes_captured"] * cfg.B * cfg.H / ATTN_TRAFFIC["heads_captured"]


# ------------------------------------------------------------------------------------------ oracle
def oracle_sample(cfg, top_p, rows=96, heads=(0,), seed_tokens=0):
    """The CPU oracle on a bounded sample of the layer: for each head in `heads`, k-means (Q and K),
    selection and permutation in full, and attention for `rows` query rows; extrapolated to the
    whole layer (attention x N/rows, the mean head x H)."""
    from oracle import oracle as O
    scale = float(np.float32(cfg.scale))
    parts = {"kmeans_q_s": 0.0, "kmeans_k_s": 0.0, "select_permute_s": 0.0, "attn_rows_s": 0.0}
    per_head = []
    w0 = time.perf_counter()
    for head in heads:
        hi = I.head_inputs(cfg, 0, head)
        t0 = time.perf_counter()
        cq, lq, count_q = O.kmeans(hi["q"], cfg.nQ, cfg.iters, hi["uq"], seed_tokens=seed_tokens)
        t1 = time.perf_counter()
        ck, lk, count_k = O.kmeans(hi["k"], cfg.nK, cfg.iters, hi["uk"], seed_tokens=seed_tokens)
        t2 = time.perf_counter()
        w = O.select_weights(cq.astype(np.float32), ck.astype(np.float32), count_k, scale)
        mask = O.topp(w, count_k, top_p)
        pq, qo = O.permute(lq, cfg.nQ)
        pk, ko = O.permute(lk, cfg.nK)
        Qp, Kp, Vp = O.gather_rows(hi["q"], pq), O.gather_rows(hi["k"], pk), O.gather_rows(hi["v"], pk)
        t3 = time.perf_counter()
        sel = np.random.default_rng(1 + head).choice(cfg.N, rows, replace=False)
        O.sparse_attention_rows(Qp, Kp, Vp, qo, ko, mask, scale, sel)
        t4 = time.perf_counter()
        for key, dt in zip(parts, (t1 - t0, t2 - t1, t3 - t2, t4 - t3)):
            parts[key] += dt
        per_head.append((t3 - t0) + (t4 - t3) * cfg.N / rows)
    parts["wall_s"] = time.perf_counter() - w0
    return float(np.mean(per_head)) * cfg.H * 1e3, parts


def sample_text(cfg, rows, heads):
    return (f"{len(heads)} of {cfg.H} heads: full k-means++ + {cfg.iters} Lloyd iterations on Q and K, selection, "
            f"permutation, and attention for {rows} of {cfg.N} query rows per head; extrapolated "
            f"x{cfg.N}/{rows} rows, mean head x{cfg.H} heads")


# One sample definition for both CPU legs (the reference arm and cpu_baseline): the first
# ORACLE_HEADS heads in full (k-means, selection, permutation) and ORACLE_ROWS query rows of attention
# per head, extrapolated to the layer.
ORACLE_HEADS, ORACLE_ROWS = 2, 128


def run_reference(args, cfg):
    cores = len(os.sched_getaffinity(0))
    heads = tuple(range(min(ORACLE_HEADS, cfg.H)))
    for _ in range(args.warmup):
        oracle_sample(cfg, args.top_p, rows=16, heads=heads[:1], seed_tokens=args.seed_tokens)
    vals = []
    for _ in range(args.steps):
        v, _ = oracle_sample(cfg, args.top_p, rows=ORACLE_ROWS, heads=heads, seed_tokens=args.seed_tokens)
        vals.append(v)
    value = statistics.median(vals)
    sample = sample_text(cfg, ORACLE_ROWS, heads)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "ms", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": value, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(cfg, args.top_p, args.seed_tokens),
            "cpu_baseline": {"value": value, "unit": "ms", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "ms", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_dict(cfg, top_p, seed_tokens, shard=None):
    """`shard` = (layer heads, world) when the ranks split one layer's heads; cfg.H is then the rank's."""
    heads, world = shard if shard else (cfg.H, 1)
    return {"workload": cfg.name, "B": cfg.B, "H": heads, "N": cfg.N, "grid": list(cfg.grid), "d": cfg.d,
            "nQ": cfg.nQ, "nK": cfg.nK, "iters": cfg.iters, "init": "kmeans++", "top_p": top_p,
            "kmeanspp_seed_tokens": seed_tokens,
            "components": cfg.components, "sigma": cfg.sigma,
            "l2": "inputs larger than L2 (each of Q, K, V is %.0f MB)" % (cfg.B * cfg.H * cfg.N * cfg.d * 2 / 1e6),
            "parallelism": f"heads/{world}" if shard else "replicas"}


def max_over_ranks(value: float, world: int, dist, device) -> float:
    """The slowest rank's time (a multi-GPU number is the max over ranks, never one rank's clock)."""
    if world <= 1:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_ms_per_layer(ms_per_step: float, world: int, sharded: bool = False) -> float:
    """Replicas (weak scaling, one layer per rank per step): the job finishes `world` layers per
    step.  Heads split across the ranks (strong scaling): one layer per step."""
    return ms_per_step if sharded else ms_per_step / world


# ------------------------------------------------------------------------------------------ clocks
class ClockSampler:
    def __init__(self, index):
        self.proc = None
        self.index = index

    def __enter__(self):
        q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                                          "-i", str(self.index), "-lms", "200"], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[0]))
                mx = float(f[1])
            except ValueError:
                continue
            for n, v in zip(names, f[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------------------------------ one layer
class LayerBench:
    """Device buffers and the timed step of one layer configuration, every stage through the C ABI:
    k-means of Q and of K, selection, the three row gathers, the attention with the inverse
    permutation fused into its epilogue."""

    names = ["kmeans_q", "kmeans_k", "select", "permute", "sparse_attn"]

    def __init__(self, svg2, torch, cfg, data, dev, seed_tokens, top_p):
        self.svg2, self.torch, self.cfg, self.dev = svg2, torch, cfg, dev
        self.seed_tokens, self.top_p = seed_tokens, top_p
        B, H, N, d = 1, cfg.H, cfg.N, cfg.d
        self.scale = float(np.float32(cfg.scale))
        self.Q = torch.from_numpy(data["q"]).to(torch.bfloat16).to(dev)
        self.K = torch.from_numpy(data["k"]).to(torch.bfloat16).to(dev)
        self.V = torch.from_numpy(data["v"]).to(torch.bfloat16).to(dev)
        self.uq = torch.from_numpy(data["uq"]).to(dev)
        self.uk = torch.from_numpy(data["uk"]).to(dev)
        self.cq = torch.zeros(B, H, cfg.nQ, d, device=dev)
        self.ck = torch.zeros(B, H, cfg.nK, d, device=dev)
        self.O = torch.empty_like(self.Q)
        self.ws = svg2.workspace(B, H, N, d, cfg.nQ, cfg.nK, device=dev)
        self.Qp, self.Kp, self.Vp = torch.empty_like(self.Q), torch.empty_like(self.K), torch.empty_like(self.V)
        i32 = dict(dtype=torch.int32, device=dev)
        self.lab_q, self.lab_k = torch.empty(B, H, N, **i32), torch.empty(B, H, N, **i32)
        self.cnt_q, self.cnt_k = torch.empty(B, H, cfg.nQ, **i32), torch.empty(B, H, cfg.nK, **i32)
        self.perm_q, self.perm_k = torch.empty(B, H, N, **i32), torch.empty(B, H, N, **i32)
        self.q_off, self.k_off = torch.empty(B, H, cfg.nQ + 1, **i32), torch.empty(B, H, cfg.nK + 1, **i32)
        self.mask = torch.empty(B, H, cfg.nQ, cfg.nK, dtype=torch.uint8, device=dev)
        self.sel_count, self.sel_idx = torch.empty(B, H, cfg.nQ, **i32), torch.empty(B, H, cfg.nQ, cfg.nK, **i32)
        self.stream_len = torch.empty(B, H, cfg.nQ, **i32)
        self.stream = torch.cuda.current_stream(dev)

    def step(self, ev=None, top_p=None):
        svg2, cfg, KPP = self.svg2, self.cfg, self.svg2.SVG2_INIT_KMEANSPP

        def mark(i):
            if ev is not None:
                ev[i].record(self.stream)
        mark(0)
        svg2.svg2_kmeans(self.Q, cfg.nQ, cfg.iters, KPP, self.cq, self.lab_q, self.cnt_q, self.ws, u=self.uq,
                         perm=self.perm_q, offsets=self.q_off, seed_tokens=self.seed_tokens)
        mark(1)
        svg2.svg2_kmeans(self.K, cfg.nK, cfg.iters, KPP, self.ck, self.lab_k, self.cnt_k, self.ws, u=self.uk,
                         perm=self.perm_k, offsets=self.k_off, seed_tokens=self.seed_tokens)
        mark(2)
        self.select(self.top_p if top_p is None else top_p)
        mark(3)
        svg2.svg2_gather(self.Q, self.perm_q, self.Qp)
        svg2.svg2_gather(self.K, self.perm_k, self.Kp)
        svg2.svg2_gather(self.V, self.perm_k, self.Vp)
        mark(4)
        self.attend()
        mark(5)

    def select(self, p):
        self.svg2.svg2_select(self.cq, self.ck, self.cnt_k, p, self.scale, self.mask, self.sel_count, self.sel_idx,
                              self.ws, stream_len=self.stream_len)

    def attend(self):
        self.svg2.svg2_sparse_attn(self.Qp, self.Kp, self.Vp, self.q_off, self.k_off, self.sel_count, self.sel_idx,
                                   self.scale, self.O, self.ws, perm_q=self.perm_q)

    def flops(self):
        """(actual, dense-equivalent, executed) attention FLOPs of the current selection."""
        cfg, d = self.cfg, self.cfg.d
        cq_h = self.cnt_q.cpu().numpy().astype(np.float64)
        sl_h = self.stream_len.cpu().numpy().astype(np.float64)
        actual = 4.0 * d * float((cq_h * sl_h).sum())
        dense = 4.0 * d * cfg.N * cfg.N * cfg.B * cfg.H
        executed = 4.0 * d * float((np.ceil(cq_h / 128.0) * 128.0 * np.ceil(sl_h / 128.0) * 128.0).sum())
        return actual, dense, executed

    def time_steps(self, steps):
        torch = self.torch
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(steps)]
        t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t_start.record(self.stream)
        for i in range(steps):
            self.step(evs[i])
        t_end.record(self.stream)
        torch.cuda.synchronize(self.dev)
        stage_ms = {n: statistics.mean(e[i].elapsed_time(e[i + 1]) for e in evs) for i, n in enumerate(self.names)}
        return t_start.elapsed_time(t_end), stage_ms

    def sweep(self, stage_ms, extra=(0.5, 1.0)):
        """Selection + attention per top-p on the step's clusters: the configuration's values plus
        labelled extension points (p = 0.5 towards the pages' 25-35 % densities on these inputs, p = 1
        every pair kept: dense attention through the sparse path)."""
        torch = self.torch
        notes = {0.5: "extension: lower density", 1.0: "extension: every pair kept (dense through the sparse path)"}
        kmeans_ms = stage_ms["kmeans_q"] + stage_ms["kmeans_k"]
        out = {}
        for p in sorted(set(self.cfg.top_p) | {self.top_p} | set(extra)):
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            self.select(p)
            self.attend()
            torch.cuda.synchronize(self.dev)
            ev[0].record(self.stream)
            self.select(p)
            ev[1].record(self.stream)
            self.attend()
            ev[2].record(self.stream)
            torch.cuda.synchronize(self.dev)
            flops, dense, _ = self.flops()
            a_ms = ev[1].elapsed_time(ev[2])
            out[str(p)] = {"density": flops / dense, "select_ms": ev[0].elapsed_time(ev[1]), "attn_ms": a_ms,
                           "attn_tflops_actual": flops / (a_ms * 1e-3) / 1e12,
                           "attn_tflops_effective": dense / (a_ms * 1e-3) / 1e12,
                           "layer_ms": kmeans_ms + ev[0].elapsed_time(ev[1]) + stage_ms["permute"] + a_ms}
            if p in notes and p not in set(self.cfg.top_p) | {self.top_p}:
                out[str(p)]["note"] = notes[p]
        self.select(self.top_p)
        return out


def time_layer_call(svg2, torch, lb, top_p, dense_ms, reps=3, attn_fp8=0):
    """The whole layer as one svg2_layer call (k-means++ and Lloyd on Q and K, selection,
    permutation, attention with the fused inverse permutation) at `top_p`, timed with CUDA events."""
    cfg = lb.cfg
    prm = svg2.LayerParams(cfg.nQ, cfg.nK, cfg.iters, svg2.SVG2_INIT_KMEANSPP, top_p, lb.scale, 1, lb.seed_tokens,
                           attn_fp8)
    cq, ck = torch.zeros_like(lb.cq), torch.zeros_like(lb.ck)
    outs = svg2.layer_output_buffers(1, cfg.H, cfg.N, cfg.nQ, cfg.nK, device=lb.dev)
    svg2.svg2_layer(lb.Q, lb.K, lb.V, prm, cq, ck, lb.O, lb.ws, lb.uq, lb.uk, outs)
    torch.cuda.synchronize(lb.dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(lb.stream)
    for _ in range(reps):
        svg2.svg2_layer(lb.Q, lb.K, lb.V, prm, cq, ck, lb.O, lb.ws, lb.uq, lb.uk, outs)
    b.record(lb.stream)
    torch.cuda.synchronize(lb.dev)
    svg2.raise_on_device_error(lb.ws)
    ms = a.elapsed_time(b) / reps
    cnt_q = outs["count_q"].cpu().numpy().astype(np.float64)
    sl = outs["stream_len"].cpu().numpy().astype(np.float64)
    density = float((cnt_q * sl).sum()) / (cfg.N * cfg.N * cfg.B * cfg.H)
    out = {"api": "svg2_layer", "top_p": top_p, "attn_fp8": attn_fp8, "density": density, "ms": ms, "reps": reps}
    if isinstance(dense_ms, float):
        out["dense_sdpa_ms"] = dense_ms
        out["speedup_vs_dense"] = dense_ms / ms
    return out


def measure_fp8(svg2, torch, lb, P, reps=5):
    """The FP8 attention variant on the step's own plan (clusters, selection, permutation): the three
    quantising gathers (E4M3 codes with per-(b,h) scales), the FP8 attention, the relative L2 of its
    output against the bf16 attention's on every element, and the whole layer as one svg2_layer call
    with attn_fp8 = 1.  The FP8 peak is the measured bf16 sustained peak times 2 (the nominal dense
    E4M3 / bf16 ratio, 4.5 / 2.25 PFLOP/s)."""
    cfg, dev = lb.cfg, lb.dev
    shape = (1, cfg.H, cfg.N, cfg.d)
    Q8, K8, V8 = (torch.empty(shape, dtype=torch.uint8, device=dev) for _ in range(3))
    sq, sk, sv = (torch.empty(1, cfg.H, dtype=torch.float32, device=dev) for _ in range(3))
    O8 = torch.empty_like(lb.O)

    def quantize():
        svg2.svg2_quantize_e4m3(lb.Q, Q8, sq, perm=lb.perm_q)
        svg2.svg2_quantize_e4m3(lb.K, K8, sk, perm=lb.perm_k)
        svg2.svg2_quantize_e4m3(lb.V, V8, sv, perm=lb.perm_k)

    def attend():
        svg2.svg2_sparse_attn_fp8(Q8, K8, V8, sq, sk, sv, lb.q_off, lb.k_off, lb.sel_count, lb.sel_idx, lb.scale,
                                  O8, lb.ws, perm_q=lb.perm_q)

    lb.step()  # the plan again: earlier records (the all-token seeding, the warm start) re-cluster in place
    quantize()
    attend()
    lb.attend()  # the bf16 output on the same plan, for the comparison
    torch.cuda.synchronize(dev)
    svg2.raise_on_device_error(lb.ws)
    diff = (O8.float() - lb.O.float()).norm() / lb.O.float().norm()
    # quantisation, then the FP8 and the bf16 attention interleaved on the same plan
    eq = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    eq[0].record(lb.stream)
    for _ in range(reps):
        quantize()
    eq[1].record(lb.stream)
    ea = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(reps)]
    for e in ea:
        e[0].record(lb.stream)
        attend()
        e[1].record(lb.stream)
        lb.attend()
        e[2].record(lb.stream)
    torch.cuda.synchronize(dev)
    svg2.raise_on_device_error(lb.ws)
    q_ms = eq[0].elapsed_time(eq[1]) / reps
    a_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ea)
    b_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ea)
    actual, _, _ = lb.flops()
    tflops = actual / (a_ms * 1e-3) / 1e12
    # per tensor: the maximum pass reads the bf16 plane, the gather reads it again and writes one byte
    # per value, and reads one permutation entry per row
    quant_bytes = 3 * (lb.Q.numel() * (2 + 2 + 1) + lb.perm_q.numel() * 4)
    out = {"kernel": "sparse_attn_kernel<128, F8> (tcgen05 kind::f8f6f4)", "top_p": lb.top_p,
           "quantize_ms": q_ms, "quantize_bytes": quant_bytes,
           "quantize_gbs": quant_bytes / (q_ms * 1e-3) / 1e9, "attn_ms": a_ms, "attn_tflops_actual": tflops,
           "peak_tflops": 2 * P["bf16_sustained"], "frac_of_fp8_sustained_peak": tflops / (2 * P["bf16_sustained"]),
           "bf16_attn_ms_same_plan": b_ms, "speedup_vs_bf16_attn": b_ms / a_ms,
           "rel_l2_vs_bf16_output": float(diff)}
    del Q8, K8, V8, O8
    out["layer_call"] = time_layer_call(svg2, torch, lb, lb.top_p, None, attn_fp8=1)
    out["layer_call_bf16"] = time_layer_call(svg2, torch, lb, lb.top_p, None)
    return out


def measure_second_config(svg2, torch, cfg, args, dev, P, steps=3, warmup=2):
    """A second configuration (by default the Hunyuan-720p layer): stage times of the step, density
    and attention throughput per top-p, and dense attention on the same tensors."""
    data = gen_inputs(cfg)
    lb = LayerBench(svg2, torch, cfg, data, dev, args.seed_tokens, args.top_p)
    del data
    for _ in range(warmup):
        lb.step()
    torch.cuda.synchronize(dev)
    svg2.raise_on_device_error(lb.ws)
    actual, dense, executed = lb.flops()
    total_ms, stage_ms = lb.time_steps(steps)
    svg2.raise_on_device_error(lb.ws)
    attn_tflops = actual / (stage_ms["sparse_attn"] * 1e-3) / 1e12
    out = {"workload": cfg.name, "H": cfg.H, "N": cfg.N, "nQ": cfg.nQ, "nK": cfg.nK, "iters": cfg.iters,
           "top_p": args.top_p, "steps": steps, "ms_per_step": total_ms / steps, "stages_ms": stage_ms,
           "density": actual / dense, "attn_tflops_actual": attn_tflops,
           "attn_frac_of_sustained_peak": attn_tflops / P["bf16_sustained"],
           "executed_over_actual": executed / actual, "top_p_sweep": lb.sweep(stage_ms, extra=(0.5,))}
    out["dense_sdpa_ms"] = time_dense(torch, lb.Q, lb.K, lb.V, lb.scale)
    out["layer_call_low_density"] = time_layer_call(svg2, torch, lb, 0.5, out["dense_sdpa_ms"])
    svg2.raise_on_device_error(lb.ws)
    return out


# ------------------------------------------------------------------------------------------ GPU arm
def main():
    args = parse()
    cfg = I.CONFIGS[args.config]
    if args.heads:
        import dataclasses
        cfg = dataclasses.replace(cfg, H=args.heads)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            run_reference(args, cfg)
        return
    sharded = args.shard == "heads" and world > 1
    shard_info = None
    if sharded:
        import dataclasses
        from sparse_attention_video_head_b200.shard import head_range
        h0, h1 = head_range(cfg.H, world, rank)
        if h1 == h0:
            raise SystemExit(f"--shard heads needs at least one head per rank ({cfg.H} heads, {world} ranks)")
        data = gen_inputs(cfg, heads=range(h0, h1))  # this rank's block of the layer's heads
        shard_info = (cfg.H, world)
        cfg = dataclasses.replace(cfg, H=h1 - h0)
    else:
        data = gen_inputs(cfg)  # before CUDA initialisation

    import torch
    import torch.distributed as dist
    from sparse_attention_video_head_b200 import svg2

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    P = peaks()
    B, H, N, d = 1, cfg.H, cfg.N, cfg.d
    BH = B * H
    scale = float(np.float32(cfg.scale))
    lb = LayerBench(svg2, torch, cfg, data, dev, args.seed_tokens, args.top_p)
    Q, K, V, O, ws = lb.Q, lb.K, lb.V, lb.O, lb.ws
    Qp, Kp, Vp = lb.Qp, lb.Kp, lb.Vp
    perm_q, perm_k, q_off, k_off = lb.perm_q, lb.perm_k, lb.q_off, lb.k_off
    cq, ck, lab_q, lab_k, cnt_q, cnt_k, uq, uk = lb.cq, lb.ck, lb.lab_q, lb.lab_k, lb.cnt_q, lb.cnt_k, lb.uq, lb.uk
    KPP = svg2.SVG2_INIT_KMEANSPP
    stream = torch.cuda.current_stream(dev)

    for _ in range(args.warmup):
        lb.step()
    torch.cuda.synchronize(dev)
    svg2.raise_on_device_error(ws)

    # algorithmic work of the attention (actual = kept pairs only, no padding)
    actual_flops, dense_flops, executed_flops = lb.flops()
    density = actual_flops / dense_flops
    waste128 = fixed128_waste(q_off.cpu().numpy(), k_off.cpu().numpy(), lb.mask.cpu().numpy(), heads=range(min(4, H)))

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        total_ms, stage_ms = lb.time_steps(args.steps)
    if world > 1:
        dist.barrier()
    svg2.raise_on_device_error(ws)
    total_ms = max_over_ranks(total_ms, world, dist, dev)
    ms_per_step = total_ms / args.steps
    attn_ms = stage_ms["sparse_attn"]
    achieved_tflops = actual_flops / (attn_ms * 1e-3) / 1e12

    # the configuration's top-p sweep on the same clusters: selection + attention per p
    sweep = None
    if not args.no_sweep:
        sweep = lb.sweep(stage_ms)
        svg2.raise_on_device_error(ws)

    # HBM stages against the measured copy bandwidth: the three row gathers (permutation) as timed
    # in the step, and the stand-alone inverse permutation (fused into the attention in the step)
    plane = BH * N * d * 2
    perm_bytes = 3 * (2 * plane + BH * N * 4)
    eu = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    for _ in range(3):
        svg2.svg2_unpermute(Qp, perm_q, Kp)  # (Kp is rebuilt by the next step's gathers)
    eu[0].record(stream)
    for _ in range(5):
        svg2.svg2_unpermute(Qp, perm_q, Kp)
    eu[1].record(stream)
    torch.cuda.synchronize(dev)
    unperm_ms = eu[0].elapsed_time(eu[1]) / 5
    unperm_bytes = 2 * plane + BH * N * 4
    hbm_stages = {
        "peak_gbs": P["hbm_gbs"], "peak_source": P["source"] + " copy bandwidth",
        "permute": {"kernel": "gather_rows_kernel x3", "ms": stage_ms["permute"], "bytes": perm_bytes,
                    "gbs": perm_bytes / (stage_ms["permute"] * 1e-3) / 1e9,
                    "frac": perm_bytes / (stage_ms["permute"] * 1e-3) / 1e9 / P["hbm_gbs"]},
        "unpermute": {"kernel": "scatter_rows_kernel (stand-alone svg2_unpermute)", "ms": unperm_ms,
                      "bytes": unperm_bytes, "gbs": unperm_bytes / (unperm_ms * 1e-3) / 1e9,
                      "frac": unperm_bytes / (unperm_ms * 1e-3) / 1e9 / P["hbm_gbs"]},
    }
    svg2.svg2_gather(K, perm_k, Kp)

    # k-means with k-means++ over all tokens (seed_tokens = 0), for comparison with the sampled seeding
    full_seed = None
    if args.seed_tokens != 0:
        ea = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        ea[0].record(stream)
        svg2.svg2_kmeans(Q, cfg.nQ, cfg.iters, KPP, cq, lab_q, cnt_q, ws, u=uq, perm=perm_q, offsets=q_off, seed_tokens=0)
        ea[1].record(stream)
        svg2.svg2_kmeans(K, cfg.nK, cfg.iters, KPP, ck, lab_k, cnt_k, ws, u=uk, perm=perm_k, offsets=k_off, seed_tokens=0)
        ea[2].record(stream)
        torch.cuda.synchronize(dev)
        full_seed = {"kmeans_q_ms": ea[0].elapsed_time(ea[1]), "kmeans_k_ms": ea[1].elapsed_time(ea[2])}

    # the same layer through the single public call with host buffers (copies inside the timed region)
    e2e = None
    if not args.no_e2e:
        e2e = measure_e2e(svg2, torch, cfg, data, args, dev, ws, world, dist)

    dense_ms = own_dense = None
    if not args.no_dense and rank == 0:
        dense_ms = time_dense(torch, Q, K, V, scale)
        own_dense = time_own_dense(svg2, torch, Q, K, V, scale)


    denoise = None
    if not args.no_denoise and rank == 0:
        denoise = measure_denoise(svg2, torch, cfg, args, dev, Q, K, V, scale)

    warm = None
    if not args.no_warm:
        warm = measure_warm(svg2, torch, cfg, args, dev, Q, K, V, ws, scale)

    # the whole layer as one svg2_layer call at a low top-p (the pages' 25-35 % densities on these
    # inputs), beside dense attention on the same tensors
    layer_call = None
    if not args.no_layer_call and rank == 0:
        layer_call = time_layer_call(svg2, torch, lb, 0.5, dense_ms)

    fp8 = None
    if not args.no_fp8 and rank == 0:
        fp8 = measure_fp8(svg2, torch, lb, P)

    second = None
    if args.second not in ("none", cfg.name) and not args.heads and rank == 0 and world == 1:
        second = measure_second_config(svg2, torch, I.CONFIGS[args.second], args, dev, P)

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        heads = tuple(range(min(ORACLE_HEADS, cfg.H)))
        v, parts = oracle_sample(cfg, args.top_p, rows=ORACLE_ROWS, heads=heads, seed_tokens=args.seed_tokens)
        cpu = {"value": v, "unit": "ms", "cores": len(os.sched_getaffinity(0)), "kind": "oracle",
               "sample": sample_text(cfg, ORACLE_ROWS, heads), "parts_s": parts}
    launches = kernel_launches(cfg)
    line = {
        "metric": METRIC, "value": whole_job_ms_per_layer(ms_per_step, world, sharded), "unit": "ms", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": False,
        "scaling": "strong" if sharded else "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config_dict(cfg, args.top_p, args.seed_tokens, shard_info),
        "roofline": {"bound": "tensor", "kernel": "sparse_attn_kernel", "achieved": achieved_tflops,
                     "peak": P["bf16_sustained"], "unit": "TFLOP/s",
                     "frac": achieved_tflops / P["bf16_sustained"],
                     "peak_source": P["source"] + " bf16 cuBLAS, sustained (kernel timed inside a long step)",
                     "traffic": attn_traffic(cfg), "traffic_unit": "bytes per launch",
                     "algorithmic_bytes": 4.0 * B * H * N * d * 2},
        "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches * args.steps,
        "clocks": clk.summary(), "stages_ms": stage_ms, "density": density,
        "attn_tflop_actual": actual_flops / 1e12, "attn_tflop_dense_equiv": dense_flops / 1e12,
        "attn_tflops_effective": dense_flops / (attn_ms * 1e-3) / 1e12,
        "layer_tflops_effective": dense_flops / (ms_per_step * 1e-3) / 1e12,
        "executed_over_actual": executed_flops / actual_flops, "fixed128_padding_waste": waste128,
        "hbm_stages": hbm_stages,
        "dense_sdpa_ms": dense_ms, "dense_sdpa_backends_enabled": sdpa_backends(torch) if dense_ms is not None else None,
        "dense_svg2_dense_attn": own_dense, "denoise_driver": denoise, "warm_start": warm, "kmeans_all_token_seeding": full_seed,
        "top_p_sweep": sweep, "layer_call_low_density": layer_call, "fp8_attention": fp8, "second_config": second,
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def measure_e2e(svg2, torch, cfg, data, args, dev, ws, world, dist):
    B, H, N, d = 1, cfg.H, cfg.N, cfg.d
    hq = torch.from_numpy(data["q"]).to(torch.bfloat16).pin_memory()
    hk = torch.from_numpy(data["k"]).to(torch.bfloat16).pin_memory()
    hv = torch.from_numpy(data["v"]).to(torch.bfloat16).pin_memory()
    huq = torch.from_numpy(data["uq"]).pin_memory()
    huk = torch.from_numpy(data["uk"]).pin_memory()
    ho = torch.empty(B, H, N, d, dtype=torch.bfloat16).pin_memory()
    Q = torch.empty(B, H, N, d, dtype=torch.bfloat16, device=dev)
    K, V, O = torch.empty_like(Q), torch.empty_like(Q), torch.empty_like(Q)
    uq = torch.empty(huq.shape, dtype=torch.float64, device=dev)
    uk = torch.empty(huk.shape, dtype=torch.float64, device=dev)
    cq = torch.zeros(B, H, cfg.nQ, d, device=dev)
    ck = torch.zeros(B, H, cfg.nK, d, device=dev)
    prm = svg2.LayerParams(cfg.nQ, cfg.nK, cfg.iters, svg2.SVG2_INIT_KMEANSPP, args.top_p, float(np.float32(cfg.scale)), 1,
                           args.seed_tokens)
    copy_stream = torch.cuda.Stream(device=dev)
    # the uniforms are tiny; they go up on the compute stream before the layer call
    def one():
        uq.copy_(huq, non_blocking=True)
        uk.copy_(huk, non_blocking=True)
        svg2.svg2_layer_host(hq, hk, hv, ho, Q, K, V, O, prm, cq, ck, ws, uq, uk,
                             heads_per_group=args.e2e_heads_per_group, copy_stream=copy_stream)

    for _ in range(max(1, args.warmup)):
        one()
    torch.cuda.synchronize(dev)
    steps = max(1, min(args.steps, 5))
    if world > 1:
        dist.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        one()
    b.record()
    torch.cuda.synchronize(dev)
    svg2.raise_on_device_error(ws)
    ms = max_over_ranks(a.elapsed_time(b) / steps, world, dist, dev)
    h2d = 3 * hq.numel() * 2 + (huq.numel() + huk.numel()) * 8
    return {"value": whole_job_ms_per_layer(ms, world, args.shard == "heads" and world > 1), "unit": "ms",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": ho.numel() * 2,
            "steps": steps, "api": "svg2_layer_host", "heads_per_group": args.e2e_heads_per_group}


def measure_warm(svg2, torch, cfg, args, dev, Q0, K0, V0, ws, scale):
    """Denoising-step sequence on the same shapes (the pages' centroid cache, section 4.3 Fig. 7(a)):
    step s uses Q_s = Q_0 + 0.05 s eps_s, K_s likewise, a fresh V_s; k-means starts from step s-1's
    centroids and runs 2 iterations (warm), and is also run cold (k-means++ + cfg.iters) on the same
    inputs.  Reports per-step warm layer ms, warm vs cold k-means ms, centroid drift, and the
    relative L2 error of both outputs against dense attention (torch SDPA) of step s."""
    B, H, N, d = Q0.shape
    i32 = dict(dtype=torch.int32, device=dev)
    bufs = {}

    def kbufs(tag, k):
        if tag not in bufs:
            bufs[tag] = (torch.empty(B, H, N, **i32), torch.empty(B, H, k, **i32), torch.empty(B, H, N, **i32),
                         torch.empty(B, H, k + 1, **i32))
        return bufs[tag]

    lab_q, cnt_q, perm_q, q_off = kbufs("q", cfg.nQ)
    lab_k, cnt_k, perm_k, k_off = kbufs("k", cfg.nK)
    mask = torch.empty(B, H, cfg.nQ, cfg.nK, dtype=torch.uint8, device=dev)
    sel_count, sel_idx = torch.empty(B, H, cfg.nQ, **i32), torch.empty(B, H, cfg.nQ, cfg.nK, **i32)
    Qp, Kp, Vp = torch.empty_like(Q0), torch.empty_like(Q0), torch.empty_like(Q0)
    O_w, O_c = torch.empty_like(Q0), torch.empty_like(Q0)
    g = torch.Generator(device=dev)
    gen_u = np.random.default_rng(12345)
    uq = torch.from_numpy(gen_u.random((B, H, cfg.nQ))).to(dev)
    uk = torch.from_numpy(gen_u.random((B, H, cfg.nK))).to(dev)
    cq = torch.zeros(B, H, cfg.nQ, d, device=dev)
    ck = torch.zeros(B, H, cfg.nK, d, device=dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)

    def layer(Q, K, V, cqx, ckx, init, iters, O):
        e = [ev() for _ in range(4)]
        e[0].record()
        svg2.svg2_kmeans(Q, cfg.nQ, iters, init, cqx, lab_q, cnt_q, ws, u=uq, perm=perm_q, offsets=q_off,
                         seed_tokens=args.seed_tokens)
        svg2.svg2_kmeans(K, cfg.nK, iters, init, ckx, lab_k, cnt_k, ws, u=uk, perm=perm_k, offsets=k_off,
                         seed_tokens=args.seed_tokens)
        e[1].record()
        svg2.svg2_select(cqx, ckx, cnt_k, args.top_p, scale, mask, sel_count, sel_idx, ws)
        svg2.svg2_gather(Q, perm_q, Qp)
        svg2.svg2_gather(K, perm_k, Kp)
        svg2.svg2_gather(V, perm_k, Vp)
        svg2.svg2_sparse_attn(Qp, Kp, Vp, q_off, k_off, sel_count, sel_idx, scale, O, ws, perm_q=perm_q)
        e[2].record()
        return e

    # step 0: cold start, fills the cache
    layer(Q0, K0, V0, cq, ck, svg2.SVG2_INIT_KMEANSPP, cfg.iters, O_c)
    out = {"steps": args.warm_steps, "warm_iters": 2, "cold": "k-means++ + %d iterations" % cfg.iters,
           "layer_ms_warm": [], "kmeans_ms_warm": [], "kmeans_ms_cold": [], "drift_q": [], "drift_k": [],
           "rel_l2_vs_dense_warm": [], "rel_l2_vs_dense_cold": []}
    for step in range(1, args.warm_steps + 1):
        g.manual_seed(1000 + step)
        Q = (Q0.float() + 0.05 * step * torch.randn(Q0.shape, device=dev, generator=g)).to(torch.bfloat16)
        K = (K0.float() + 0.05 * step * torch.randn(K0.shape, device=dev, generator=g)).to(torch.bfloat16)
        V = torch.randn(V0.shape, device=dev, generator=g).to(torch.bfloat16)
        cq_prev, ck_prev = cq.clone(), ck.clone()
        ew = layer(Q, K, V, cq, ck, svg2.SVG2_INIT_GIVEN, 2, O_w)
        cq_c, ck_c = torch.zeros_like(cq), torch.zeros_like(ck)
        ec = layer(Q, K, V, cq_c, ck_c, svg2.SVG2_INIT_KMEANSPP, cfg.iters, O_c)
        dense = torch.nn.functional.scaled_dot_product_attention(Q, K, V, scale=scale).float()
        torch.cuda.synchronize(dev)
        dn = dense.norm()
        out["layer_ms_warm"].append(ew[0].elapsed_time(ew[2]))
        out["kmeans_ms_warm"].append(ew[0].elapsed_time(ew[1]))
        out["kmeans_ms_cold"].append(ec[0].elapsed_time(ec[1]))
        out["drift_q"].append(float((cq - cq_prev).norm() / cq_prev.norm()))
        out["drift_k"].append(float((ck - ck_prev).norm() / ck_prev.norm()))
        out["rel_l2_vs_dense_warm"].append(float((O_w.float() - dense).norm() / dn))
        out["rel_l2_vs_dense_cold"].append(float((O_c.float() - dense).norm() / dn))
    svg2.raise_on_device_error(ws)
    med = lambda v: float(statistics.median(v))
    out["summary"] = {"layer_ms_warm": med(out["layer_ms_warm"]), "kmeans_ms_warm": med(out["kmeans_ms_warm"]),
                      "kmeans_ms_cold": med(out["kmeans_ms_cold"]),
                      "kmeans_speedup": med(out["kmeans_ms_cold"]) / med(out["kmeans_ms_warm"])}
    return out


def sdpa_backends(torch):
    """The scaled_dot_product_attention backends torch has enabled (it picks among them per call)."""
    b = torch.backends.cuda
    names = {"flash": b.flash_sdp_enabled, "cudnn": getattr(b, "cudnn_sdp_enabled", None),
             "mem_efficient": b.mem_efficient_sdp_enabled, "math": b.math_sdp_enabled}
    return [n for n, f in names.items() if f is not None and f()]


def time_dense(torch, Q, K, V, scale, reps=3):
    try:
        f = torch.nn.functional.scaled_dot_product_attention
        f(Q, K, V, scale=scale)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            f(Q, K, V, scale=scale)
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps
    except Exception as e:  # library baseline only; never part of the product path
        return f"unavailable: {type(e).__name__}"


def measure_denoise(svg2, torch, cfg, args, dev, Q, K, V, scale, steps=6, dense_steps=1):
    """The denoising-loop driver over a short schedule of one layer: `dense_steps` dense steps, then
    a cold k-means step, then warm steps (2 iterations from the layer's cached centroids).  The
    inputs are the step's tensors re-used each step (the k-means work per warm step is fixed at 2
    iterations whatever the drift).  Reports ms per step kind and the schedule's mean per step."""
    B, H, N, d = Q.shape
    p = svg2.LayerParams(nQ=cfg.nQ, nK=cfg.nK, iters=cfg.iters, top_p=args.top_p, scale=scale,
                         seed_tokens=args.seed_tokens)
    drv = svg2.Driver(B, H, N, d, num_steps=steps, num_layers=1, dense_steps=dense_steps, warm_iters=2, params=p,
                      device=dev)
    rng = np.random.default_rng(4321)
    uq = torch.from_numpy(rng.random((B, H, cfg.nQ))).to(dev)
    uk = torch.from_numpy(rng.random((B, H, cfg.nK))).to(dev)
    O = torch.empty_like(Q)
    names = {svg2.SVG2_STEP_DENSE: "dense", svg2.SVG2_STEP_COLD: "cold", svg2.SVG2_STEP_WARM: "warm"}
    for s in range(steps):  # warm-up pass over the schedule
        drv.layer(s, 0, Q, K, V, O, uq, uk)
    drv.reset()
    per = {}
    total = 0.0
    for s in range(steps):
        kind = names[drv.plan(s, 0)]
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        drv.layer(s, 0, Q, K, V, O, uq, uk)
        b.record()
        torch.cuda.synchronize(dev)
        ms = a.elapsed_time(b)
        per.setdefault(kind, []).append(ms)
        total += ms
    svg2.raise_on_device_error(drv.ws)
    out = {"steps": steps, "dense_steps": dense_steps, "warm_iters": 2,
           "ms": {k: statistics.mean(v) for k, v in per.items()}, "mean_ms_per_step": total / steps,
           "api": "svg2_driver_layer"}
    drv.close()
    return out


def time_own_dense(svg2, torch, Q, K, V, scale, reps=3):
    """This library's dense attention (the one-cluster case of the same tcgen05 kernel)."""
    B, H, N, d = Q.shape
    O = torch.empty_like(Q)
    ws = svg2.dense_workspace(B, H, N, d, device=Q.device)
    svg2.svg2_dense_attn(Q, K, V, scale, O, ws)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        svg2.svg2_dense_attn(Q, K, V, scale, O, ws)
    b.record()
    torch.cuda.synchronize()
    svg2.raise_on_device_error(ws)
    ms = a.elapsed_time(b) / reps
    flops = 4.0 * N * N * d * B * H
    return {"ms": ms, "tflops": flops / (ms * 1e-3) / 1e12}


def fixed128_waste(q_off, k_off, mask, heads):
    """Fraction of a fixed 128x128 block-sparse kernel's work that would be padding for the same
    kept cluster pairs (the pages' Fig. 7(b) comparison)."""
    act, fixed = 0.0, 0.0
    for h in heads:
        qo, ko, m = q_off[0, h], k_off[0, h], mask[0, h]
        nQ, nK = m.shape
        nb_q = (qo[-1] + 127) // 128
        nb_k = (ko[-1] + 127) // 128
        blocks = np.zeros((nb_q, nb_k), bool)
        for i in range(nQ):
            if qo[i + 1] == qo[i]:
                continue
            js = np.nonzero(m[i])[0]
            rq = slice(qo[i] // 128, (qo[i + 1] - 1) // 128 + 1)
            for j in js:
                if ko[j + 1] == ko[j]:
                    continue
                blocks[rq, ko[j] // 128:(ko[j + 1] - 1) // 128 + 1] = True
                act += float(qo[i + 1] - qo[i]) * float(ko[j + 1] - ko[j])
        fixed += float(blocks.sum()) * 128.0 * 128.0
    return 1.0 - act / fixed if fixed > 0 else None


def kernel_launches(cfg):
    per_role = 1 + 1 + cfg.iters * (2 + 3 + 1)   # k-means++, split prep, per iteration: assign + re-rank, 3 sort, update
    return 2 * per_role + 1 + 3 + 4               # select, 3 gathers, plan (3) + attention


if __name__ == "__main__":
    main()
