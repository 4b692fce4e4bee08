#!/usr/bin/env python
"""Throughput of the block-hybrid attention decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode|commit|sweep|cycle]

Default workload ("decode"): one denoising step of one block-hybrid layer for 128 requests
with 32-token active blocks, 16 query / 4 KV heads, head dim 128, feature dim 256 (W is
128 x 128 per KV head), each request's 1024-token prefix held only as fp32 states
S [4, 256, 128] and Z [4, 256]; bf16 activations ~ N(0, 1), W ~ N(0, 1/128), states built
by committing 32 random blocks through the library.  A step is one library call that runs
the whole fused decode step (feature map of the queries, block scores, block softmax,
cross-block state read, P.V and the shared-normaliser merge) for all 4096 block tokens.

Metric: tokens per second per denoise step (block tokens / step time), one JSON line on
rank 0.  Timing: W eager warm-up steps, then exactly K steps replayed from CUDA graphs,
bracketed by a barrier and a synchronize, timed with CUDA events on the launching stream,
max over ranks.  L2 is defeated by rotating 4 independent input/state sets (4 x 110 MB
against a 126 MB L2).  Multi-GPU runs are independent replicas (no collective on the path).

Other workloads print their own JSON line: "commit" (the block-commit update for 128
requests x 4 KV heads), "sweep" (the decode step vs the in-run full-prefix softmax teacher
at 64 requests over prefixes of 512..32768 tokens) and "cycle" (a ragged serving mix of 128
requests, 6 hybrid layers, 8 denoising steps then a commit, as one CUDA graph).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "hybrid-attn tokens/s per denoise step @128 reqs; % HBM roofline (1×B200)"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# decode-step workload
R, HQ, HKV, D, F, B, PREFIX = 128, 16, 4, 128, 256, 32, 1024
NSETS = 4


def step_bytes(R=R, Hq=HQ, Hkv=HKV, d=D, F=F, B=B):
    """Algorithmic HBM bytes of one decode step: Q, K, V, O once (bf16), S and Z once (fp32),
    W once per KV head (bf16).  phi, scores and partial sums never reach HBM."""
    G = Hq // Hkv
    per_unit = F * d * 4 + F * 4 + G * B * d * 2 + 2 * B * d * 2 + G * B * d * 2
    return R * Hkv * per_unit + Hkv * d * (F // 2) * 2


def step_flops(R=R, Hq=HQ, Hkv=HKV, d=D, F=F, B=B):
    """FLOPs of one decode step (2 per multiply-add): q.W, q.k, P.V, phi.S and phi.Z per query."""
    per_q = d * (F // 2) + B * d + B * d + F * d + F
    return 2 * R * Hq * B * per_q


def commit_bytes(R=R, Hkv=HKV, d=D, F=F, B=B):
    """S and Z read and written once (fp32), K and V of the block read once, W once."""
    return R * Hkv * (2 * F * d * 4 + 2 * F * 4 + 2 * B * d * 2) + Hkv * d * (F // 2) * 2


def teacher_bytes(R, Hq, Hkv, d, B, P):
    """Full-prefix softmax: Q and O once, the whole K/V cache (P + B tokens) once (bf16)."""
    return R * Hq * B * d * 2 * 2 + R * Hkv * (P + B) * d * 2 * 2


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def code_of(text):
    """Source text with comments and blank space removed, so that a capture recorded for a
    kernel stays valid across comment-only edits but not across code changes."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def source_hash(*names):
    h = hashlib.sha1()
    for n in names:
        with open(os.path.join(ROOT, "linear_attention_diffusion_hedgehog_b200", "csrc", n)) as f:
            h.update(code_of(f.read()).encode())
    return h.hexdigest()[:12]


def profiled_traffic(kernel_key, src_hash):
    """DRAM bytes per launch recorded by an ncu capture in profiles/, if the capture was
    taken of the current kernel source (same hash); else None."""
    pdir = os.path.join(ROOT, "profiles")
    if not os.path.isdir(pdir):
        return None
    pat = re.compile(r"^traffic\s+(\S+)\s+src=(\S+)\s+bytes_per_launch=(\d+)", re.M)
    for fn in sorted(os.listdir(pdir)):
        if not fn.endswith((".md", ".txt")):
            continue
        with open(os.path.join(pdir, fn)) as f:
            for m in pat.finditer(f.read()):
                if m.group(1) == kernel_key and m.group(2) == src_hash:
                    return int(m.group(3))
    return None


# ------------------------------------------------------------------ clocks sampler
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self):
        return time.time()

    def stop(self, t0, t1):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = [l for (ts, l) in self.lines if t0 - 0.05 <= ts <= t1 + 0.05] or \
               [l for (ts, l) in self.lines][-3:]
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in rows:
            p = [x.strip() for x in l.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                smax.append(float(p[2]))
            except ValueError:
                continue
            for n, v in zip(names, p[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ distributed plumbing
def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x, world, device="cuda"):
    """The largest of the ranks' values (each rank's device time); the job's time is the
    slowest rank's.  device is where the reduction tensor lives (cpu for gloo)."""
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank_step, steps, max_ms, world):
    """Units per second of the whole job: every rank processes units_per_rank_step units per
    step (independent replicas, weak scaling) and the job takes the slowest rank's time."""
    return units_per_rank_step * world * steps / (max_ms / 1e3)


# ------------------------------------------------------------------ graph timing
def time_graphed(fn_step, K, W, world, stream):
    """Run W eager warm-up steps, capture K steps into CUDA graphs (chunks of <= 512), replay
    once untimed, then time exactly K replayed steps.  fn_step(i) enqueues step i."""
    for i in range(W):
        fn_step(i)
    torch.cuda.synchronize()
    chunk = min(K, 512)
    graphs = []
    done = 0
    while done < K:
        n = min(chunk, K - done)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(done, done + n):
                fn_step(i)
        graphs.append(g)
        done += n
    for g in graphs:
        g.replay()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for g in graphs:
            g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = e0.elapsed_time(e1)
    del graphs
    return ms


# ------------------------------------------------------------------ workloads
def make_decode_sets(gen, nsets=NSETS, R=R, Hq=HQ, Hkv=HKV, d=D, F=F, B=B, prefix=PREFIX,
                     states_from_commits=True):
    from linear_attention_diffusion_hedgehog_b200 import bha

    dev = torch.device("cuda")
    bf = torch.bfloat16
    W = (torch.randn((Hkv, d, F // 2), generator=gen, device=dev) / d ** 0.5).to(bf)
    cu = torch.arange(0, (R + 1) * B, B, dtype=torch.int32, device=dev)
    S0 = torch.zeros((R, Hkv, F, d), device=dev)
    Z0 = torch.zeros((R, Hkv, F), device=dev)
    if states_from_commits and prefix > 0:
        for _ in range(prefix // B):
            Kb = torch.randn((R * B, Hkv, d), generator=gen, device=dev).to(bf)
            Vb = torch.randn((R * B, Hkv, d), generator=gen, device=dev).to(bf)
            bha.commit_block(cu, Kb, Vb, W, S0, Z0, max_block=B)
    sets = []
    for s in range(nsets):
        sets.append(dict(
            Q=torch.randn((R * B, Hq, d), generator=gen, device=dev).to(bf),
            K=torch.randn((R * B, Hkv, d), generator=gen, device=dev).to(bf),
            V=torch.randn((R * B, Hkv, d), generator=gen, device=dev).to(bf),
            S=S0.clone(), Z=Z0.clone(), O=torch.empty((R * B, Hq, d), device=dev, dtype=bf)))
    torch.cuda.synchronize()
    return W, cu, sets


def cpu_oracle_decode(budget_s, seed=0):
    """Time the float64 oracle on a bounded sample of the decode-step workload: whole
    requests (all 16 query heads, 32 block tokens) with directly drawn states, one request's
    computation repeated until about budget_s seconds of CPU work have run."""
    from linear_attention_diffusion_hedgehog_b200 import inputs
    from oracle import bha_ref as ref

    c = inputs.decode_case(R=1, Hq=HQ, Hkv=HKV, d=D, F=F, block_lens=B, prefix_lens=0, seed=seed)
    S, Z = inputs.random_states(1, HKV, F, D, PREFIX, seed=seed)
    S64, Z64 = S.astype(np.float64), Z.astype(np.float64)

    def one():
        ref.hybrid_attn(c.cu_blk, c.Q, c.K, c.V, S64, Z64, c.W)

    t = time.perf_counter()
    one()
    t1 = time.perf_counter() - t
    n = int(max(1, budget_s // max(t1, 1e-6)))
    t = time.perf_counter()
    for _ in range(n):
        one()
    el = time.perf_counter() - t
    try:
        import threadpoolctl

        cores = max(i.get("num_threads", 1) for i in threadpoolctl.threadpool_info()) or 1
    except Exception:  # noqa: BLE001
        cores = 1
    return n, el, cores


def bench_reference(args, world, rank):
    """The float64 CPU oracle as the reference arm: same metric and workload, each step a
    bounded sample (whole requests of the decode step) so the run stays within minutes."""
    if rank != 0:
        return
    from linear_attention_diffusion_hedgehog_b200 import inputs
    from oracle import bha_ref as ref

    c = inputs.decode_case(R=1, Hq=HQ, Hkv=HKV, d=D, F=F, block_lens=B, prefix_lens=0, seed=0)
    S, Z = inputs.random_states(1, HKV, F, D, PREFIX, seed=0)
    S64, Z64 = S.astype(np.float64), Z.astype(np.float64)

    def one_request():
        ref.hybrid_attn(c.cu_blk, c.Q, c.K, c.V, S64, Z64, c.W)

    t = time.perf_counter()
    one_request()
    t1 = time.perf_counter() - t
    budget = 150.0 / max(1, args.steps + args.warmup)
    per_step = int(max(1, min(R, budget // max(t1, 1e-6))))
    for _ in range(args.warmup):
        for _ in range(per_step):
            one_request()
    t = time.perf_counter()
    for _ in range(args.steps):
        for _ in range(per_step):
            one_request()
    el = time.perf_counter() - t
    tokens = args.steps * per_step * B
    value = tokens / el
    try:
        import threadpoolctl

        cores = max(i.get("num_threads", 1) for i in threadpoolctl.threadpool_info()) or 1
    except Exception:  # noqa: BLE001
        cores = 1
    sample = f"{per_step} of 128 requests per step (all 16 query heads, 32 block tokens each)"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": decode_config(),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def decode_config():
    return {"workload": "decode step, one layer: 128 requests x 32-token blocks, 16 query / 4 KV "
                        "heads, head dim 128, feature dim 256, fp32 states of 1024-token prefixes",
            "requests": R, "q_heads": HQ, "kv_heads": HKV, "head_dim": D, "feature_dim": F,
            "block": B, "prefix_tokens": PREFIX, "parallelism": "replicas",
            "l2": f"rotating {NSETS} independent input/state sets of ~110 MB each, together larger "
                  f"than the 126 MB L2"}


def bench_decode(args, world, rank, local):
    from linear_attention_diffusion_hedgehog_b200 import bha

    peaks, peak_src = load_peaks()
    gen = torch.Generator(device="cuda")
    gen.manual_seed(1234 + rank)
    W, cu, sets = make_decode_sets(gen)
    stream = torch.cuda.Stream()
    dims = bha.make_dims(R, HQ, HKV, D, F, B, R * B, R, torch.bfloat16)
    variant = bha.kernel_variant(dims, 1)

    def step(i):
        s = sets[i % NSETS]
        bha.hybrid_attn(cu, s["Q"], s["K"], s["V"], s["S"], s["Z"], W, max_block=B, out=s["O"],
                        stream=stream)

    sampler = ClockSampler(local)
    if rank == 0:
        sampler.start()
    torch.cuda.synchronize()
    t0 = time.time()
    ms = time_graphed(step, args.steps, args.warmup, world, stream)
    t1 = time.time()
    clocks = sampler.stop(t0, t1) if rank == 0 else None
    ms = max_over_ranks(ms, world)
    step_ms = ms / args.steps
    value = whole_job_rate(R * B, args.steps, ms, world)

    # end to end through the public API: pinned host Q/K/V in, O back to pinned host
    e2e_steps = min(args.steps, 200)
    hsets = [{k: sets[i][k].cpu().pin_memory() for k in ("Q", "K", "V")} for i in range(NSETS)]
    hout = torch.empty(sets[0]["O"].shape, dtype=torch.bfloat16).pin_memory()
    dQ = torch.empty_like(sets[0]["Q"])
    dK = torch.empty_like(sets[0]["K"])
    dV = torch.empty_like(sets[0]["V"])
    h2d = sum(hsets[0][k].numel() * 2 for k in ("Q", "K", "V"))
    d2h = hout.numel() * 2

    def e2e_step(i):
        s, h = sets[i % NSETS], hsets[i % NSETS]
        with torch.cuda.stream(stream):
            dQ.copy_(h["Q"], non_blocking=True)
            dK.copy_(h["K"], non_blocking=True)
            dV.copy_(h["V"], non_blocking=True)
            bha.hybrid_attn(cu, dQ, dK, dV, s["S"], s["Z"], W, max_block=B, out=s["O"],
                            stream=stream)
            hout.copy_(s["O"], non_blocking=True)

    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(e2e_steps):
        e2e_step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    e2e_value = whole_job_rate(R * B, e2e_steps, e2e_ms, world)

    if rank != 0:
        return
    nbytes = step_bytes()
    achieved = nbytes / (step_ms / 1e3) / 1e9
    peak = peaks["hbm_gbs"]
    src = source_hash("hybrid_tc.cu") if variant == 1 and os.path.exists(
        os.path.join(ROOT, "linear_attention_diffusion_hedgehog_b200", "csrc", "hybrid_tc.cu")) \
        else source_hash("simt.cu")
    traffic = profiled_traffic("hybrid_decode", src)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16",
        "precision": ("bf16 activations; fp32 states read as tf32 by the tensor cores; fp32 "
                      "accumulation" if variant == 1 else "bf16 activations; fp32 arithmetic"),
        "data": "synthetic", "config": decode_config(),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "peak_source": f"{peak_src} hbm_gbs",
                     "algorithmic_bytes_per_launch": nbytes, "flops_per_launch": step_flops(),
                     "kernel": "hybrid tensor-core" if variant == 1 else "hybrid generic"},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps},
        "gpu_launches": args.steps,
        "clocks": clocks,
        "kernel_variant": variant,
    }
    if world == 1 and not args.no_cpu_baseline:
        n, el, cores = cpu_oracle_decode(budget_s=12.0)
        line["cpu_baseline"] = {"value": n * B / el, "unit": UNIT, "cores": cores,
                                "kind": "oracle",
                                "sample": f"{n} whole requests of the decode step (16 query heads x "
                                          f"32 tokens, states given; one request repeated), "
                                          f"{el:.1f} s"}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ other workloads
def _line(metric, value, unit, args, world, ms_step, higher, config, **extra):
    d = {"metric": metric, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
         "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": higher,
         "scaling": "weak", "vs_baseline": None, "data": "synthetic", "config": config}
    d.update(extra)
    return d


def _roof(nbytes, ms, peaks, peak_src, kernel, flops=None, traffic=None):
    achieved = nbytes / (ms / 1e3) / 1e9
    r = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
         "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
         "peak_source": f"{peak_src} hbm_gbs", "algorithmic_bytes_per_launch": nbytes,
         "kernel": kernel}
    if flops is not None:
        r["flops_per_launch"] = flops
    return r


def bench_commit(args, world, rank, local):
    """Block commit for 128 requests x 4 KV heads (d 128, F 256, 32-token blocks): S and Z
    updated in place; 4 rotating state sets (75 MB each) keep L2 from holding them."""
    from linear_attention_diffusion_hedgehog_b200 import bha

    peaks, src = load_peaks()
    gen = torch.Generator(device="cuda")
    gen.manual_seed(99 + rank)
    dev, bf = torch.device("cuda"), torch.bfloat16
    W = (torch.randn((HKV, D, F // 2), generator=gen, device=dev) / D ** 0.5).to(bf)
    cu = torch.arange(0, (R + 1) * B, B, dtype=torch.int32, device=dev)
    sets = [dict(K=torch.randn((R * B, HKV, D), generator=gen, device=dev).to(bf),
                 V=torch.randn((R * B, HKV, D), generator=gen, device=dev).to(bf),
                 S=torch.randn((R, HKV, F, D), generator=gen, device=dev),
                 Z=torch.rand((R, HKV, F), generator=gen, device=dev) * 8) for _ in range(NSETS)]
    stream = torch.cuda.Stream()
    dims = bha.make_dims(R, HKV, HKV, D, F, B, R * B, R, bf)

    def step(i):
        s = sets[i % NSETS]
        bha.commit_block(cu, s["K"], s["V"], W, s["S"], s["Z"], max_block=B, stream=stream)

    ms = max_over_ranks(time_graphed(step, args.steps, args.warmup, world, stream), world)
    if rank == 0:
        ms_step = ms / args.steps
        cfg = {"workload": "block commit: fold a 32-token block into S/Z for 128 requests x 4 KV "
                           "heads, head dim 128, feature dim 256", "requests": R, "kv_heads": HKV,
               "head_dim": D, "feature_dim": F, "block": B,
               "l2": f"rotating {NSETS} state sets of ~75 MB each, together larger than the 126 MB L2"}
        print(json.dumps(_line("block-commit tokens/s (128 reqs x 4 KV heads)",
                               R * B * world / (ms_step / 1e3), UNIT, args, world, ms_step, True, cfg,
                               dtype="bf16", precision="bf16 activations; fp32 states and accumulation",
                               kernel_variant=bha.kernel_variant(dims, 2),
                               roofline=_roof(commit_bytes(), ms_step, peaks, src, "commit",
                                              flops=2 * R * HKV * B * (D * (F // 2) + F * D + F),
                                              traffic=profiled_traffic("commit", source_hash("commit_tc.cu"))
                                              if bha.kernel_variant(dims, 2) == 1 else None),
                               gpu_launches=args.steps)), flush=True)


def bench_featuremap(args, world, rank, local):
    """Standalone feature map phi(x) on the decode step's queries: x [4096, 16, 128] bf16 ->
    phi [4096, 16, 256] fp32, 4 KV-head weight matrices; 2 rotating sets (84 MB each)."""
    from linear_attention_diffusion_hedgehog_b200 import bha

    peaks, src = load_peaks()
    gen = torch.Generator(device="cuda")
    gen.manual_seed(7 + rank)
    dev, bf = torch.device("cuda"), torch.bfloat16
    W = (torch.randn((HKV, D, F // 2), generator=gen, device=dev) / D ** 0.5).to(bf)
    sets = [dict(x=torch.randn((R * B, HQ, D), generator=gen, device=dev).to(bf),
                 o=torch.empty((R * B, HQ, F), device=dev)) for _ in range(2)]
    stream = torch.cuda.Stream()

    def step(i):
        s = sets[i % 2]
        bha.featuremap(s["x"], W, out=s["o"], stream=stream)

    ms = max_over_ranks(time_graphed(step, args.steps, args.warmup, world, stream), world)
    if rank == 0:
        ms_step = ms / args.steps
        rows = R * B * HQ
        nbytes = rows * D * 2 + rows * F * 4 + HKV * D * (F // 2) * 2
        cfg = {"workload": "feature map phi(x) of 4096 tokens x 16 heads, head dim 128, feature dim "
                           "256, fp32 output", "tokens": R * B, "heads": HQ, "head_dim": D,
               "feature_dim": F, "l2": "2 rotating sets of ~84 MB each, together larger than the 126 MB L2"}
        print(json.dumps(_line("feature-map rows/s", rows * world / (ms_step / 1e3), "rows/s", args,
                               world, ms_step, True, cfg, dtype="bf16", precision="bf16 x and W; fp32 u and phi",
                               roofline=_roof(nbytes, ms_step, peaks, src, "featuremap",
                                              flops=2 * rows * D * (F // 2),
                                              traffic=profiled_traffic("featuremap",
                                                                       source_hash("featuremap_tc.cu"))),
                               gpu_launches=args.steps)), flush=True)


def bench_sweep(args, world, rank, local):
    """Decode step vs the full-prefix softmax teacher at 64 requests (16 query / 4 KV heads,
    head dim 128, 32-token blocks) over prefixes of 512 .. 32768 tokens.  The hybrid reads only
    the fixed-size states; the teacher reads a bf16 KV cache of prefix + block tokens."""
    from linear_attention_diffusion_hedgehog_b200 import bha

    peaks, src = load_peaks()
    dev, bf = torch.device("cuda"), torch.bfloat16
    Rs = 64
    gen = torch.Generator(device="cuda")
    gen.manual_seed(5 + rank)
    W, cu, hsets = make_decode_sets(gen, nsets=NSETS, R=Rs, prefix=0, states_from_commits=False)
    for s in hsets:
        s["S"].normal_(generator=gen)
        s["Z"].uniform_(0.5, 1.5, generator=gen)
    stream = torch.cuda.Stream()
    steps = args.steps

    def hstep(i):
        s = hsets[i % NSETS]
        bha.hybrid_attn(cu, s["Q"], s["K"], s["V"], s["S"], s["Z"], W, max_block=B, out=s["O"],
                        stream=stream)

    h_ms = max_over_ranks(time_graphed(hstep, steps, args.warmup, world, stream), world) / steps
    out = []
    for P in (512, 2048, 8192, 32768):
        L = P + B
        cap = L
        nsets = max(1, min(NSETS, int(np.ceil(400e6 / (Rs * HKV * L * D * 2 * 2)))))
        tsets = []
        for _ in range(nsets):
            Kc = torch.randn((Rs, HKV, cap, D), generator=gen, device=dev).to(bf)
            Vc = torch.randn((Rs, HKV, cap, D), generator=gen, device=dev).to(bf)
            tsets.append(dict(Kc=Kc, Vc=Vc, Q=hsets[0]["Q"], O=torch.empty_like(hsets[0]["O"])))
        kv_len = torch.full((Rs,), L, dtype=torch.int32, device=dev)
        ws_bytes = bha.full_prefix_workspace_bytes(Rs, HQ, HKV, D, B, Rs * B, cap)
        ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)

        def tstep(i):
            s = tsets[i % nsets]
            bha.full_prefix_attn(cu, kv_len, s["Q"], s["Kc"], s["Vc"], max_block=B, workspace=ws,
                                 out=s["O"], stream=stream)

        tsteps = max(3, min(steps, int(2e5 // max(P, 1))))
        t_ms = max_over_ranks(time_graphed(tstep, tsteps, args.warmup, world, stream), world) / tsteps
        del tsets
        torch.cuda.empty_cache()
        hb = step_bytes(R=Rs)
        tb = teacher_bytes(Rs, HQ, HKV, D, B, P)
        out.append({"prefix": P, "hybrid_ms": h_ms, "teacher_ms": t_ms, "speedup": t_ms / h_ms,
                    "hybrid_hbm_frac": hb / (h_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                    "teacher_hbm_frac": tb / (t_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                    "teacher_steps": tsteps})
    if rank == 0:
        cfg = {"workload": "hybrid decode step (states only) vs full-prefix softmax teacher, 64 "
                           "requests, 16 query / 4 KV heads, head dim 128, 32-token blocks",
               "requests": Rs, "prefixes": [o["prefix"] for o in out]}
        print(json.dumps(_line("hybrid vs teacher per-block latency over prefix length",
                               out[-1]["speedup"], "x (teacher/hybrid at 32K prefix)", args, world,
                               h_ms, True, cfg, dtype="bf16", sweep=out)), flush=True)


def bench_cycle(args, world, rank, local):
    """Ragged serving mix: 128 requests with prefix lengths uniform on {0, 32, ..., 8192},
    32-token blocks, 6 hybrid layers (16 query / 4 KV heads, head dim 128, F 256, independent
    W), 8 denoising steps per block then a commit of every layer, captured as one CUDA graph.
    A step of this workload is one whole block cycle."""
    from linear_attention_diffusion_hedgehog_b200 import bha, inputs

    peaks, src = load_peaks()
    dev, bf = torch.device("cuda"), torch.bfloat16
    layers, nsteps = 6, 8
    gen = torch.Generator(device="cuda")
    gen.manual_seed(11 + rank)
    plen = inputs.ragged_prefix_lengths(R, seed=5)
    cu = torch.arange(0, (R + 1) * B, B, dtype=torch.int32, device=dev)
    Ws = [(torch.randn((HKV, D, F // 2), generator=gen, device=dev) / D ** 0.5).to(bf)
          for _ in range(layers)]
    Ss = [torch.zeros((R, HKV, F, D), device=dev) for _ in range(layers)]
    Zs = [torch.zeros((R, HKV, F), device=dev) for _ in range(layers)]
    # prefix states: one commit call per 128-token slice of each request's prefix
    for l in range(layers):
        for j in range(0, int(plen.max()), 128):
            lens = np.clip(plen - j, 0, 128)
            if lens.sum() == 0:
                break
            cuj = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device=dev)
            T = int(lens.sum())
            Kb = torch.randn((T, HKV, D), generator=gen, device=dev).to(bf)
            Vb = torch.randn((T, HKV, D), generator=gen, device=dev).to(bf)
            bha.commit_block(cuj, Kb, Vb, Ws[l], Ss[l], Zs[l], max_block=128)
    acts = [[dict(Q=torch.randn((R * B, HQ, D), generator=gen, device=dev).to(bf),
                  K=torch.randn((R * B, HKV, D), generator=gen, device=dev).to(bf),
                  V=torch.randn((R * B, HKV, D), generator=gen, device=dev).to(bf))
             for _ in range(layers)] for _ in range(nsteps)]
    O = torch.empty((R * B, HQ, D), device=dev, dtype=bf)
    stream = torch.cuda.Stream()

    def cycle(i):
        for st in range(nsteps):
            for l in range(layers):
                a = acts[st][l]
                bha.hybrid_attn(cu, a["Q"], a["K"], a["V"], Ss[l], Zs[l], Ws[l], max_block=B,
                                out=O, stream=stream)
        for l in range(layers):
            a = acts[nsteps - 1][l]
            bha.commit_block(cu, a["K"], a["V"], Ws[l], Ss[l], Zs[l], max_block=B, stream=stream)

    ms = max_over_ranks(time_graphed(cycle, args.steps, args.warmup, world, stream), world)
    if rank == 0:
        ms_cycle = ms / args.steps
        nbytes = nsteps * layers * step_bytes() + layers * commit_bytes()
        cfg = {"workload": "ragged serving mix: 128 requests, prefixes uniform on {0,32,...,8192}, "
                           "32-token blocks, 6 hybrid layers, 8 denoising steps then a commit per "
                           "block cycle (one CUDA graph)", "requests": R, "layers": layers,
               "steps_per_block": nsteps, "prefix_mean": float(plen.mean())}
        print(json.dumps(_line("serving-cycle tokens/s per denoise step (6 hybrid layers)",
                               nsteps * R * B * world / (ms_cycle / 1e3), UNIT, args, world,
                               ms_cycle, True, cfg, dtype="bf16", precision="bf16 activations; fp32 states",
                               roofline=_roof(nbytes, ms_cycle, peaks, src, "block cycle"),
                               committed_tokens_per_s=R * B * world / (ms_cycle / 1e3),
                               gpu_launches=args.steps * (nsteps * layers + layers))), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["decode", "commit", "featuremap", "sweep", "cycle"],
                    default="decode")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    assert args.warmup >= 3, "at least 3 warm-up steps"
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        bench_reference(args, int(os.environ.get("WORLD_SIZE", "1")), rank)
        return
    world, rank, local = dist_setup(args.gpus)
    try:
        if args.workload == "decode":
            bench_decode(args, world, rank, local)
        else:
            {"commit": bench_commit, "featuremap": bench_featuremap, "sweep": bench_sweep,
             "cycle": bench_cycle}[args.workload](args, world, rank, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
