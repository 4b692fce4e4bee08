#!/usr/bin/env python
"""Throughput of the block-hybrid attention decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload all|decode|commit|fused|featuremap|per_qhead|sweep|cycle]

Headline workload ("decode"): one denoising step of one block-hybrid layer for 128 requests
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

The default run ("all") adds, under "workloads", one record per other workload, each timed
the same way with its own roofline: the gated decode step, the block commit (128 requests x
4 KV heads), the last step of a block fused with its commit, the standalone feature map, the per-query-head layout (16 state heads), the prefix sweep (decode step on states committed
from each prefix vs the in-run softmax teacher over the same cache, 64 requests, prefixes
512..32768, with the teacher's linear fit) and the serving cycle (ragged mix of 128 requests,
6 layers, 8 denoising steps then a commit, as one CUDA graph, and again with each layer's
last step fused with its commit), plus the state-vs-KV-cache
capacity figures.  --workload X runs one of them alone.
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


def commit_flops(R=R, Hkv=HKV, d=D, F=F, B=B):
    """FLOPs of one commit (2 per multiply-add): k.W, phi(k) v^T and the phi sum per token."""
    return 2 * R * Hkv * B * (d * (F // 2) + F * d + F)


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


def host_info():
    """CPU model, logical core count and the BLAS pool size the float64 oracle runs with."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    blas = None
    try:
        import threadpoolctl

        blas = max(i.get("num_threads", 1) for i in threadpoolctl.threadpool_info())
    except Exception:  # noqa: BLE001
        pass
    return {"cpu_model": model, "cpu_count": os.cpu_count(), "blas_threads": blas}


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
                         "sample": sample, **host_info()},
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


def _roof(nbytes, ms, peaks, peak_src, kernel, flops=None, traffic=None):
    achieved = nbytes / (ms / 1e3) / 1e9
    r = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
         "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
         "peak_source": f"{peak_src} hbm_gbs", "algorithmic_bytes_per_launch": nbytes,
         "kernel": kernel}
    if flops is not None:
        r["flops_per_launch"] = flops
    return r


def _record(metric, value, unit, steps, ms_step, config, **extra):
    d = {"metric": metric, "value": value, "unit": unit, "steps": steps, "ms_per_step": ms_step,
         "higher_is_better": True, "config": config}
    d.update(extra)
    return d


def _traffic_for(kernel_key, variant, src_file):
    return profiled_traffic(kernel_key, source_hash(src_file)) if variant == 1 else None


def e2e_pipelined(sets, cu, W, steps, world, stream, alpha=None):
    """Decode steps end to end through the public API with pinned host buffers: every step
    copies its Q, K, V host -> device, runs the step and copies O device -> host.  Three
    streams pipeline consecutive steps (step i+1's inputs go up while step i computes and step
    i-1's output comes down, so both PCIe directions run at once), with two device buffer sets
    and events ordering each reuse.  Returns (ms, h2d bytes, d2h bytes) per the whole run."""
    from linear_attention_diffusion_hedgehog_b200 import bha

    hsets = [{k: sets[i][k].cpu().pin_memory() for k in ("Q", "K", "V")} for i in range(len(sets))]
    dbuf = [{k: torch.empty_like(sets[0][k]) for k in ("Q", "K", "V", "O")} for _ in range(2)]
    hout = [torch.empty(sets[0]["O"].shape, dtype=sets[0]["O"].dtype).pin_memory() for _ in range(2)]
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def step(i):
        b, s, h = i % 2, sets[i % len(sets)], hsets[i % len(hsets)]
        with torch.cuda.stream(up):
            if i >= 2:
                up.wait_event(ev_done[b])      # step i-2 has read this buffer set
            for k in ("Q", "K", "V"):
                dbuf[b][k].copy_(h[k], non_blocking=True)
            ev_in[b].record(up)
        stream.wait_event(ev_in[b])
        if i >= 2:
            stream.wait_event(ev_out[b])       # step i-2's output has left this buffer
        bha.hybrid_attn(cu, dbuf[b]["Q"], dbuf[b]["K"], dbuf[b]["V"], s["S"], s["Z"], W,
                        max_block=B, alpha=alpha, out=dbuf[b]["O"], stream=stream)
        ev_done[b].record(stream)
        with torch.cuda.stream(down):
            down.wait_event(ev_done[b])
            hout[b].copy_(dbuf[b]["O"], non_blocking=True)
            ev_out[b].record(down)

    for i in range(4):
        step(i)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(up)
    for i in range(steps):
        step(i)
    down.wait_stream(stream)
    e1.record(down)
    torch.cuda.synchronize()
    barrier(world)
    h2d = sum(hsets[0][k].numel() * hsets[0][k].element_size() for k in ("Q", "K", "V"))
    d2h = hout[0].numel() * hout[0].element_size()
    return e0.elapsed_time(e1), h2d, d2h


def capacity_record(S, Z, Hkv=HKV, d=D, act_bytes=2):
    """State bytes of one request in one hybrid layer, from the state buffers themselves,
    against the KV cache the softmax teacher keeps for the same request (K and V per token)."""
    state = S[0].numel() * S.element_size() + Z[0].numel() * Z.element_size()
    kv_per_token = 2 * Hkv * d * act_bytes
    rec = {"state_bytes_per_request_layer": state, "kv_bytes_per_token_layer": kv_per_token,
           "break_even_prefix_tokens": state / kv_per_token}
    for P in (1024, 4096, 32768):
        rec[f"kv_over_state_at_{P}"] = P * kv_per_token / state
    return rec


def bench_decode(args, world, rank, local, gen):
    """The headline: one decode step of one layer, 128 requests (see the module docstring)."""
    from linear_attention_diffusion_hedgehog_b200 import bha

    peaks, peak_src = load_peaks()
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

    e2e_steps = min(args.steps, 200)
    e2e_ms, h2d, d2h = e2e_pipelined(sets, cu, W, e2e_steps, world, stream)
    e2e_ms = max_over_ranks(e2e_ms, world)
    e2e_value = whole_job_rate(R * B, e2e_steps, e2e_ms, world)

    # the same step with the sigmoid gate on (alpha ~ N(0, 1) per query head)
    alpha = torch.randn((HQ,), generator=gen, device="cuda")
    gsteps = min(args.steps, 2000)

    def gstep(i):
        s = sets[i % NSETS]
        bha.hybrid_attn(cu, s["Q"], s["K"], s["V"], s["S"], s["Z"], W, max_block=B, alpha=alpha,
                        out=s["O"], stream=stream)

    g_ms = max_over_ranks(time_graphed(gstep, gsteps, args.warmup, world, stream), world) / gsteps
    src = "hybrid_tc.cu" if variant == 1 else "simt.cu"
    nbytes = step_bytes() + HQ * 4
    gated = _record("hybrid-attn tokens/s per denoise step, gated merge (alpha ~ N(0,1))",
                    whole_job_rate(R * B, gsteps, g_ms * gsteps, world), UNIT, gsteps, g_ms,
                    dict(decode_config(), gate="alpha ~ N(0, 1) per query head"),
                    roofline=_roof(nbytes, g_ms, peaks, peak_src, "hybrid tensor-core" if variant == 1
                                   else "hybrid generic", flops=step_flops()),
                    gpu_launches=gsteps)
    capacity = capacity_record(sets[0]["S"], sets[0]["Z"])
    del sets
    torch.cuda.empty_cache()
    if rank != 0:
        return None
    nbytes = step_bytes()
    achieved = nbytes / (step_ms / 1e3) / 1e9
    peak = peaks["hbm_gbs"]
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16",
        "precision": ("bf16 activations; fp32 states read as tf32 by the tensor cores; fp32 "
                      "accumulation" if variant == 1 else "bf16 activations; fp32 arithmetic"),
        "data": "synthetic", "config": decode_config(),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": _traffic_for("hybrid_decode", variant, src),
                     "peak_source": f"{peak_src} hbm_gbs",
                     "algorithmic_bytes_per_launch": nbytes, "flops_per_launch": step_flops(),
                     "kernel": "hybrid tensor-core" if variant == 1 else "hybrid generic"},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "pipelining": "3 streams: next step's H2D and previous step's D2H overlap this "
                              "step's kernel"},
        "gpu_launches": args.steps,
        "clocks": clocks,
        "kernel_variant": variant,
        "workloads": {"decode_gated": gated, "capacity": capacity},
    }
    if world == 1 and not args.no_cpu_baseline:
        n, el, cores = cpu_oracle_decode(budget_s=12.0)
        line["cpu_baseline"] = {"value": n * B / el, "unit": UNIT, "cores": cores,
                                "kind": "oracle",
                                "sample": f"{n} whole requests of the decode step (16 query heads x "
                                          f"32 tokens, states given; one request repeated), "
                                          f"{el:.1f} s", **host_info()}
    return line


def bench_commit(args, world, rank, local, steps, block=B):
    """Block commit for 128 requests x 4 KV heads (d 128, F 256, `block`-token blocks: 32, the
    serving shape, or 128, the large-block variant whose contractions are 4x deeper): S and Z
    updated in place; 4 rotating state sets (75 MB and more each) keep L2 from holding them."""
    from linear_attention_diffusion_hedgehog_b200 import bha

    peaks, src = load_peaks()
    gen = torch.Generator(device="cuda")
    gen.manual_seed(99 + rank)
    dev, bf = torch.device("cuda"), torch.bfloat16
    W = (torch.randn((HKV, D, F // 2), generator=gen, device=dev) / D ** 0.5).to(bf)
    cu = torch.arange(0, (R + 1) * block, block, dtype=torch.int32, device=dev)
    sets = [dict(K=torch.randn((R * block, HKV, D), generator=gen, device=dev).to(bf),
                 V=torch.randn((R * block, HKV, D), generator=gen, device=dev).to(bf),
                 S=torch.randn((R, HKV, F, D), generator=gen, device=dev),
                 Z=torch.rand((R, HKV, F), generator=gen, device=dev) * 8) for _ in range(NSETS)]
    stream = torch.cuda.Stream()
    dims = bha.make_dims(R, HKV, HKV, D, F, block, R * block, R, bf)
    variant = bha.kernel_variant(dims, 2)

    def step(i):
        s = sets[i % NSETS]
        bha.commit_block(cu, s["K"], s["V"], W, s["S"], s["Z"], max_block=block, stream=stream)

    ms = max_over_ranks(time_graphed(step, steps, args.warmup, world, stream), world)
    del sets
    torch.cuda.empty_cache()
    ms_step = ms / steps
    cfg = {"workload": f"block commit: fold a {block}-token block into S/Z for 128 requests x 4 KV "
                       "heads, head dim 128, feature dim 256", "requests": R, "kv_heads": HKV,
           "head_dim": D, "feature_dim": F, "block": block,
           "l2": f"rotating {NSETS} state sets of ~{commit_bytes(B=block) / 2 / 1e6:.0f} MB each, "
                 "together larger than the 126 MB L2"}
    key = "commit" if block == B else f"commit_b{block}"
    return _record(f"block-commit tokens/s (128 reqs x 4 KV heads, {block}-token blocks)",
                   whole_job_rate(R * block, steps, ms, world),
                   UNIT, steps, ms_step, cfg, dtype="bf16",
                   precision="bf16 activations; fp32 states and accumulation", kernel_variant=variant,
                   roofline=_roof(commit_bytes(B=block), ms_step, peaks, src, "commit",
                                  flops=commit_flops(B=block),
                                  traffic=_traffic_for(key, variant, "commit_tc.cu")),
                   gpu_launches=steps)


def bench_commit_b128(args, world, rank, local, steps):
    """The large-block variant of the commit: 128-token blocks (one request per 128-row tile,
    dS^T contracted over 128 tokens)."""
    return bench_commit(args, world, rank, local, steps, block=128)


def bench_featuremap(args, world, rank, local, steps):
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

    ms = max_over_ranks(time_graphed(step, steps, args.warmup, world, stream), world)
    del sets
    torch.cuda.empty_cache()
    ms_step = ms / steps
    rows = R * B * HQ
    nbytes = rows * D * 2 + rows * F * 4 + HKV * D * (F // 2) * 2
    cfg = {"workload": "feature map phi(x) of 4096 tokens x 16 heads, head dim 128, feature dim "
                       "256, fp32 output", "tokens": R * B, "heads": HQ, "head_dim": D,
           "feature_dim": F, "l2": "2 rotating sets of ~84 MB each, together larger than the 126 MB L2"}
    return _record("feature-map rows/s", whole_job_rate(rows, steps, ms, world), "rows/s", steps,
                   ms_step, cfg, dtype="bf16", precision="bf16 x and W; fp32 u and phi",
                   roofline=_roof(nbytes, ms_step, peaks, src, "featuremap", flops=2 * rows * D * (F // 2),
                                  traffic=_traffic_for("featuremap", 1, "featuremap_tc.cu")),
                   gpu_launches=steps)


def fused_bytes(R=R, Hq=HQ, Hkv=HKV, d=D, F=F, B=B):
    """The last step of a block fused with its commit: the decode step's bytes plus S and Z
    written back once (the commit's K, V and W are the step's own, already counted)."""
    return step_bytes(R, Hq, Hkv, d, F, B) + R * Hkv * (F * d * 4 + F * 4)


def bench_fused(args, world, rank, local, steps):
    """The last denoising step of a block fused with its commit (one call), at the decode
    step's shape: 128 requests, 16 query / 4 KV heads, 32-token blocks; S and Z updated in
    place, 4 rotating sets."""
    from linear_attention_diffusion_hedgehog_b200 import bha

    peaks, src = load_peaks()
    gen = torch.Generator(device="cuda")
    gen.manual_seed(29 + rank)
    W, cu, sets = make_decode_sets(gen)
    stream = torch.cuda.Stream()
    dims = bha.make_dims(R, HQ, HKV, D, F, B, R * B, R, torch.bfloat16)
    variant = bha.kernel_variant(dims, 4)

    def step(i):
        s = sets[i % NSETS]
        bha.hybrid_attn_commit(cu, s["Q"], s["K"], s["V"], s["S"], s["Z"], W, max_block=B,
                               out=s["O"], stream=stream)

    ms = max_over_ranks(time_graphed(step, steps, args.warmup, world, stream), world)
    del sets
    torch.cuda.empty_cache()
    ms_step = ms / steps
    cfg = dict(decode_config(), workload="last denoising step of a block fused with its commit: 128 "
               "requests x 32-token blocks, 16 query / 4 KV heads, head dim 128, feature dim 256; "
               "S and Z updated in place")
    return _record("block-end step + commit tokens/s (128 reqs)", whole_job_rate(R * B, steps, ms, world),
                   UNIT, steps, ms_step, cfg, dtype="bf16", kernel_variant=variant,
                   separate_calls_bytes=step_bytes() + commit_bytes(),
                   roofline=_roof(fused_bytes(), ms_step, peaks, src,
                                  "hybrid + commit tensor-core" if variant == 1 else "generic",
                                  traffic=_traffic_for("fused", variant, "hybrid_commit_tc.cu")),
                   gpu_launches=steps)


def linear_fit(xs, ys):
    """Least-squares y = a + b x and its coefficient of determination R^2."""
    xs, ys = np.asarray(xs, np.float64), np.asarray(ys, np.float64)
    b, a = np.polyfit(xs, ys, 1)
    pred = a + b * xs
    ss_res = float(((ys - pred) ** 2).sum())
    ss_tot = float(((ys - ys.mean()) ** 2).sum())
    return float(a), float(b), 1.0 - ss_res / ss_tot if ss_tot > 0 else 1.0


def bench_sweep(args, world, rank, local, steps):
    """Decode step vs the full-prefix softmax teacher at 64 requests (16 query / 4 KV heads,
    head dim 128, 32-token blocks) over prefixes of 512 .. 32768 tokens.  At each prefix length
    one KV cache of prefix + block tokens is drawn; the hybrid's states are committed from that
    cache's prefix tokens (32 at a time, through the library) and the block's own K/V are the
    cache's last 32 rows, so both kernels see the same request; each is timed at that prefix."""
    from linear_attention_diffusion_hedgehog_b200 import bha

    peaks, src = load_peaks()
    dev, bf = torch.device("cuda"), torch.bfloat16
    Rs = 64
    gen = torch.Generator(device="cuda")
    gen.manual_seed(5 + rank)
    W = (torch.randn((HKV, D, F // 2), generator=gen, device=dev) / D ** 0.5).to(bf)
    cu = torch.arange(0, (Rs + 1) * B, B, dtype=torch.int32, device=dev)
    stream = torch.cuda.Stream()
    out = []
    for P in (512, 2048, 8192, 32768):
        L = P + B
        Kc = torch.randn((Rs, HKV, L, D), generator=gen, device=dev).to(bf)
        Vc = torch.randn((Rs, HKV, L, D), generator=gen, device=dev).to(bf)
        S = torch.zeros((Rs, HKV, F, D), device=dev)
        Z = torch.zeros((Rs, HKV, F), device=dev)
        for j in range(0, P, B):
            bha.commit_block(cu, Kc[:, :, j:j + B].transpose(1, 2).reshape(Rs * B, HKV, D).contiguous(),
                             Vc[:, :, j:j + B].transpose(1, 2).reshape(Rs * B, HKV, D).contiguous(),
                             W, S, Z, max_block=B)
        Kb = Kc[:, :, P:L].transpose(1, 2).reshape(Rs * B, HKV, D).contiguous()
        Vb = Vc[:, :, P:L].transpose(1, 2).reshape(Rs * B, HKV, D).contiguous()
        hsets = [dict(Q=torch.randn((Rs * B, HQ, D), generator=gen, device=dev).to(bf), K=Kb.clone(),
                      V=Vb.clone(), S=S.clone(), Z=Z.clone(),
                      O=torch.empty((Rs * B, HQ, D), device=dev, dtype=bf)) for _ in range(NSETS)]

        def hstep(i):
            s = hsets[i % NSETS]
            bha.hybrid_attn(cu, s["Q"], s["K"], s["V"], s["S"], s["Z"], W, max_block=B, out=s["O"],
                            stream=stream)

        h_ms = max_over_ranks(time_graphed(hstep, steps, args.warmup, world, stream), world) / steps
        kv_len = torch.full((Rs,), L, dtype=torch.int32, device=dev)
        ws_bytes = bha.full_prefix_workspace_bytes(Rs, HQ, HKV, D, B, Rs * B, L)
        ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
        nsets = max(1, min(NSETS, int(np.ceil(400e6 / (Rs * HKV * L * D * 2 * 2)))))
        tsets = [dict(Kc=Kc, Vc=Vc)] + [dict(Kc=Kc.clone(), Vc=Vc.clone()) for _ in range(nsets - 1)]
        tO = torch.empty((Rs * B, HQ, D), device=dev, dtype=bf)

        def tstep(i):
            s = tsets[i % nsets]
            bha.full_prefix_attn(cu, kv_len, hsets[i % NSETS]["Q"], s["Kc"], s["Vc"], max_block=B,
                                 workspace=ws, out=tO, stream=stream)

        tsteps = max(3, min(steps, int(2e5 // max(P, 1))))
        t_ms = max_over_ranks(time_graphed(tstep, tsteps, args.warmup, world, stream), world) / tsteps
        del tsets, hsets, Kc, Vc, S, Z
        torch.cuda.empty_cache()
        hb = step_bytes(R=Rs)
        tb = teacher_bytes(Rs, HQ, HKV, D, B, P)
        out.append({"prefix": P, "hybrid_ms": h_ms, "teacher_ms": t_ms, "speedup": t_ms / h_ms,
                    "hybrid_hbm_frac": hb / (h_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                    "teacher_hbm_frac": tb / (t_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                    "hybrid_steps": steps, "teacher_steps": tsteps})
    hs = [o["hybrid_ms"] for o in out]
    a, b, r2 = linear_fit([o["prefix"] for o in out], [o["teacher_ms"] for o in out])
    cfg = {"workload": "hybrid decode step (states committed from each prefix) vs full-prefix softmax "
                       "teacher over the same cache, 64 requests, 16 query / 4 KV heads, head dim 128, "
                       "32-token blocks", "requests": Rs, "prefixes": [o["prefix"] for o in out],
           "l2": "hybrid: 4 rotating state sets (55 MB each); teacher: caches of 88 MB to 4.3 GB, "
                 "rotated up to 400 MB"}
    return _record("hybrid vs teacher per-block latency over prefix length", out[-1]["speedup"],
                   "x (teacher/hybrid at 32K prefix)", steps, float(np.mean(hs)), cfg, dtype="bf16",
                   sweep=out,
                   hybrid_spread=(max(hs) - min(hs)) / float(np.mean(hs)),
                   teacher_fit={"a_ms": a, "b_ms_per_prefix_token": b, "r2": r2},
                   roofline=_roof(step_bytes(R=Rs), float(np.mean(hs)), peaks, src,
                                  "hybrid tensor-core (64 requests, mean over the prefixes)"),
                   gpu_launches=steps * len(out) + sum(o["teacher_steps"] for o in out))


def bench_cycle(args, world, rank, local, steps):
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

    def cycle_fused(i):
        # the same cycle with each layer's last step and commit in one call
        for st in range(nsteps):
            for l in range(layers):
                a = acts[st][l]
                if st < nsteps - 1:
                    bha.hybrid_attn(cu, a["Q"], a["K"], a["V"], Ss[l], Zs[l], Ws[l], max_block=B,
                                    out=O, stream=stream)
                else:
                    bha.hybrid_attn_commit(cu, a["Q"], a["K"], a["V"], Ss[l], Zs[l], Ws[l],
                                           max_block=B, out=O, stream=stream)

    ms = max_over_ranks(time_graphed(cycle, steps, args.warmup, world, stream), world)
    ms_fused = max_over_ranks(time_graphed(cycle_fused, steps, args.warmup, world, stream), world)
    del acts, Ss, Zs
    torch.cuda.empty_cache()
    ms_cycle = ms / steps
    ms_cycle_fused = ms_fused / steps
    nbytes = nsteps * layers * step_bytes() + layers * commit_bytes()
    nbytes_fused = (nsteps - 1) * layers * step_bytes() + layers * fused_bytes()
    fused = {"ms_per_cycle": ms_cycle_fused,
             "tokens_per_s_per_step": whole_job_rate(nsteps * R * B, steps, ms_fused, world),
             "roofline": _roof(nbytes_fused, ms_cycle_fused, peaks, src,
                               "block cycle, last step fused with the commit"),
             "gpu_launches": steps * nsteps * layers}
    cfg = {"workload": "ragged serving mix: 128 requests, prefixes uniform on {0,32,...,8192}, "
                       "32-token blocks, 6 hybrid layers, 8 denoising steps then a commit per "
                       "block cycle (one CUDA graph)", "requests": R, "layers": layers,
           "steps_per_block": nsteps, "prefix_mean": float(plen.mean())}
    return _record("serving-cycle tokens/s per denoise step (6 hybrid layers)",
                   whole_job_rate(nsteps * R * B, steps, ms, world), UNIT, steps, ms_cycle, cfg,
                   dtype="bf16", precision="bf16 activations; fp32 states",
                   roofline=_roof(nbytes, ms_cycle, peaks, src, "block cycle"),
                   committed_tokens_per_s=whole_job_rate(R * B, steps, ms, world),
                   fused_last_step=fused,
                   gpu_launches=steps * (nsteps * layers + layers))


def bench_per_qhead(args, world, rank, local, steps):
    """The decode step in the per-query-head layout (a W and a state per query head: 16 query
    and 16 state heads), 128 requests, 32-token blocks, fp32 states of 1024-token prefixes
    built through the library: four times the state bytes of the grouped layout."""
    from linear_attention_diffusion_hedgehog_b200 import bha

    peaks, src = load_peaks()
    gen = torch.Generator(device="cuda")
    gen.manual_seed(23 + rank)
    W, cu, sets = make_decode_sets(gen, nsets=NSETS, Hkv=HQ)
    stream = torch.cuda.Stream()
    dims = bha.make_dims(R, HQ, HQ, D, F, B, R * B, R, torch.bfloat16)
    variant = bha.kernel_variant(dims, 1)

    def step(i):
        s = sets[i % NSETS]
        bha.hybrid_attn(cu, s["Q"], s["K"], s["V"], s["S"], s["Z"], W, max_block=B, out=s["O"],
                        stream=stream)

    ms = max_over_ranks(time_graphed(step, steps, args.warmup, world, stream), world)
    del sets
    torch.cuda.empty_cache()
    ms_step = ms / steps
    cfg = dict(decode_config(), workload="decode step, per-query-head layout: 128 requests x 32-token "
               "blocks, 16 query heads each with its own W and fp32 state (16 state heads), head dim "
               "128, feature dim 256, states of 1024-token prefixes", kv_heads=HQ,
               l2=f"rotating {NSETS} input/state sets of ~340 MB each")
    return _record("hybrid-attn tokens/s per denoise step, per-query-head states", whole_job_rate(R * B, steps, ms, world),
                   UNIT, steps, ms_step, cfg, dtype="bf16", kernel_variant=variant,
                   roofline=_roof(step_bytes(Hkv=HQ), ms_step, peaks, src,
                                  "hybrid tensor-core" if variant == 1 else "hybrid generic",
                                  flops=step_flops(Hkv=HQ),
                                  traffic=_traffic_for("hybrid_per_qhead", variant, "hybrid_tc.cu")),
                   gpu_launches=steps)


SUB_STEPS = {"commit": 1000, "commit_b128": 1000, "fused": 1000, "featuremap": 1000,
             "per_qhead": 1000, "sweep": 500, "cycle": 50}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["all", "decode", "commit", "commit_b128", "fused", "featuremap",
                                           "per_qhead", "sweep", "cycle"],
                    default="all")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    assert args.warmup >= 3, "at least 3 warm-up steps"
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        bench_reference(args, int(os.environ.get("WORLD_SIZE", "1")), rank)
        return
    world, rank, local = dist_setup(args.gpus)
    subs = {"commit": bench_commit, "commit_b128": bench_commit_b128, "fused": bench_fused,
            "featuremap": bench_featuremap, "per_qhead": bench_per_qhead, "sweep": bench_sweep,
            "cycle": bench_cycle}
    try:
        if args.workload in subs:
            rec = subs[args.workload](args, world, rank, local, args.steps)
            if rank == 0:
                rec.update({"n_gpus": world, "warmup": args.warmup, "scaling": "weak",
                            "vs_baseline": None, "data": "synthetic"})
                print(json.dumps(rec), flush=True)
            return
        gen = torch.Generator(device="cuda")
        gen.manual_seed(1234 + rank)
        line = bench_decode(args, world, rank, local, gen)
        if args.workload == "all":
            for name, fn in subs.items():
                rec = fn(args, world, rank, local, min(args.steps, SUB_STEPS[name]))
                if rank == 0:
                    line["workloads"][name] = rec
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
