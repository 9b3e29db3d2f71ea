#!/usr/bin/env python
"""Benchmark of the tree verification step on B200.

A step is one pass of the whole hot path over one batch of synthetic inputs:
tree_build_mask, tree_attention over every layer of the workload (distinct
per-layer buffers), tree_accept and kv_commit_realign.  Default workload:
single-sequence 7B-like verify (batch 1, 32 q / 32 kv heads, head dim 128,
prefix 2048, 65-row tree of depth <= 6, vocab 32000, 32 layers).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl reference]

Prints one JSON line (rank 0).  For N > 1 launch with torchrun: every rank runs
an independent replica (the sequences of the step are independent; there is no
exchange step), timing is the maximum over ranks and the value counts the work
of all ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "verified tree nodes/sec + KV-commit GB/s on 1 B200; fraction of roofline"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attention_traffic.json")
# the sources of the tensor-core attention kernel: its traffic figure holds only
# for the exact sources it was measured on
ATTN_SRCS = [os.path.join(ROOT, "tree_speculative_decoding_04_b200", "csrc", f)
             for f in ("attention_tc.cu", "attention_common.cuh", "tv_common.cuh", "attention.cu")]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="mha7b", choices=list(W.CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=20.0, help="CPU work budget of the oracle baseline sample")
    ap.add_argument("--layers", type=int, default=0, help="override the layer count (profiling runs only)")
    ap.add_argument("--no-e2e", action="store_true")
    return ap.parse_args()


# ----------------------------------------------------------------------------- distributed plumbing

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x, world, device):
    """The largest x over all ranks (device: where the reduction tensor lives --
    the rank's GPU under NCCL, the CPU under gloo)."""
    if world == 1:
        return x
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world, units_per_rank, ms_total_max, steps):
    """Units per second over all ranks: every rank did the same work, the job
    took as long as the slowest rank."""
    return world * units_per_rank / (ms_total_max / steps * 1e-3)


def config_dict(cfg, world, kv_len):
    return {"workload": f"{cfg.name}: {W.describe(cfg)}", "global_batch": cfg.B * world,
            "prefix": cfg.prefix, "tree_rows": cfg.M + 1, "layers": cfg.L, "parallelism": f"replicas x{world}",
            "l2": "inputs larger than L2: every step streams %.2f GB of distinct per-layer KV" %
                  (cfg.L * attention_bytes(cfg, kv_len) / 1e9),
            "timing": "CUDA graph of one step replayed K times; CUDA events on the launching stream"}


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, device):
        self.samples, self.reasons, self.ok = [], 0, False
        self._stop = threading.Event()
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _sample(self):
        self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
        try:
            self.reasons |= self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            self.reasons |= self.nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self._sample()
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()
            self._sample()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        names = [v for k, v in self.REASONS.items() if self.reasons & k and k != 0x1]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


# ----------------------------------------------------------------------------- inputs

def build_workload(cfg, seed, device):
    """A TreeVerifier holding a seeded synthetic step of the workload."""
    from tree_speculative_decoding_04_b200.verifier import TreeVerifier

    rng = np.random.default_rng(seed)
    parent = W.make_parents(cfg, rng)
    P = W.make_prefix_lengths(cfg, rng)
    ks, kl, S_cap = W.cache_geometry(cfg, P)
    ver = TreeVerifier(cfg.B, cfg.M, cfg.Hq, cfg.Hkv, cfg.D, cfg.V, cfg.L, S_cap, cfg.max_depth,
                       realign=cfg.left_padded, device=device)
    g = W.torch_generator(seed, device)
    for layer in range(cfg.L):
        ver.q[layer].copy_(W.randn_bf16(ver.q[layer].shape, g, device))
        ver.k[layer].copy_(W.randn_bf16(ver.k[layer].shape, g, device))
        ver.v[layer].copy_(W.randn_bf16(ver.v[layer].shape, g, device))
    ver.logits.copy_(W.randn_f32(ver.logits.shape, g, device, cfg.logit_sigma))
    draft = W.plant_drafts(ver.logits, parent, cfg.p_plant, rng)
    ver.parent.copy_(torch.as_tensor(parent))
    ver.draft.copy_(torch.as_tensor(draft))
    ver.kv_start.copy_(torch.as_tensor(ks))
    ver.kv_len.copy_(torch.as_tensor(kl))
    host = dict(parent=parent, draft=draft, P=P, kv_start=ks, kv_len=kl, S_cap=S_cap)
    return ver, host


def attention_bytes(cfg, kv_len):
    """Algorithmic bytes of one tree_attention launch: every key/value row of every
    sequence's range once (prefix + M+1 tree rows), q in and out once."""
    kv = sum(cfg.Hkv * (int(p) + cfg.M + 1) * cfg.D * 2 * 2 for p in kv_len)
    qo = cfg.B * (cfg.M + 1) * cfg.Hq * cfg.D * 2 * 2
    return kv + qo


def attention_flops(cfg, kv_len, depth):
    pre = sum(4 * cfg.D * cfg.Hq * (cfg.M + 1) * int(p) for p in kv_len)
    tree = int(4 * cfg.D * cfg.Hq * (depth + 1).sum())
    return pre + tree


def commit_bytes(cfg, path, accept_len, kv_len, realign, shift):
    """Algorithmic bytes of kv_commit_realign: rows that must move, read + write."""
    row = cfg.D * 2
    total = 0
    for b in range(cfg.B):
        a = int(accept_len[b])
        if realign and shift[b] != 0:
            total += cfg.L * cfg.Hkv * 2 * (int(kv_len[b]) + max(a, -1) + 1) * row * 2
        elif a >= 0:
            moved = sum(1 for j in range(a + 1) if int(path[b, j]) != j)
            total += cfg.L * cfg.Hkv * 2 * moved * row * 2
    return total


def event_time(fn, reps, stream):
    """Mean device time (ms) of fn(), launched on `stream`, over reps back-to-back calls."""
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
    e1.synchronize()
    return e0.elapsed_time(e1) / reps


def capture(fn, stream):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    torch.cuda.synchronize()
    return g


def attention_source_sha256():
    h = hashlib.sha256()
    for path in ATTN_SRCS:
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def read_traffic(workload):
    """DRAM bytes per attention launch from the committed ncu summary, only for the
    workload it was captured on and only if the kernel sources have not changed
    since the counters were taken."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
        sha = attention_source_sha256()
        if rec.get("source_sha256") == sha and rec.get("workload") == workload:
            return rec
    except Exception:
        pass
    return None


def roofline_entry(a_bytes, a_flops, attn_ms, hbm, tflops, peak_kind, traffic, kernel):
    """Roofline of one attention launch: roofline time = max(bytes / bandwidth,
    flops / tensor peak); the larger term names the bound, and achieved / peak
    are given in that term's unit."""
    attn_s = attn_ms * 1e-3
    tensor_bound = a_flops / (tflops * 1e12) > a_bytes / (hbm * 1e9)
    r = {
        "bound": "tensor" if tensor_bound else "hbm",
        "kernel": kernel,
        "achieved": a_flops / attn_s / 1e12 if tensor_bound else a_bytes / attn_s / 1e9,
        "peak": tflops if tensor_bound else hbm,
        "unit": "TFLOP/s" if tensor_bound else "GB/s",
        "peak_kind": f"{peak_kind} sustained bf16 GEMM" if tensor_bound else f"{peak_kind} copy bandwidth",
        "traffic": traffic,
        "algorithmic_bytes_per_launch": a_bytes, "algorithmic_flops_per_launch": a_flops, "launch_us": attn_ms * 1e3,
        "hbm_gbs": a_bytes / attn_s / 1e9, "tensor_tflops": a_flops / attn_s / 1e12,
    }
    r["frac"] = r["achieved"] / r["peak"]
    return r


def peaks():
    """(HBM copy GB/s, sustained bf16 TFLOP/s, "measured" | "fallback").  The
    attention launches are timed inside a long step, so a tensor-bound launch is
    held to the sustained GEMM figure."""
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p["hbm_gbs"], p.get("bf16_tflops_sustained", p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1400.0, "fallback"


# ----------------------------------------------------------------------------- CPU oracle baseline

def cpu_oracle_step(cfg, ver, host, layers, rows_frac=1.0, rng=None):
    """Time the oracle on a bounded sample of one step: the mask, attention on
    `layers` layers (optionally a fraction of the rows), accept and the commit
    of those layers.  Returns (seconds for the full step, by scaling, description)."""
    import oracle

    oracle.build()
    t_mask0 = time.perf_counter()
    anc, depth, st = oracle.tree_build_mask(host["parent"], cfg.max_depth)
    t_mask = time.perf_counter() - t_mask0
    ks, kl = host["kv_start"], host["kv_len"]
    t_attn = 0.0
    n_rows_total = cfg.B * (cfg.M + 1) * cfg.Hq
    for layer in range(layers):
        q = W.bf16_bits(ver.q[layer])
        k = W.bf16_bits(ver.k[layer])
        v = W.bf16_bits(ver.v[layer])
        if rows_frac >= 1.0:
            t0 = time.perf_counter()
            oracle.tree_attention(q, k, v, ks, kl, host["parent"], st, cfg.Hkv)
            t_attn += time.perf_counter() - t0
        else:
            nsel = max(1, int(round(rows_frac * n_rows_total)))
            sel = np.stack([rng.integers(cfg.B, size=nsel), rng.integers(cfg.M + 1, size=nsel),
                            rng.integers(cfg.Hq, size=nsel)], axis=1).astype(np.int32)
            t0 = time.perf_counter()
            oracle.tree_attention_rows(q, k, v, ks, kl, host["parent"], st, cfg.Hkv, sel)
            t_attn += (time.perf_counter() - t0) * n_rows_total / nsel
    logits = ver.logits.cpu().numpy()
    t0 = time.perf_counter()
    am, al, path, bonus = oracle.tree_accept(logits, host["draft"], host["parent"], st, cfg.max_depth)
    t_acc = time.perf_counter() - t0
    kh = [W.bf16_bits(ver.k[l]).copy() for l in range(layers)]
    vh = [W.bf16_bits(ver.v[l]).copy() for l in range(layers)]
    t0 = time.perf_counter()
    oracle.kv_commit_realign(kh, vh, cfg.M, path, al, st, cfg.max_depth, ks, kl, int(cfg.left_padded))
    t_com = time.perf_counter() - t0
    scale = cfg.L / layers
    total = t_mask + t_attn * scale + t_acc + t_com * scale
    desc = (f"mask+accept in full; attention on {layers} of {cfg.L} layers"
            + (f" ({rows_frac:.3%} of the rows, sampled)" if rows_frac < 1.0 else "")
            + f" and commit on {layers} layers, both scaled x{scale:g}; single-threaded C oracle")
    return total, desc


def run_reference(args, cfg, world, rank):
    """The reference arm: the oracle, as it stands, timed on the host cores."""
    if rank != 0:
        return
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0"))) if torch.cuda.is_available() else "cpu"
    ver, host = build_workload(cfg, args.seed, dev)
    rng = np.random.default_rng(1)
    # calibrate: attention cost per output row on this host
    import oracle

    oracle.build()
    anc, depth, st = oracle.tree_build_mask(host["parent"], cfg.max_depth)
    q, k, v = W.bf16_bits(ver.q[0]), W.bf16_bits(ver.k[0]), W.bf16_bits(ver.v[0])
    sel = np.zeros((16, 3), np.int32)
    sel[:, 1] = np.arange(16) % (cfg.M + 1)
    sel[:, 2] = np.arange(16) % cfg.Hq
    t0 = time.perf_counter()
    oracle.tree_attention_rows(q, k, v, host["kv_start"], host["kv_len"], host["parent"], st, cfg.Hkv, sel)
    per_row = (time.perf_counter() - t0) / 16
    budget = 150.0 / max(1, args.steps + args.warmup)  # seconds of CPU per step
    n_rows_total = cfg.B * (cfg.M + 1) * cfg.Hq
    frac = min(1.0, max(1.0 / n_rows_total, 0.5 * budget / max(per_row * n_rows_total, 1e-9)))
    times = []
    desc = ""
    for i in range(args.warmup + args.steps):
        t, desc = cpu_oracle_step(cfg, ver, host, 1, frac, rng)
        if i >= args.warmup:
            times.append(t)
    t_step = sum(times) / len(times)
    value = cfg.B * cfg.M / t_step
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "nodes/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_step * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(cfg, world, host["kv_len"]),
        "cpu_baseline": {"value": value, "unit": "nodes/s", "cores": 1, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "nodes/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- our arm

def physical_layers(cfg, device):
    """Layers of KV cache that fit in 60% of the free device memory (all of them
    for every workload except the 80-layer ragged stress case)."""
    P = W.make_prefix_lengths(cfg, np.random.default_rng(0))
    _, _, S_cap = W.cache_geometry(cfg, P)
    per_layer = 2 * cfg.B * cfg.Hkv * S_cap * cfg.D * 2
    free, _ = torch.cuda.mem_get_info(device)
    return max(1, min(cfg.L, int(0.6 * free // per_layer)))


def run_ours(args, cfg, world, rank, local):
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    import tree_speculative_decoding_04_b200 as tvpkg

    tvpkg.load()
    L_cfg = cfg.L
    L_phys = physical_layers(cfg, device)
    if L_phys < cfg.L:
        import dataclasses

        cfg = dataclasses.replace(cfg, L=L_phys)
    ver, host = build_workload(cfg, args.seed, device)
    stream = torch.cuda.Stream(device)
    ks0 = ver.kv_start.clone()
    kl0 = ver.kv_len.clone()

    def reset():
        ver.kv_start.copy_(ks0, non_blocking=True)
        ver.kv_len.copy_(kl0, non_blocking=True)

    def step():
        reset()
        ver.step(stream)

    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        step()  # eager once (plans launches, checks errors)
    torch.cuda.synchronize()
    g_step = capture(step, stream)

    # ---- the timed region: K whole steps, graph replays, L2 never warm (1+ GB of KV per step)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            g_step.replay()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(device) as clk, torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(args.steps):
            g_step.replay()
        e1.record(stream)
        e1.synchronize()
    torch.cuda.synchronize()
    barrier(world)
    ms_total = max_over_ranks(e0.elapsed_time(e1), world, device)
    ms_step = ms_total / args.steps
    value = whole_job_rate(world, cfg.B * cfg.M, ms_total, args.steps)

    # ---- results of one step (for the algorithmic byte counts)
    with torch.cuda.stream(stream):
        step()
    torch.cuda.synchronize()
    al = ver.accept_len.cpu().numpy()
    path = ver.path.cpu().numpy()
    depth = ver.depth.cpu().numpy()
    kl_h = host["kv_len"]
    shift = (ver.kv_start.cpu().numpy() - host["kv_start"]) if cfg.left_padded else np.zeros(cfg.B, np.int64)

    # ---- per-call timings (graphs, inputs resident, CUDA events on the launching stream)
    L = cfg.L
    reps = max(5, args.steps // 2)
    g_attn = capture(lambda: [ver.attention(layer, stream) for layer in range(L)], stream)
    with torch.cuda.stream(stream):
        for _ in range(3):
            g_attn.replay()
    attn_ms = event_time(g_attn.replay, reps, stream) / L
    g_mask = capture(lambda: ver.build_mask(stream), stream)
    mask_ms = event_time(g_mask.replay, reps, stream)
    g_acc = capture(lambda: ver.accept(stream), stream)
    acc_ms = event_time(g_acc.replay, reps, stream)

    def commit_only():
        reset()
        ver.commit(stream)

    g_com = capture(commit_only, stream)
    com_ms = event_time(g_com.replay, reps, stream)
    g_reset = capture(reset, stream)
    reset_ms = event_time(g_reset.replay, reps, stream)
    com_ms = max(com_ms - reset_ms, 1e-6)

    # one attention launch alone (eager, not overlapped with a neighbour), median of 20
    singles = []
    for r in range(20):
        with torch.cuda.stream(stream):
            a0 = torch.cuda.Event(enable_timing=True)
            a1 = torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            ver.attention(r % L, stream)
            a1.record(stream)
        a1.synchronize()
        singles.append(a0.elapsed_time(a1))
    attn_single_ms = statistics.median(singles)

    hbm, tflops, peak_kind = peaks()
    a_bytes = attention_bytes(cfg, kl_h)
    a_flops = attention_flops(cfg, kl_h, depth)
    traffic = read_traffic(cfg.name)
    roofline = roofline_entry(a_bytes, a_flops, attn_ms, hbm, tflops, peak_kind,
                              traffic["dram_bytes_per_launch"] if traffic else None,
                              "tree_attn_tc_kernel" if cfg.D == 128 else "tree_attn_mma_kernel")
    c_bytes = commit_bytes(cfg, path, al, kl_h, cfg.left_padded, shift)
    kv_commit = {"gbs": c_bytes / (com_ms * 1e-3) / 1e9, "bytes_per_step": c_bytes, "us": com_ms * 1e3,
                 "frac_hbm": c_bytes / (com_ms * 1e-3) / 1e9 / hbm}

    # ---- end to end: pinned host inputs -> device, step, results -> host, every step
    e2e = run_e2e(args, cfg, ver, host, reset, stream, world, device) if not args.no_e2e else None

    # ---- CPU oracle baseline (rank 0, one GPU only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rng = np.random.default_rng(2)
        probe, _ = cpu_oracle_step(cfg, ver, host, 1, min(1.0, 64.0 / (cfg.B * (cfg.M + 1) * cfg.Hq)), rng)
        layers = int(max(1, min(cfg.L, args.cpu_seconds / max(probe / cfg.L, 1e-6))))
        t_step, desc = cpu_oracle_step(cfg, ver, host, layers)
        cpu = {"value": cfg.B * cfg.M / t_step, "unit": "nodes/s", "cores": 1, "kind": "oracle", "sample": desc,
               "host_threads_available": os.cpu_count()}
    return finish(args, cfg, world, rank, value, ms_step, roofline, kv_commit, mask_ms, attn_ms, attn_single_ms,
                  acc_ms, com_ms, reset_ms, al, cpu, e2e, ver, clk, kl_h, device, L_cfg)


def run_e2e(args, cfg, ver, host, reset, stream, world, device):
    L = cfg.L
    h = ver.pinned_inputs()
    h["parent"].copy_(torch.as_tensor(host["parent"]))
    h["draft"].copy_(torch.as_tensor(host["draft"]))
    h["logits"].copy_(ver.logits.cpu())
    for layer in range(L):
        h["q"][layer].copy_(ver.q[layer].cpu())
        for b in range(cfg.B):
            c0 = int(host["kv_start"][b] + host["kv_len"][b])
            h["tree_k"][layer, b].copy_(ver.k[layer][b, :, c0:c0 + cfg.M + 1].cpu())
            h["tree_v"][layer, b].copy_(ver.v[layer][b, :, c0:c0 + cfg.M + 1].cpu())

    def e2e_step():
        reset()
        ver.step_from_host(h, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(max(1, args.warmup // 2)):
            e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    e2e_steps = max(3, min(args.steps, 20))
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        t1.record(stream)
    t1.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(t0.elapsed_time(t1), world, device) / e2e_steps
    return {"value": world * cfg.B * cfg.M / (e2e_ms * 1e-3), "unit": "nodes/s", "ms_per_step": e2e_ms,
            "h2d_bytes_per_step": ver.h2d_bytes(), "d2h_bytes_per_step": ver.d2h_bytes()}


def finish(args, cfg, world, rank, value, ms_step, roofline, kv_commit, mask_ms, attn_ms, attn_single_ms, acc_ms,
           com_ms, reset_ms, al, cpu, e2e, ver, clk, kl_h, device, L_cfg):
    L = cfg.L
    if rank != 0:
        return
    accept_stats = {"mean_accept_len": float(np.mean(al)), "accept_len": al.tolist()}
    line = {
        "metric": METRIC, "value": value, "unit": "nodes/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(config_dict(cfg, world, kl_h), layers_in_workload=L_cfg,
                       layers_measured=cfg.L),
        "roofline": roofline,
        "kv_commit": kv_commit,
        "breakdown_us": {"tree_build_mask": mask_ms * 1e3, "tree_attention_per_layer": attn_ms * 1e3,
                         "tree_attention_all_layers": attn_ms * 1e3 * L,
                         "tree_attention_single_launch": attn_single_ms * 1e3, "tree_accept": acc_ms * 1e3,
                         "kv_commit_realign": com_ms * 1e3, "geometry_reset_copies": reset_ms * 1e3},
        "accept": accept_stats,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": ver.launches_per_step() * args.steps,
        "clocks": clk.summary(),
        "gpu": torch.cuda.get_device_name(device),
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    cfg = W.CONFIGS[args.config]
    if args.layers > 0:
        import dataclasses

        cfg = dataclasses.replace(cfg, L=args.layers)
    world, rank, local = dist_setup(args) if args.impl == "ours" else (
        int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")))
    try:
        if args.impl == "reference":
            run_reference(args, cfg, world, rank)
        else:
            run_ours(args, cfg, world, rank, local)
    finally:
        if world > 1 and args.impl == "ours":
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
