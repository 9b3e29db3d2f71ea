#!/usr/bin/env python
"""Benchmark of the tree verification step on B200.

A step is one pass of the whole hot path over one batch of synthetic inputs:
tree_build_mask, tree_attention over every layer of the workload, tree_accept
and kv_commit_realign.  Default workload: the stress case (batch 16, 64 q / 8
kv heads, head dim 128, ragged left-padded prefixes of 4096-32768 tokens,
129-row trees of depth <= 12, vocab 128256, 80 layers).

Layers that do not fit on the GPU: attention runs on all of the workload's
layers, cycling over the distinct layer buffers that fit (every launch reads a
whole layer of KV, far larger than L2); kv_commit_realign moves the cache of
the distinct layers only, and its share of the step is scaled to the full layer
count (reported as scaled, with the measured figures beside it).

The EQSPEC workload replays its rounds for real: every round writes fresh tree
rows, reads fresh q and logits, and commits and repads on the state the
previous round left (nothing is reset between the rounds of one replay).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl reference]

Prints one JSON line (rank 0).  For N > 1 launch with torchrun: every rank runs
an independent replica (the sequences of the step are independent; there is no
exchange step), timing is the maximum over ranks and the value counts the work
of all ranks.  With N = 1 the line also carries a record per other workload
(``per_config``).
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import platform
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
NOMINAL_HBM_GBS = 8000.0  # the "about 8 TB/s" HBM3e figure, for context beside the measured copy bandwidth
# the sources of the tensor-core attention kernel: its traffic figure holds only
# for the exact sources it was measured on
ATTN_SRCS = [os.path.join(ROOT, "tree_speculative_decoding_04_b200", "csrc", f)
             for f in ("attention_tc.cu", "attention_common.cuh", "tv_common.cuh", "attention.cu")]
# a commit that moves less than this is a handful of launches, not a stream of HBM traffic
COMMIT_HBM_REGIME_BYTES = 256 << 20
PER_CONFIG = ["tiny", "mha7b", "eqspec", "b32gqa", "stress"]


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="stress", choices=list(W.CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="CPU work budget of each oracle baseline sample (one thread and all cores)")
    ap.add_argument("--layers", type=int, default=0,
                    help="cap on the distinct layer buffers; with --profile commit, the layers committed")
    ap.add_argument("--rounds", type=int, default=0, help="rounds of a multi-round workload (0: the workload's own)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-per-config", action="store_true")
    ap.add_argument("--profile", choices=["attention", "lm_head", "commit"], default=None,
                    help="profiling run: a few launches of one kernel on one layer of the workload, no timing")
    ap.add_argument("--batch", type=int, default=0, help="profiling run: sequences (0: the workload's)")
    return ap.parse_args(argv)


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
    """The workload description shared by both arms (identical keys and values)."""
    return {"workload": f"{cfg.name}: {W.describe(cfg)}", "global_batch": cfg.B * world,
            "prefix": list(cfg.prefix), "tree_rows": cfg.M + 1, "layers": cfg.L,
            "rounds": cfg.rounds, "parallelism": f"replicas x{world}",
            "l2": l2_note(cfg, kv_len)}


def l2_note(cfg, kv_len):
    nbytes = cfg.L * attention_bytes(cfg, kv_len)
    if nbytes > (126 << 20):
        return ("inputs larger than L2: every step streams %.2f GB of KV and q, one whole layer per attention "
                "launch" % (nbytes / 1e9))
    return "inputs fit in L2 (%.2f MB per step, not flushed): a launch-latency case" % (nbytes / 1e6)


GPU_TIMING = "CUDA graph of whole steps replayed K times; CUDA events on the launching stream"
CPU_TIMING = "host wall clock (time.perf_counter) around each oracle call on the host cores"


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


# ----------------------------------------------------------------------------- algorithmic work

def attention_bytes(cfg, kv_len):
    """Algorithmic bytes of one tree_attention launch: every key/value row of every
    sequence's range once (prefix + M+1 tree rows), q in and out once."""
    kv = sum(cfg.Hkv * (int(p) + cfg.M + 1) * cfg.D * 2 * 2 for p in kv_len)
    qo = cfg.B * (cfg.M + 1) * cfg.Hq * cfg.D * 2 * 2
    return kv + qo


def attention_flops(cfg, kv_len, depth):
    pre = sum(4 * cfg.D * cfg.Hq * (cfg.M + 1) * int(p) for p in kv_len)
    tree = int(4 * cfg.D * cfg.Hq * (np.asarray(depth) + 1).sum())
    return pre + tree


def accept_bytes(cfg):
    return cfg.B * (cfg.M + 1) * cfg.V * 4


def commit_bytes(cfg, path, accept_len, kv_len, realign, shift, layers=None):
    """Algorithmic bytes of kv_commit_realign over `layers` layers (default the
    workload's): rows that must move, read + write."""
    L = cfg.L if layers is None else layers
    row = cfg.D * 2
    total = 0
    for b in range(cfg.B):
        a = int(accept_len[b])
        if realign and shift[b] != 0:
            total += L * cfg.Hkv * 2 * (int(kv_len[b]) + max(a, -1) + 1) * row * 2
        elif a >= 0:
            moved = sum(1 for j in range(a + 1) if int(path[b, j]) != j)
            total += L * cfg.Hkv * 2 * moved * row * 2
    return total


def realign_geometry(kv_start, kv_len, accept_len, realign):
    """kv_start', kv_len' after one commit (the left-padded repad rule: content
    ends at the new batch maximum) -- bookkeeping for the byte counts."""
    ks = np.asarray(kv_start, np.int64)
    kl = np.asarray(kv_len, np.int64)
    n = np.where(np.asarray(accept_len) >= 0, np.asarray(accept_len) + 1, 0)
    kl2 = kl + n
    if not realign:
        return ks.copy(), kl2
    lmax = int(kl2.max())
    return lmax - kl2, kl2


# ----------------------------------------------------------------------------- timing helpers

def event_time(fn, reps, stream):
    """Mean device time (ms) of fn(), launched on `stream`, over reps back-to-back
    calls, after one untimed call (the first replay of a captured graph also
    uploads it)."""
    with torch.cuda.stream(stream):
        fn()
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
            recs = json.load(f)
        if isinstance(recs, dict):
            recs = [recs]
        sha = attention_source_sha256()
        for rec in recs:
            if rec.get("source_sha256") == sha and rec.get("workload") == workload:
                return rec
    except Exception:
        pass
    return None


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
        "hbm_frac_of_nominal_8tbs": a_bytes / attn_s / 1e9 / NOMINAL_HBM_GBS,
        "roofline_us": 1e6 * max(a_bytes / (hbm * 1e9), a_flops / (tflops * 1e12)),
    }
    r["frac"] = r["achieved"] / r["peak"]
    return r


def commit_entry(c_bytes, com_ms, hbm, layers_measured, layers_workload, peak_kind):
    gbs = c_bytes / (com_ms * 1e-3) / 1e9 if com_ms > 0 else 0.0
    return {"gbs": gbs, "bytes_per_step": c_bytes, "us": com_ms * 1e3, "frac_hbm": gbs / hbm,
            "peak_kind": f"{peak_kind} copy bandwidth", "frac_of_nominal_8tbs": gbs / NOMINAL_HBM_GBS,
            "layers_measured": layers_measured, "layers_in_workload": layers_workload,
            "regime": "hbm" if c_bytes >= COMMIT_HBM_REGIME_BYTES else
            "launch-latency bound (%.1f MB moved: the fraction is not an HBM figure)" % (c_bytes / 1e6)}


# ----------------------------------------------------------------------------- GPU workloads

def physical_layers(cfg, device, cap=0, frac=0.6):
    """Distinct layer buffers of KV cache that fit in `frac` of the free device
    memory (all of the workload's layers except for the stress case)."""
    P = W.make_prefix_lengths(cfg, np.random.default_rng(0))
    _, _, S_cap = W.cache_geometry(cfg, P, extra_rows=cfg.rounds * (cfg.M + 1) if cfg.rounds > 1 else 0)
    per_layer = 2 * cfg.B * cfg.Hkv * S_cap * cfg.D * 2
    free, _ = torch.cuda.mem_get_info(device)
    n = max(1, min(cfg.L, int(frac * free // per_layer)))
    return min(n, cap) if cap > 0 else n


def build_workload(cfg, seed, device, L_phys=None, extra_rows=0):
    """A TreeVerifier holding a seeded synthetic step of the workload.  With
    L_phys < cfg.L, layer l's cache is distinct buffer l % L_phys."""
    from tree_speculative_decoding_04_b200.verifier import TreeVerifier

    L_phys = cfg.L if L_phys is None else L_phys
    rng = np.random.default_rng(seed)
    parent = W.make_parents(cfg, rng)
    P = W.make_prefix_lengths(cfg, rng)
    ks, kl, S_cap = W.cache_geometry(cfg, P, extra_rows=extra_rows)
    g = W.torch_generator(seed, device)
    kbuf = [W.randn_bf16((cfg.B, cfg.Hkv, S_cap, cfg.D), g, device) for _ in range(L_phys)]
    vbuf = [W.randn_bf16((cfg.B, cfg.Hkv, S_cap, cfg.D), g, device) for _ in range(L_phys)]
    ver = TreeVerifier(cfg.B, cfg.M, cfg.Hq, cfg.Hkv, cfg.D, cfg.V, cfg.L, S_cap, cfg.max_depth,
                       realign=cfg.left_padded, device=device,
                       k_layers=[kbuf[l % L_phys] for l in range(cfg.L)],
                       v_layers=[vbuf[l % L_phys] for l in range(cfg.L)], commit_layers=list(range(L_phys)))
    for layer in range(cfg.L):
        ver.q[layer].copy_(W.randn_bf16(ver.q[layer].shape, g, device))
    ver.logits.copy_(W.randn_f32(ver.logits.shape, g, device, cfg.logit_sigma))
    draft = W.plant_drafts(ver.logits, parent, cfg.p_plant, rng)
    ver.parent.copy_(torch.as_tensor(parent))
    ver.draft.copy_(torch.as_tensor(draft))
    ver.kv_start.copy_(torch.as_tensor(ks))
    ver.kv_len.copy_(torch.as_tensor(kl))
    host = dict(parent=parent, draft=draft, P=P, kv_start=ks, kv_len=kl, S_cap=S_cap)
    return ver, host


def per_call_times(ver, cfg, stream, reps, reset):
    """Device time (ms) of each call alone: graphs, inputs resident."""
    L = cfg.L
    g_attn = capture(lambda: [ver.attention(layer, stream) for layer in range(L)], stream)
    with torch.cuda.stream(stream):
        for _ in range(3):
            g_attn.replay()
    attn_ms = event_time(g_attn.replay, reps, stream) / L
    del g_attn
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
    # the fused rotary embedding: attention with the query rotation, and the
    # tree-row append with and without the K rotation (graphs of L launches)
    ver.rope_theta = 10000.0
    attn_rope_ms = None
    if cfg.D == 128:  # the rotation is fused into the head dim 128 kernel only
        g_r = capture(lambda: [ver.attention(layer, stream) for layer in range(L)], stream)
        attn_rope_ms = event_time(g_r.replay, reps, stream) / L
        del g_r
    g_w = capture(lambda: [ver.write_tree_rows(layer, stream) for layer in range(L)], stream)
    kvw_rope_ms = event_time(g_w.replay, reps, stream) / L
    ver.rope_theta = 0.0
    g_w0 = capture(lambda: [ver.write_tree_rows(layer, stream) for layer in range(L)], stream)
    kvw_ms = event_time(g_w0.replay, reps, stream) / L
    del g_w, g_w0
    # one attention launch alone (eager, after a synchronisation), median of 10
    singles = []
    for r in range(10):
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            a0 = torch.cuda.Event(enable_timing=True)
            a1 = torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            ver.attention(r % L, stream)
            a1.record(stream)
        a1.synchronize()
        singles.append(a0.elapsed_time(a1))
    return dict(attn_ms=attn_ms, mask_ms=mask_ms, acc_ms=acc_ms, com_ms=com_ms, reset_ms=reset_ms,
                attn_single_ms=statistics.median(singles), attn_rope_ms=attn_rope_ms, kvw_rope_ms=kvw_rope_ms,
                kvw_ms=kvw_ms)


def commit_modes(ver, cfg, stream, reps, reset, L_phys, al, path, com_ms, kv_start0, kv_len0):
    """The commit modes of "EAGLE-Pangu", methodology A, timed on B200 over the
    distinct layers and scaled to the workload's layers:
    - fast reorder (this library): kv_commit_realign with the step's path --
      only the new segment moves, in place;
    - length-based (this library): the same call with every accepted row
      already in place (a chain accepted in order) -- nothing moves;
    - branch cache (the pages' prior art, torch copies here): every step clones
      the committed cache of every layer into a branch cache, and the accepted
      rows are then copied from the branch back into the main cache;
    - full path-index reorder (prior art): the whole content is gathered by an
      index map (prefix in order, then the accepted rows) instead of only the
      new segment."""
    import tree_speculative_decoding_04_b200 as tvpkg  # noqa: F401

    scale = cfg.L / L_phys
    # length-based: the chain path 0..a, every row already in place
    saved = ver.path.clone()
    chain = torch.zeros_like(ver.path)
    for b in range(cfg.B):
        a = int(al[b])
        if a >= 0:
            chain[b, :a + 1] = torch.arange(a + 1, dtype=torch.int32, device=chain.device)
    ver.path.copy_(chain)

    def commit_only():
        reset()
        ver.commit(stream)

    g = capture(commit_only, stream)
    len_ms = event_time(g.replay, reps, stream)
    del g
    ver.path.copy_(saved)
    g_reset = capture(reset, stream)
    reset_ms = event_time(g_reset.replay, reps, stream)
    len_ms = max(len_ms - reset_ms, 1e-6)
    # branch cache: clone every layer (one scratch layer, rotated), then copy back
    # the accepted rows of every sequence from the branch
    kb = [ver.k[i] for i in range(L_phys)]
    vb = [ver.v[i] for i in range(L_phys)]
    scratch = torch.empty_like(kb[0])
    kl = [int(x) for x in kv_len0]  # the geometry before the commit
    ks = [int(x) for x in kv_start0]
    n_acc = [int(a) + 1 if a >= 0 else 0 for a in al]
    src_idx = [torch.as_tensor([ks[b] + kl[b] + int(path[b, j]) for j in range(n_acc[b])], dtype=torch.long,
                               device=scratch.device) for b in range(cfg.B)]
    dst_idx = [torch.as_tensor([ks[b] + kl[b] + j for j in range(n_acc[b])], dtype=torch.long,
                               device=scratch.device) for b in range(cfg.B)]

    def clone_all():
        for i in range(L_phys):
            scratch.copy_(kb[i])
            scratch.copy_(vb[i])

    def commit_back():
        for i in range(L_phys):
            for cache in (kb[i], vb[i]):
                for b in range(cfg.B):
                    if n_acc[b]:
                        cache[b].index_copy_(1, dst_idx[b], scratch[b].index_select(1, src_idx[b]))

    def full_reorder():
        for i in range(L_phys):
            for cache in (kb[i], vb[i]):
                for b in range(cfg.B):
                    idx = torch.cat([torch.arange(ks[b], ks[b] + kl[b], device=scratch.device), src_idx[b]])
                    scratch[b, :, :len(idx)].copy_(cache[b].index_select(1, idx))

    with torch.cuda.stream(stream):
        clone_ms = event_time(clone_all, 2, stream)
        back_ms = event_time(commit_back, 2, stream)
        full_ms = event_time(full_reorder, 2, stream)
    del scratch
    clone_bytes = L_phys * 2 * kb[0].numel() * 2 * 2  # read + write of each layer's K and V
    branch_ms = (clone_ms + back_ms) * scale
    return {
        "layers_measured": L_phys, "scaled_to_layers": cfg.L,
        "fast_reorder_us": com_ms * scale * 1e3,
        "length_based_us": len_ms * scale * 1e3,
        "branch_cache_us": branch_ms * 1e3,
        "branch_cache_clone_gbs": clone_bytes / (clone_ms * 1e-3) / 1e9,
        "full_path_index_reorder_us": full_ms * scale * 1e3,
        "fast_reorder_speedup_vs_branch_cache": branch_ms / (com_ms * scale),
        "fast_reorder_speedup_vs_full_reorder": full_ms / com_ms,
        "note": "branch cache and full reorder are the pages' prior art written with torch copies / index ops "
                "(comparison arms, not this library's path)",
    }


def measure_step(args, cfg, world, device, steps, warmup, with_clock=False, with_e2e=False):
    """Whole-step timing of a single-step workload.  Returns (record, state)."""
    import tree_speculative_decoding_04_b200 as tvpkg

    tvpkg.load()
    L_phys = physical_layers(cfg, device, cap=args.layers)
    ver, host = build_workload(cfg, args.seed, device, L_phys=L_phys)
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
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            g_step.replay()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    clk = ClockSampler(device) if with_clock else None
    with (clk if clk else _Null()), torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(steps):
            g_step.replay()
        e1.record(stream)
        e1.synchronize()
    torch.cuda.synchronize()
    barrier(world)
    ms_total = max_over_ranks(e0.elapsed_time(e1), world, device)
    del g_step
    ms_meas = ms_total / steps

    # results of one step (for the algorithmic byte counts)
    with torch.cuda.stream(stream):
        step()
    torch.cuda.synchronize()
    al = ver.accept_len.cpu().numpy()
    path = ver.path.cpu().numpy()
    depth = ver.depth.cpu().numpy()
    kl_h = host["kv_len"]
    shift = (ver.kv_start.cpu().numpy() - host["kv_start"]) if cfg.left_padded else np.zeros(cfg.B, np.int64)

    t = per_call_times(ver, cfg, stream, max(5, steps // 2), reset)
    modes = commit_modes(ver, cfg, stream, max(5, steps // 2), reset, L_phys, al, path, t["com_ms"],
                         host["kv_start"], host["kv_len"]) if cfg.name in ("mha7b", "b32gqa", "stress") else None
    # the commit ran on the distinct layers only: scale its share to every layer
    scale = cfg.L / L_phys
    ms_step = ms_meas + (scale - 1.0) * t["com_ms"]
    value = whole_job_rate(world, cfg.B * cfg.M, ms_step * steps, steps)

    hbm, tflops, peak_kind = peaks()
    a_bytes = attention_bytes(cfg, kl_h)
    a_flops = attention_flops(cfg, kl_h, depth)
    traffic = read_traffic(cfg.name)
    roof = roofline_entry(a_bytes, a_flops, t["attn_ms"], hbm, tflops, peak_kind,
                          traffic["dram_bytes_per_launch"] if traffic else None,
                          "tree_attn_tc_kernel" if cfg.D == 128 else "tree_attn_mma_kernel")
    c_bytes = commit_bytes(cfg, path, al, kl_h, cfg.left_padded, shift, layers=L_phys)
    kvc = commit_entry(c_bytes, t["com_ms"], hbm, L_phys, cfg.L, peak_kind)
    acc_gbs = accept_bytes(cfg) / (t["acc_ms"] * 1e-3) / 1e9
    rec = {
        "workload": f"{cfg.name}: {W.describe(cfg)}",
        "nodes_per_s": value, "ms_per_step": ms_step, "ms_per_step_measured": ms_meas,
        "layers_in_workload": cfg.L, "layers_physical": L_phys,
        "step_scaling": None if L_phys == cfg.L else
        f"measured step ({cfg.L} attention launches over {L_phys} distinct layer buffers, commit on "
        f"{L_phys} layers) + ({cfg.L}/{L_phys} - 1) x the measured commit time",
        "roofline": roof, "kv_commit": kvc,
        "accept": {"us": t["acc_ms"] * 1e3, "gbs": acc_gbs, "frac_hbm": acc_gbs / hbm,
                   "mean_accept_len": float(np.mean(al)), "accept_len": al.tolist()},
        "breakdown_us": {"tree_build_mask": t["mask_ms"] * 1e3, "tree_attention_per_layer": t["attn_ms"] * 1e3,
                         "tree_attention_all_layers": t["attn_ms"] * 1e3 * cfg.L,
                         "tree_attention_single_launch": t["attn_single_ms"] * 1e3,
                         "tree_accept": t["acc_ms"] * 1e3, "kv_commit_realign": t["com_ms"] * 1e3,
                         "geometry_reset_copies": t["reset_ms"] * 1e3},
        "commit_modes": modes,
        "rope": {"attention_per_layer_us": t["attn_rope_ms"] * 1e3 if t["attn_rope_ms"] else None,
                 "attention_plain_per_layer_us": t["attn_ms"] * 1e3,
                 "attention_overhead_frac": t["attn_rope_ms"] / t["attn_ms"] - 1.0 if t["attn_rope_ms"] else None,
                 "tree_kv_write_per_layer_us": t["kvw_rope_ms"] * 1e3,
                 "tree_kv_write_plain_per_layer_us": t["kvw_ms"] * 1e3,
                 "note": "query rows rotated to kv_len + depth while staged (TV_ATTN_ROPE); tree K rows rotated "
                         "by tree_kv_write; base 10000"},
        "gpu_launches_per_step": ver.launches_per_step(),
        "_kv_len": [int(x) for x in kl_h],
    }
    if with_e2e:
        rec["e2e"] = run_e2e(args, cfg, ver, host, reset, stream, world, device, L_phys)
    state = dict(ver=ver, host=host, clk=clk, stream=stream)
    return rec, state


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def run_e2e(args, cfg, ver, host, reset, stream, world, device, L_phys):
    """The same step through TreeVerifier.step_from_host: every step the inputs are
    copied in from pinned host memory and the accept results copied out.  With
    L_phys < L the commit's share is scaled as for the device-resident step."""
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
        for _ in range(2):
            e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    e2e_steps = max(3, min(args.steps, 10))
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
    # pinned host -> device copy bandwidth of this machine, for the bound of the copies
    nb = min(ver.layout.nbytes, 1 << 30)
    src = h["_buf"][:nb]
    dst = torch.empty(nb, dtype=torch.uint8, device=device)
    pcie_ms = event_time(lambda: dst.copy_(src, non_blocking=True), 3, stream)
    del dst
    return {"value": world * cfg.B * cfg.M / (e2e_ms * 1e-3), "unit": "nodes/s", "ms_per_step": e2e_ms,
            "h2d_bytes_per_step": ver.h2d_bytes(), "d2h_bytes_per_step": ver.d2h_bytes(),
            "pinned_h2d_gbs": nb / (pcie_ms * 1e-3) / 1e9,
            "copy_bound_ms": ver.h2d_bytes() / (nb / (pcie_ms * 1e-3)) * 1e3,
            "path": "TreeVerifier.step_from_host: one pinned staging buffer, per-layer sections on a copy "
                    "stream, tree_kv_write + attention per landed layer, accept results copied back"}


def measure_rounds(args, cfg, world, device, rounds, replays, warmup, with_clock=False):
    """A multi-round workload (EQSPEC): `rounds` real rounds per replay, every
    round with its own tree rows, q, logits and drafts, the cache geometry and
    content carried from round to round.  One CUDA graph holds all rounds; the
    geometry is reset before each replay of the whole sequence of rounds."""
    import tree_speculative_decoding_04_b200 as tvpkg
    from tree_speculative_decoding_04_b200 import _lib as tv

    tvpkg.load()
    extra = rounds * (cfg.M + 1)
    L_phys = physical_layers(cfg, device, cap=args.layers)
    if L_phys < cfg.L:
        raise RuntimeError("multi-round workload does not fit")
    ver, host = build_workload(cfg, args.seed, device, extra_rows=extra)
    stream = torch.cuda.Stream(device)
    B, n, L = cfg.B, cfg.M + 1, cfg.L
    rng = np.random.default_rng(args.seed + 1)
    g = W.torch_generator(args.seed + 1, device)
    # per-round inputs, all resident
    q_r = W.randn_bf16((rounds, L, B, n, cfg.Hq, cfg.D), g, device)
    tk_r = W.randn_bf16((rounds, L, B, cfg.Hkv, n, cfg.D), g, device)
    tv_r = W.randn_bf16((rounds, L, B, cfg.Hkv, n, cfg.D), g, device)
    lg_r = W.randn_f32((rounds, B, n, cfg.V), g, device, cfg.logit_sigma)
    dr_r = torch.stack([torch.as_tensor(W.plant_drafts(lg_r[r], host["parent"], cfg.p_plant, rng))
                        for r in range(rounds)]).to(device)
    i32 = dict(dtype=torch.int32, device=device)
    al_r = torch.zeros((rounds, B), **i32)
    path_r = torch.zeros((rounds, B, cfg.max_depth + 1), **i32)
    bonus_r = torch.zeros((rounds, B), **i32)
    am = torch.zeros((B, n), **i32)
    ks0, kl0 = ver.kv_start.clone(), ver.kv_len.clone()

    def reset():
        ver.kv_start.copy_(ks0, non_blocking=True)
        ver.kv_len.copy_(kl0, non_blocking=True)

    def one_round(r):
        ver.build_mask(stream)
        for layer in range(L):
            tv.tree_kv_write(ver.k_ptrs[layer:layer + 1], ver.v_ptrs[layer:layer + 1], tk_r[r, layer:layer + 1],
                             tv_r[r, layer:layer + 1], ver.S_cap, ver.kv_start, ver.kv_len, stream)
            tv.tree_attention(q_r[r, layer], ver.k[layer], ver.v[layer], ver.kv_start, ver.kv_len, ver.anc,
                              ver.status, ver.out[layer], ver.workspace, stream=stream)
        tv.tree_accept(lg_r[r], dr_r[r], ver.parent, ver.depth, ver.anc, ver.status, cfg.max_depth, am, al_r[r],
                       path_r[r], bonus_r[r], stream)
        tv.kv_commit_realign(ver.k_commit_ptrs, ver.v_commit_ptrs, B, cfg.Hkv, cfg.D, ver.S_cap, cfg.M, path_r[r],
                             al_r[r], ver.status, cfg.max_depth, ver.kv_start, ver.kv_len, ver.max_len,
                             int(cfg.left_padded), ver.attn_mask, ver.pos_ids, stream)

    def all_rounds():
        reset()
        for r in range(rounds):
            one_round(r)

    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        all_rounds()
    torch.cuda.synchronize()
    g_all = capture(all_rounds, stream)
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            g_all.replay()
    torch.cuda.synchronize()
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    clk = ClockSampler(device) if with_clock else None
    with (clk if clk else _Null()), torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(replays):
            g_all.replay()
        e1.record(stream)
        e1.synchronize()
    barrier(world)
    ms_total = max_over_ranks(e0.elapsed_time(e1), world, device)
    del g_all
    ms_round = ms_total / (replays * rounds)
    value = whole_job_rate(world, B * cfg.M, ms_round * replays * rounds, replays * rounds)

    # per-round bookkeeping for the byte counts (accept results of the last replay)
    al_h, path_h = al_r.cpu().numpy(), path_r.cpu().numpy()
    ks_h, kl_h = host["kv_start"].astype(np.int64), host["kv_len"].astype(np.int64)
    c_bytes, a_bytes, a_flops = 0, 0, 0
    depth = np.tile(np.arange(n), (B, 1))
    for r in range(rounds):
        a_bytes += attention_bytes(cfg, kl_h) * L
        a_flops += attention_flops(cfg, kl_h, depth) * L
        ks2, kl2 = realign_geometry(ks_h, kl_h, al_h[r], cfg.left_padded)
        c_bytes += commit_bytes(cfg, path_h[r], al_h[r], kl_h, cfg.left_padded, ks2 - ks_h)
        ks_h, kl_h = ks2, kl2
    ok_geometry = bool(np.array_equal(ver.kv_len.cpu().numpy(), kl_h))

    # the commits alone: the same sequence of per-round accept results, replayed
    def commits_only():
        reset()
        for r in range(rounds):
            tv.kv_commit_realign(ver.k_commit_ptrs, ver.v_commit_ptrs, B, cfg.Hkv, cfg.D, ver.S_cap, cfg.M,
                                 path_r[r], al_r[r], ver.status, cfg.max_depth, ver.kv_start, ver.kv_len,
                                 ver.max_len, int(cfg.left_padded), ver.attn_mask, ver.pos_ids, stream)

    g_c = capture(commits_only, stream)
    with torch.cuda.stream(stream):
        g_c.replay()
    com_ms = event_time(g_c.replay, 3, stream) / rounds
    del g_c
    g_reset = capture(reset, stream)
    reset_ms = event_time(g_reset.replay, 10, stream)
    com_ms = max(com_ms - reset_ms / rounds, 1e-6)

    # attention alone: the layers of one round (round 0's state), back to back
    reset()

    def attn_round0():
        for layer in range(L):
            tv.tree_attention(q_r[0, layer], ver.k[layer], ver.v[layer], ver.kv_start, ver.kv_len, ver.anc,
                              ver.status, ver.out[layer], ver.workspace, stream=stream)

    g_a = capture(attn_round0, stream)
    with torch.cuda.stream(stream):
        g_a.replay()
    attn_ms = event_time(g_a.replay, 10, stream) / L
    del g_a
    hbm, tflops, peak_kind = peaks()
    a0_bytes = attention_bytes(cfg, host["kv_len"])
    a0_flops = attention_flops(cfg, host["kv_len"], depth)
    traffic = read_traffic(cfg.name)
    roof = roofline_entry(a0_bytes, a0_flops, attn_ms, hbm, tflops, peak_kind,
                          traffic["dram_bytes_per_launch"] if traffic else None, "tree_attn_tc_kernel")
    kvc = commit_entry(c_bytes / rounds, com_ms, hbm, L, L, peak_kind)
    kvc["rounds"] = rounds
    rec = {
        "workload": f"{cfg.name}: {W.describe(cfg)}, {rounds} rounds",
        "nodes_per_s": value, "ms_per_step": ms_round, "ms_per_round": ms_round, "rounds": rounds,
        "ms_per_replay_of_all_rounds": ms_total / replays,
        "layers_in_workload": L, "layers_physical": L, "step_scaling": None,
        "roofline": roof, "kv_commit": kvc,
        "attention_all_rounds": {"gbs": a_bytes / (attn_ms * 1e-3 * L * rounds) / 1e9},
        "accept": {"mean_accept_len": float(al_h.mean()), "accept_len_hist": np.bincount(
            al_h.ravel() + 1, minlength=cfg.M + 2).tolist()},
        "geometry_matches_bookkeeping": ok_geometry,
        "breakdown_us": {"round": ms_round * 1e3, "tree_attention_per_layer": attn_ms * 1e3,
                         "kv_commit_realign_per_round": com_ms * 1e3},
        "gpu_launches_per_step": 1 + 2 * L + 2 + 2,
        "steps_timed": replays * rounds,
        "_kv_len": [int(x) for x in host["kv_len"]],
    }
    return rec, dict(ver=ver, host=host, clk=clk, stream=stream)


def measure_lm_head(args, cfg, device, reps=5):
    """tree_accept_lm_head on the workload's tree rows: hidden states [B][M+1][H]
    (H = Hq * D) against synthetic LM-head weights [V][H], the argmax fused into
    the GEMM's epilogue, then the acceptance walk.  Beside it, the unfused path
    it replaces: the logits written by a cuBLAS bf16 GEMM (through torch),
    widened to fp32, then tree_accept."""
    import tree_speculative_decoding_04_b200 as tv

    H = cfg.Hq * cfg.D
    n = cfg.M + 1
    rng = np.random.default_rng(args.seed + 3)
    g = W.torch_generator(args.seed + 3, device)
    parent = W.make_parents(cfg, rng)
    hidden = W.randn_bf16((cfg.B, n, H), g, device)
    w = W.randn_bf16((cfg.V, H), g, device, sigma=H ** -0.5)
    rows = cfg.B * n
    i32 = dict(dtype=torch.int32, device=device)
    par = torch.as_tensor(parent, device=device)
    anc = torch.zeros((cfg.B, n, (n + 31) // 32), **i32)
    depth = torch.zeros((cfg.B, n), **i32)
    status = torch.zeros((cfg.B,), **i32)
    tv.tree_build_mask(par, cfg.max_depth, anc, depth, status)
    logits = torch.matmul(hidden.reshape(rows, H), w.T).float().reshape(cfg.B, n, cfg.V)
    draft = torch.as_tensor(W.plant_drafts(logits, parent, cfg.p_plant, rng), device=device)
    am = torch.zeros((cfg.B, n), **i32)
    al = torch.zeros((cfg.B,), **i32)
    path = torch.zeros((cfg.B, cfg.max_depth + 1), **i32)
    bonus = torch.zeros((cfg.B,), **i32)
    ws = tv.lm_head_workspace(cfg.B, cfg.M, device)
    stream = torch.cuda.Stream(device)

    def fused():
        tv.tree_accept_lm_head(hidden, w, draft, par, depth, anc, status, cfg.max_depth, am, al, path, bonus, ws,
                               stream)

    def unfused():
        lg = torch.matmul(hidden.reshape(rows, H), w.T).float().reshape(cfg.B, n, cfg.V)
        tv.tree_accept(lg, draft, par, depth, anc, status, cfg.max_depth, am, al, path, bonus, stream)

    with torch.cuda.stream(stream):
        fused()
        unfused()
    torch.cuda.synchronize()
    g_f = capture(fused, stream)
    with torch.cuda.stream(stream):
        g_f.replay()
    f_ms = event_time(g_f.replay, reps, stream)
    del g_f
    with torch.cuda.stream(stream):
        u_ms = event_time(unfused, reps, stream)
    same = None
    with torch.cuda.stream(stream):
        fused()
    torch.cuda.synchronize()
    a_f = am.clone()
    with torch.cuda.stream(stream):
        unfused()
    torch.cuda.synchronize()
    same = float((a_f == am).float().mean().item())
    hbm, tflops, peak_kind = peaks()
    flops = 2 * rows * H * cfg.V
    nbytes = cfg.V * H * 2 + rows * H * 2
    r = roofline_entry(nbytes, flops, f_ms, hbm, tflops, peak_kind, None, "lm_head_argmax_kernel")
    del hidden, w, logits
    torch.cuda.empty_cache()
    return {"rows": rows, "H": H, "V": cfg.V, "fused_us": f_ms * 1e3, "unfused_us": u_ms * 1e3,
            "speedup_vs_unfused": u_ms / f_ms, "argmax_agreement_with_unfused": same,
            "logits_bytes_not_written": rows * cfg.V * 4, "roofline": r,
            "note": "fused: tree_accept_lm_head (GEMM + argmax epilogue + walk); unfused: cuBLAS bf16 logits "
                    "widened to fp32, then tree_accept"}


def measure_exspec(args, cfg, device, rounds=64, n_slots=32, buckets=4, repad=True):
    """Cross-batch scheduling (EXSPEC) on the EQSPEC shapes: a pool of n_slots
    sequences whose prefix lengths come from a few length buckets (drawn from the
    workload's range), batches of up to B picked every round by SequencePool
    (equal lengths: no realignment; else the EQSPEC repad), each round with fresh
    tree rows, q and logits.  The scheduler needs each round's accept lengths, so
    every round ends with a host synchronisation; device time (CUDA events
    around each step) and wall time are both reported, with the share of the
    device time spent in kv_commit_realign beside the EQSPEC figure."""
    from tree_speculative_decoding_04_b200.pool import FALLBACK, PoolVerifier, SequencePool

    rng = np.random.default_rng(args.seed + 7)
    g = W.torch_generator(args.seed + 7, device)
    B, n, L = cfg.B, cfg.M + 1, cfg.L
    lo, hi = cfg.prefix[1], cfg.prefix[2]
    bucket_len = rng.integers(lo, hi + 1, size=buckets)
    lengths0 = np.sort(rng.choice(bucket_len, size=n_slots)).astype(np.int32)
    S_cap = int(lengths0.max()) + (rounds + 1) * n + 8
    S_cap = (S_cap + 7) // 8 * 8
    pv = PoolVerifier(n_slots, B, cfg.M, cfg.Hq, cfg.Hkv, cfg.D, cfg.V, L, S_cap, cfg.max_depth, device=device,
                      with_mask_outputs=True)
    for layer in range(L):
        pv.k[layer].copy_(W.randn_bf16(pv.k[layer].shape, g, device))
        pv.v[layer].copy_(W.randn_bf16(pv.v[layer].shape, g, device))
    pv.kv_len.copy_(torch.as_tensor(lengths0))
    parent = np.stack([W.make_tree(cfg, rng) for _ in range(B)]).astype(np.int32)
    pv.parent.copy_(torch.as_tensor(parent))
    pv.q.copy_(W.randn_bf16(pv.q.shape, g, device))
    pv.tree_k.copy_(W.randn_bf16(pv.tree_k.shape, g, device))
    pv.tree_v.copy_(W.randn_bf16(pv.tree_v.shape, g, device))
    lg = W.randn_f32((rounds, B, n, cfg.V), g, device, cfg.logit_sigma)
    drafts = [torch.as_tensor(W.plant_drafts(lg[r], parent, cfg.p_plant, rng)).to(device) for r in range(rounds)]
    pool = SequencePool(lengths0, batch=B)
    stream = torch.cuda.Stream(device)
    dev_ms, com_ms, wall = 0.0, 0.0, 0.0
    n_grouped = n_fallback = 0
    nodes = 0
    com_by_mode = {"grouped": 0.0, "fallback": 0.0}
    torch.cuda.synchronize()
    for r in range(rounds + 2):  # two untimed warm-up rounds
        t0 = time.perf_counter()
        slots, mode = pool.next_batch()
        Bb = len(slots)
        pv.logits[:Bb].copy_(lg[r % rounds, :Bb])
        pv.draft[:Bb].copy_(drafts[r % rounds][:Bb])
        pv.set_slots(slots, stream)
        e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        realign = 1 if (mode == FALLBACK and repad) else 0
        pv.graphs(Bb, realign, stream)  # captured on first use, before the timed region
        stream.wait_stream(torch.cuda.current_stream(device))  # this round's logits and drafts
        with torch.cuda.stream(stream):
            e0.record(stream)
            pv.step_graphed(Bb, realign, stream, between=lambda: e1.record(stream))
            e2.record(stream)
        e2.synchronize()
        al = pv.accept_len[:Bb].cpu().numpy()
        pool.commit(slots, al)
        t1 = time.perf_counter()
        if r >= 2:
            wall += t1 - t0
            dev_ms += e0.elapsed_time(e2)
            c = e1.elapsed_time(e2)
            com_ms += c
            com_by_mode[mode] += c
            n_grouped += mode != FALLBACK
            n_fallback += mode == FALLBACK
            nodes += Bb * cfg.M
    rec = {
        "workload": f"exspec: pool of {n_slots} sequences of the eqspec shapes, prefix lengths from {buckets} buckets "
                    f"of {lo}-{hi}, batches of up to {B}, {rounds} rounds",
        "nodes_per_s_device": nodes / (dev_ms * 1e-3), "nodes_per_s_wall": nodes / wall,
        "ms_per_round_device": dev_ms / rounds, "ms_per_round_wall": wall * 1e3 / rounds,
        "grouped_rounds": n_grouped, "fallback_rounds": n_fallback,
        "commit_share_of_device_time": com_ms / dev_ms,
        "commit_ms_per_round": {k: v / max(1, n_grouped if k == "grouped" else n_fallback)
                                for k, v in com_by_mode.items()},
        "fallback_commit": "EQSPEC repad (the pages' EXSPEC)" if repad else
                           "per sequence, no repad (the slot map's per-sequence geometry; beyond the pages)",
        "gpu_launches_per_round": pv.launches_per_step(),
        "note": "each round replays the step's CUDA graphs (captured once per batch size and mode) with its slot "
                "map; every round ends with a host synchronisation (the scheduler needs the accept lengths)",
    }
    del pv, lg, drafts
    return rec


# ----------------------------------------------------------------------------- CPU oracle

def cpu_oracle_sample(cfg, q, k, v, logits, host, budget_s, rng, layers_cap=None):
    """Time the oracle on a bounded sample of one step: the mask and accept in
    full, attention on a sample of output rows of one layer, the commit of one
    layer.  Returns (seconds of one full step by extrapolation, seconds actually
    timed, fraction of the step's work actually run, description)."""
    import oracle

    t_run = 0.0
    t0 = time.perf_counter()
    anc, depth, st = oracle.tree_build_mask(host["parent"], cfg.max_depth)
    t_mask = time.perf_counter() - t0
    ks, kl = host["kv_start"], host["kv_len"]
    n_rows = cfg.B * (cfg.M + 1) * cfg.Hq
    # calibrate the cost of one attention row on a few rows
    nprobe = max(4, oracle.threads())
    probe = np.stack([rng.integers(cfg.B, size=nprobe), rng.integers(cfg.M + 1, size=nprobe),
                      rng.integers(cfg.Hq, size=nprobe)], axis=1).astype(np.int32)
    t0 = time.perf_counter()
    oracle.tree_attention_rows(q, k, v, ks, kl, host["parent"], st, cfg.Hkv, probe)
    per_row = (time.perf_counter() - t0) / nprobe  # wall time per row with every thread busy
    nsel = int(max(oracle.threads(), min(n_rows, 0.7 * budget_s / max(per_row, 1e-9))))
    if nsel >= n_rows:
        sel = np.stack(np.meshgrid(np.arange(cfg.B), np.arange(cfg.M + 1), np.arange(cfg.Hq), indexing="ij"),
                       axis=-1).reshape(-1, 3).astype(np.int32)
    else:
        sel = np.stack([rng.integers(cfg.B, size=nsel), rng.integers(cfg.M + 1, size=nsel),
                        rng.integers(cfg.Hq, size=nsel)], axis=1).astype(np.int32)
    t0 = time.perf_counter()
    oracle.tree_attention_rows(q, k, v, ks, kl, host["parent"], st, cfg.Hkv, sel)
    t_attn_sample = time.perf_counter() - t0
    t_attn_layer = t_attn_sample * n_rows / len(sel)
    t0 = time.perf_counter()
    am, al, path, bonus = oracle.tree_accept(logits, host["draft"], host["parent"], st, cfg.max_depth)
    t_acc = time.perf_counter() - t0
    kh, vh = k[:, :1].copy(), v[:, :1].copy()  # one kv head of one layer
    t0 = time.perf_counter()
    oracle.kv_commit_realign([kh], [vh], cfg.M, path, al, st, cfg.max_depth, ks, kl, int(cfg.left_padded))
    t_com = time.perf_counter() - t0
    t_run = t_mask + t_attn_sample + t_acc + t_com
    total = t_mask + t_attn_layer * cfg.L + t_acc + t_com * cfg.L * cfg.Hkv
    frac = (t_mask + t_attn_sample + t_acc + t_com) / total
    desc = (f"mask and accept in full; attention on {len(sel)} of {n_rows} output rows of one layer "
            f"({len(sel) / n_rows:.3%}, {'all' if len(sel) == n_rows else 'sampled'}), scaled to {n_rows} rows x "
            f"{cfg.L} layers; commit on one kv head of one layer scaled x{cfg.L * cfg.Hkv}; C oracle, "
            f"{oracle.threads()} host thread(s)")
    return total, t_run, frac, desc


def host_bulk(cfg, seed, device):
    """One layer's q/k/v and the logits of the workload as host arrays, drawn with
    torch only (no part of the CUDA library is loaded)."""
    rng = np.random.default_rng(seed)
    parent = W.make_parents(cfg, rng)
    P = W.make_prefix_lengths(cfg, rng)
    ks, kl, S_cap = W.cache_geometry(cfg, P)
    g = W.torch_generator(seed, device)
    n = cfg.M + 1
    k = W.bf16_bits(W.randn_bf16((cfg.B, cfg.Hkv, S_cap, cfg.D), g, device))
    v = W.bf16_bits(W.randn_bf16((cfg.B, cfg.Hkv, S_cap, cfg.D), g, device))
    q = W.bf16_bits(W.randn_bf16((cfg.B, n, cfg.Hq, cfg.D), g, device))
    lg = W.randn_f32((cfg.B, n, cfg.V), g, device, cfg.logit_sigma)
    draft = W.plant_drafts(lg, parent, cfg.p_plant, rng)
    host = dict(parent=parent, draft=draft, P=P, kv_start=ks, kv_len=kl, S_cap=S_cap)
    return q, k, v, lg.cpu().numpy(), host


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return platform.processor() or "unknown"


def cpu_baseline(args, cfg, device):
    """The oracle on the host cores, single thread and all cores (each build loaded
    in a child process of its own, so that the choice of build is clean)."""
    import subprocess

    out = {}
    for mode in ("single", "all"):
        cmd = [sys.executable, os.path.abspath(__file__), "--impl", "reference", "--config", cfg.name,
               "--steps", "1", "--warmup", "0", "--seed", str(args.seed), "--cpu-seconds", str(args.cpu_seconds),
               "--_cpu-mode", mode]
        env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
        try:
            r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, env=env)
            lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
            out[mode] = json.loads(lines[-1])["cpu_baseline"] if r.returncode == 0 and lines else {
                "error": r.stderr[-400:]}
        except Exception as e:  # a baseline failure must not void the GPU line
            out[mode] = {"error": repr(e)}
    best = out.get("all") if "value" in out.get("all", {}) else out.get("single")
    res = dict(best) if best and "value" in best else {"value": None, "unit": "nodes/s", "cores": 0,
                                                        "kind": "oracle", "sample": "failed"}
    res["single_thread"] = out.get("single")
    res["all_cores"] = out.get("all")
    res["cpu_model"] = cpu_model()
    res["nproc"] = os.cpu_count()
    return res


def run_reference(args, cfg, world, rank):
    """The reference arm: the oracle, as it stands, timed on the host cores; each
    step is a bounded sample of the workload's step (see cpu_oracle_sample)."""
    if rank != 0:
        return
    import oracle

    mode = getattr(args, "_cpu_mode", None) or "all"
    oracle.use_openmp(mode == "all")
    oracle.build(openmp=(mode == "all"))
    dev = "cpu"
    q, k, v, logits, host = host_bulk(cfg, args.seed, dev)
    rng = np.random.default_rng(1)
    # the whole --steps/--warmup run stays within about a minute of sampled work
    budget = min(args.cpu_seconds, max(0.5, 60.0 / max(1, args.steps + args.warmup)))
    totals, runs, fracs = [], [], []
    desc = ""
    for i in range(args.warmup + args.steps):
        total, t_run, frac, desc = cpu_oracle_sample(cfg, q, k, v, logits, host, budget, rng)
        if i >= args.warmup:
            totals.append(total)
            runs.append(t_run)
            fracs.append(frac)
    t_step = statistics.mean(totals)
    value = cfg.B * cfg.M / t_step
    cores = oracle.threads()
    cpu = {"value": value, "unit": "nodes/s", "cores": cores, "kind": "oracle", "sample": desc,
           "seconds_timed_per_step": statistics.mean(runs), "work_fraction_per_step": statistics.mean(fracs),
           "extrapolated": True, "seconds_per_full_step": t_step, "cpu_model": cpu_model(),
           "nproc": os.cpu_count()}
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "nodes/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.mean(runs) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "value_note": "nodes/s of a full step, extrapolated from the bounded sample that each step runs; "
                      "ms_per_step is the time of that sample",
        "config": config_dict(cfg, world, host["kv_len"]),
        "timing": CPU_TIMING,
        "cpu_baseline": cpu,
        "e2e": {"value": value, "unit": "nodes/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- our arm

def free_state(state):
    for key in list(state):
        state[key] = None
    import gc

    gc.collect()
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def measure(args, cfg, world, device, headline):
    if cfg.rounds > 1:
        rounds = args.rounds or cfg.rounds
        cfg = dataclasses.replace(cfg, rounds=rounds)
        return measure_rounds(args, cfg, world, device, rounds, replays=max(2, args.steps // 4) if headline else 2,
                              warmup=max(1, args.warmup // 2), with_clock=headline)
    steps = args.steps if headline else max(5, args.steps // 2)
    warm = args.warmup if headline else 3
    return measure_step(args, cfg, world, device, steps, warm, with_clock=headline,
                        with_e2e=headline and not args.no_e2e)


def run_ours(args, cfg, world, rank, local):
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    rec, state = measure(args, cfg, world, device, headline=True)
    clk = state["clk"]
    free_state(state)
    per_config = {}
    if world == 1 and not args.no_per_config:
        for name in PER_CONFIG:
            if name == cfg.name:
                continue
            try:
                r, st = measure(args, W.CONFIGS[name], world, device, headline=False)
                free_state(st)
                per_config[name] = r
            except Exception as e:  # a secondary workload must not void the headline line
                per_config[name] = {"error": repr(e)[:300]}
                torch.cuda.empty_cache()
        for name in ("mha7b", "eqspec", "b32gqa", "stress"):
            try:
                per_config.setdefault(name, {})["lm_head"] = measure_lm_head(args, W.CONFIGS[name], device)
            except Exception as e:
                per_config.setdefault(name, {})["lm_head"] = {"error": repr(e)[:300]}
                torch.cuda.empty_cache()
        try:
            per_config["exspec"] = measure_exspec(args, W.CONFIGS["eqspec"], device)
            if "eqspec" in per_config and "kv_commit" in per_config["eqspec"]:
                eq = per_config["eqspec"]
                per_config["exspec"]["eqspec_commit_share"] = (
                    eq["kv_commit"]["us"] * 1e-3 / eq["ms_per_round"])
        except Exception as e:
            per_config["exspec"] = {"error": repr(e)[:300]}
        try:
            per_config["exspec_ragged_fallback"] = measure_exspec(args, W.CONFIGS["eqspec"], device, repad=False)
        except Exception as e:
            per_config["exspec_ragged_fallback"] = {"error": repr(e)[:300]}
        free_state({})
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args, cfg, device)
    if rank != 0:
        return
    steps = args.steps
    kv_len0 = rec.pop("_kv_len")
    for r in per_config.values():
        r.pop("_kv_len", None)
    steps = rec.get("steps_timed", args.steps)
    line = {
        "metric": METRIC, "value": rec["nodes_per_s"], "unit": "nodes/s", "n_gpus": world, "steps": steps,
        "warmup": args.warmup, "ms_per_step": rec["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_dict(dataclasses.replace(cfg, rounds=rec.get("rounds", cfg.rounds)), world, kv_len0),
        "timing": GPU_TIMING,
        "layers_physical": rec["layers_physical"], "step_scaling": rec["step_scaling"],
        "ms_per_step_measured": rec.get("ms_per_step_measured", rec["ms_per_step"]),
        "roofline": rec["roofline"],
        "kv_commit": rec["kv_commit"],
        "accept": rec["accept"],
        "breakdown_us": rec["breakdown_us"],
        "cpu_baseline": cpu,
        "e2e": rec.get("e2e"),
        "gpu_launches": rec["gpu_launches_per_step"] * steps,
        "clocks": clk.summary() if clk else None,
        "gpu": torch.cuda.get_device_name(device),
        "per_config": per_config,
    }
    print(json.dumps(line), flush=True)


def run_profile(args, cfg):
    """A few launches of one kernel on one layer of the workload (optionally
    fewer sequences), for an ncu capture: small enough to capture, inputs still
    larger than L2 for the DRAM counters.  Prints the launch's algorithmic
    bytes and flops so that the captured counters can be set against them."""
    import tree_speculative_decoding_04_b200 as tv

    device = torch.device("cuda", 0)
    if args.batch:
        cfg = dataclasses.replace(cfg, B=args.batch)
    # one layer, or with --layers that many for the commit (its launch moves
    # every layer's rows: a few layers keep the moved bytes above L2)
    cfg = dataclasses.replace(cfg, L=args.layers if (args.profile == "commit" and args.layers > 0) else 1)
    stream = torch.cuda.current_stream(device)
    if args.profile == "lm_head":
        H = cfg.Hq * cfg.D
        g = W.torch_generator(args.seed, device)
        rng = np.random.default_rng(args.seed)
        parent = W.make_parents(cfg, rng)
        n = cfg.M + 1
        hidden = W.randn_bf16((cfg.B, n, H), g, device)
        w = W.randn_bf16((cfg.V, H), g, device, sigma=H ** -0.5)
        par = torch.as_tensor(parent, device=device)
        anc = torch.zeros((cfg.B, n, (n + 31) // 32), dtype=torch.int32, device=device)
        depth = torch.zeros((cfg.B, n), dtype=torch.int32, device=device)
        status = torch.zeros((cfg.B,), dtype=torch.int32, device=device)
        tv.tree_build_mask(par, cfg.max_depth, anc, depth, status)
        draft = torch.zeros((cfg.B, n), dtype=torch.int32, device=device)
        am = torch.zeros((cfg.B, n), dtype=torch.int32, device=device)
        al = torch.zeros((cfg.B,), dtype=torch.int32, device=device)
        path = torch.zeros((cfg.B, cfg.max_depth + 1), dtype=torch.int32, device=device)
        bonus = torch.zeros((cfg.B,), dtype=torch.int32, device=device)
        ws = tv.lm_head_workspace(cfg.B, cfg.M, device)
        for _ in range(3):
            tv.tree_accept_lm_head(hidden, w, draft, par, depth, anc, status, cfg.max_depth, am, al, path, bonus, ws)
        torch.cuda.synchronize()
        rows = cfg.B * n
        print(json.dumps({"profile": "lm_head", "workload": cfg.name, "B": cfg.B, "rows": rows, "H": H, "V": cfg.V,
                          "flops_per_launch": 2 * rows * H * cfg.V,
                          "bytes_per_launch": cfg.V * H * 2 + rows * H * 2}))
        return
    ver, host = build_workload(cfg, args.seed, device)
    with torch.cuda.stream(stream):
        ver.build_mask(stream)
        for _ in range(3):
            if args.profile == "attention":
                ver.attention(0, stream)
            else:
                ver.kv_start.copy_(torch.as_tensor(host["kv_start"], device=device))
                ver.kv_len.copy_(torch.as_tensor(host["kv_len"], device=device))
                ver.accept(stream)
                ver.commit(stream)
    torch.cuda.synchronize()
    depth = ver.depth.cpu().numpy()
    print(json.dumps({"profile": args.profile, "workload": cfg.name, "B": cfg.B,
                      "attention_bytes_per_launch": attention_bytes(cfg, host["kv_len"]),
                      "attention_flops_per_launch": attention_flops(cfg, host["kv_len"], depth)}))


def main(argv=None):
    ap_args = parse(argv)
    cfg = W.CONFIGS[ap_args.config]
    if ap_args.profile:
        run_profile(ap_args, cfg)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ap_args.impl == "ours":
        world, rank, local = dist_setup(ap_args)
    try:
        if ap_args.impl == "reference":
            run_reference(ap_args, cfg, world, rank)
        else:
            run_ours(ap_args, cfg, world, rank, local)
    finally:
        if world > 1 and ap_args.impl == "ours":
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    # internal: which oracle build a CPU-baseline child process times
    if "--_cpu-mode" in sys.argv:
        i = sys.argv.index("--_cpu-mode")
        _mode = sys.argv[i + 1]
        del sys.argv[i:i + 2]
        _args = parse()
        _args._cpu_mode = _mode
        _cfg = W.CONFIGS[_args.config]
        run_reference(_args, _cfg, 1, 0)
    else:
        main()
