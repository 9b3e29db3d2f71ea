"""Helpers for the GPU parity tests: run the CUDA calls through the C ABI on
seeded inputs and fetch everything back to the host for comparison with the
oracle."""
import numpy as np
import torch

import tree_speculative_decoding_04_b200 as tv
import workloads as W


def dev():
    return torch.device("cuda:0")


def i32(a):
    return torch.as_tensor(np.ascontiguousarray(a, dtype=np.int32), device=dev())


def gpu_mask(parent, max_depth):
    parent = np.ascontiguousarray(parent, np.int32)
    B, n = parent.shape
    Wd = (n + 31) // 32
    par = i32(parent)
    anc = torch.full((B, n, Wd), -1, dtype=torch.int32, device=dev())
    depth = torch.full((B, n), -1, dtype=torch.int32, device=dev())
    status = torch.full((B,), -1, dtype=torch.int32, device=dev())
    tv.tree_build_mask(par, max_depth, anc, depth, status)
    return par, anc, depth, status


def host_u32(t):
    return t.cpu().numpy().view(np.uint32)


def gpu_attention(q, k, v, kv_start, kv_len, anc, status, scale=None, flags=0):
    out = torch.full_like(q, float("nan"))
    B, n, Hq, D = q.shape
    ws = tv.attention_workspace(B, n - 1, Hq, k.shape[1], D, k.shape[2], q.device)
    if ws is not None:
        ws.fill_(0xFF)  # NaN patterns: the kernel must not depend on the workspace contents
    tv.tree_attention(q, k, v, i32(kv_start), i32(kv_len), anc, status, out, ws, scale=scale, flags=flags)
    return out


def gpu_accept(logits, draft, par, depth, anc, status, max_depth):
    B, n = par.shape
    am = torch.full((B, n), -7, dtype=torch.int32, device=dev())
    al = torch.full((B,), -7, dtype=torch.int32, device=dev())
    path = torch.full((B, max_depth + 1), -7, dtype=torch.int32, device=dev())
    bonus = torch.full((B,), -7, dtype=torch.int32, device=dev())
    tv.tree_accept(logits, i32(draft), par, depth, anc, status, max_depth, am, al, path, bonus)
    return am, al, path, bonus


def random_parents(B, M, max_depth, rng):
    return np.stack([W.tree_uniform_depth(M, max_depth, rng) for _ in range(B)]).astype(np.int32)
