"""Seeded synthetic inputs for the tree verification step.

This module is shared by the tests, the smoke check and the benchmark.  It holds
no arithmetic of the method itself: it draws trees, prefix lengths, bulk
tensors and draft tokens, nothing more.  Trees follow the shapes the pages
describe (dummy root row 0, parent pointers into earlier rows, a node / depth
budget such as 16 nodes at depth 10 from "EAGLE-Pangu: Accelerator-Safe Tree
Speculative Decoding on Ascend NPUs", results section); ragged left-padded
batches follow "Batch Speculative Decoding Done Right" (ragged-tensor problem).

Structure (parents, lengths, planting coins) comes from numpy
``default_rng(seed)``; bulk tensors come from a seeded torch generator on the
requested device, so host and device runs of one seed see the same structure.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    M: int  # draft nodes; arrays have M+1 rows (row 0 = dummy root)
    max_depth: int
    V: int
    L: int  # layers of KV cache touched by the commit
    prefix: tuple  # ("fixed", P) or ("uniform", lo, hi)
    tree: str  # "uniform_depth" | "bfs14" | "bfs_skewed" | "chain"
    p_plant: float
    logit_sigma: float
    left_padded: bool
    rounds: int = 1

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv


# The five workloads (sizes, distributions and structure of the pages' settings).
CONFIGS = {
    "tiny": Config("tiny", B=1, Hq=4, Hkv=4, D=64, M=16, max_depth=10, V=1024, L=1,
                   prefix=("fixed", 128), tree="uniform_depth", p_plant=0.7, logit_sigma=1.0,
                   left_padded=False),
    "mha7b": Config("mha7b", B=1, Hq=32, Hkv=32, D=128, M=64, max_depth=6, V=32000, L=32,
                    prefix=("fixed", 2048), tree="bfs14", p_plant=0.7, logit_sigma=2.0,
                    left_padded=False),
    "eqspec": Config("eqspec", B=8, Hq=32, Hkv=8, D=128, M=5, max_depth=5, V=151936, L=36,
                     prefix=("uniform", 512, 4096), tree="chain", p_plant=0.6, logit_sigma=1.0,
                     left_padded=True, rounds=64),
    "b32gqa": Config("b32gqa", B=32, Hq=32, Hkv=2, D=128, M=16, max_depth=10, V=151552, L=40,
                     prefix=("fixed", 8192), tree="uniform_depth", p_plant=0.7, logit_sigma=1.0,
                     left_padded=False),
    "stress": Config("stress", B=16, Hq=64, Hkv=8, D=128, M=128, max_depth=12, V=128256, L=80,
                     prefix=("uniform", 4096, 32768), tree="bfs_skewed", p_plant=0.75,
                     logit_sigma=2.0, left_padded=True),
}

# The eqspec shapes in per-sequence-length mode (every sequence's content starts
# at column 0, no padding): the commit appends in place and nothing is realigned,
# which is what cross-batch grouping of equal lengths buys a padded batch.
CONFIGS["eqspec_ragged"] = dataclasses.replace(CONFIGS["eqspec"], name="eqspec_ragged", left_padded=False)

CONFIG_ORDER = ["tiny", "mha7b", "eqspec", "b32gqa", "stress"]


def describe(cfg: Config) -> str:
    G = cfg.Hq // cfg.Hkv
    return (f"B{cfg.B} Hq{cfg.Hq}/Hkv{cfg.Hkv} (G={G}) D{cfg.D} M{cfg.M} depth<={cfg.max_depth} "
            f"V{cfg.V} L{cfg.L} prefix={cfg.prefix} tree={cfg.tree}"
            f"{' left-padded' if cfg.left_padded else ''}")


# ----------------------------------------------------------------------------- trees

def tree_chain(M: int) -> np.ndarray:
    p = np.arange(-1, M, dtype=np.int32)
    p[0] = 0
    return p


def tree_uniform_depth(M: int, max_depth: int, rng: np.random.Generator) -> np.ndarray:
    """parent[i] uniform over the earlier rows whose depth is below max_depth."""
    par = np.zeros(M + 1, np.int32)
    dep = np.zeros(M + 1, np.int32)
    for i in range(1, M + 1):
        cand = np.nonzero(dep[:i] < max_depth)[0]
        par[i] = cand[rng.integers(len(cand))]
        dep[i] = dep[par[i]] + 1
    return par


def _tree_bfs(M: int, max_depth: int, rng: np.random.Generator, n_children) -> np.ndarray | None:
    par = [0]
    dep = [0]
    queue = [0]
    while len(par) < M + 1:
        if not queue:
            return None
        x = queue.pop(0)
        if dep[x] >= max_depth:
            continue
        for _ in range(n_children(rng)):
            if len(par) == M + 1:
                break
            par.append(x)
            dep.append(dep[x] + 1)
            queue.append(len(par) - 1)
    return np.asarray(par, np.int32)


def tree_bfs14(M: int, max_depth: int, rng: np.random.Generator) -> np.ndarray:
    """Breadth-first tree, every expanded node gets U{1..4} children, stop at M nodes."""
    while True:
        t = _tree_bfs(M, max_depth, rng, lambda r: int(r.integers(1, 5)))
        if t is not None:
            return t


def tree_bfs_skewed(M: int, max_depth: int, rng: np.random.Generator, frac_wide: float = 0.2) -> np.ndarray:
    """Breadth-first tree with skewed branching: an expanded node gets 4-5 children
    with probability 0.6, else 1-2; redrawn until at least frac_wide of the rows
    have four or more children."""
    need = math.ceil(frac_wide * (M + 1))

    def nch(r):
        return int(r.integers(4, 6)) if r.random() < 0.6 else int(r.integers(1, 3))

    while True:
        t = _tree_bfs(M, max_depth, rng, nch)
        if t is None:
            continue
        counts = np.bincount(t[1:], minlength=M + 1)
        if int((counts >= 4).sum()) >= need:
            return t


def make_tree(cfg: Config, rng: np.random.Generator) -> np.ndarray:
    if cfg.tree == "chain":
        return tree_chain(cfg.M)
    if cfg.tree == "uniform_depth":
        return tree_uniform_depth(cfg.M, cfg.max_depth, rng)
    if cfg.tree == "bfs14":
        return tree_bfs14(cfg.M, cfg.max_depth, rng)
    if cfg.tree == "bfs_skewed":
        return tree_bfs_skewed(cfg.M, cfg.max_depth, rng)
    raise ValueError(cfg.tree)


def make_parents(cfg: Config, rng: np.random.Generator) -> np.ndarray:
    return np.stack([make_tree(cfg, rng) for _ in range(cfg.B)]).astype(np.int32)


def make_prefix_lengths(cfg: Config, rng: np.random.Generator) -> np.ndarray:
    if cfg.prefix[0] == "fixed":
        return np.full(cfg.B, cfg.prefix[1], np.int32)
    lo, hi = cfg.prefix[1], cfg.prefix[2]
    return rng.integers(lo, hi + 1, size=cfg.B).astype(np.int32)


def cache_geometry(cfg: Config, P: np.ndarray, extra_rows: int = 0):
    """(kv_start, kv_len, S_cap).  Left-padded batches end every prefix at the
    batch maximum; per-sequence batches start every prefix at column 0.
    S_cap leaves room for the M+1 tree rows plus extra_rows of growth."""
    P = np.asarray(P, np.int32)
    pmax = int(P.max()) if len(P) else 0
    if cfg.left_padded:
        kv_start = (pmax - P).astype(np.int32)
    else:
        kv_start = np.zeros_like(P)
    S_cap = pmax + cfg.M + 1 + extra_rows
    S_cap = (S_cap + 7) // 8 * 8
    return kv_start, P.copy(), S_cap


# ----------------------------------------------------------------------------- bulk tensors

def torch_generator(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def randn_bf16(shape, gen: torch.Generator, device, sigma: float = 1.0) -> torch.Tensor:
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if sigma != 1.0:
        x.mul_(sigma)
    return x.to(torch.bfloat16)


def randn_f32(shape, gen: torch.Generator, device, sigma: float = 1.0) -> torch.Tensor:
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if sigma != 1.0:
        x.mul_(sigma)
    return x


def plant_drafts(logits: torch.Tensor, parent: np.ndarray, p_plant: float, rng: np.random.Generator) -> np.ndarray:
    """draft[b][i] = the first maximum of logits[b][parent[b][i]] with probability
    p_plant, else a uniform token.  Row 0 (the root's own token) is 0."""
    B, n, V = logits.shape
    top = torch.argmax(logits, dim=-1).cpu().numpy().astype(np.int64)  # [B][n]
    coins = rng.random((B, n))
    unif = rng.integers(0, V, size=(B, n))
    draft = np.where(coins < p_plant, np.take_along_axis(top, parent.astype(np.int64), axis=1), unif)
    draft[:, 0] = 0
    return draft.astype(np.int32)


# ----------------------------------------------------------------------------- self-describing rows

_MASK32 = 0xFFFFFFFF


def _mix32_np(x: np.ndarray) -> np.ndarray:
    x = x.astype(np.int64) & _MASK32
    x = ((x >> 16) ^ x) * 0x45D9F3B & _MASK32
    x = ((x >> 16) ^ x) * 0x45D9F3B & _MASK32
    return (x >> 16) ^ x


def _mix32_torch(x: torch.Tensor) -> torch.Tensor:
    x = x & _MASK32
    x = (((x >> 16) ^ x) * 0x45D9F3B) & _MASK32
    x = (((x >> 16) ^ x) * 0x45D9F3B) & _MASK32
    return (x >> 16) ^ x


def tagged_rows(layer: int, kvsel: int, B: int, Hkv: int, S_cap: int, D: int, device="cpu",
                salt: int = 0) -> torch.Tensor:
    """A [B][Hkv][S_cap][D] bf16 tensor whose every 16-bit word is a hash of
    (salt, layer, K|V, b, h, column, d), with exponent-all-ones patterns (Inf/NaN)
    remapped to finite values, so each moved row proves where it came from."""
    out = torch.empty((B, Hkv, S_cap, D), dtype=torch.int16, device=device)
    base = ((salt * 131 + layer) * 2 + kvsel) * 1_000_003
    per_b = Hkv * S_cap * D
    for b in range(B):  # one sequence at a time keeps the int64 temporaries small
        idx = torch.arange(b * per_b, (b + 1) * per_b, device=device, dtype=torch.int64)
        h = _mix32_torch(idx * 2654435761 % (1 << 32) + base)
        bits = (h & 0xFFFF).to(torch.int32)
        bad = (bits & 0x7F80) == 0x7F80
        bits = torch.where(bad, bits & ~0x0080, bits)
        bits = torch.where(bits >= 0x8000, bits - 0x10000, bits).to(torch.int16)
        out[b] = bits.reshape(Hkv, S_cap, D)
    return out.view(torch.bfloat16)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Host uint16 view of a bf16 tensor's bits."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


# ----------------------------------------------------------------------------- one verify step

@dataclasses.dataclass
class Step:
    cfg: Config
    parent: np.ndarray  # [B][M+1] int32
    draft: np.ndarray  # [B][M+1] int32
    prefix: np.ndarray  # [B] int32
    kv_start: np.ndarray
    kv_len: np.ndarray
    S_cap: int
    q: torch.Tensor  # [B][M+1][Hq][D] bf16
    k: torch.Tensor  # [B][Hkv][S_cap][D] bf16 (one layer)
    v: torch.Tensor
    logits: torch.Tensor  # [B][M+1][V] fp32


def make_step(cfg: Config, seed: int = 0, device="cpu", extra_rows: int = 0, with_logits: bool = True) -> Step:
    rng = np.random.default_rng(seed)
    parent = make_parents(cfg, rng)
    P = make_prefix_lengths(cfg, rng)
    kv_start, kv_len, S_cap = cache_geometry(cfg, P, extra_rows)
    gen = torch_generator(seed, device)
    n = cfg.M + 1
    q = randn_bf16((cfg.B, n, cfg.Hq, cfg.D), gen, device)
    k = randn_bf16((cfg.B, cfg.Hkv, S_cap, cfg.D), gen, device)
    v = randn_bf16((cfg.B, cfg.Hkv, S_cap, cfg.D), gen, device)
    if with_logits:
        logits = randn_f32((cfg.B, n, cfg.V), gen, device, cfg.logit_sigma)
        draft = plant_drafts(logits, parent, cfg.p_plant, rng)
    else:
        logits = torch.empty((0,), device=device)
        draft = np.zeros((cfg.B, n), np.int32)
    return Step(cfg, parent, draft, P, kv_start, kv_len, S_cap, q, k, v, logits)
