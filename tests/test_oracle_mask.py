"""Pins for the oracle's tree validation and ancestor bitmask (CPU only).

The mask is pinned by: a hand-worked fixture, exhaustive enumeration of every
sentinel-free tree with M <= 6 against a top-down reachability computation, the
closed forms of a chain (lower triangular) and a star, and the invariant checks
(bad parents, depth budget) of "EAGLE-Pangu: Accelerator-Safe Tree Speculative
Decoding on Ascend NPUs", methodology B.
"""
import itertools

import numpy as np
import pytest

from helpers import load_golden
import workloads as W


def _all_trees(M):
    """Every parent array with parent[0] = 0 and parent[i] in [0, i)."""
    for rest in itertools.product(*[range(i) for i in range(1, M + 1)]):
        yield (0,) + rest


def _mask_rows_to_sets(anc, M):
    n = M + 1
    out = []
    for u in range(n):
        s = set()
        for r in range(n):
            if (int(anc[u][r // 32]) >> (r % 32)) & 1:
                s.add(r)
        out.append(s)
    return out


def _descendants(parent, v):
    """Rows reachable from v by following child links (v included) -- top-down,
    a different route from the oracle's bottom-up parent walk."""
    n = len(parent)
    children = [[] for _ in range(n)]
    for i in range(1, n):
        children[parent[i]].append(i)
    seen, stack = {v}, [v]
    while stack:
        x = stack.pop()
        for c in children[x]:
            if c not in seen:
                seen.add(c)
                stack.append(c)
    return seen


def test_golden_tree6(orc):
    g = load_golden("mask_tree6.txt")
    anc, depth, st = orc.tree_build_mask(g["parent"][None, :], max_depth=10)
    assert st.tolist() == [0]
    assert depth[0].tolist() == g["depth"].tolist()
    assert anc[0, :, 0].tolist() == g["mask"].tolist()


@pytest.mark.parametrize("M", [0, 1, 2, 3, 4, 5, 6])
def test_exhaustive_small_trees(orc, M):
    trees = np.array(list(_all_trees(M)), np.int32)
    anc, depth, st = orc.tree_build_mask(trees, max_depth=M)
    assert (st == 0).all()
    for t in range(len(trees)):
        par = trees[t].tolist()
        sets = _mask_rows_to_sets(anc[t], M)
        for u in range(M + 1):
            assert 0 in sets[u] and u in sets[u]
            assert len(sets[u]) == depth[t][u] + 1
            if u > 0:
                assert sets[u] == sets[par[u]] | {u}
                assert depth[t][u] == depth[t][par[u]] + 1
        for v in range(M + 1):
            below = _descendants(par, v)
            for u in range(M + 1):
                assert (v in sets[u]) == (u in below)


def test_high_bits_are_zero(orc):
    rng = np.random.default_rng(1)
    for M in (31, 32, 33, 63, 64, 100, 255):
        par = W.tree_uniform_depth(M, 10_000, rng)[None, :]
        anc, _, st = orc.tree_build_mask(par, max_depth=10_000)
        assert st[0] == 0
        W_ = (M + 1 + 31) // 32
        assert anc.shape == (1, M + 1, W_)
        n = M + 1
        if n % 32:
            hi = ~np.uint32((1 << (n % 32)) - 1)
            assert not (anc[0, :, -1] & hi).any()


def test_chain_is_lower_triangular(orc):
    M = 40
    anc, depth, _ = orc.tree_build_mask(W.tree_chain(M)[None, :], max_depth=M)
    sets = _mask_rows_to_sets(anc[0], M)
    for u in range(M + 1):
        assert sets[u] == set(range(u + 1))
        assert depth[0][u] == u


def test_star_is_diagonal_plus_root(orc):
    M = 9
    par = np.zeros((1, M + 1), np.int32)
    anc, depth, _ = orc.tree_build_mask(par, max_depth=1)
    sets = _mask_rows_to_sets(anc[0], M)
    assert sets[0] == {0}
    for u in range(1, M + 1):
        assert sets[u] == {0, u} and depth[0][u] == 1


def test_invalid_parents_flagged(orc):
    M = 5
    good = np.array([0, 0, 1, 2, 1, 4], np.int32)
    cases = []
    bad_root = good.copy(); bad_root[0] = 1; cases.append(bad_root)
    self_loop = good.copy(); self_loop[3] = 3; cases.append(self_loop)
    forward = good.copy(); forward[2] = 4; cases.append(forward)
    negative = good.copy(); negative[4] = -1; cases.append(negative)
    too_big = good.copy(); too_big[5] = 99; cases.append(too_big)
    batch = np.stack([good] + cases)
    anc, depth, st = orc.tree_build_mask(batch, max_depth=M)
    assert st[0] == 0
    assert (st[1:] & orc.BAD_PARENT).all()
    assert not anc[1:].any() and not depth[1:].any()
    assert anc[0].any()


def test_depth_budget_flagged(orc):
    par = W.tree_chain(8)[None, :]
    _, _, st = orc.tree_build_mask(par, max_depth=8)
    assert st[0] == 0
    anc, depth, st = orc.tree_build_mask(par, max_depth=7)
    assert st[0] == orc.TOO_DEEP and not anc.any() and not depth.any()


def test_config_trees_valid(orc):
    rng = np.random.default_rng(0)
    for name in W.CONFIG_ORDER:
        cfg = W.CONFIGS[name]
        par = W.make_parents(cfg, rng)
        assert par.shape == (cfg.B, cfg.M + 1)
        anc, depth, st = orc.tree_build_mask(par, cfg.max_depth)
        assert (st == 0).all(), name
        assert depth.max() <= cfg.max_depth
    # skewed stress trees: at least 20% of rows have four or more children
    par = W.tree_bfs_skewed(128, 12, np.random.default_rng(3))
    assert (np.bincount(par[1:], minlength=129) >= 4).sum() >= 26
