"""GPU parity of tree_build_mask against the oracle: bit-exact masks, depths and
status, over every small tree, random trees of every supported size, invalid
trees and depth budgets."""
import itertools

import numpy as np
import pytest

from gpu_helpers import gpu_mask, host_u32, random_parents
import workloads as W

pytestmark = pytest.mark.gpu


def _compare(orc, parents, max_depth):
    _, anc, depth, status = gpu_mask(parents, max_depth)
    o_anc, o_dep, o_st = orc.tree_build_mask(parents, max_depth)
    np.testing.assert_array_equal(host_u32(anc), o_anc)
    np.testing.assert_array_equal(depth.cpu().numpy(), o_dep)
    np.testing.assert_array_equal(status.cpu().numpy(), o_st)
    return o_st


@pytest.mark.parametrize("M", [0, 1, 2, 3, 4, 5, 6])
def test_every_small_tree(orc, M):
    trees = np.array([(0,) + r for r in itertools.product(*[range(i) for i in range(1, M + 1)])], np.int32)
    for md in (M, max(0, M - 2)):
        _compare(orc, trees, md)


@pytest.mark.parametrize("n", [1, 2, 17, 31, 32, 33, 63, 64, 65, 100, 129, 200, 255, 256])
def test_random_trees_all_sizes(orc, n):
    rng = np.random.default_rng(n)
    M = n - 1
    for md in (3, 12, M):
        par = random_parents(37, M, max(md, 1) if M else 0, rng)
        _compare(orc, par, md)
    chains = np.stack([W.tree_chain(M)] * 3)
    st = _compare(orc, chains, M)
    assert (st == 0).all()
    if M > 0:
        st = _compare(orc, chains, M - 1)
        assert (st == orc.TOO_DEEP).all()


@pytest.mark.parametrize("n", [9, 32, 33, 129])
def test_invalid_parents(orc, n):
    rng = np.random.default_rng(7)
    M = n - 1
    par = random_parents(12, M, 100, rng)
    par[1, 0] = 3
    par[2, M] = M  # self loop
    par[3, 1] = -5
    par[4, M // 2 + 1] = M  # forward pointer
    par[5, M] = 10_000
    st = _compare(orc, par, 100)
    assert (st[1:6] & orc.BAD_PARENT).all() and (st[6:] == 0).all() and st[0] == 0


def test_config_trees(orc):
    rng = np.random.default_rng(0)
    for name in W.CONFIG_ORDER:
        cfg = W.CONFIGS[name]
        par = W.make_parents(cfg, rng)
        st = _compare(orc, par, cfg.max_depth)
        assert (st == 0).all()


def test_large_batch(orc):
    rng = np.random.default_rng(3)
    par = random_parents(1000, 16, 10, rng)
    _compare(orc, par, 10)
    par = random_parents(300, 128, 12, rng)
    _compare(orc, par, 12)
