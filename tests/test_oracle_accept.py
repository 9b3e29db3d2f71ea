"""Pins for the oracle's argmax and greedy tree acceptance (CPU only).

"EAGLE-Pangu: Accelerator-Safe Tree Speculative Decoding on Ascend NPUs",
results section: the accepted length counts the speculative tokens that the
teacher's greedy choice agrees with in one verification step.  Pins: a
hand-worked fixture with ties, numpy's argmax (first maximum), the chain closed
form (first mismatch), exhaustive small trees (the oracle also checks its
recurrence against brute-force path enumeration internally), and greedy
equivalence with token-by-token decoding of a toy language model.
"""
import itertools

import numpy as np
import pytest

from helpers import load_golden
import workloads as W


def _status(orc, parent, max_depth):
    return orc.tree_build_mask(parent, max_depth)[2]


def test_golden_tree6(orc):
    g = load_golden("accept_tree6.txt")
    par = g["parent"][None].astype(np.int32)
    logits = np.stack([g[f"logits{i}"] for i in range(7)])[None].astype(np.float32)
    md = int(g["max_depth"][0])
    st = _status(orc, par, md)
    for case in "AB":
        am, al, path, bonus = orc.tree_accept(logits, g[f"{case}.draft"][None], par, st, md)
        assert am[0].tolist() == g["argmax"].tolist()
        assert al.tolist() == g[f"{case}.accept_len"].tolist()
        assert path[0].tolist() == g[f"{case}.path"].tolist()
        assert bonus.tolist() == g[f"{case}.bonus"].tolist()


def test_argmax_first_maximum(orc):
    rng = np.random.default_rng(0)
    for V in (1, 2, 3, 5, 1024, 1027, 32000):
        x = rng.standard_normal((9, V)).astype(np.float32)
        # plant ties of the maximum in some rows
        for r in range(0, 9, 2):
            j = rng.integers(V, size=3)
            x[r, j] = x[r].max() + 1.0
        x[8] = 0.0  # all equal
        np.testing.assert_array_equal(orc.argmax_rows(x), np.argmax(x, axis=1))
    x = np.full((2, 7), -np.inf, np.float32)
    x[1, 3] = -1e30
    assert orc.argmax_rows(x).tolist() == [0, 3]


@pytest.mark.parametrize("M", [1, 5, 9])
def test_chain_accepts_up_to_first_mismatch(orc, M):
    rng = np.random.default_rng(M)
    V = 17
    par = W.tree_chain(M)[None]
    st = _status(orc, par, M)
    for trial in range(40):
        logits = rng.standard_normal((1, M + 1, V)).astype(np.float32)
        am = np.argmax(logits[0], axis=1)
        mism = int(rng.integers(1, M + 2))  # first wrong row (M+1 = none)
        draft = np.zeros((1, M + 1), np.int32)
        for i in range(1, M + 1):
            draft[0, i] = am[i - 1] if i < mism else (am[i - 1] + 1) % V
        _, al, path, bonus = orc.tree_accept(logits, draft, par, st, M)
        a = mism - 1
        assert al[0] == a
        assert path[0, : a + 1].tolist() == list(range(a + 1)) and not path[0, a + 1 :].any()
        assert bonus[0] == am[a]


@pytest.mark.parametrize("M", [2, 3, 4, 5])
def test_exhaustive_small_trees_with_ties(orc, M):
    """Every tree shape, drafts drawn from a vocabulary of 2 so siblings often share
    tokens; the oracle raises if recurrence and brute force ever disagree."""
    rng = np.random.default_rng(M)
    V = 2
    trees = [(0,) + r for r in itertools.product(*[range(i) for i in range(1, M + 1)])]
    par = np.array(trees, np.int32)
    B = len(trees)
    st = _status(orc, par, M)
    logits = rng.standard_normal((B, M + 1, V)).astype(np.float32)
    draft = rng.integers(0, V, size=(B, M + 1)).astype(np.int32)
    am, al, path, bonus = orc.tree_accept(logits, draft, par, st, M)
    for b in range(B):
        a = int(al[b])
        e = int(path[b, a])
        # the path is a root chain of the tree
        assert path[b, 0] == 0
        for j in range(1, a + 1):
            assert par[b, path[b, j]] == path[b, j - 1]
            assert draft[b, path[b, j]] == am[b, path[b, j - 1]]
        assert bonus[b] == am[b, e]


def _toy_lm_row(tokens, V, salt=7):
    """A fixed function of the token history: identical histories give identical rows."""
    r = np.random.default_rng([salt] + list(tokens))
    return r.standard_normal(V).astype(np.float32)


@pytest.mark.parametrize("seed", range(6))
def test_greedy_equivalence(orc, seed):
    """Tree acceptance emits exactly the first a+1 tokens of plain greedy decoding,
    where a is the longest greedy prefix present in the tree as a root path."""
    rng = np.random.default_rng(seed)
    M, V = 24, 4
    par = W.tree_uniform_depth(M, 8, rng)
    root_tok = 1
    hist = {0: (root_tok,)}
    draft = np.zeros(M + 1, np.int32)
    logits = np.zeros((M + 1, V), np.float32)
    logits[0] = _toy_lm_row(hist[0], V)
    for i in range(1, M + 1):
        p = int(par[i])
        greedy = int(np.argmax(logits[p]))
        draft[i] = greedy if rng.random() < 0.7 else int(rng.integers(V))
        hist[i] = hist[p] + (int(draft[i]),)
        logits[i] = _toy_lm_row(hist[i], V)
    st = _status(orc, par[None], 8)
    _, al, path, bonus = orc.tree_accept(logits[None], draft[None], par[None], st, 8)
    a = int(al[0])
    emitted = [int(draft[path[0, j]]) for j in range(1, a + 1)] + [int(bonus[0])]
    # plain greedy decoding with the same toy model
    seq = (root_tok,)
    greedy = []
    for _ in range(12):
        t = int(np.argmax(_toy_lm_row(seq, V)))
        greedy.append(t)
        seq = seq + (t,)
    assert emitted == greedy[: a + 1]
    # a is maximal: no root path spells the first a+1 greedy tokens
    present = set(hist.values())
    assert (root_tok,) + tuple(greedy[: a + 1]) not in present


def test_invalid_sequence_rejected(orc):
    par = np.array([[0, 0, 1], [0, 2, 1]], np.int32)  # second one is malformed
    st = _status(orc, par, 4)
    assert st.tolist()[0] == 0 and st[1] & orc.BAD_PARENT
    logits = np.zeros((2, 3, 5), np.float32)
    draft = np.zeros((2, 3), np.int32)
    am, al, path, bonus = orc.tree_accept(logits, draft, par, st, 4)
    assert al.tolist() == [2, -1] and not path[1].any() and bonus[1] == 0
