"""Pins for the oracle's KV commit and EQSPEC realignment (CPU only).

"Batch Speculative Decoding Done Right", methodology: the synchronization
invariants (rectangular alignment; position IDs contiguous from 0 over the
attended positions) and unpad-append-repad; "EAGLE-Pangu: Accelerator-Safe Tree
Speculative Decoding on Ascend NPUs", methodology A: path-index commit of the new
segment.  Pins: a hand-worked fixture, the two invariants, padding invariance
(a padded batch holds what unpadded single-sequence runs hold, over many
rounds), an independent list model of the cache contents using self-describing
rows, and the chain special case (length-based and path-index commits agree).
"""
import numpy as np
import pytest

from helpers import load_golden
import workloads as W


def _ids_cache(B, Hkv, S_cap, D):
    """uint16 cache whose row (b, h, c) holds words (100*b + c, h, d) -- readable ids."""
    a = np.zeros((B, Hkv, S_cap, D), np.uint16)
    for b in range(B):
        for c in range(S_cap):
            a[b, :, c, 0] = 100 * b + c
    a[:, :, :, 1:] = np.arange(1, D, dtype=np.uint16)
    for h in range(Hkv):
        a[:, h, :, 1] += 1000 * h
    return a


def test_golden_realign_b2(orc):
    g = load_golden("realign_b2.txt")
    S_cap, M, md = int(g["S_cap"][0]), int(g["M"][0]), int(g["max_depth"][0])
    k = _ids_cache(2, 1, S_cap, 2)
    v = k.copy()
    path = np.stack([g["path0"], g["path1"]]).astype(np.int32)
    ks, kl, ml, mask, pos = orc.kv_commit_realign(
        [k], [v], M, path, g["accept_len"], np.zeros(2, np.int32), md, g["kv_start"], g["kv_len"], realign=1
    )
    assert ks.tolist() == g["new.kv_start"].tolist()
    assert kl.tolist() == g["new.kv_len"].tolist()
    assert ml == int(g["new.max_len"][0])
    for b in range(2):
        content = k[b, 0, ks[b] : ks[b] + kl[b], 0].tolist()
        assert content == g[f"new.content{b}"].tolist()
        assert v[b, 0, ks[b] : ks[b] + kl[b], 0].tolist() == content
        assert mask[b].tolist() == g[f"new.mask{b}"].tolist()
        assert pos[b].tolist() == g[f"new.pos{b}"].tolist()


def _random_round(rng, B, M, md, kl):
    """A random accepted path per sequence: a root chain of a random tree."""
    par = np.stack([W.tree_uniform_depth(M, md, rng) for _ in range(B)])
    path = np.zeros((B, md + 1), np.int32)
    al = np.zeros(B, np.int32)
    for b in range(B):
        e = int(rng.integers(M + 1))
        chain = []
        x = e
        while True:
            chain.append(x)
            if x == 0:
                break
            x = int(par[b, x])
        chain = chain[::-1]
        al[b] = len(chain) - 1
        path[b, : len(chain)] = chain
    return par, path, al


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_rounds_match_list_model_and_invariants(orc, seed):
    """Many EQSPEC rounds on a ragged left-padded batch: each round the tree rows are
    freshly written behind the content, a random path is committed and the batch is
    repadded.  An independent list-of-ids model predicts every content row."""
    rng = np.random.default_rng(seed)
    B, Hkv, D, M, md, R = 5, 2, 4, 6, 6, 12
    P = rng.integers(0, 20, size=B).astype(np.int32)
    pmax = int(P.max())
    S_cap = pmax + R * (md + 1) + M + 1 + 2
    ks = (pmax - P).astype(np.int32)
    kl = P.copy()
    k = np.zeros((B, Hkv, S_cap, D), np.uint16)
    v = np.zeros_like(k)
    model = [[(b, -1, c) for c in range(int(P[b]))] for b in range(B)]  # ids of content rows
    tag = 1

    def write_row(arr, b, c, ident, which):
        arr[b, :, c, 0] = ident & 0xFFFF
        arr[b, :, c, 1] = (ident >> 16) & 0xFFFF
        arr[b, :, c, 2] = np.arange(Hkv)
        arr[b, :, c, 3] = which

    ids = {}
    for b in range(B):
        for c in range(int(P[b])):
            ids[(b, -1, c)] = tag
            write_row(k, b, ks[b] + c, tag, 0)
            write_row(v, b, ks[b] + c, tag, 1)
            tag += 1
    for rnd in range(R):
        par, path, al = _random_round(rng, B, M, md, kl)
        st = np.zeros(B, np.int32)
        if rnd % 5 == 4:
            st[rnd % B] = orc.BAD_PARENT  # a rejected tree commits nothing but still shifts
        for b in range(B):
            for r in range(M + 1):
                ids[(b, rnd, r)] = tag
                write_row(k, b, ks[b] + kl[b] + r, tag, 0)
                write_row(v, b, ks[b] + kl[b] + r, tag, 1)
                tag += 1
        ks, kl, ml, mask, pos = orc.kv_commit_realign([k], [v], M, path, al, st, md, ks, kl, realign=1)
        for b in range(B):
            if st[b] == 0:
                model[b] += [(b, rnd, int(path[b, j])) for j in range(al[b] + 1)]
        # rectangular alignment and position-ID contiguity
        assert (ks + kl == ml).all()
        assert ml == max(len(m) for m in model)
        for b in range(B):
            sel = mask[b] == 1
            assert sel.sum() == kl[b] and sel[ks[b] : ks[b] + kl[b]].all()
            assert pos[b][sel].tolist() == list(range(kl[b]))
            assert not pos[b][~sel].any()
            got = [int(k[b, 0, c, 0]) | (int(k[b, 0, c, 1]) << 16) for c in range(ks[b], ks[b] + kl[b])]
            assert got == [ids[t] for t in model[b]]
            gotv = [int(v[b, 1, c, 0]) | (int(v[b, 1, c, 1]) << 16) for c in range(ks[b], ks[b] + kl[b])]
            assert gotv == got and (v[b, :, ks[b] : ks[b] + kl[b], 3] == 1).all()


@pytest.mark.parametrize("seed", [0, 1])
def test_padding_invariance(orc, seed):
    """After several rounds, each sequence of the padded batch holds exactly what the
    same sequence holds when run alone (batch of one, never padded)."""
    rng = np.random.default_rng(seed)
    B, Hkv, D, M, md, R = 4, 1, 8, 5, 5, 6
    P = rng.integers(1, 15, size=B).astype(np.int32)
    pmax = int(P.max())
    S_cap = pmax + R * (md + 1) + M + 1
    kb = [W.bf16_bits(W.tagged_rows(0, 0, B, Hkv, S_cap, D, salt=seed))]
    vb = [W.bf16_bits(W.tagged_rows(0, 1, B, Hkv, S_cap, D, salt=seed))]
    kb = [a.copy() for a in kb]
    vb = [a.copy() for a in vb]
    ks_b = (pmax - P).astype(np.int32)
    kl_b = P.copy()
    # batch-of-one copies hold the same rows without padding
    singles = []
    for b in range(B):
        k1 = np.zeros((1, Hkv, S_cap, D), np.uint16)
        v1 = np.zeros_like(k1)
        k1[0, :, : P[b] + M + 1] = kb[0][b, :, ks_b[b] : ks_b[b] + P[b] + M + 1]
        v1[0, :, : P[b] + M + 1] = vb[0][b, :, ks_b[b] : ks_b[b] + P[b] + M + 1]
        singles.append([k1, v1, np.zeros(1, np.int32), P[b : b + 1].copy()])
    for rnd in range(R):
        _, path, al = _random_round(rng, B, M, md, kl_b)
        st = np.zeros(B, np.int32)
        fresh_k = rng.integers(0, 0x7F00, size=(B, Hkv, M + 1, D), dtype=np.uint16)
        fresh_v = rng.integers(0, 0x7F00, size=(B, Hkv, M + 1, D), dtype=np.uint16)
        for b in range(B):
            c0 = ks_b[b] + kl_b[b]
            kb[0][b, :, c0 : c0 + M + 1] = fresh_k[b]
            vb[0][b, :, c0 : c0 + M + 1] = fresh_v[b]
            k1, v1, s1, l1 = singles[b]
            k1[0, :, l1[0] : l1[0] + M + 1] = fresh_k[b]
            v1[0, :, l1[0] : l1[0] + M + 1] = fresh_v[b]
        ks_b, kl_b, _, _, _ = orc.kv_commit_realign(kb, vb, M, path, al, st, md, ks_b, kl_b, realign=1)
        for b in range(B):
            k1, v1, s1, l1 = singles[b]
            s1n, l1n, _, _, _ = orc.kv_commit_realign(
                [k1], [v1], M, path[b : b + 1], al[b : b + 1], st[b : b + 1], md, s1, l1, realign=1
            )
            singles[b][2], singles[b][3] = s1n, l1n
    for b in range(B):
        k1, v1, s1, l1 = singles[b]
        assert s1[0] == 0 and l1[0] == kl_b[b]
        np.testing.assert_array_equal(kb[0][b, :, ks_b[b] : ks_b[b] + kl_b[b]], k1[0, :, : l1[0]])
        np.testing.assert_array_equal(vb[0][b, :, ks_b[b] : ks_b[b] + kl_b[b]], v1[0, :, : l1[0]])


def test_chain_commit_moves_nothing(orc):
    """Length-based commit (keep the prefix, append the first a steps of the branch)
    and path-index commit coincide on a chain: path[j] = j moves no byte."""
    B, Hkv, D, M, md, L = 3, 2, 8, 5, 5, 2
    S_cap = 40
    ks = np.zeros(B, np.int32)
    kl = np.array([10, 3, 20], np.int32)
    ks_ = [W.bf16_bits(W.tagged_rows(l, 0, B, Hkv, S_cap, D)).copy() for l in range(L)]
    vs_ = [W.bf16_bits(W.tagged_rows(l, 1, B, Hkv, S_cap, D)).copy() for l in range(L)]
    before = [a.copy() for a in ks_ + vs_]
    al = np.array([5, 0, 2], np.int32)
    path = np.tile(np.arange(md + 1, dtype=np.int32), (B, 1))
    for b in range(B):
        path[b, al[b] + 1 :] = 0
    ks2, kl2, ml, _, _ = orc.kv_commit_realign(ks_, vs_, M, path, al, np.zeros(B, np.int32), md, ks, kl, realign=0)
    for a, bef in zip(ks_ + vs_, before):
        np.testing.assert_array_equal(a, bef)
    assert kl2.tolist() == [16, 4, 23] and ks2.tolist() == [0, 0, 0] and ml == 23


def test_per_sequence_mode_reorders_only_tail(orc):
    B, Hkv, D, M, md = 2, 1, 4, 6, 4
    S_cap = 30
    k = _ids_cache(B, Hkv, S_cap, D)
    v = k.copy()
    before = k.copy()
    ks = np.array([0, 0], np.int32)
    kl = np.array([7, 12], np.int32)
    path = np.array([[0, 2, 5, 0, 0], [0, 1, 3, 4, 6]], np.int32)
    al = np.array([2, 4], np.int32)
    ks2, kl2, ml, mask, pos = orc.kv_commit_realign([k], [v], M, path, al, np.zeros(B, np.int32), md, ks, kl, realign=0)
    assert kl2.tolist() == [10, 17] and ml == 17
    for b in range(B):
        np.testing.assert_array_equal(k[b, :, : kl[b]], before[b, :, : kl[b]])
        for j in range(al[b] + 1):
            np.testing.assert_array_equal(k[b, :, kl[b] + j], before[b, :, kl[b] + path[b, j]])
        assert mask[b].sum() == kl2[b] and pos[b][: kl2[b]].tolist() == list(range(kl2[b]))


def test_bad_geometry_left_untouched(orc):
    B, Hkv, D, M, md = 2, 1, 4, 3, 3
    S_cap = 16
    k = _ids_cache(B, Hkv, S_cap, D)
    v = k.copy()
    before = k.copy()
    ks = np.array([2, 0], np.int32)
    kl = np.array([5, 14], np.int32)  # second: 14 + 4 tree rows > 16 columns
    path = np.array([[0, 1, 0, 0], [0, 1, 2, 3]], np.int32)
    al = np.array([1, 3], np.int32)
    ks2, kl2, ml, mask, pos = orc.kv_commit_realign([k], [v], M, path, al, np.zeros(B, np.int32), md, ks, kl, realign=1)
    np.testing.assert_array_equal(k[1], before[1])
    assert ks2[1] == 0 and kl2[1] == 14 and not mask[1].any()
    assert ks2[0] == 0 and kl2[0] == 7 and ml == 7


def test_out_of_tree_path_commits_nothing(orc):
    B, Hkv, D, M, md = 2, 1, 4, 3, 3
    S_cap = 20
    k = _ids_cache(B, Hkv, S_cap, D)
    v = k.copy()
    before = k.copy()
    ks = np.array([0, 0], np.int32)
    kl = np.array([5, 6], np.int32)
    path = np.array([[0, 1, 9, 0], [0, 2, 0, 0]], np.int32)  # row 9 does not exist (M = 3)
    al = np.array([2, 1], np.int32)
    ks2, kl2, ml, _, _, st = orc.kv_commit_realign(
        [k], [v], M, path, al, np.zeros(B, np.int32), md, ks, kl, realign=0, with_status=True
    )
    assert kl2.tolist() == [5, 8] and ml == 8 and st.tolist() == [0, 0]
    np.testing.assert_array_equal(k[0], before[0])
    np.testing.assert_array_equal(k[1, :, 6 + 1], before[1, :, 6 + 2])
