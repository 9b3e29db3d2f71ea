"""Pins for the oracle's tree-row append (CPU only).

The cache layout these calls share puts the M+1 tree rows of the current step
right behind each sequence's committed prefix, in every layer ("EAGLE-Pangu:
Accelerator-Safe Tree Speculative Decoding on Ascend NPUs", methodology C: one
teacher pass over all speculative tokens against the cached prefix).  Pins:
self-describing rows (each source row carries its own layer, sequence, head,
row and K/V marker, decoded independently of the write's index arithmetic),
every cell outside the destination windows unchanged, sequences with a
geometry that does not fit left untouched, and the composition with the
length-based commit (a chain path commits the first a+1 rows in order).
"""
import numpy as np

MARK_K, MARK_V = 0x4B00, 0x5600


def _tagged_tree(L, B, Hkv, n, D, mark):
    """uint16 [L][B][Hkv][n][D]: words 0..4 = (row, head, seq, layer, mark), then d."""
    t = np.zeros((L, B, Hkv, n, D), np.uint16)
    t[..., 0] = np.arange(n, dtype=np.uint16)[None, None, None, :]
    t[..., 1] = np.arange(Hkv, dtype=np.uint16)[None, None, :, None]
    t[..., 2] = np.arange(B, dtype=np.uint16)[None, :, None, None]
    t[..., 3] = np.arange(L, dtype=np.uint16)[:, None, None, None]
    t[..., 4] = mark
    t[..., 5:] = np.arange(5, D, dtype=np.uint16)
    return t


def _case(orc, L, B, Hkv, D, S_cap, M, ks, kl, seed=0):
    rng = np.random.default_rng(seed)
    n = M + 1
    k = [rng.integers(0, 1 << 16, (B, Hkv, S_cap, D), dtype=np.uint16) for _ in range(L)]
    v = [rng.integers(0, 1 << 16, (B, Hkv, S_cap, D), dtype=np.uint16) for _ in range(L)]
    k0 = [a.copy() for a in k]
    v0 = [a.copy() for a in v]
    tk = _tagged_tree(L, B, Hkv, n, D, MARK_K)
    tv = _tagged_tree(L, B, Hkv, n, D, MARK_V)
    orc.tree_kv_write(k, v, tk, tv, np.asarray(ks, np.int32), np.asarray(kl, np.int32))
    return k, v, k0, v0


def _fits(ks, kl, M, S_cap):
    return ks >= 0 and kl >= 0 and ks + kl + M + 1 <= S_cap


def test_rows_land_behind_the_prefix_and_nothing_else_moves(orc):
    L, B, Hkv, D, M, S_cap = 3, 4, 2, 8, 5, 40
    ks, kl = [0, 3, 10, 0], [7, 20, 0, 34]
    k, v, k0, v0 = _case(orc, L, B, Hkv, D, S_cap, M, ks, kl)
    for l in range(L):
        for b in range(B):
            lo = ks[b] + kl[b]
            for h in range(Hkv):
                for c in range(S_cap):
                    for cache, base, mark in ((k, k0, MARK_K), (v, v0, MARK_V)):
                        row = cache[l][b, h, c]
                        if lo <= c < lo + M + 1:
                            # decode the provenance carried by the row itself
                            assert (int(row[0]), int(row[1]), int(row[2]), int(row[3]), int(row[4])) == \
                                (c - lo, h, b, l, mark)
                            assert row[5:].tolist() == list(range(5, D))
                        else:
                            assert np.array_equal(row, base[l][b, h, c])


def test_geometry_that_does_not_fit_is_left_untouched(orc):
    L, B, Hkv, D, M, S_cap = 2, 4, 1, 8, 6, 24
    ks, kl = [0, 10, -1, 5], [17, 8, 3, 0]  # b0 fits exactly; b1 one column short; b2 negative
    assert [_fits(a, c, M, S_cap) for a, c in zip(ks, kl)] == [True, False, False, True]
    k, v, k0, v0 = _case(orc, L, B, Hkv, D, S_cap, M, ks, kl, seed=1)
    for l in range(L):
        for b in (1, 2):
            assert np.array_equal(k[l][b], k0[l][b]) and np.array_equal(v[l][b], v0[l][b])
        assert int(k[l][0, 0, S_cap - 1, 0]) == M  # the last tree row fills the last column
        assert not np.array_equal(k[l][3], k0[l][3])


def test_chain_commit_after_append_keeps_rows_in_order(orc):
    """Append, then a length-based commit (path[j] = j): the committed content is
    the old prefix followed by tree rows 0..a, in order."""
    L, B, Hkv, D, M, S_cap, md = 2, 3, 2, 8, 4, 30, 4
    ks, kl = [0, 0, 0], [5, 9, 0]
    k, v, k0, v0 = _case(orc, L, B, Hkv, D, S_cap, M, ks, kl, seed=2)
    al = np.array([2, 0, 4], np.int32)
    path = np.tile(np.arange(md + 1, dtype=np.int32), (B, 1))
    for b in range(B):
        path[b, al[b] + 1:] = 0
    ks2, kl2, _, _, _ = orc.kv_commit_realign(k, v, M, path, al, np.zeros(B, np.int32), md, ks, kl, realign=0)
    assert kl2.tolist() == [kl[b] + al[b] + 1 for b in range(B)]
    for l in range(L):
        for b in range(B):
            for h in range(Hkv):
                assert np.array_equal(k[l][b, h, :kl[b]], k0[l][b, h, :kl[b]])
                rows = k[l][b, h, kl[b]:kl2[b]]
                assert rows[:, 0].tolist() == list(range(al[b] + 1))
                assert (rows[:, 4] == MARK_K).all() and (v[l][b, h, kl[b]:kl2[b], 4] == MARK_V).all()
