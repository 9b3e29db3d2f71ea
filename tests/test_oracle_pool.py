"""Pin of the oracle's cache-slot pools (cross-batch scheduling, "Batch
Speculative Decoding Done Right", methodology: EXSPEC) against an independent
list model.

A pool of sequences runs many rounds; every round the scheduler picks a batch
(equal lengths: per-sequence-length commit; otherwise: EQSPEC repad), the
batch's tree rows are appended, and an accepted path is committed.  Every KV
row is self-describing (sequence, origin, layer, K|V, head), so after every
round each slot's content must decode to the list of rows the list model
appended for that sequence alone: grouping, fallback batches and repadding
are invisible to every sequence (the padding-invariance of the batch
algorithms, extended to batches drawn from a pool).  Fallback batches must also
leave their sequences rectangular (pad + length = the batch maximum) with
contiguous position IDs.
"""
import numpy as np

from tree_speculative_decoding_04_b200.pool import FALLBACK, SequencePool

import workloads as W


def _row(slot, kind, a, b, layer, kv, h, D):
    r = np.zeros(D, np.uint16)
    r[:7] = [slot, kind, a, b, layer, kv, h]
    r[7:] = 0x5A5A
    return r


def test_pool_rounds_match_per_sequence_lists(orc):
    rng = np.random.default_rng(0)
    n_slots, B, L, Hkv, D, M, max_depth = 7, 4, 2, 2, 8, 5, 5
    lengths0 = rng.choice([6, 9, 13], size=n_slots)
    rounds = 40
    S_cap = int(lengths0.max()) + rounds * (M + 1) + M + 1 + 8
    k_pool = [np.zeros((n_slots, Hkv, S_cap, D), np.uint16) for _ in range(L)]
    v_pool = [np.zeros((n_slots, Hkv, S_cap, D), np.uint16) for _ in range(L)]
    kv_start = np.zeros(n_slots, np.int32)
    kv_len = lengths0.astype(np.int32).copy()
    content = [[(1, i, 0) for i in range(lengths0[s])] for s in range(n_slots)]
    for s in range(n_slots):
        for layer in range(L):
            for h in range(Hkv):
                for i in range(lengths0[s]):
                    k_pool[layer][s, h, i] = _row(s, 1, i, 0, layer, 0, h, D)
                    v_pool[layer][s, h, i] = _row(s, 1, i, 0, layer, 1, h, D)
    mask = np.zeros((n_slots, S_cap), np.uint8)
    pos = np.zeros((n_slots, S_cap), np.int32)
    pool = SequencePool(lengths0, batch=B, max_wait=5)
    modes = set()
    for rnd in range(rounds):
        slots, mode = pool.next_batch()
        modes.add(mode)
        Bb = len(slots)
        parent = np.stack([W.tree_uniform_depth(M, max_depth, rng) for _ in range(Bb)]).astype(np.int32)
        anc, depth, st = orc.tree_build_mask(parent, max_depth)
        tk = np.zeros((L, Bb, Hkv, M + 1, D), np.uint16)
        tv = np.zeros((L, Bb, Hkv, M + 1, D), np.uint16)
        for layer in range(L):
            for b in range(Bb):
                for h in range(Hkv):
                    for r in range(M + 1):
                        tk[layer, b, h, r] = _row(slots[b], 2, rnd, r, layer, 0, h, D)
                        tv[layer, b, h, r] = _row(slots[b], 2, rnd, r, layer, 1, h, D)
        orc.pool_tree_kv_write(k_pool, v_pool, slots, tk, tv, kv_start, kv_len)
        # an accepted path: root .. a random node (sometimes the sequence is rejected)
        path = np.zeros((Bb, max_depth + 1), np.int32)
        accept = np.zeros(Bb, np.int32)
        status = np.zeros(Bb, np.int32)
        for b in range(Bb):
            if rng.random() < 0.1:
                status[b] = 1
                accept[b] = -1
                continue
            e = int(rng.integers(M + 1))
            x = e
            while True:
                path[b, depth[b, x]] = x
                if x == 0:
                    break
                x = parent[b, x]
            accept[b] = depth[b, e]
        realign = 1 if mode == FALLBACK else 0
        ml, st2 = orc.pool_kv_commit_realign(k_pool, v_pool, slots, M, path, accept, status, max_depth, kv_start,
                                             kv_len, realign, mask, pos)
        for b, s in enumerate(slots):
            if accept[b] >= 0:
                content[s] += [(2, rnd, int(path[b, j])) for j in range(accept[b] + 1)]
        pool.commit(slots, accept)
        # every slot: content = its own list, in every layer / head / K|V
        for s in range(n_slots):
            assert kv_len[s] == len(content[s]) == pool.length[s]
            for layer in range(L):
                for kvsel, arr in ((0, k_pool[layer]), (1, v_pool[layer])):
                    for h in range(Hkv):
                        rows = arr[s, h, kv_start[s]:kv_start[s] + kv_len[s]]
                        want = np.stack([_row(s, kd, a, bb, layer, kvsel, h, D) for kd, a, bb in content[s]])
                        np.testing.assert_array_equal(rows, want)
        if mode == FALLBACK:
            ends = {int(kv_start[s] + kv_len[s]) for s in slots}
            assert ends == {ml}  # rectangular alignment over the batch
            for s in slots:
                on = mask[s].astype(bool)
                np.testing.assert_array_equal(np.nonzero(on)[0], np.arange(kv_start[s], kv_start[s] + kv_len[s]))
                np.testing.assert_array_equal(pos[s][on], np.arange(kv_len[s]))
    assert modes == {"grouped", "fallback"}  # both kinds of batch were exercised


def test_pool_attention_reads_each_rows_slot(orc):
    """Batch row b attends over slot slots[b]: equal to the batch function on the
    gathered slots, and rows whose slot is outside the pool are zero."""
    rng = np.random.default_rng(1)
    n_slots, Hq, Hkv, D, M = 5, 4, 2, 16, 3
    S_cap = 40
    k = orc.round_bf16(rng.standard_normal((n_slots, Hkv, S_cap, D)))
    v = orc.round_bf16(rng.standard_normal((n_slots, Hkv, S_cap, D)))
    ks = np.array([0, 3, 1, 0, 2], np.int32)
    kl = np.array([10, 20, 5, 30, 7], np.int32)
    slots = np.array([3, 0, 9, 2], np.int32)  # 9 is outside the pool
    parent = np.stack([W.tree_chain(M)] * 4).astype(np.int32)
    q = orc.round_bf16(rng.standard_normal((4, M + 1, Hq, D)))
    st = np.zeros(4, np.int32)
    got = orc.pool_tree_attention(q, k, v, slots, ks, kl, parent, st, Hkv)
    for b, s in enumerate(slots):
        if s >= n_slots:
            assert not got[b].any()
            continue
        one = orc.tree_attention(q[b:b + 1], k[s:s + 1], v[s:s + 1], ks[s:s + 1], kl[s:s + 1], parent[b:b + 1],
                                 st[b:b + 1], Hkv)
        np.testing.assert_array_equal(got[b], one[0])
