"""Host logic of the cross-batch scheduler (SequencePool, EXSPEC): grouped
batches hold sequences of one length only, the largest group goes first, a
pool with no group falls back to an EQSPEC batch, and no sequence waits longer
than the bound ("Batch Speculative Decoding Done Right", methodology: EXSPEC)."""
import numpy as np

from tree_speculative_decoding_04_b200.pool import FALLBACK, GROUPED, SequencePool


def test_grouped_batches_share_one_length_and_the_largest_group_goes_first():
    pool = SequencePool([10, 12, 10, 12, 12, 7], batch=8)
    slots, mode = pool.next_batch()
    assert mode == GROUPED and slots == [1, 3, 4]
    pool.commit(slots, [0, 1, 2])  # 12 -> 13, 14, 15
    slots, mode = pool.next_batch()
    assert mode == GROUPED and slots == [0, 2]


def test_batch_size_is_capped_and_ties_go_to_the_shorter_length():
    pool = SequencePool([5] * 5 + [3] * 5, batch=4)
    slots, mode = pool.next_batch()
    assert mode == GROUPED and len(slots) == 4 and all(pool.length[s] == 3 for s in slots)


def test_no_group_falls_back_to_an_eqspec_batch():
    pool = SequencePool([1, 2, 3, 4, 5], batch=3)
    slots, mode = pool.next_batch()
    assert mode == FALLBACK and len(slots) == 3 and len({pool.length[s] for s in slots}) == 3


def test_min_group_one_never_falls_back():
    pool = SequencePool([1, 2, 3], batch=3, min_group=1)
    _, mode = pool.next_batch()
    assert mode == GROUPED


def test_waiting_is_bounded_over_many_rounds():
    rng = np.random.default_rng(0)
    n, B = 24, 8
    pool = SequencePool(rng.integers(100, 104, size=n), batch=B, max_wait=6)
    last = [-1] * n
    for r in range(300):
        slots, mode = pool.next_batch()
        assert 0 < len(slots) <= B and len(set(slots)) == len(slots)
        lens = {pool.length[s] for s in slots}
        assert (mode == GROUPED) == (len(lens) == 1)
        for s in range(n):
            assert r - last[s] <= 6 + 2, (s, r, last[s])
        for s in slots:
            last[s] = r
        pool.commit(slots, rng.integers(-1, 6, size=len(slots)))


def test_commit_adds_accepted_rows_plus_the_root():
    pool = SequencePool([10, 10], batch=2)
    pool.commit([0, 1], [3, -1])
    assert pool.length == [14, 10]
