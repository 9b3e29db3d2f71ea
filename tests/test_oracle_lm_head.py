"""Pins of the oracle's LM-head logits and their argmax ("EAGLE-Pangu", section
2.C: the teacher's greedy choice at each node is the argmax of its logits, here
computed from the final hidden state and the LM-head weights).  Pins: numpy's
float64 matrix product, exact integer products (small-integer bf16 inputs give
integer logits that an int64 matrix product reproduces exactly), and the
first-maximum rule on planted ties (duplicated weight rows)."""
import numpy as np


def _bf16(x):
    return (np.asarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _f64(b):
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_logits_match_numpy_float64_matmul(orc):
    rng = np.random.default_rng(0)
    R, H, V = 7, 96, 301
    hid = _bf16(rng.standard_normal((R, H)))
    w = _bf16(rng.standard_normal((V, H)))
    got = orc.lm_head_logits(hid, w)
    want = _f64(hid) @ _f64(w).T
    np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-12)
    sub = orc.lm_head_logits(hid, w, rows=[6, 2])
    np.testing.assert_array_equal(sub, got[[6, 2]])


def test_integer_inputs_give_exact_integer_logits(orc):
    rng = np.random.default_rng(1)
    R, H, V = 4, 256, 50
    hi = rng.integers(-8, 9, size=(R, H))
    wi = rng.integers(-8, 9, size=(V, H))
    got = orc.lm_head_logits(_bf16(hi), _bf16(wi))
    np.testing.assert_array_equal(got, (hi.astype(np.int64) @ wi.astype(np.int64).T).astype(np.float64))


def test_argmax_takes_the_first_maximum_on_ties(orc):
    rng = np.random.default_rng(2)
    R, H, V = 6, 32, 40
    hid = _bf16(rng.standard_normal((R, H)))
    w = _bf16(rng.standard_normal((V, H)))
    logits = orc.lm_head_logits(hid, w)
    best = logits.argmax(axis=1)
    w2 = w.copy()
    for r in range(R):  # copy the winning row to a lower index: a tie the lower index must win
        lo = int(rng.integers(0, best[r])) if best[r] > 0 else 0
        w2[lo] = w[best[r]]
    l2 = orc.lm_head_logits(hid, w2)
    am = orc.argmax_rows_f64(l2)
    np.testing.assert_array_equal(am, np.argmax(l2, axis=1))  # numpy returns the first occurrence
    assert (l2[np.arange(R), am] == l2.max(axis=1)).all()
