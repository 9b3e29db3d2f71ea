"""Small helpers shared by the test modules (fixture parsing, tolerances)."""
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

# Attention tolerance: pass iff |gpu - ref| <= ATOL + RTOL * |ref| elementwise.
ATOL = 1e-2
RTOL = 2e-2


def load_golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = line.split(":", 1)
            vals = val.split()
            try:
                out[key.strip()] = np.array([int(x) for x in vals], np.int64)
            except ValueError:
                out[key.strip()] = np.array([float(x) for x in vals], np.float64)
    return out


# Raw error statistics of every attention comparison of the session, by label:
# max |gpu - ref| over all elements, and max |gpu - ref| / |ref| over the
# elements with |ref| >= 0.1 (the max-abs 1e-2 / max-rel 2e-2 figures of the
# attention tolerance, which the allclose bar above combines).  Printed at the
# end of the session.
ERR_STATS = {}


def error_stats(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(got - ref)
    big = np.abs(ref) >= 0.1
    return {"max_abs": float(err.max()) if err.size else 0.0,
            "max_rel_ref_ge_0.1": float((err[big] / np.abs(ref[big])).max()) if big.any() else 0.0,
            "elements": int(err.size)}


def assert_attn_close(got, ref, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    ERR_STATS[what or "attention"] = error_stats(got, ref)
    err = np.abs(got - ref)
    bad = err > ATOL + RTOL * np.abs(ref)
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(
            f"{what}: {int(bad.sum())} elements out of tolerance; first at {tuple(i)}: "
            f"got {got[tuple(i)]!r} ref {ref[tuple(i)]!r}; max abs err {err.max():.3e}"
        )
    return float(err.max()) if err.size else 0.0
