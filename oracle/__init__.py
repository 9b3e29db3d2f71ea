"""CPU oracle for the tree speculative-decoding verification step.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference arm are the only callers.  The product
package never imports this module, and this module never imports the product
package.  The arithmetic lives in ``oracle.c`` (plain C, no CUDA headers); this
file only compiles it with gcc and marshals numpy arrays through ctypes.

Sources: "EAGLE-Pangu: Accelerator-Safe Tree Speculative Decoding on Ascend
NPUs" (methodology A-C, results) and "Batch Speculative Decoding Done Right"
(methodology: synchronization invariants, EQSPEC).  Each C function names the
passage it follows.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

BAD_PARENT = 1
TOO_DEEP = 2
BAD_GEOMETRY = 8


_LIB_OMP = os.path.join(_HERE, "liboracle_omp.so")


def build(force: bool = False, openmp: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, -O2, no fast-math).
    openmp=True builds the same source with -fopenmp into liboracle_omp.so: the
    loops over independent output rows then run on every host core (the
    arithmetic of each row is unchanged).  Only the benchmark's CPU arms use it."""
    out = _LIB_OMP if openmp else _LIB
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(_SRC):
        tmp = out + ".tmp%d" % os.getpid()
        extra = ["-fopenmp"] if openmp else []
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math"] + extra + ["-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, out)
    return out


_lib = None
_use_openmp = False


def use_openmp(on: bool = True) -> None:
    """Select the all-cores build for every later call (must be chosen before
    the first call; the benchmark's CPU arms only)."""
    global _use_openmp
    if _lib is not None and bool(on) != _use_openmp:
        raise RuntimeError("oracle library already loaded")
    _use_openmp = bool(on)


def threads() -> int:
    """Host threads the loaded oracle build uses (1 unless the all-cores build is in use)."""
    if not _use_openmp:
        return 1
    n = os.environ.get("OMP_NUM_THREADS")
    return int(n) if n else (len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count())


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build(openmp=_use_openmp))
        P = ctypes.c_void_p
        i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
        _lib.oracle_tree_build_mask.argtypes = [P, i32, i32, i32, P, P, P]
        _lib.oracle_tree_attention_rows.argtypes = [P, P, P, i64, P, P, P, P, i32, i32, i32, i32, i32, f64, f64, P,
                                                    i64, P]
        _lib.oracle_tree_attention.argtypes = [P, P, P, i64, P, P, P, P, i32, i32, i32, i32, i32, f64, f64, P]
        _lib.oracle_argmax_rows.argtypes = [P, i64, i32, P]
        _lib.oracle_tree_accept.argtypes = [P, P, P, P, i32, i32, i32, i32, P, P, P, P]
        _lib.oracle_kv_commit_realign.argtypes = [P, P, i32, i32, i32, i32, i64, i32, P, P, P, i32, P, P, P, i32, P, P]
        _lib.oracle_tree_kv_write.argtypes = [P, P, P, P, i32, i32, i32, i32, i64, i32, P, P, P, f64]
        _lib.oracle_rope_rows.argtypes = [P, P, i64, i32, f64]
        _lib.oracle_lm_head_logits.argtypes = [P, P, P, i64, i32, i32, P]
        _lib.oracle_argmax_rows_f64.argtypes = [P, i64, i32, P]
        _lib.oracle_round_bf16.argtypes = [P, i64, P]
        for f in (
            _lib.oracle_tree_build_mask,
            _lib.oracle_tree_attention_rows,
            _lib.oracle_tree_attention,
            _lib.oracle_argmax_rows,
            _lib.oracle_tree_accept,
            _lib.oracle_kv_commit_realign,
        ):
            f.restype = ctypes.c_int
    return _lib


def _c(a: np.ndarray, dtype) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=dtype)
    return a


def _p(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def _bits16(a: np.ndarray) -> np.ndarray:
    """bf16 payload as uint16 bits (accepts uint16 bits or torch-exported int16 views)."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return a
    if a.dtype == np.int16:
        return a.view(np.uint16)
    raise TypeError("bf16 tensors must be passed as uint16 bit patterns")


def tree_build_mask(parent: np.ndarray, max_depth: int):
    """parent int32 [B][M+1] -> (anc_mask uint32 [B][M+1][W], depth int32 [B][M+1], status int32 [B])."""
    parent = _c(parent, np.int32)
    B, n = parent.shape
    M = n - 1
    W = (n + 31) // 32
    anc = np.zeros((B, n, W), np.uint32)
    depth = np.zeros((B, n), np.int32)
    status = np.zeros((B,), np.int32)
    rc = lib().oracle_tree_build_mask(_p(parent), B, M, max_depth, _p(anc), _p(depth), _p(status))
    if rc:
        raise ValueError("oracle_tree_build_mask rc=%d" % rc)
    return anc, depth, status


def tree_attention(q, k, v, kv_start, kv_len, parent, status, Hkv: int, scale: float | None = None,
                   rope_base: float = 0.0):
    """q bf16-bits [B][M+1][Hq][D]; k, v bf16-bits [B][Hkv][S_cap][D] -> float64 [B][M+1][Hq][D].
    rope_base > 0: each query row is first rotated to position kv_len + depth(u)."""
    q, k, v = _bits16(q), _bits16(k), _bits16(v)
    B, n, Hq, D = q.shape
    S_cap = k.shape[2]
    assert k.shape == (B, Hkv, S_cap, D) and v.shape == k.shape
    ks, kl = _c(kv_start, np.int32), _c(kv_len, np.int32)
    par, st = _c(parent, np.int32), _c(status, np.int32)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    out = np.zeros((B, n, Hq, D), np.float64)
    rc = lib().oracle_tree_attention(
        _p(q), _p(k), _p(v), S_cap, _p(ks), _p(kl), _p(par), _p(st), B, n - 1, Hq, Hkv, D, scale,
        float(rope_base), _p(out)
    )
    if rc:
        raise ValueError("oracle_tree_attention rc=%d" % rc)
    return out


def tree_attention_rows(q, k, v, kv_start, kv_len, parent, status, Hkv: int, sel, scale: float | None = None,
                        rope_base: float = 0.0):
    """Only the rows listed in sel ([n][3] of (b, u, q_head)) -> float64 [n][D]."""
    q, k, v = _bits16(q), _bits16(k), _bits16(v)
    B, n, Hq, D = q.shape
    S_cap = k.shape[2]
    ks, kl = _c(kv_start, np.int32), _c(kv_len, np.int32)
    par, st = _c(parent, np.int32), _c(status, np.int32)
    sel = _c(sel, np.int32).reshape(-1, 3)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    out = np.zeros((sel.shape[0], D), np.float64)
    rc = lib().oracle_tree_attention_rows(
        _p(q), _p(k), _p(v), S_cap, _p(ks), _p(kl), _p(par), _p(st), B, n - 1, Hq, Hkv, D, scale,
        float(rope_base), _p(sel), sel.shape[0], _p(out),
    )
    if rc:
        raise ValueError("oracle_tree_attention_rows rc=%d" % rc)
    return out


def argmax_rows(logits):
    logits = _c(logits, np.float32)
    V = logits.shape[-1]
    rows = logits.size // V
    out = np.zeros((rows,), np.int32)
    lib().oracle_argmax_rows(_p(logits), rows, V, _p(out))
    return out.reshape(logits.shape[:-1])


def tree_accept(logits, draft, parent, status, max_depth: int):
    """-> (argmax [B][M+1], accept_len [B], path [B][max_depth+1], bonus [B])."""
    logits = _c(logits, np.float32)
    B, n, V = logits.shape
    dr, par, st = _c(draft, np.int32), _c(parent, np.int32), _c(status, np.int32)
    am = np.zeros((B, n), np.int32)
    al = np.zeros((B,), np.int32)
    path = np.zeros((B, max_depth + 1), np.int32)
    bonus = np.zeros((B,), np.int32)
    rc = lib().oracle_tree_accept(
        _p(logits), _p(dr), _p(par), _p(st), B, n - 1, V, max_depth, _p(am), _p(al), _p(path), _p(bonus)
    )
    if rc:
        raise AssertionError("oracle_tree_accept: recurrence and brute force disagree (rc=%d)" % rc)
    return am, al, path, bonus


def kv_commit_realign(k_layers, v_layers, M: int, path, accept_len, status, max_depth: int,
                      kv_start, kv_len, realign: int, with_mask: bool = True, with_status: bool = False):
    """In place on the uint16 arrays in k_layers / v_layers (each [B][Hkv][S_cap][D]).

    Returns (kv_start', kv_len', max_len', attn_mask or None, pos_ids or None);
    with_status=True appends status' (input status with TV_SEQ_BAD_GEOMETRY OR-ed in)."""
    L = len(k_layers)
    assert L == len(v_layers) and L >= 1
    B, Hkv, S_cap, D = k_layers[0].shape
    for a in list(k_layers) + list(v_layers):
        assert a.dtype == np.uint16 and a.flags.c_contiguous and a.shape == (B, Hkv, S_cap, D)
    kp = (ctypes.c_void_p * L)(*[a.ctypes.data for a in k_layers])
    vp = (ctypes.c_void_p * L)(*[a.ctypes.data for a in v_layers])
    ks = _c(kv_start, np.int32).copy()
    kl = _c(kv_len, np.int32).copy()
    pth, al = _c(path, np.int32), _c(accept_len, np.int32)
    st = _c(status, np.int32).copy()
    ml = np.zeros((1,), np.int32)
    am = np.zeros((B, S_cap), np.uint8) if with_mask else None
    pos = np.zeros((B, S_cap), np.int32) if with_mask else None
    rc = lib().oracle_kv_commit_realign(
        ctypes.cast(kp, ctypes.c_void_p), ctypes.cast(vp, ctypes.c_void_p), L, B, Hkv, D, S_cap, M,
        _p(pth), _p(al), _p(st), max_depth, _p(ks), _p(kl), _p(ml), int(realign),
        _p(am) if with_mask else None, _p(pos) if with_mask else None,
    )
    if rc:
        raise ValueError("oracle_kv_commit_realign rc=%d" % rc)
    if with_status:
        return ks, kl, int(ml[0]), am, pos, st
    return ks, kl, int(ml[0]), am, pos


def tree_kv_write(k_layers, v_layers, tree_k, tree_v, kv_start, kv_len, depth=None, rope_base: float = 0.0):
    """In place on the uint16 arrays in k_layers / v_layers (each [B][Hkv][S_cap][D]):
    tree_k / tree_v uint16 [L][B][Hkv][M+1][D] go to columns kv_start + kv_len + r.
    depth [B][M+1] with rope_base > 0: K rows are rotated to position kv_len + depth
    and stored as the nearest bf16."""
    L = len(k_layers)
    assert L == len(v_layers) and L >= 1
    B, Hkv, S_cap, D = k_layers[0].shape
    for a in list(k_layers) + list(v_layers):
        assert a.dtype == np.uint16 and a.flags.c_contiguous and a.shape == (B, Hkv, S_cap, D)
    tk, tv = _c(tree_k, np.uint16), _c(tree_v, np.uint16)
    assert tk.shape == tv.shape and tk.shape[:3] == (L, B, Hkv) and tk.shape[4] == D
    M = tk.shape[3] - 1
    kp = (ctypes.c_void_p * L)(*[a.ctypes.data for a in k_layers])
    vp = (ctypes.c_void_p * L)(*[a.ctypes.data for a in v_layers])
    ks, kl = _c(kv_start, np.int32), _c(kv_len, np.int32)  # kept alive across the call
    dep = None if depth is None else _c(depth, np.int32)
    rc = lib().oracle_tree_kv_write(ctypes.cast(kp, ctypes.c_void_p), ctypes.cast(vp, ctypes.c_void_p), _p(tk),
                                    _p(tv), L, B, Hkv, D, S_cap, M, _p(ks), _p(kl),
                                    None if dep is None else _p(dep), float(rope_base))
    if rc:
        raise ValueError("oracle_tree_kv_write rc=%d" % rc)


def rope_rows(x, pos, base: float):
    """Rotary embedding: rows x [n][D] (float64) rotated by the angles of their
    positions pos [n]; returns a new array."""
    x = np.array(x, np.float64, copy=True, order="C")
    n, D = x.shape
    pos = _c(pos, np.float64)
    assert pos.shape == (n,)
    rc = lib().oracle_rope_rows(_p(x), _p(pos), n, D, float(base))
    if rc:
        raise ValueError("oracle_rope_rows rc=%d" % rc)
    return x


def round_bf16(x):
    """Nearest bf16 (ties to even) of each float64, as uint16 bits."""
    x = _c(x, np.float64)
    out = np.zeros(x.shape, np.uint16)
    lib().oracle_round_bf16(_p(x), x.size, _p(out))
    return out


# ----------------------------------------------------------------------------- cache-slot pools
# "Batch Speculative Decoding Done Right", methodology: EXSPEC keeps a pool of
# sequences and batches any of them together (same-length groups need no
# realignment).  With a slot map, batch row b's cache is slot slots[b] of a pool
# whose layers are [n_slots][Hkv][S_cap][D] and whose geometry is [n_slots].  The
# pool versions below are the plainest reading of that: gather the batch's
# slots, run the batch function above unchanged, scatter the result back.  A
# slot outside [0, n_slots) is skipped and flagged like a bad geometry.

def _valid_slots(slots, n_slots):
    slots = np.asarray(slots, np.int64)
    return slots, (slots >= 0) & (slots < n_slots)


def pool_tree_kv_write(k_pool, v_pool, slots, tree_k, tree_v, kv_start, kv_len, depth=None, rope_base: float = 0.0):
    """tree_kv_write on the batch rows' slots of a pool (in place)."""
    n_slots = k_pool[0].shape[0]
    slots, ok = _valid_slots(slots, n_slots)
    idx = np.nonzero(ok)[0]
    if len(idx) == 0:
        return
    s = slots[idx]
    kb = [np.ascontiguousarray(k[s]) for k in k_pool]
    vb = [np.ascontiguousarray(v[s]) for v in v_pool]
    tree_kv_write(kb, vb, np.asarray(tree_k)[:, idx], np.asarray(tree_v)[:, idx], np.asarray(kv_start)[s],
                  np.asarray(kv_len)[s], None if depth is None else np.asarray(depth)[idx], rope_base)
    for layer in range(len(k_pool)):
        k_pool[layer][s] = kb[layer]
        v_pool[layer][s] = vb[layer]


def pool_tree_attention(q, k_pool, v_pool, slots, kv_start, kv_len, parent, status, Hkv: int,
                        rope_base: float = 0.0):
    """tree_attention with batch row b reading cache slot slots[b]; rows whose slot
    is outside the pool are zero."""
    n_slots = k_pool.shape[0]
    slots, ok = _valid_slots(slots, n_slots)
    st = np.asarray(status, np.int32).copy()
    st[~ok] |= BAD_GEOMETRY
    s = np.where(ok, slots, 0)
    return tree_attention(q, np.ascontiguousarray(k_pool[s]), np.ascontiguousarray(v_pool[s]),
                          np.asarray(kv_start)[s], np.asarray(kv_len)[s], parent, st, Hkv, rope_base=rope_base)


def pool_kv_commit_realign(k_pool, v_pool, slots, M: int, path, accept_len, status, max_depth: int, kv_start, kv_len,
                           realign: int, attn_mask=None, pos_ids=None):
    """kv_commit_realign of a batch of pool slots, in place on the pool layers and
    on the pool geometry kv_start / kv_len ([n_slots], int32, modified).  Returns
    (max_len, status') ; attn_mask / pos_ids ([n_slots][S_cap]) rows of the
    batch's slots are rewritten when given."""
    n_slots = k_pool[0].shape[0]
    slots, ok = _valid_slots(slots, n_slots)
    st = np.asarray(status, np.int32).copy()
    st[~ok] |= BAD_GEOMETRY
    idx = np.nonzero(ok)[0]
    if len(idx) == 0:
        return 0, st
    s = slots[idx]
    kb = [np.ascontiguousarray(k[s]) for k in k_pool]
    vb = [np.ascontiguousarray(v[s]) for v in v_pool]
    ks2, kl2, ml, am, pos, st2 = kv_commit_realign(kb, vb, M, np.asarray(path)[idx], np.asarray(accept_len)[idx],
                                                   st[idx], max_depth, np.asarray(kv_start)[s],
                                                   np.asarray(kv_len)[s], realign, with_mask=True, with_status=True)
    for layer in range(len(k_pool)):
        k_pool[layer][s] = kb[layer]
        v_pool[layer][s] = vb[layer]
    kv_start[s] = ks2
    kv_len[s] = kl2
    st[idx] = st2
    if attn_mask is not None:
        attn_mask[s] = am
    if pos_ids is not None:
        pos_ids[s] = pos
    return ml, st


# ----------------------------------------------------------------------------- LM head
def lm_head_logits(hidden, w, rows=None):
    """Exact (double) logits of the selected rows: hidden bf16-bits [R][H], w bf16-bits
    [V][H] -> float64 [len(rows)][V] (all rows by default)."""
    hidden, w = _bits16(hidden), _bits16(w)
    H = hidden.shape[-1]
    hidden = hidden.reshape(-1, H)
    V = w.shape[0]
    assert w.shape == (V, H)
    rows = np.arange(hidden.shape[0], dtype=np.int32) if rows is None else _c(rows, np.int32)
    out = np.zeros((len(rows), V), np.float64)
    rc = lib().oracle_lm_head_logits(_p(hidden), _p(w), _p(rows), len(rows), H, V, _p(out))
    if rc:
        raise ValueError("oracle_lm_head_logits rc=%d" % rc)
    return out


def argmax_rows_f64(x):
    """First maximum of each row of a float64 array."""
    x = _c(x, np.float64)
    V = x.shape[-1]
    out = np.zeros((x.size // V,), np.int32)
    lib().oracle_argmax_rows_f64(_p(x), x.size // V, V, _p(out))
    return out.reshape(x.shape[:-1])
