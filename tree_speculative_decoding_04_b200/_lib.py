"""ctypes binding of libtreeverify.so -- argument marshalling only.

Each function has the name of the C entry point it calls and takes torch tensors
that already live on the GPU; every step of the computation runs in the CUDA
library.  There is no fallback: if the library is missing or a call fails, an
exception is raised.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtreeverify.so")

TV_OK = 0
SEQ_BAD_PARENT = 1
SEQ_TOO_DEEP = 2
SEQ_TIMEOUT = 4
SEQ_BAD_GEOMETRY = 8
MAX_TREE_ROWS = 256
ATTN_PREFIX_READY = 1
ATTN_ROPE = 2

EXPORTS = (
    "tree_build_mask",
    "tree_attention_workspace_size",
    "tree_attention",
    "tree_attention_noalloc_max_scratch",
    "tree_attention_noalloc",
    "tree_accept",
    "tree_accept_lm_head_workspace_size",
    "tree_accept_lm_head",
    "kv_commit_realign",
    "tree_kv_write",
    "tv_status_string",
    "tv_last_cuda_error",
    "tv_version",
    "tv_set_wait_limit_ns",
)


class TVError(RuntimeError):
    pass


_lib = None


def load(path: str = LIB_PATH):
    """Load the shared library (built by build.py) and declare its signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise TVError(f"CUDA library not built: {path} (run __graft_entry__.build())")
    lib = ctypes.CDLL(path)
    P, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
    lib.tree_build_mask.argtypes = [P, i32, i32, i32, P, P, P, P]
    lib.tree_attention_workspace_size.argtypes = [i32, i32, i32, i32, i32, i64]
    lib.tree_attention_workspace_size.restype = ctypes.c_size_t
    lib.tree_attention.argtypes = [P, P, P, i64, P, P, P, P, i32, i32, i32, i32, i32, f32, P, P, ctypes.c_size_t,
                                   ctypes.c_uint, P, f32, P, i32, P]
    lib.tree_attention_noalloc_max_scratch.argtypes = []
    lib.tree_attention_noalloc_max_scratch.restype = ctypes.c_size_t
    lib.tree_attention_noalloc.argtypes = [P, P, P, i64, P, P, P, P, i32, i32, i32, i32, i32, f32, P, P]
    lib.tree_attention_noalloc.restype = ctypes.c_int
    lib.tree_accept.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, P, P, P, P, P]
    lib.tree_accept_lm_head_workspace_size.argtypes = [i32, i32]
    lib.tree_accept_lm_head_workspace_size.restype = ctypes.c_size_t
    lib.tree_accept_lm_head.argtypes = [P, P, P, P, P, P, P, i32, i32, i32, i32, i32, P, P, P, P, P, ctypes.c_size_t,
                                        P]
    lib.kv_commit_realign.argtypes = [P, P, i32, i32, i32, i32, i64, i32, P, P, P, i32, P, P, P, i32, P, P, P, i32, P]
    lib.tree_kv_write.argtypes = [P, P, P, P, i32, i32, i32, i32, i64, i32, P, P, P, f32, P, i32, P]
    for name in ("tree_build_mask", "tree_attention", "tree_accept", "tree_accept_lm_head", "kv_commit_realign",
                 "tree_kv_write"):
        getattr(lib, name).restype = ctypes.c_int
    lib.tv_status_string.argtypes = [ctypes.c_int]
    lib.tv_status_string.restype = ctypes.c_char_p
    lib.tv_last_cuda_error.restype = ctypes.c_int
    lib.tv_version.restype = ctypes.c_int
    lib.tv_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    lib.tv_set_wait_limit_ns.restype = None
    _lib = lib
    return lib


def _check(rc: int, what: str):
    if rc != TV_OK:
        lib = load()
        msg = lib.tv_status_string(rc).decode()
        if msg == "TV_ERR_CUDA":
            msg += f" (cudaError {lib.tv_last_cuda_error()})"
        raise TVError(f"{what}: {msg}")


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise TVError("tensor must live on the GPU")
    if not t.is_contiguous():
        raise TVError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t: torch.Tensor, dtype, shape, name):
    if t.dtype != dtype:
        raise TVError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise TVError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")


def tree_build_mask(parent, max_depth, anc_mask, depth, status, stream=None):
    """parent int32 [B][M+1] -> anc_mask uint32-as-int32 [B][M+1][W], depth [B][M+1], status [B]."""
    B, n = parent.shape
    W = (n + 31) // 32
    _need(parent, torch.int32, (B, n), "parent")
    _need(anc_mask, torch.int32, (B, n, W), "anc_mask")
    _need(depth, torch.int32, (B, n), "depth")
    _need(status, torch.int32, (B,), "status")
    rc = load().tree_build_mask(_ptr(parent), B, n - 1, int(max_depth), _ptr(anc_mask), _ptr(depth),
                                _ptr(status), _stream(stream))
    _check(rc, "tree_build_mask")


def tree_attention_workspace_size(B, M, Hq, Hkv, D, S_cap) -> int:
    """Bytes of device scratch tree_attention needs for this shape (0 = none)."""
    return int(load().tree_attention_workspace_size(B, M, Hq, Hkv, D, int(S_cap)))


def attention_workspace(B, M, Hq, Hkv, D, S_cap, device) -> torch.Tensor | None:
    """A device buffer of the workspace size (None when no workspace is needed)."""
    nbytes = tree_attention_workspace_size(B, M, Hq, Hkv, D, S_cap)
    if nbytes == 0:
        return None
    return torch.empty((nbytes + 15) // 16 * 16, dtype=torch.uint8, device=device)


def tree_attention(q, k, v, kv_start, kv_len, anc_mask, status, out, workspace=None, scale=None, stream=None,
                   flags=0, depth=None, rope_theta=0.0, slot=None):
    """q [B][M+1][Hq][D] bf16; k, v [B][Hkv][S_cap][D] bf16 (one layer) -> out like q.
    workspace: a uint8 device tensor of at least tree_attention_workspace_size bytes.
    flags: an OR of ATTN_PREFIX_READY (the launch just before this one on the
    stream writes neither the geometry, the slot map nor any prefix K/V column)
    and ATTN_ROPE (q is rotated to kv_len + depth[b][u] with base rope_theta).
    slot: int32 [B] cache slots; k, v are then a pool [n_slots][Hkv][S_cap][D]
    and kv_start / kv_len are [n_slots]."""
    B, n, Hq, D = q.shape
    Hkv, S_cap = k.shape[1], k.shape[2]
    NS = k.shape[0] if slot is not None else B
    _need(q, torch.bfloat16, (B, n, Hq, D), "q")
    _need(k, torch.bfloat16, (NS, Hkv, S_cap, D), "k")
    _need(v, torch.bfloat16, (NS, Hkv, S_cap, D), "v")
    _need(kv_start, torch.int32, (NS,), "kv_start")
    _need(kv_len, torch.int32, (NS,), "kv_len")
    if slot is not None:
        _need(slot, torch.int32, (B,), "slot")
    if flags & ATTN_ROPE:
        _need(depth, torch.int32, (B, n), "depth")
    _need(anc_mask, torch.int32, (B, n, (n + 31) // 32), "anc_mask")
    _need(status, torch.int32, (B,), "status")
    _need(out, torch.bfloat16, (B, n, Hq, D), "out")
    if scale is None:
        scale = D ** -0.5
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = load().tree_attention(_ptr(q), _ptr(k), _ptr(v), S_cap, _ptr(kv_start), _ptr(kv_len), _ptr(anc_mask),
                               _ptr(status), B, n - 1, Hq, Hkv, D, float(scale), _ptr(out), _ptr(workspace),
                               ws_bytes, int(flags), _ptr(depth) if flags & ATTN_ROPE else None,
                               float(rope_theta), _ptr(slot), NS, _stream(stream))
    _check(rc, "tree_attention")


def tree_accept(logits, draft, parent, depth, anc_mask, status, max_depth, argmax, accept_len, path, bonus,
                stream=None):
    B, n, V = logits.shape
    _need(logits, torch.float32, (B, n, V), "logits")
    for t, name in ((draft, "draft"), (parent, "parent"), (depth, "depth"), (argmax, "argmax")):
        _need(t, torch.int32, (B, n), name)
    _need(anc_mask, torch.int32, (B, n, (n + 31) // 32), "anc_mask")
    _need(status, torch.int32, (B,), "status")
    _need(accept_len, torch.int32, (B,), "accept_len")
    _need(path, torch.int32, (B, int(max_depth) + 1), "path")
    _need(bonus, torch.int32, (B,), "bonus")
    rc = load().tree_accept(_ptr(logits), _ptr(draft), _ptr(parent), _ptr(depth), _ptr(anc_mask), _ptr(status),
                            B, n - 1, V, int(max_depth), _ptr(argmax), _ptr(accept_len), _ptr(path), _ptr(bonus),
                            _stream(stream))
    _check(rc, "tree_accept")


def lm_head_workspace(B, M, device) -> torch.Tensor:
    """A device buffer of tree_accept_lm_head_workspace_size bytes."""
    nbytes = int(load().tree_accept_lm_head_workspace_size(B, M))
    return torch.empty((max(nbytes, 8) + 15) // 16 * 16, dtype=torch.uint8, device=device)


def tree_accept_lm_head(hidden, w_lm, draft, parent, depth, anc_mask, status, max_depth, argmax, accept_len, path,
                        bonus, workspace, stream=None):
    """hidden bf16 [B][M+1][H], w_lm bf16 [V][H] -> argmax of hidden @ w_lm^T per node
    (the logits are never stored), then the acceptance walk (as tree_accept)."""
    B, n, H = hidden.shape
    V = w_lm.shape[0]
    _need(hidden, torch.bfloat16, (B, n, H), "hidden")
    _need(w_lm, torch.bfloat16, (V, H), "w_lm")
    for t, name in ((draft, "draft"), (parent, "parent"), (depth, "depth"), (argmax, "argmax")):
        _need(t, torch.int32, (B, n), name)
    _need(anc_mask, torch.int32, (B, n, (n + 31) // 32), "anc_mask")
    _need(status, torch.int32, (B,), "status")
    _need(accept_len, torch.int32, (B,), "accept_len")
    _need(path, torch.int32, (B, int(max_depth) + 1), "path")
    _need(bonus, torch.int32, (B,), "bonus")
    ws_bytes = workspace.numel() * workspace.element_size()
    rc = load().tree_accept_lm_head(_ptr(hidden), _ptr(w_lm), _ptr(draft), _ptr(parent), _ptr(depth), _ptr(anc_mask),
                                    _ptr(status), B, n - 1, H, V, int(max_depth), _ptr(argmax), _ptr(accept_len),
                                    _ptr(path), _ptr(bonus), _ptr(workspace), ws_bytes, _stream(stream))
    _check(rc, "tree_accept_lm_head")


def kv_commit_realign(k_layer_ptrs, v_layer_ptrs, B, Hkv, D, S_cap, M, path, accept_len, status, max_depth,
                      kv_start, kv_len, max_len, realign, attn_mask=None, pos_ids=None, stream=None, slot=None):
    """k_layer_ptrs / v_layer_ptrs: int64 CUDA tensors [L] of layer base addresses
    (each layer a bf16 [B][Hkv][S_cap][D] buffer, or a pool [n_slots][Hkv][S_cap][D]
    with slot: int32 [B] cache slots, kv_start / kv_len / mask rows per slot)."""
    L = k_layer_ptrs.numel()
    NS = kv_start.shape[0] if slot is not None else B
    _need(k_layer_ptrs, torch.int64, (L,), "k_layer_ptrs")
    _need(v_layer_ptrs, torch.int64, (L,), "v_layer_ptrs")
    _need(path, torch.int32, (B, int(max_depth) + 1), "path")
    for t, name in ((accept_len, "accept_len"), (status, "status")):
        _need(t, torch.int32, (B,), name)
    for t, name in ((kv_start, "kv_start"), (kv_len, "kv_len")):
        _need(t, torch.int32, (NS,), name)
    if slot is not None:
        _need(slot, torch.int32, (B,), "slot")
    _need(max_len, torch.int32, (1,), "max_len")
    if attn_mask is not None:
        _need(attn_mask, torch.uint8, (NS, S_cap), "attn_mask")
    if pos_ids is not None:
        _need(pos_ids, torch.int32, (NS, S_cap), "pos_ids")
    rc = load().kv_commit_realign(_ptr(k_layer_ptrs), _ptr(v_layer_ptrs), L, B, Hkv, D, int(S_cap), M, _ptr(path),
                                  _ptr(accept_len), _ptr(status), int(max_depth), _ptr(kv_start), _ptr(kv_len),
                                  _ptr(max_len), int(realign), _ptr(attn_mask), _ptr(pos_ids), _ptr(slot), NS,
                                  _stream(stream))
    _check(rc, "kv_commit_realign")


def tree_kv_write(k_layer_ptrs, v_layer_ptrs, tree_k, tree_v, S_cap, kv_start, kv_len, stream=None, depth=None,
                  rope_theta=0.0, slot=None):
    """tree_k / tree_v bf16 [L][B][Hkv][M+1][D] -> the cache of every layer, at
    columns kv_start + kv_len + r (k_layer_ptrs / v_layer_ptrs as for
    kv_commit_realign).  depth int32 [B][M+1]: K rows are rotated to kv_len +
    depth with base rope_theta.  slot: int32 [B] cache slots of a pool (kv_start /
    kv_len then [n_slots])."""
    L, B, Hkv, n, D = tree_k.shape
    NS = kv_start.shape[0] if slot is not None else B
    _need(k_layer_ptrs, torch.int64, (L,), "k_layer_ptrs")
    _need(v_layer_ptrs, torch.int64, (L,), "v_layer_ptrs")
    _need(tree_k, torch.bfloat16, (L, B, Hkv, n, D), "tree_k")
    _need(tree_v, torch.bfloat16, (L, B, Hkv, n, D), "tree_v")
    _need(kv_start, torch.int32, (NS,), "kv_start")
    _need(kv_len, torch.int32, (NS,), "kv_len")
    if depth is not None:
        _need(depth, torch.int32, (B, n), "depth")
    if slot is not None:
        _need(slot, torch.int32, (B,), "slot")
    rc = load().tree_kv_write(_ptr(k_layer_ptrs), _ptr(v_layer_ptrs), _ptr(tree_k), _ptr(tree_v), L, B, Hkv, D,
                              int(S_cap), n - 1, _ptr(kv_start), _ptr(kv_len), _ptr(depth), float(rope_theta),
                              _ptr(slot), NS, _stream(stream))
    _check(rc, "tree_kv_write")


def set_wait_limit_ns(ns: int) -> None:
    """Testing hook: limit (ns) of tree_attention's pipeline waits for later
    launches; 0 restores the default (1 s)."""
    load().tv_set_wait_limit_ns(int(ns))


def layer_pointers(layers, device=None) -> torch.Tensor:
    """Device int64 tensor of the base addresses of a list of layer tensors."""
    dev = device or layers[0].device
    return torch.tensor([t.data_ptr() for t in layers], dtype=torch.int64, device=dev)
