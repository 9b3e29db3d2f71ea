"""GPU test of tree_attention_noalloc, the allocation-free variant of tree attention.

Some callers cannot allocate device memory -- a serving process whose memory
pool already owns the whole GPU, or a plugin whose host framework gives it no
device allocator.  tree_attention_noalloc serves them: the key-split partials go
to a fixed scratch array inside the library instead of a caller workspace.
This file checks, through the C ABI, that two calls in a row give the same
output as tree_attention with a caller-provided workspace (within the attention
tolerance of the other tests), and that every split plan of this GPU fits the
fixed scratch.  It runs last so that a failure here leaves every other test run.
"""
import ctypes

import numpy as np
import pytest
import torch

import tree_speculative_decoding_04_b200 as tv
import workloads as W
from helpers import assert_attn_close

pytestmark = pytest.mark.gpu


def _p(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _inputs(name, seed):
    cfg = W.CONFIGS[name]
    dev = torch.device("cuda:0")
    st = W.make_step(cfg, seed=seed, device=dev, with_logits=False)
    B, n = cfg.B, cfg.M + 1
    par = torch.as_tensor(st.parent, device=dev)
    anc = torch.empty((B, n, (n + 31) // 32), dtype=torch.int32, device=dev)
    depth = torch.empty((B, n), dtype=torch.int32, device=dev)
    status = torch.empty((B,), dtype=torch.int32, device=dev)
    tv.tree_build_mask(par, cfg.max_depth, anc, depth, status)
    ks = torch.as_tensor(st.kv_start, device=dev)
    kl = torch.as_tensor(st.kv_len, device=dev)
    return cfg, st, anc, status, ks, kl


def _noalloc(lib, cfg, st, anc, status, ks, kl, out, stream):
    return lib.tree_attention_noalloc(
        _p(st.q), _p(st.k), _p(st.v), st.S_cap, _p(ks), _p(kl), _p(anc), _p(status), cfg.B, cfg.M, cfg.Hq,
        cfg.Hkv, cfg.D, ctypes.c_float(cfg.D ** -0.5), _p(out), ctypes.c_void_p(stream))


def _with_workspace(lib, cfg, st, anc, status, ks, kl, out, stream):
    nbytes = lib.tree_attention_workspace_size(cfg.B, cfg.M, cfg.Hq, cfg.Hkv, cfg.D, st.S_cap)
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=out.device)
    rc = lib.tree_attention(
        _p(st.q), _p(st.k), _p(st.v), st.S_cap, _p(ks), _p(kl), _p(anc), _p(status), cfg.B, cfg.M, cfg.Hq,
        cfg.Hkv, cfg.D, ctypes.c_float(cfg.D ** -0.5), _p(out), _p(ws), nbytes, 0, None, ctypes.c_float(0.0), None, 0,
        ctypes.c_void_p(stream))
    return rc, ws


def test_noalloc_matches_the_workspace_entry_point_on_two_calls(orc):
    lib = tv.load()
    cap = lib.tree_attention_noalloc_max_scratch()
    first = _inputs("mha7b", seed=3)
    second = _inputs("eqspec", seed=4)
    for cfg, st, *_ in (first, second):
        need = lib.tree_attention_workspace_size(cfg.B, cfg.M, cfg.Hq, cfg.Hkv, cfg.D, st.S_cap)
        assert 0 < need <= cap  # both shapes go through the scratch array
    stream = torch.cuda.current_stream().cuda_stream
    outs = []
    # two calls in a row, no synchronisation in between: the second reuses the scratch
    for cfg, st, anc, status, ks, kl in (first, second):
        out = torch.full_like(st.q, float("nan"))
        assert _noalloc(lib, cfg, st, anc, status, ks, kl, out, stream) == 0
        outs.append(out)
    torch.cuda.synchronize()
    for (cfg, st, anc, status, ks, kl), got in zip((first, second), outs):
        ref = torch.full_like(st.q, float("nan"))
        rc, ws = _with_workspace(lib, cfg, st, anc, status, ks, kl, ref, stream)
        assert rc == 0
        torch.cuda.synchronize()
        g = got.float().cpu().numpy()
        r = ref.float().cpu().numpy()
        assert np.isfinite(g).all()
        assert_attn_close(g, r, f"noalloc vs workspace ({cfg.name})")
        # and against the oracle itself, so that a fault the two entry points
        # share cannot pass: every row of sequence 0 and a seeded sample
        rng = np.random.default_rng(7)
        n = cfg.M + 1
        sel = [(0, u, h) for u in range(n) for h in range(cfg.Hq)]
        sel += [(int(rng.integers(cfg.B)), int(rng.integers(n)), int(rng.integers(cfg.Hq))) for _ in range(64)]
        sel = np.array(sel, np.int32)
        st_h = status.cpu().numpy()
        o = orc.tree_attention_rows(W.bf16_bits(st.q), W.bf16_bits(st.k), W.bf16_bits(st.v), st.kv_start,
                                    st.kv_len, st.parent, st_h, cfg.Hkv, sel)
        assert_attn_close(np.stack([g[b, u, h] for b, u, h in sel]), o, f"noalloc vs oracle ({cfg.name})")


def test_noalloc_scratch_holds_every_split_plan():
    """The key-split plan adds splits only while (query tiles x splits) stays
    within 2 CTAs per SM, so the partials never exceed 2 x SMs x 128 rows x 130
    floats (19.7 MB on 148 SMs): on this GPU every shape that tree_attention
    serves fits the fixed scratch, and the size check that refuses larger
    workspaces is never reached.  The sweep reaches that bound exactly."""
    lib = tv.load()
    cap = lib.tree_attention_noalloc_max_scratch()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    bound = 2 * sms * 128 * 130 * 4
    worst = 0
    for Hq, Hkv in ((1, 1), (8, 8), (32, 32), (32, 8), (28, 4), (64, 8)):
        for M in (3, 16, 63, 127, 255):
            for S_cap in (64, 4096, 65536):
                for B in range(1, 301):
                    need = lib.tree_attention_workspace_size(B, M, Hq, Hkv, 128, S_cap)
                    assert need <= min(cap, bound), (B, M, Hq, Hkv, S_cap, need, cap, bound)
                    worst = max(worst, need)
    assert worst == bound
