"""Whole verification steps through TreeVerifier (the four C-ABI calls chained on
one stream with programmatic dependent launches), compared with the oracle run
step by step on the same inputs: every layer's attention output, the accept
results, the committed cache and the new geometry -- over several EQSPEC rounds
on a ragged left-padded batch, and inside a CUDA graph."""
import numpy as np
import pytest
import torch

from helpers import assert_attn_close
from tree_speculative_decoding_04_b200.verifier import TreeVerifier
import workloads as W

pytestmark = pytest.mark.gpu


def _dev():
    return torch.device("cuda:0")


def _oracle_step(orc, cfg, kh, vh, qh, logits, parent, draft, ks, kl):
    anc, depth, st = orc.tree_build_mask(parent, cfg.max_depth)
    outs = [orc.tree_attention(qh[l], kh[l], vh[l], ks, kl, parent, st, cfg.Hkv) for l in range(len(kh))]
    am, al, path, bonus = orc.tree_accept(logits, draft, parent, st, cfg.max_depth)
    ks2, kl2, ml, mask, pos = orc.kv_commit_realign(kh, vh, cfg.M, path, al, st, cfg.max_depth, ks, kl,
                                                    int(cfg.left_padded))
    return outs, (al, path, bonus), (ks2, kl2, ml, mask, pos)


def _fill_round(ver, cfg, rng, g, kh, vh, qh, ks, kl):
    """New tree rows, queries, logits, tree and drafts for one round."""
    B, n = cfg.B, cfg.M + 1
    parent = W.make_parents(cfg, rng)
    for l in range(ver.L):
        ver.q[l].copy_(W.randn_bf16(ver.q[l].shape, g, _dev()))
        qh[l] = W.bf16_bits(ver.q[l]).copy()
        for which, dev_t, host_t in ((0, ver.k[l], kh[l]), (1, ver.v[l], vh[l])):
            rows = W.randn_bf16((B, cfg.Hkv, n, cfg.D), g, _dev())
            for b in range(B):
                c0 = int(ks[b] + kl[b])
                dev_t[b, :, c0:c0 + n].copy_(rows[b])
                host_t[b, :, c0:c0 + n] = W.bf16_bits(rows[b])
    ver.logits.copy_(W.randn_f32(ver.logits.shape, g, _dev(), cfg.logit_sigma))
    draft = W.plant_drafts(ver.logits, parent, cfg.p_plant, rng)
    ver.parent.copy_(torch.as_tensor(parent))
    ver.draft.copy_(torch.as_tensor(draft))
    return parent, draft


@pytest.mark.parametrize("name,L,rounds,graph", [("tiny", 1, 3, False), ("eqspec", 2, 6, False),
                                                 ("eqspec", 2, 4, True), ("mha7b", 3, 1, True)])
def test_rounds(orc, name, L, rounds, graph):
    cfg = W.CONFIGS[name]
    rng = np.random.default_rng(0)
    g = W.torch_generator(0, _dev())
    P = W.make_prefix_lengths(cfg, rng)
    ks, kl, S_cap = W.cache_geometry(cfg, P, extra_rows=rounds * (cfg.max_depth + 1))
    ver = TreeVerifier(cfg.B, cfg.M, cfg.Hq, cfg.Hkv, cfg.D, cfg.V, L, S_cap, cfg.max_depth,
                       realign=cfg.left_padded, device=_dev(), with_mask_outputs=True)
    for l in range(L):
        ver.k[l].copy_(W.randn_bf16(ver.k[l].shape, g, _dev()))
        ver.v[l].copy_(W.randn_bf16(ver.v[l].shape, g, _dev()))
    kh = [W.bf16_bits(t).copy() for t in ver.k]
    vh = [W.bf16_bits(t).copy() for t in ver.v]
    qh = [None] * L
    ver.kv_start.copy_(torch.as_tensor(ks))
    ver.kv_len.copy_(torch.as_tensor(kl))
    stream = torch.cuda.Stream()
    cg = None
    for rnd in range(rounds):
        parent, draft = _fill_round(ver, cfg, rng, g, kh, vh, qh, ks, kl)
        torch.cuda.synchronize()
        if graph:
            if cg is None:
                cg = torch.cuda.CUDAGraph()
                with torch.cuda.graph(cg, stream=stream):
                    ver.step(stream)
            cg.replay()  # capture does not run the work; replay does
        else:
            with torch.cuda.stream(stream):
                ver.step(stream)
        torch.cuda.synchronize()
        outs, (al, path, bonus), (ks2, kl2, ml, mask, pos) = _oracle_step(
            orc, cfg, kh, vh, qh, ver.logits.cpu().numpy(), parent, draft, ks, kl)
        for l in range(L):
            assert_attn_close(ver.out[l].float().cpu().numpy(), outs[l], f"{name} round {rnd} layer {l}")
        np.testing.assert_array_equal(ver.accept_len.cpu().numpy(), al)
        np.testing.assert_array_equal(ver.path.cpu().numpy(), path)
        np.testing.assert_array_equal(ver.bonus.cpu().numpy(), bonus)
        np.testing.assert_array_equal(ver.kv_start.cpu().numpy(), ks2)
        np.testing.assert_array_equal(ver.kv_len.cpu().numpy(), kl2)
        assert int(ver.max_len.item()) == ml
        np.testing.assert_array_equal(ver.attn_mask.cpu().numpy(), mask)
        np.testing.assert_array_equal(ver.pos_ids.cpu().numpy(), pos)
        for l in range(L):
            gk, gv = W.bf16_bits(ver.k[l]), W.bf16_bits(ver.v[l])
            for b in range(cfg.B):
                lo, hi = int(ks2[b]), int(ks2[b] + kl2[b])
                np.testing.assert_array_equal(gk[b, :, lo:hi], kh[l][b, :, lo:hi])
                np.testing.assert_array_equal(gv[b, :, lo:hi], vh[l][b, :, lo:hi])
            kh[l][:] = gk
            vh[l][:] = gv
        ks, kl = ks2, kl2


@pytest.mark.parametrize("name,L,rounds", [("tiny", 1, 2), ("eqspec", 2, 4), ("mha7b", 1, 1)])
def test_rounds_from_host(orc, name, L, rounds):
    """The end-to-end path: inputs staged in pinned host memory, copied in a
    section at a time on a copy stream, tree rows placed by tree_kv_write, results
    copied back -- against the oracle round by round."""
    cfg = W.CONFIGS[name]
    rng = np.random.default_rng(1)
    g = W.torch_generator(1, _dev())
    B, n = cfg.B, cfg.M + 1
    P = W.make_prefix_lengths(cfg, rng)
    ks, kl, S_cap = W.cache_geometry(cfg, P, extra_rows=rounds * (cfg.max_depth + 1))
    ver = TreeVerifier(cfg.B, cfg.M, cfg.Hq, cfg.Hkv, cfg.D, cfg.V, L, S_cap, cfg.max_depth,
                       realign=cfg.left_padded, device=_dev(), with_mask_outputs=True)
    for l in range(L):
        ver.k[l].copy_(W.randn_bf16(ver.k[l].shape, g, _dev()))
        ver.v[l].copy_(W.randn_bf16(ver.v[l].shape, g, _dev()))
    kh = [W.bf16_bits(t).copy() for t in ver.k]
    vh = [W.bf16_bits(t).copy() for t in ver.v]
    ver.kv_start.copy_(torch.as_tensor(ks))
    ver.kv_len.copy_(torch.as_tensor(kl))
    h = ver.pinned_inputs()
    stream = torch.cuda.Stream(_dev())
    for rnd in range(rounds):
        parent = W.make_parents(cfg, rng)
        q = W.randn_bf16((L, B, n, cfg.Hq, cfg.D), g, _dev())
        tk = W.randn_bf16((L, B, cfg.Hkv, n, cfg.D), g, _dev())
        tvv = W.randn_bf16((L, B, cfg.Hkv, n, cfg.D), g, _dev())
        logits = W.randn_f32((B, n, cfg.V), g, _dev(), cfg.logit_sigma)
        draft = W.plant_drafts(logits, parent, cfg.p_plant, rng)
        h["parent"].copy_(torch.as_tensor(parent))
        h["draft"].copy_(torch.as_tensor(draft))
        h["q"].copy_(q.cpu())
        h["tree_k"].copy_(tk.cpu())
        h["tree_v"].copy_(tvv.cpu())
        h["logits"].copy_(logits.cpu())
        res = ver.step_from_host(h, stream=stream)
        torch.cuda.synchronize()
        qh = [W.bf16_bits(q[l]) for l in range(L)]
        orc.tree_kv_write(kh, vh, W.bf16_bits(tk), W.bf16_bits(tvv), ks, kl)
        outs, (al, path, bonus), (ks2, kl2, ml, mask, pos) = _oracle_step(
            orc, cfg, kh, vh, qh, logits.cpu().numpy(), parent, draft, ks, kl)
        for l in range(L):
            assert_attn_close(ver.out[l].float().cpu().numpy(), outs[l], f"{name} host round {rnd} layer {l}")
        np.testing.assert_array_equal(res.accept_len.numpy(), al)
        np.testing.assert_array_equal(res.path.numpy(), path)
        np.testing.assert_array_equal(res.bonus.numpy(), bonus)
        np.testing.assert_array_equal(ver.kv_start.cpu().numpy(), ks2)
        np.testing.assert_array_equal(ver.kv_len.cpu().numpy(), kl2)
        for l in range(L):
            gk, gv = W.bf16_bits(ver.k[l]), W.bf16_bits(ver.v[l])
            for b in range(B):
                lo, hi = int(ks2[b]), int(ks2[b] + kl2[b])
                np.testing.assert_array_equal(gk[b, :, lo:hi], kh[l][b, :, lo:hi])
                np.testing.assert_array_equal(gv[b, :, lo:hi], vh[l][b, :, lo:hi])
            kh[l][:] = gk
            vh[l][:] = gv
        ks, kl = ks2, kl2
