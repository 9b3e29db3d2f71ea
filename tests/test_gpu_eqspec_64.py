"""The EQSPEC workload as written: 64 rounds from the seed on the eqspec shapes
(batch 8, GQA 32/8, head dim 128, prefixes U[512, 4096] left-padded, chain of 5
draft tokens, vocabulary 151936), two layers, the same calls the benchmark's
round replay makes (tree_kv_write, tree_attention with the prefix-ready flag,
tree_accept, kv_commit_realign with the repad), every round checked against
the oracle on the same inputs: accept results, geometry, attention mask and
position IDs bit for bit every round, attention on a seeded sample of rows
every round, and every content row of both layers every 8th round and at the
end ("Batch Speculative Decoding Done Right", methodology: EQSPEC)."""
import numpy as np
import pytest
import torch

import tree_speculative_decoding_04_b200 as tv
import workloads as W
from gpu_helpers import dev
from helpers import assert_attn_close
from tree_speculative_decoding_04_b200.verifier import TreeVerifier

pytestmark = pytest.mark.gpu


@pytest.mark.timeout(900)
def test_eqspec_64_rounds(orc):
    cfg = W.CONFIGS["eqspec"]
    L, rounds = 2, 64
    rng = np.random.default_rng(0)
    g = W.torch_generator(0, dev())
    B, n = cfg.B, cfg.M + 1
    parent = W.make_parents(cfg, rng)
    P = W.make_prefix_lengths(cfg, rng)
    ks, kl, S_cap = W.cache_geometry(cfg, P, extra_rows=rounds * n)
    ver = TreeVerifier(B, cfg.M, cfg.Hq, cfg.Hkv, cfg.D, cfg.V, L, S_cap, cfg.max_depth, realign=True,
                       device=dev(), with_mask_outputs=True)
    for layer in range(L):
        ver.k[layer].copy_(W.randn_bf16(ver.k[layer].shape, g, dev()))
        ver.v[layer].copy_(W.randn_bf16(ver.v[layer].shape, g, dev()))
    kh = [W.bf16_bits(t).copy() for t in ver.k]
    vh = [W.bf16_bits(t).copy() for t in ver.v]
    ver.kv_start.copy_(torch.as_tensor(ks))
    ver.kv_len.copy_(torch.as_tensor(kl))
    ver.parent.copy_(torch.as_tensor(parent))
    stream = torch.cuda.Stream(dev())
    am = torch.zeros((B, n), dtype=torch.int32, device=dev())
    sums = []
    for rnd in range(rounds):
        q = W.randn_bf16((L, B, n, cfg.Hq, cfg.D), g, dev())
        tk = W.randn_bf16((L, B, cfg.Hkv, n, cfg.D), g, dev())
        tvv = W.randn_bf16((L, B, cfg.Hkv, n, cfg.D), g, dev())
        logits = W.randn_f32((B, n, cfg.V), g, dev(), cfg.logit_sigma)
        draft = W.plant_drafts(logits, parent, cfg.p_plant, rng)
        ver.draft.copy_(torch.as_tensor(draft))
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            ver.build_mask(stream)
            for layer in range(L):
                tv.tree_kv_write(ver.k_ptrs[layer:layer + 1], ver.v_ptrs[layer:layer + 1], tk[layer:layer + 1],
                                 tvv[layer:layer + 1], S_cap, ver.kv_start, ver.kv_len, stream)
                tv.tree_attention(q[layer], ver.k[layer], ver.v[layer], ver.kv_start, ver.kv_len, ver.anc,
                                  ver.status, ver.out[layer], ver.workspace, stream=stream,
                                  flags=tv.ATTN_PREFIX_READY)
            tv.tree_accept(logits, ver.draft, ver.parent, ver.depth, ver.anc, ver.status, cfg.max_depth, am,
                           ver.accept_len, ver.path, ver.bonus, stream)
            ver.commit(stream)
        torch.cuda.synchronize()
        # the oracle, the same round
        anc, depth, st = orc.tree_build_mask(parent, cfg.max_depth)
        orc.tree_kv_write(kh, vh, W.bf16_bits(tk), W.bf16_bits(tvv), ks, kl)
        sel = np.stack([rng.integers(B, size=24), rng.integers(n, size=24), rng.integers(cfg.Hq, size=24)],
                       axis=1).astype(np.int32)
        for layer in range(L):
            ref = orc.tree_attention_rows(W.bf16_bits(q[layer]), kh[layer], vh[layer], ks, kl, parent, st, cfg.Hkv,
                                          sel)
            got = ver.out[layer].float().cpu().numpy()
            assert_attn_close(np.stack([got[b, u, h] for b, u, h in sel]), ref, f"eqspec 64 rounds, layer {layer}")
        o_am, al, path, bonus = orc.tree_accept(logits.cpu().numpy(), draft, parent, st, cfg.max_depth)
        np.testing.assert_array_equal(am.cpu().numpy(), o_am)
        np.testing.assert_array_equal(ver.accept_len.cpu().numpy(), al)
        np.testing.assert_array_equal(ver.path.cpu().numpy(), path)
        np.testing.assert_array_equal(ver.bonus.cpu().numpy(), bonus)
        ks2, kl2, ml, mask, pos = orc.kv_commit_realign(kh, vh, cfg.M, path, al, st, cfg.max_depth, ks, kl, 1)
        np.testing.assert_array_equal(ver.kv_start.cpu().numpy(), ks2)
        np.testing.assert_array_equal(ver.kv_len.cpu().numpy(), kl2)
        assert int(ver.max_len.item()) == ml
        np.testing.assert_array_equal(ver.attn_mask.cpu().numpy(), mask)
        np.testing.assert_array_equal(ver.pos_ids.cpu().numpy(), pos)
        assert ((ks2 + kl2) == ml).all()  # rectangular after every round
        if rnd % 8 == 7 or rnd == rounds - 1:
            for layer in range(L):
                gk, gv = W.bf16_bits(ver.k[layer]), W.bf16_bits(ver.v[layer])
                for b in range(B):
                    lo, hi = int(ks2[b]), int(ks2[b] + kl2[b])
                    np.testing.assert_array_equal(gk[b, :, lo:hi], kh[layer][b, :, lo:hi])
                    np.testing.assert_array_equal(gv[b, :, lo:hi], vh[layer][b, :, lo:hi])
        sums.append(int(al.sum()))
        ks, kl = ks2, kl2
    assert min(sums) >= 0 and len(set(sums)) > 1  # accept lengths vary over the rounds
