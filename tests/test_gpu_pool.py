"""GPU parity of cross-batch scheduling (EXSPEC) against the oracle: a pool of
sequences, each in its own cache slot, runs several rounds; every round the
SequencePool picks a batch (equal lengths: per-sequence-length commit; else the
EQSPEC repad), and the GPU step through the slot map (tree_kv_write,
tree_attention, tree_accept, kv_commit_realign) is compared with the oracle's
pool functions on the same inputs: accept results, geometry, mask / position
rows and every content row of the batch's slots bit for bit, attention at the
usual tolerance.  ("Batch Speculative Decoding Done Right", methodology:
EXSPEC.)"""
import numpy as np
import pytest
import torch

import workloads as W
from gpu_helpers import dev
from helpers import assert_attn_close
from tree_speculative_decoding_04_b200.pool import FALLBACK, PoolVerifier, SequencePool

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize(
    "tree,graphed,repad",
    [("uniform_depth", False, True), ("chain", False, True), ("uniform_depth", True, True), ("chain", True, True),
     ("uniform_depth", True, False)],
    ids=["uniform_depth-eager", "chain-eager", "uniform_depth-graphs", "chain-graphs", "ragged_fallback-graphs"])
def test_pool_rounds_against_the_oracle(orc, tree, graphed, repad):
    """Eager launches, or the step's CUDA graphs captured once per (batch size,
    mode) and replayed with each round's slot map.  repad: fallback batches take
    the EQSPEC repad (the pages' EXSPEC); else they commit per sequence like
    grouped ones (the slot map's per-sequence geometry needs no alignment)."""
    rng = np.random.default_rng(3 if tree == "chain" else 4)
    g = W.torch_generator(5, dev())
    n_slots, B, L, Hq, Hkv, D, M, max_depth, V = 10, 4, 2, 8, 2, 128, 5, 5, 2048
    rounds = 12
    lengths0 = rng.choice([300, 517, 1000], size=n_slots).astype(np.int32)
    S_cap = int(lengths0.max()) + (rounds + 1) * (M + 1) + 8
    pv = PoolVerifier(n_slots, B, M, Hq, Hkv, D, V, L, S_cap, max_depth, device=dev())
    for layer in range(L):
        pv.k[layer].copy_(W.randn_bf16(pv.k[layer].shape, g, dev()))
        pv.v[layer].copy_(W.randn_bf16(pv.v[layer].shape, g, dev()))
    pv.kv_len.copy_(torch.as_tensor(lengths0))
    kh = [W.bf16_bits(t).copy() for t in pv.k]
    vh = [W.bf16_bits(t).copy() for t in pv.v]
    ks_h = np.zeros(n_slots, np.int32)
    kl_h = lengths0.copy()
    mask_h = np.zeros((n_slots, S_cap), np.uint8)
    pos_h = np.zeros((n_slots, S_cap), np.int32)
    pool = SequencePool(lengths0, batch=B, max_wait=4)
    side = torch.cuda.Stream(dev())
    modes = set()
    for rnd in range(rounds):
        slots, mode = pool.next_batch()
        modes.add(mode)
        Bb = len(slots)
        if tree == "chain":
            parent = np.stack([W.tree_chain(M)] * Bb).astype(np.int32)
        else:
            parent = np.stack([W.tree_uniform_depth(M, max_depth, rng) for _ in range(Bb)]).astype(np.int32)
        pv.parent[:Bb].copy_(torch.as_tensor(parent))
        pv.logits[:Bb].copy_(W.randn_f32((Bb, M + 1, V), g, dev()))
        draft = W.plant_drafts(pv.logits[:Bb], parent, 0.7, rng)
        pv.draft[:Bb].copy_(torch.as_tensor(draft))
        pv.q[:, :Bb].copy_(W.randn_bf16((L, Bb, M + 1, Hq, D), g, dev()))
        pv.tree_k[:, :Bb].copy_(W.randn_bf16((L, Bb, Hkv, M + 1, D), g, dev()))
        pv.tree_v[:, :Bb].copy_(W.randn_bf16((L, Bb, Hkv, M + 1, D), g, dev()))
        realign = 1 if (mode == FALLBACK and repad) else 0
        if graphed:
            torch.cuda.synchronize()  # the inputs above are on the default stream
            pv.set_slots(slots, side)
            pv.step_graphed(Bb, realign, side)
        else:
            pv.set_slots(slots)
            pv.step(Bb, realign)
        torch.cuda.synchronize()
        # the oracle on the same inputs
        anc, depth, st = orc.tree_build_mask(parent, max_depth)
        orc.pool_tree_kv_write(kh, vh, slots, W.bf16_bits(pv.tree_k[:, :Bb]), W.bf16_bits(pv.tree_v[:, :Bb]),
                               ks_h, kl_h)
        for layer in range(L):
            ref = orc.pool_tree_attention(W.bf16_bits(pv.q[layer, :Bb]), kh[layer], vh[layer], slots, ks_h, kl_h,
                                          parent, st, Hkv)
            assert_attn_close(pv.out[layer, :Bb].float().cpu().numpy(), ref, f"pool attention ({tree})")
        am, al, path, bonus = orc.tree_accept(pv.logits[:Bb].cpu().numpy(), draft, parent, st, max_depth)
        np.testing.assert_array_equal(pv.accept_len[:Bb].cpu().numpy(), al)
        np.testing.assert_array_equal(pv.path[:Bb].cpu().numpy(), path)
        np.testing.assert_array_equal(pv.bonus[:Bb].cpu().numpy(), bonus)
        ml, st2 = orc.pool_kv_commit_realign(kh, vh, slots, M, path, al, st, max_depth, ks_h, kl_h, realign,
                                             mask_h, pos_h)
        np.testing.assert_array_equal(pv.kv_start.cpu().numpy(), ks_h)
        np.testing.assert_array_equal(pv.kv_len.cpu().numpy(), kl_h)
        np.testing.assert_array_equal(pv.status[:Bb].cpu().numpy(), st2)
        assert int(pv.max_len.item()) == ml
        gm, gp = pv.attn_mask.cpu().numpy(), pv.pos_ids.cpu().numpy()
        for s in slots:
            np.testing.assert_array_equal(gm[s], mask_h[s])
            np.testing.assert_array_equal(gp[s], pos_h[s])
        for layer in range(L):
            gk, gv = W.bf16_bits(pv.k[layer]), W.bf16_bits(pv.v[layer])
            for s in range(n_slots):  # every slot's content, batched this round or not
                lo, hi = ks_h[s], ks_h[s] + kl_h[s]
                np.testing.assert_array_equal(gk[s, :, lo:hi], kh[layer][s, :, lo:hi])
                np.testing.assert_array_equal(gv[s, :, lo:hi], vh[layer][s, :, lo:hi])
        pool.commit(slots, al)
    assert FALLBACK in modes and "grouped" in modes
