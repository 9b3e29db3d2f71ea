"""GPU parity of tree_accept against the oracle: argmax rows, accepted length,
path and bonus token bit-exact, on every workload shape (full size), with ties,
odd vocabulary sizes (unaligned rows), single-token vocabularies, the largest
tree, and rejected sequences."""
import numpy as np
import pytest
import torch

from gpu_helpers import dev, gpu_accept, gpu_mask, i32, random_parents
import workloads as W

pytestmark = pytest.mark.gpu


def _check(orc, logits, draft, parent, max_depth, status_override=None):
    par, anc, depth, status = gpu_mask(parent, max_depth)
    if status_override is not None:
        status.copy_(i32(status_override))
    st_h = status.cpu().numpy()
    am, al, path, bonus = gpu_accept(logits, draft, par, depth, anc, status, max_depth)
    torch.cuda.synchronize()
    o_am, o_al, o_path, o_bonus = orc.tree_accept(logits.cpu().numpy(), draft, parent, st_h, max_depth)
    np.testing.assert_array_equal(am.cpu().numpy(), o_am)
    np.testing.assert_array_equal(al.cpu().numpy(), o_al)
    np.testing.assert_array_equal(path.cpu().numpy(), o_path)
    np.testing.assert_array_equal(bonus.cpu().numpy(), o_bonus)
    return o_al


@pytest.mark.parametrize("name", W.CONFIG_ORDER)
def test_config_full(orc, name):
    cfg = W.CONFIGS[name]
    rng = np.random.default_rng(0)
    parent = W.make_parents(cfg, rng)
    g = W.torch_generator(0, dev())
    logits = W.randn_f32((cfg.B, cfg.M + 1, cfg.V), g, dev(), cfg.logit_sigma)
    draft = W.plant_drafts(logits, parent, cfg.p_plant, rng)
    al = _check(orc, logits, draft, parent, cfg.max_depth)
    assert (al >= 0).all()


@pytest.mark.parametrize("V", [1, 2, 3, 5, 7, 1023, 2049, 4097, 32001, 151937])
def test_odd_vocab_and_ties(orc, V):
    rng = np.random.default_rng(V)
    B, M, md = 6, 20, 8
    parent = random_parents(B, M, md, rng)
    g = W.torch_generator(V, dev())
    logits = W.randn_f32((B, M + 1, V), g, dev())
    # plant ties of the row maximum at random columns in half of the rows
    lh = logits.cpu().numpy()
    for b in range(B):
        for u in range(0, M + 1, 2):
            cols = rng.integers(0, V, size=3)
            lh[b, u, cols] = lh[b, u].max() + 0.5
    logits = torch.as_tensor(lh, device=dev())
    draft = W.plant_drafts(logits, parent, 0.8, rng)
    _check(orc, logits, draft, parent, md)


def test_sibling_ties_and_small_vocab(orc):
    """Vocabulary of 2: siblings often carry the same token, so equal-depth accepted
    nodes are common and the lowest-row rule decides."""
    rng = np.random.default_rng(5)
    B, M, md = 64, 30, 10
    parent = random_parents(B, M, md, rng)
    g = W.torch_generator(5, dev())
    logits = W.randn_f32((B, M + 1, 2), g, dev())
    draft = rng.integers(0, 2, size=(B, M + 1)).astype(np.int32)
    _check(orc, logits, draft, parent, md)


def test_largest_tree(orc):
    rng = np.random.default_rng(9)
    B, M, md = 3, 255, 40
    parent = random_parents(B, M, md, rng)
    g = W.torch_generator(9, dev())
    logits = W.randn_f32((B, M + 1, 3000), g, dev())
    draft = W.plant_drafts(logits, parent, 0.9, rng)
    _check(orc, logits, draft, parent, md)


def test_rejected_sequences(orc):
    rng = np.random.default_rng(4)
    B, M, md = 5, 12, 6
    parent = random_parents(B, M, md, rng)
    parent[2, 5] = 9  # malformed
    g = W.torch_generator(4, dev())
    logits = W.randn_f32((B, M + 1, 500), g, dev())
    draft = W.plant_drafts(logits, parent, 0.9, rng)
    al = _check(orc, logits, draft, parent, md, status_override=[0, 0, 1, 8, 0])
    assert al[2] == -1 and al[3] == -1


def test_chain_accepts_prefix(orc):
    rng = np.random.default_rng(8)
    B, M = 16, 5
    parent = np.stack([W.tree_chain(M)] * B)
    g = W.torch_generator(8, dev())
    logits = W.randn_f32((B, M + 1, 151936), g, dev())
    draft = W.plant_drafts(logits, parent, 0.6, rng)
    _check(orc, logits, draft, parent, M)
