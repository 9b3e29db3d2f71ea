"""GPU parity of tree_accept_lm_head (the LM-head GEMM with the argmax fused into
its epilogue, then the acceptance walk) against the oracle's exact logits.

The oracle forms every logit in double from the bf16 inputs (each product is
exact); the kernel accumulates in fp32 on the tensor cores, so the two argmax
decisions can differ only where the two largest logits lie within the fp32
accumulation bound of each other:  eps = 2 H 2^-24 sum_h |hidden_h w_h|.
Rows whose top two exact logits are more than 2 eps apart must give the
oracle's index exactly; every row's index must reach the exact maximum within
eps.  The acceptance results must equal the oracle walk on the kernel's argmax,
and the oracle's own argmax where no row is that close.
"""
import numpy as np
import pytest
import torch

import tree_speculative_decoding_04_b200 as tv
import workloads as W
from gpu_helpers import dev, gpu_mask, i32

pytestmark = pytest.mark.gpu

CASES = [
    # name, B, M, H, V, max_depth, sampled rows (None: all)
    ("small", 2, 16, 256, 1000, 10, None),
    ("mha7b", 1, 64, 4096, 32000, 6, None),
    ("eqspec", 8, 5, 4096, 151936, 5, 12),
    ("stress", 16, 128, 8192, 128256, 12, 6),
]


def _abs_bits(b):
    return np.asarray(b, np.uint16) & np.uint16(0x7FFF)


@pytest.mark.parametrize("name,B,M,H,V,max_depth,nsample", CASES, ids=[c[0] for c in CASES])
def test_lm_head_argmax_and_accept(orc, name, B, M, H, V, max_depth, nsample):
    rng = np.random.default_rng(11)
    g = W.torch_generator(12, dev())
    n = M + 1
    parent = np.stack([W.tree_uniform_depth(M, max_depth, rng) for _ in range(B)]).astype(np.int32)
    hidden = W.randn_bf16((B, n, H), g, dev())
    w = W.randn_bf16((V, H), g, dev(), sigma=H ** -0.5)
    # planted drafts from fp32 logits (input generation only)
    lg32 = (hidden.float().reshape(B * n, H) @ w.float().T).reshape(B, n, V)
    draft = W.plant_drafts(lg32, parent, 0.7, rng)
    del lg32
    par, anc, depth, status = gpu_mask(parent, max_depth)
    am = torch.full((B, n), -7, dtype=torch.int32, device=dev())
    al = torch.full((B,), -7, dtype=torch.int32, device=dev())
    path = torch.full((B, max_depth + 1), -7, dtype=torch.int32, device=dev())
    bonus = torch.full((B,), -7, dtype=torch.int32, device=dev())
    ws = tv.lm_head_workspace(B, M, dev())
    ws.fill_(0xAB)  # the kernel clears what it needs
    tv.tree_accept_lm_head(hidden, w, i32(draft), par, depth, anc, status, max_depth, am, al, path, bonus, ws)
    torch.cuda.synchronize()
    assert int(status.abs().sum()) == 0
    g_am = am.cpu().numpy().reshape(-1)
    hb, wb = W.bf16_bits(hidden).reshape(-1, H), W.bf16_bits(w)
    rows = np.arange(B * n, dtype=np.int32)
    if nsample is not None:
        rows = np.unique(np.concatenate([np.arange(min(n, nsample)), rng.integers(0, B * n, size=nsample)]))
        rows = rows.astype(np.int32)
    exact = orc.lm_head_logits(hb, wb, rows)
    absb = orc.lm_head_logits(_abs_bits(hb), _abs_bits(wb), rows)
    eps = 2.0 * H * 2.0 ** -24 * absb.max(axis=1)
    o_am = orc.argmax_rows_f64(exact)
    top = exact.max(axis=1)
    srt = np.sort(exact, axis=1)
    gap = srt[:, -1] - srt[:, -2]
    chosen = exact[np.arange(len(rows)), g_am[rows]]
    assert (chosen >= top - eps).all(), "an argmax misses the exact maximum by more than the fp32 bound"
    clear = gap > 2 * eps
    np.testing.assert_array_equal(g_am[rows][clear], o_am[clear])
    # the bound is a worst case, several times the real error: still, the test
    # must not be vacuous
    assert clear.mean() > 0.4, clear.mean()
    # the walk, on the kernel's argmax and (where nothing is close) on the oracle's
    st_h = np.zeros(B, np.int32)
    onehot = np.zeros((B, n, V), np.float32)
    onehot[np.arange(B)[:, None], np.arange(n)[None, :], g_am.reshape(B, n)] = 1.0
    o = orc.tree_accept(onehot, draft, parent, st_h, max_depth)
    np.testing.assert_array_equal(al.cpu().numpy(), o[1])
    np.testing.assert_array_equal(path.cpu().numpy(), o[2])
    np.testing.assert_array_equal(bonus.cpu().numpy(), o[3])


def test_lm_head_matches_tree_accept_on_materialised_logits():
    """The fused path and tree_accept over the same logits written out (here from
    an fp32 matrix product, ties being the only possible difference) agree."""
    rng = np.random.default_rng(13)
    g = W.torch_generator(14, dev())
    B, M, H, V, md = 4, 20, 512, 3000, 8
    n = M + 1
    parent = np.stack([W.tree_uniform_depth(M, md, rng) for _ in range(B)]).astype(np.int32)
    hidden = W.randn_bf16((B, n, H), g, dev())
    w = W.randn_bf16((V, H), g, dev(), sigma=H ** -0.5)
    lg = (hidden.float().reshape(B * n, H) @ w.float().T).reshape(B, n, V).contiguous()
    draft = i32(W.plant_drafts(lg, parent, 0.8, rng))
    par, anc, depth, status = gpu_mask(parent, md)
    outs = []
    for fused in (True, False):
        am = torch.zeros((B, n), dtype=torch.int32, device=dev())
        al = torch.zeros((B,), dtype=torch.int32, device=dev())
        pth = torch.zeros((B, md + 1), dtype=torch.int32, device=dev())
        bn = torch.zeros((B,), dtype=torch.int32, device=dev())
        if fused:
            tv.tree_accept_lm_head(hidden, w, draft, par, depth, anc, status, md, am, al, pth, bn,
                                   tv.lm_head_workspace(B, M, dev()))
        else:
            tv.tree_accept(lg, draft, par, depth, anc, status, md, am, al, pth, bn)
        torch.cuda.synchronize()
        outs.append((am.cpu(), al.cpu(), pth.cpu(), bn.cpu()))
    same = (outs[0][0] == outs[1][0]).float().mean().item()
    assert same > 0.98
    if torch.equal(outs[0][0], outs[1][0]):
        for a, b in zip(outs[0], outs[1]):
            assert torch.equal(a, b)
