"""Pins for the oracle's tree-masked attention (CPU only).

"EAGLE-Pangu: Accelerator-Safe Tree Speculative Decoding on Ascend NPUs",
methodology C: a query node sees the committed prefix and, inside the tree, only
its ancestors and itself.  The oracle is checked against torch's
scaled_dot_product_attention (an independent textbook routine, in float64 with an
explicit boolean mask) through reductions that the definition fixes:
  * a chain tree is ordinary causal attention over prefix ++ chain,
  * a single-node tree (M = 0) is plain decode attention,
  * any node equals the last query of causal attention over prefix ++ its root path,
plus a leak test, relabelling invariance, the GQA head map, and the equal-keys
closed form.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import workloads as W


def _bits(t):
    return W.bf16_bits(t)


def _f64(t):
    return t.to(torch.float64)


def _setup(B, M, Hq, Hkv, D, P, seed, parent=None, left_pad=0):
    g = W.torch_generator(seed, "cpu")
    rng = np.random.default_rng(seed)
    S_cap = left_pad + P + M + 1 + 3
    q = W.randn_bf16((B, M + 1, Hq, D), g, "cpu")
    k = W.randn_bf16((B, Hkv, S_cap, D), g, "cpu")
    v = W.randn_bf16((B, Hkv, S_cap, D), g, "cpu")
    if parent is None:
        parent = np.stack([W.tree_uniform_depth(M, 100, rng) for _ in range(B)])
    ks = np.full(B, left_pad, np.int32)
    kl = np.full(B, P, np.int32)
    st = np.zeros(B, np.int32)
    return q, k, v, parent.astype(np.int32), ks, kl, st, S_cap


def _oracle(orc, q, k, v, parent, ks, kl, st, Hkv):
    return orc.tree_attention(_bits(q), _bits(k), _bits(v), ks, kl, parent, st, Hkv)


def _sdpa_rows(qrows, keys, vals, mask):
    """qrows [n][D], keys/vals [t][D], mask [n][t] bool -> [n][D] float64."""
    return F.scaled_dot_product_attention(
        _f64(qrows)[None, None], _f64(keys)[None, None], _f64(vals)[None, None], attn_mask=torch.as_tensor(mask)[None, None]
    )[0, 0].numpy()


@pytest.mark.parametrize("P,D", [(0, 64), (7, 64), (33, 128)])
def test_chain_equals_causal(orc, P, D):
    M, Hq, Hkv = 9, 2, 2
    q, k, v, par, ks, kl, st, S_cap = _setup(1, M, Hq, Hkv, D, P, 11, parent=W.tree_chain(M)[None])
    out = _oracle(orc, q, k, v, par, ks, kl, st, Hkv)
    n = M + 1
    for h in range(Hq):
        keys = k[0, h, : P + n]
        vals = v[0, h, : P + n]
        mask = np.zeros((n, P + n), bool)
        for u in range(n):
            mask[u, : P + u + 1] = True  # causal: prefix and chain rows up to itself
        ref = _sdpa_rows(q[0, :, h], keys, vals, mask)
        np.testing.assert_allclose(out[0, :, h], ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("P", [1, 64, 300])
def test_single_node_equals_decode(orc, P):
    M, Hq, Hkv, D = 0, 4, 4, 64
    q, k, v, par, ks, kl, st, S_cap = _setup(2, M, Hq, Hkv, D, P, 5)
    out = _oracle(orc, q, k, v, par, ks, kl, st, Hkv)
    for b in range(2):
        for h in range(Hq):
            ref = F.scaled_dot_product_attention(
                _f64(q[b, 0, h])[None, None, None], _f64(k[b, h, : P + 1])[None, None], _f64(v[b, h, : P + 1])[None, None]
            )[0, 0, 0].numpy()
            np.testing.assert_allclose(out[b, 0, h], ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_node_equals_causal_over_its_path(orc, seed):
    B, M, Hq, Hkv, D, P = 2, 14, 4, 2, 64, 20
    q, k, v, par, ks, kl, st, S_cap = _setup(B, M, Hq, Hkv, D, P, seed, left_pad=5)
    out = _oracle(orc, q, k, v, par, ks, kl, st, Hkv)
    G = Hq // Hkv
    for b in range(B):
        for u in range(M + 1):
            path = []
            x = u
            while True:
                path.append(x)
                if x == 0:
                    break
                x = int(par[b][x])
            path = path[::-1]
            cols = list(range(5, 5 + P)) + [5 + P + r for r in path]
            for h in range(Hq):
                kk = k[b, h // G, cols]
                vv = v[b, h // G, cols]
                ref = F.scaled_dot_product_attention(
                    _f64(q[b, u, h])[None, None, None], _f64(kk)[None, None], _f64(vv)[None, None]
                )[0, 0, 0].numpy()
                np.testing.assert_allclose(out[b, u, h], ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("P", [0, 3])
def test_no_leak_across_branches(orc, P):
    """Non-ancestor tree rows carry V = 1e4: any leak would show at O(1)."""
    M, Hq, Hkv, D = 12, 2, 2, 64
    q, k, v, par, ks, kl, st, S_cap = _setup(1, M, Hq, Hkv, D, P, 3)
    anc, _, _ = orc.tree_build_mask(par, 100)
    out_clean = _oracle(orc, q, k, v, par, ks, kl, st, Hkv)
    for u in range(M + 1):
        vv = v.clone()
        for r in range(M + 1):
            if not (int(anc[0, u, 0]) >> r) & 1:
                vv[0, :, P + r] = 1e4
        o = _oracle(orc, q, k, vv, par, ks, kl, st, Hkv)
        np.testing.assert_allclose(o[0, u], out_clean[0, u], rtol=0, atol=1e-12)
        assert np.abs(o[0, u]).max() < 10


def test_relabelling_permutes_outputs(orc):
    """Renumber the nodes in another topological order; outputs follow the nodes."""
    M, Hq, Hkv, D, P = 10, 2, 1, 64, 9
    par = np.array([[0, 0, 0, 1, 1, 2, 3, 3, 5, 0, 9]], np.int32)
    q, k, v, _, ks, kl, st, S_cap = _setup(1, M, Hq, Hkv, D, P, 8, parent=par)
    out = _oracle(orc, q, k, v, par, ks, kl, st, Hkv)
    # new order: a breadth-first relabelling; new row i holds old node perm[i]
    perm = [0, 9, 2, 1, 10, 5, 4, 3, 8, 7, 6]
    inv = {old: new for new, old in enumerate(perm)}
    par2 = np.array([[0] + [inv[int(par[0, perm[i]])] for i in range(1, M + 1)]], np.int32)
    assert all(par2[0, i] < i for i in range(1, M + 1))
    q2 = q[:, perm]
    k2, v2 = k.clone(), v.clone()
    k2[0, :, P : P + M + 1] = k[0, :, [P + perm[i] for i in range(M + 1)]]
    v2[0, :, P : P + M + 1] = v[0, :, [P + perm[i] for i in range(M + 1)]]
    out2 = _oracle(orc, q2, k2, v2, par2, ks, kl, st, Hkv)
    np.testing.assert_allclose(out2[0], out[0, perm], rtol=1e-12, atol=1e-12)


def test_gqa_head_map(orc):
    B, M, Hq, Hkv, D, P = 1, 6, 8, 2, 64, 17
    q, k, v, par, ks, kl, st, S_cap = _setup(B, M, Hq, Hkv, D, P, 4, parent=W.tree_chain(M)[None])
    out = _oracle(orc, q, k, v, par, ks, kl, st, Hkv)
    n = M + 1
    mask = np.zeros((n, P + n), bool)
    for u in range(n):
        mask[u, : P + u + 1] = True
    kk = k[0, :, : P + n].repeat_interleave(Hq // Hkv, dim=0)  # q head h -> kv head h // G
    vv = v[0, :, : P + n].repeat_interleave(Hq // Hkv, dim=0)
    ref = F.scaled_dot_product_attention(
        _f64(q[0].transpose(0, 1)), _f64(kk), _f64(vv), attn_mask=torch.as_tensor(mask)[None]
    ).transpose(0, 1).numpy()
    np.testing.assert_allclose(out[0], ref, rtol=1e-12, atol=1e-12)


def test_equal_keys_give_mean_of_values(orc):
    """All keys equal -> uniform softmax -> the mean of the attended values."""
    M, Hq, Hkv, D, P = 5, 1, 1, 64, 4
    par = np.array([[0, 0, 1, 1, 3, 0]], np.int32)
    q, k, v, _, ks, kl, st, S_cap = _setup(1, M, Hq, Hkv, D, P, 2, parent=par)
    k[:] = k[0, 0, 0]
    out = _oracle(orc, q, k, v, par, ks, kl, st, Hkv)
    anc_rows = {0: [0], 1: [0, 1], 2: [0, 1, 2], 3: [0, 1, 3], 4: [0, 1, 3, 4], 5: [0, 5]}
    vv = v.to(torch.float64).numpy()
    for u, rows in anc_rows.items():
        cols = list(range(P)) + [P + r for r in rows]
        np.testing.assert_allclose(out[0, u, 0], vv[0, 0, cols].mean(axis=0), rtol=1e-12, atol=1e-12)


def test_invalid_sequences_give_zero_rows(orc):
    B, M, Hq, Hkv, D, P = 3, 4, 2, 2, 64, 6
    q, k, v, par, ks, kl, st, S_cap = _setup(B, M, Hq, Hkv, D, P, 9)
    st[1] = orc.BAD_PARENT
    kl2 = kl.copy()
    kl2[2] = S_cap  # tree rows would run past the cache
    out = _oracle(orc, q, k, v, par, ks, kl2, st, Hkv)
    assert not out[1].any() and not out[2].any() and out[0].any()


def test_left_padding_is_invisible(orc):
    """The same sequence, once at column 0 and once behind 11 pad columns of garbage."""
    M, Hq, Hkv, D, P = 7, 2, 2, 64, 13
    q, k, v, par, ks, kl, st, S_cap = _setup(1, M, Hq, Hkv, D, P, 6)
    out0 = _oracle(orc, q, k, v, par, ks, kl, st, Hkv)
    pad = 11
    g = W.torch_generator(99, "cpu")
    kp = torch.cat([W.randn_bf16((1, Hkv, pad, D), g, "cpu", 50.0), k], dim=2)
    vp = torch.cat([W.randn_bf16((1, Hkv, pad, D), g, "cpu", 50.0), v], dim=2)
    out1 = _oracle(orc, q, kp, vp, par, ks + pad, kl, st, Hkv)
    np.testing.assert_array_equal(out0, out1)
