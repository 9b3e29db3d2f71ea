"""Pins of the oracle's rotary position embedding of tree rows and its use in
tree attention and in the tree-row append.

The pages fix only that position IDs must run contiguously over the attended
positions ("Batch Speculative Decoding Done Right", section 2, position-ID
contiguity); the rotation is the published rotary embedding (RoFormer) in the
half-split arrangement, and a tree node u sits at position kv_len + depth(u).
Pins: hand-worked values (tests/golden/rope_d4_d8.txt), the identity at
position 0, norm preservation, the relative-position property, the bf16
rounding against torch's own conversion, and tree attention with rotation
against causal attention (torch SDPA, float64) over each node's root path.
"""
import math

import numpy as np
import torch

from helpers import load_golden


def test_rope_hand_worked_values(orc):
    g = load_golden("rope_d4_d8.txt")
    out4 = orc.rope_rows(g["d4_x"].astype(np.float64)[None], [3.0], 10000.0)[0]
    np.testing.assert_allclose(out4, g["d4_out"], rtol=0, atol=1e-14)
    out8 = orc.rope_rows(g["d8_x"].astype(np.float64)[None], [1.0], 10000.0)[0]
    np.testing.assert_allclose(out8, g["d8_out"], rtol=0, atol=1e-14)


def test_rope_position_zero_is_identity_and_norms_are_kept(orc):
    rng = np.random.default_rng(0)
    x = rng.standard_normal((6, 128))
    np.testing.assert_array_equal(orc.rope_rows(x, np.zeros(6), 10000.0), x)
    y = orc.rope_rows(x, rng.integers(0, 40000, size=6).astype(np.float64), 500000.0)
    h = 64
    np.testing.assert_allclose(x[:, :h] ** 2 + x[:, h:] ** 2, y[:, :h] ** 2 + y[:, h:] ** 2, rtol=1e-12, atol=1e-12)


def test_rope_relative_position_property(orc):
    """<R(m) q, R(n) k> = <R(m - n) q, k>: the score depends on the distance only."""
    rng = np.random.default_rng(1)
    D = 128
    for m, n in ((5, 3), (9000, 8990), (70, 700), (32768, 0)):
        q = rng.standard_normal(D)
        k = rng.standard_normal(D)
        lhs = orc.rope_rows(q[None], [m], 10000.0)[0] @ orc.rope_rows(k[None], [n], 10000.0)[0]
        rhs = orc.rope_rows(q[None], [m - n], 10000.0)[0] @ k
        assert abs(lhs - rhs) <= 1e-9 * max(1.0, abs(rhs)), (m, n, lhs, rhs)


def test_bf16_rounding_matches_torch(orc):
    rng = np.random.default_rng(2)
    # values exactly representable in float32, so torch's float32 -> bf16
    # conversion (round to nearest, ties to even) rounds them once as well
    x = rng.standard_normal(4096).astype(np.float32).astype(np.float64)
    ties = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8), 2.5 + 2.0 ** -7, 0.0, -0.0])
    x = np.concatenate([x, ties])
    want = torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(orc.round_bf16(x), want)
    assert list(orc.round_bf16(ties[:2])) == [0x3F80, 0x3F82]


def _bits_to_f64(u16):
    return (np.asarray(u16, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_kv_write_rotates_k_rows_only(orc):
    rng = np.random.default_rng(3)
    B, Hkv, D, M, L = 2, 2, 64, 6, 1
    par = np.array([[0, 0, 1, 1, 2, 4, 0], [0, 0, 0, 2, 3, 4, 5]], np.int32)
    depth = np.array([[0, 1, 2, 2, 3, 3, 1], [0, 1, 1, 2, 3, 4, 5]], np.int32)
    ks, kl = np.array([0, 3], np.int32), np.array([10, 4], np.int32)
    S_cap = 24
    tk = orc.round_bf16(rng.standard_normal((L, B, Hkv, M + 1, D)))
    tv = orc.round_bf16(rng.standard_normal((L, B, Hkv, M + 1, D)))
    k = [np.zeros((B, Hkv, S_cap, D), np.uint16)]
    v = [np.zeros((B, Hkv, S_cap, D), np.uint16)]
    orc.tree_kv_write(k, v, tk, tv, ks, kl, depth=depth, rope_base=10000.0)
    for b in range(B):
        for h in range(Hkv):
            c0 = ks[b] + kl[b]
            pos = (kl[b] + depth[b]).astype(np.float64)
            want = orc.round_bf16(orc.rope_rows(_bits_to_f64(tk[0, b, h]), pos, 10000.0))
            np.testing.assert_array_equal(k[0][b, h, c0:c0 + M + 1], want)
            np.testing.assert_array_equal(v[0][b, h, c0:c0 + M + 1], tv[0, b, h])
    del par


def test_tree_attention_with_rope_is_causal_attention_on_each_path(orc):
    """Node u with rotation = the last query of causal attention over the prefix
    followed by u's root path, every path row placed at its position (prefix
    kv_len + depth): torch SDPA in float64 on explicitly rotated inputs."""
    import workloads as W

    rng = np.random.default_rng(4)
    B, Hq, Hkv, D, M, P = 1, 4, 2, 64, 12, 9
    base = 10000.0
    par = W.tree_uniform_depth(M, 5, rng)[None].astype(np.int32)
    anc, depth, st = orc.tree_build_mask(par, 100)
    S_cap = P + M + 1
    q = orc.round_bf16(rng.standard_normal((B, M + 1, Hq, D)))
    k = orc.round_bf16(rng.standard_normal((B, Hkv, S_cap, D)))  # prefix rows: stored as they are
    v = orc.round_bf16(rng.standard_normal((B, Hkv, S_cap, D)))
    tk = orc.round_bf16(rng.standard_normal((1, B, Hkv, M + 1, D)))
    tv = orc.round_bf16(rng.standard_normal((1, B, Hkv, M + 1, D)))
    ks, kl = np.zeros(B, np.int32), np.full(B, P, np.int32)
    kk, vv = [k.copy()], [v.copy()]
    orc.tree_kv_write(kk, vv, tk, tv, ks, kl, depth=depth, rope_base=base)
    out = orc.tree_attention(q, kk[0], vv[0], ks, kl, par, st, Hkv, rope_base=base)
    G = Hq // Hkv
    for u in range(M + 1):
        path = []
        x = u
        while True:
            path.append(x)
            if x == 0:
                break
            x = par[0, x]
        path = path[::-1]
        for h in range(Hq):
            hk = h // G
            qr = orc.rope_rows(_bits_to_f64(q[0, u, h])[None], [P + depth[0, u]], base)
            keys = np.concatenate([_bits_to_f64(kk[0][0, hk, :P]), _bits_to_f64(kk[0][0, hk, [P + r for r in path]])])
            vals = np.concatenate([_bits_to_f64(vv[0][0, hk, :P]), _bits_to_f64(vv[0][0, hk, [P + r for r in path]])])
            ref = torch.nn.functional.scaled_dot_product_attention(
                torch.tensor(qr)[None, None], torch.tensor(keys)[None, None], torch.tensor(vals)[None, None],
                scale=1.0 / math.sqrt(D))[0, 0, 0].numpy()
            np.testing.assert_allclose(out[0, u, h], ref, rtol=1e-10, atol=1e-12)
            # the rotated path keys are the raw tree rows turned to kv_len + depth
            for j, r in enumerate(path):
                assert depth[0, r] == j  # positions along the path run on from the prefix without a gap
