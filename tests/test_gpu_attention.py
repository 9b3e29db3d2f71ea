"""GPU parity of tree_attention against the oracle.

Tolerance (bf16 inputs, fp32 accumulation, bf16 output): |gpu - ref| <= 1e-2 +
2e-2 |ref| elementwise.  Small and mid-size workloads are compared on every
output row; the two largest are compared on a seeded sample of rows (plus every
row of sequence 0) in the launch configuration the benchmark uses.  Also: the
leak test (non-ancestor V rows = 1e4), invalid sequences give zero rows, GQA
groups, head dims 64/128, empty prefixes, single-node trees and the largest
tree the kernels take.
"""
import numpy as np
import pytest
import torch

from gpu_helpers import dev, gpu_attention, gpu_mask, i32
from helpers import assert_attn_close
import workloads as W

pytestmark = pytest.mark.gpu


def _run(orc, q, k, v, parent, kv_start, kv_len, max_depth=1000, status_override=None, sel=None, flags=0):
    par, anc, depth, status = gpu_mask(parent, max_depth)
    if status_override is not None:
        status.copy_(i32(status_override))
    st_h = status.cpu().numpy()
    out = gpu_attention(q, k, v, kv_start, kv_len, anc, status, flags=flags)
    torch.cuda.synchronize()
    qb, kb, vb = W.bf16_bits(q), W.bf16_bits(k), W.bf16_bits(v)
    Hkv = k.shape[1]
    got = out.float().cpu().numpy()
    if sel is None:
        ref = orc.tree_attention(qb, kb, vb, kv_start, kv_len, parent, st_h, Hkv)
        return got, ref, status
    ref = orc.tree_attention_rows(qb, kb, vb, kv_start, kv_len, parent, st_h, Hkv, sel)
    got = np.stack([got[b, u, h] for b, u, h in sel])
    return got, ref, status


def _inputs(B, M, Hq, Hkv, D, P, seed, left_padded=False, tree="uniform", max_depth=1000, slack=5):
    rng = np.random.default_rng(seed)
    g = W.torch_generator(seed, dev())
    if np.isscalar(P):
        P = np.full(B, P, np.int32)
    P = np.asarray(P, np.int32)
    pmax = int(P.max())
    kv_start = (pmax - P).astype(np.int32) if left_padded else np.zeros(B, np.int32)
    S_cap = pmax + M + 1 + slack
    if tree == "chain":
        parent = np.stack([W.tree_chain(M)] * B)
    else:
        parent = np.stack([W.tree_uniform_depth(M, max_depth, rng) for _ in range(B)])
    q = W.randn_bf16((B, M + 1, Hq, D), g, dev())
    k = W.randn_bf16((B, Hkv, S_cap, D), g, dev())
    v = W.randn_bf16((B, Hkv, S_cap, D), g, dev())
    return q, k, v, parent.astype(np.int32), kv_start, P.copy()


@pytest.mark.parametrize(
    "B,M,Hq,Hkv,D,P",
    [
        (1, 16, 4, 4, 64, 128),  # tiny
        (1, 0, 4, 4, 64, 77),  # single node = decode
        (2, 5, 8, 2, 128, 0),  # empty prefix: tree only
        (3, 9, 6, 3, 64, [1, 100, 333]),  # ragged, odd G
        (1, 31, 16, 16, 128, 1000),
        (2, 33, 8, 1, 128, 500),  # MQA, two mask words
        (1, 255, 2, 1, 128, 200),  # largest tree
        (4, 20, 12, 4, 128, [64, 65, 127, 129]),  # tile edges
        (2, 85, 6, 2, 128, [70, 300]),  # 258 query rows: three query tiles, the last with 2 rows
    ],
)
def test_parity_full(orc, B, M, Hq, Hkv, D, P):
    q, k, v, par, ks, kl = _inputs(B, M, Hq, Hkv, D, P, seed=B * 1000 + M)
    got, ref, _ = _run(orc, q, k, v, par, ks, kl)
    assert not np.isnan(got).any()
    assert_attn_close(got, ref, f"B{B} M{M} Hq{Hq} Hkv{Hkv} D{D} P{P}")


# Grids of more than one wave (320 CTAs of 2 query tiles on 148 SMs x 2): they
# run the instance that starts (sequence, kv head) blocks longest prefix first.
# B > 32 keeps row order; B = 1 ranks one row; the ragged batches put the
# longest sequences in the middle and last, so the order moves rows around.
@pytest.mark.parametrize("flags", [0, 1], ids=["plain", "prefix_ready"])
@pytest.mark.parametrize(
    "B,M,Hq,Hkv,P,left",
    [
        (40, 16, 32, 4, "ragged", False),  # more rows than one warp ranks: row order
        (1, 130, 160, 160, [100], False),  # one sequence, many heads
        (20, 40, 32, 8, "ragged", True),  # longest first changes which row each block serves
    ],
    ids=["B40", "B1", "B20_left_padded"],
)
def test_multi_wave_block_order(orc, B, M, Hq, Hkv, P, left, flags):
    if P == "ragged":
        rng = np.random.default_rng(B)
        P = rng.integers(16, 300, size=B).astype(np.int32)
        P[B // 2] = 500  # the longest in the middle ...
        P[-1] = 499  # ... and the second longest last
    q, k, v, par, ks, kl = _inputs(B, M, Hq, Hkv, 128, P, seed=7000 + B, left_padded=left)
    got, ref, status = _run(orc, q, k, v, par, ks, kl, flags=flags)
    assert not status.any().item()
    assert not np.isnan(got).any()
    assert_attn_close(got, ref, f"multi-wave B{B} M{M} Hq{Hq} Hkv{Hkv} flags{flags}")


def test_left_padded_ragged(orc):
    q, k, v, par, ks, kl = _inputs(5, 7, 16, 4, 128, [10, 700, 64, 1, 1500], seed=3, left_padded=True)
    got, ref, _ = _run(orc, q, k, v, par, ks, kl)
    assert_attn_close(got, ref, "left-padded attention")


def test_garbage_outside_key_range_is_ignored(orc):
    """Pad columns and columns past the tree rows hold Inf/NaN: nothing may leak."""
    B, M, Hq, Hkv, D = 3, 6, 4, 2, 128
    q, k, v, par, ks, kl = _inputs(B, M, Hq, Hkv, D, [5, 90, 40], seed=5, left_padded=True, slack=70)
    ref_k, ref_v = k.clone(), v.clone()
    for b in range(B):
        lo, hi = int(ks[b]), int(ks[b] + kl[b] + M + 1)
        k[b, :, :lo] = float("nan")
        v[b, :, :lo] = float("inf")
        k[b, :, hi:] = float("inf")
        v[b, :, hi:] = float("nan")
    got, _, _ = _run(orc, q, k, v, par, ks, kl)
    _, ref, _ = _run(orc, q, ref_k, ref_v, par, ks, kl)
    assert np.isfinite(got).all()
    assert_attn_close(got, ref, "attention with garbage outside the key range")


@pytest.mark.parametrize("P", [0, 3, 200])
def test_no_leak_between_branches(orc, P):
    B, M, Hq, Hkv, D = 1, 40, 4, 2, 128
    q, k, v, par, ks, kl = _inputs(B, M, Hq, Hkv, D, P, seed=11)
    _, anc, _, status = gpu_mask(par, 1000)
    anc_h = anc.cpu().numpy().view(np.uint32)
    base = gpu_attention(q, k, v, ks, kl, anc, status).float().cpu().numpy()
    for u in (0, 7, 23, 40):
        vv = v.clone()
        for r in range(M + 1):
            if not (int(anc_h[0, u, r // 32]) >> (r % 32)) & 1:
                vv[0, :, P + r] = 1e4
        o = gpu_attention(q, k, vv, ks, kl, anc, status).float().cpu().numpy()
        np.testing.assert_array_equal(o[0, u], base[0, u])


@pytest.mark.parametrize("D", [64, 128])
def test_single_row_maximum_jumps(orc, D):
    """A key that only one query row scores highly, far into the prefix: that row's
    running maximum jumps by far more than the lazy-rescale threshold while the
    other rows of its warp keep theirs, so the O rescale runs for some rows of a
    warp and not for others (it must stay warp-collective)."""
    B, M, Hq, Hkv = 1, 63, 2, 1
    P = 1000
    q, k, v, par, ks, kl = _inputs(B, M, Hq, Hkv, D, P, seed=21)
    spikes = [(5, 0, 700, 3), (40, 1, 300, 17), (63, 0, 900, 40)]  # (row, q-head, key, channel)
    for u, h, key, ch in spikes:
        q[0, :, :, ch] = 0.0  # only the spiking row sees the spike key's channel
    for u, h, key, ch in spikes:
        q[0, u, h, ch] = 1.0
        k[0, 0, key, :] = 0.0
        k[0, 0, key, ch] = 16.0 * D ** 0.5  # score 16 / ln 2 = 23 in the log2 domain
    got, ref, _ = _run(orc, q, k, v, par, ks, kl)
    assert np.isfinite(got).all()
    assert_attn_close(got, ref, "attention with single-row maximum jumps")
    for u, h, key, ch in spikes:  # the spiking row is (almost) the spike key's value row
        np.testing.assert_allclose(got[0, u, h], v[0, 0, key].float().cpu().numpy(), atol=2e-2, rtol=2e-2)


def test_invalid_sequences_zero_rows(orc):
    B, M, Hq, Hkv, D = 4, 10, 8, 4, 128
    q, k, v, par, ks, kl = _inputs(B, M, Hq, Hkv, D, 300, seed=2)
    par[1, 3] = 7  # forward pointer: flagged by the mask kernel
    kl_bad = kl.copy()
    kl_bad[2] = 10_000  # tree rows would run past the cache
    got, ref, status = _run(orc, q, k, v, par, ks, kl_bad)
    assert not got[1].any() and not got[2].any()
    assert_attn_close(got, ref, "attention with invalid sequences")


PREFIX_READY = 1


@pytest.mark.parametrize("flags", [0, PREFIX_READY], ids=["plain", "prefix_ready"])
@pytest.mark.parametrize("name", ["tiny", "mha7b", "eqspec"])
def test_config_full(orc, name, flags):
    """Every output row; with TV_ATTN_PREFIX_READY (tree_build_mask is the launch
    just before) the prefix tiles are requested before the grid dependency, and
    the result must not change."""
    cfg = W.CONFIGS[name]
    st = W.make_step(cfg, seed=0, device=dev(), with_logits=False)
    got, ref, _ = _run(orc, st.q, st.k, st.v, st.parent, st.kv_start, st.kv_len, cfg.max_depth, flags=flags)
    assert_attn_close(got, ref, f"{name} ({'prefix_ready' if flags else 'plain'})")


@pytest.mark.parametrize("flags", [0, PREFIX_READY], ids=["plain", "prefix_ready"])
@pytest.mark.parametrize("name", ["b32gqa", "stress"])
def test_config_sampled(orc, name, flags):
    cfg = W.CONFIGS[name]
    st = W.make_step(cfg, seed=0, device=dev(), with_logits=False)
    rng = np.random.default_rng(1)
    n = cfg.M + 1
    sel = [(0, u, h) for u in range(n) for h in range(0, cfg.Hq, max(1, cfg.Hq // 8))]
    sel += [(int(rng.integers(cfg.B)), int(rng.integers(n)), int(rng.integers(cfg.Hq))) for _ in range(96)]
    sel = np.array(sel, np.int32)
    got, ref, _ = _run(orc, st.q, st.k, st.v, st.parent, st.kv_start, st.kv_len, cfg.max_depth, sel=sel,
                       flags=flags)
    assert_attn_close(got, ref, f"{name} sampled ({'prefix_ready' if flags else 'plain'})")


def test_prefix_ready_is_bit_identical(orc):
    """The launch flag changes when the prefix tiles are requested, not what is
    computed: outputs with and without it are equal bit for bit (eqspec shapes,
    left-padded ragged prefixes; a ring's worth of tiles is requested early)."""
    cfg = W.CONFIGS["eqspec"]
    st = W.make_step(cfg, seed=5, device=dev(), with_logits=False)
    par, anc, depth, status = gpu_mask(st.parent, cfg.max_depth)
    a = gpu_attention(st.q, st.k, st.v, st.kv_start, st.kv_len, anc, status, flags=0)
    b = gpu_attention(st.q, st.k, st.v, st.kv_start, st.kv_len, anc, status, flags=PREFIX_READY)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert int(status.abs().sum()) == 0
