"""GPU parity of kv_commit_realign against the oracle: every cache byte of the
new content of every layer, the new geometry, the attention mask and position
IDs, bit-exact, in both modes; multi-round EQSPEC replay on ragged batches;
shifts in both directions; rejected sequences and bad geometry."""
import numpy as np
import pytest
import torch

import tree_speculative_decoding_04_b200 as tv
from gpu_helpers import dev, i32
import workloads as W

pytestmark = pytest.mark.gpu


def _random_paths(rng, B, M, md):
    path = np.zeros((B, md + 1), np.int32)
    al = np.zeros(B, np.int32)
    for b in range(B):
        par = W.tree_uniform_depth(M, md, rng)
        e = int(rng.integers(M + 1))
        chain = []
        x = e
        while True:
            chain.append(x)
            if x == 0:
                break
            x = int(par[x])
        chain = chain[::-1]
        al[b] = len(chain) - 1
        path[b, : len(chain)] = chain
    return path, al


class Cache:
    """L layers of K and V on the GPU plus host copies for the oracle."""

    def __init__(self, L, B, Hkv, S_cap, D, salt=0):
        self.k = [W.tagged_rows(l, 0, B, Hkv, S_cap, D, dev(), salt) for l in range(L)]
        self.v = [W.tagged_rows(l, 1, B, Hkv, S_cap, D, dev(), salt) for l in range(L)]
        self.kh = [W.bf16_bits(t).copy() for t in self.k]
        self.vh = [W.bf16_bits(t).copy() for t in self.v]
        self.kp = tv.layer_pointers(self.k)
        self.vp = tv.layer_pointers(self.v)
        self.shape = (B, Hkv, S_cap, D)

    def write_tree_rows(self, ks, kl, M, rng):
        """Fresh tree rows behind every sequence's content (as the caller would)."""
        B, Hkv, S_cap, D = self.shape
        for l in range(len(self.k)):
            for kv, dv, hv in ((0, self.k[l], self.kh[l]), (1, self.v[l], self.vh[l])):
                rows = rng.integers(0, 0x7F00, size=(B, Hkv, M + 1, D), dtype=np.uint16)
                for b in range(B):
                    c0 = int(ks[b] + kl[b])
                    hv[b, :, c0 : c0 + M + 1] = rows[b]
                dv.copy_(torch.as_tensor(hv.view(np.int16)).view(torch.bfloat16).to(dev()))


def _step(orc, cache, M, md, path, al, status, ks, kl, realign, with_mask=True):
    B, Hkv, S_cap, D = cache.shape
    g_ks, g_kl, g_st = i32(ks), i32(kl), i32(status)
    ml = torch.full((1,), -1, dtype=torch.int32, device=dev())
    mask = torch.full((B, S_cap), 7, dtype=torch.uint8, device=dev()) if with_mask else None
    pos = torch.full((B, S_cap), -1, dtype=torch.int32, device=dev()) if with_mask else None
    tv.kv_commit_realign(cache.kp, cache.vp, B, Hkv, D, S_cap, M, i32(path), i32(al), g_st, md, g_ks, g_kl, ml,
                         realign, mask, pos)
    torch.cuda.synchronize()
    o_ks, o_kl, o_ml, o_mask, o_pos, o_st = orc.kv_commit_realign(
        cache.kh, cache.vh, M, path, al, status, md, ks, kl, realign, with_mask=with_mask, with_status=True
    )
    np.testing.assert_array_equal(g_ks.cpu().numpy(), o_ks)
    np.testing.assert_array_equal(g_kl.cpu().numpy(), o_kl)
    assert int(ml.item()) == o_ml
    np.testing.assert_array_equal(g_st.cpu().numpy(), o_st)
    if with_mask:
        np.testing.assert_array_equal(mask.cpu().numpy(), o_mask)
        np.testing.assert_array_equal(pos.cpu().numpy(), o_pos)
    # content of every sequence, every layer, K and V: bit-exact
    for l in range(len(cache.k)):
        gk, gv = W.bf16_bits(cache.k[l]), W.bf16_bits(cache.v[l])
        for b in range(B):
            lo, hi = int(o_ks[b]), int(o_ks[b] + o_kl[b])
            np.testing.assert_array_equal(gk[b, :, lo:hi], cache.kh[l][b, :, lo:hi])
            np.testing.assert_array_equal(gv[b, :, lo:hi], cache.vh[l][b, :, lo:hi])
        # keep host copies identical outside the content too (pad bytes are don't-care)
        cache.kh[l][:] = gk
        cache.vh[l][:] = gv
    return o_ks, o_kl


@pytest.mark.parametrize("D", [64, 128])
def test_per_sequence_mode(orc, D):
    rng = np.random.default_rng(D)
    L, B, Hkv, M, md = 3, 5, 4, 16, 10
    kl = rng.integers(0, 300, size=B).astype(np.int32)
    ks = np.zeros(B, np.int32)
    S_cap = int(kl.max()) + M + 1 + 8
    cache = Cache(L, B, Hkv, S_cap, D)
    path, al = _random_paths(rng, B, M, md)
    _step(orc, cache, M, md, path, al, np.zeros(B, np.int32), ks, kl, 0)


@pytest.mark.parametrize("seed", [0, 1])
def test_eqspec_rounds(orc, seed):
    """Left-padded ragged batch over many rounds: shifts go both ways."""
    rng = np.random.default_rng(seed)
    L, B, Hkv, D, M, md, R = 2, 8, 2, 128, 5, 5, 12
    P = rng.integers(1, 700, size=B).astype(np.int32)
    pmax = int(P.max())
    S_cap = pmax + R * (md + 1) + M + 1
    ks = (pmax - P).astype(np.int32)
    kl = P.copy()
    cache = Cache(L, B, Hkv, S_cap, D, salt=seed)
    for rnd in range(R):
        cache.write_tree_rows(ks, kl, M, rng)
        parent = np.stack([W.tree_chain(M)] * B)
        path, al = _random_paths(rng, B, M, md)
        # a chain tree accepts a prefix: path[j] = j
        for b in range(B):
            path[b] = 0
            path[b, : al[b] + 1] = np.arange(al[b] + 1)
        status = np.zeros(B, np.int32)
        if rnd % 4 == 3:
            status[rnd % B] = 1
        ks, kl = _step(orc, cache, M, md, path, al, status, ks, kl, 1)
        assert (ks + kl == (ks + kl).max()).all()


def test_tree_paths_realign(orc):
    rng = np.random.default_rng(3)
    L, B, Hkv, D, M, md = 3, 6, 3, 128, 40, 12
    P = np.array([0, 1, 513, 64, 1000, 77], np.int32)
    pmax = int(P.max())
    S_cap = pmax + 2 * (M + 1) + 4
    ks = (pmax - P).astype(np.int32)
    kl = P.copy()
    cache = Cache(L, B, Hkv, S_cap, D, salt=9)
    for _ in range(2):
        path, al = _random_paths(rng, B, M, md)
        ks, kl = _step(orc, cache, M, md, path, al, np.zeros(B, np.int32), ks, kl, 1)
        cache.write_tree_rows(ks, kl, M, rng)


def test_bad_geometry_and_bad_path(orc):
    rng = np.random.default_rng(6)
    L, B, Hkv, D, M, md = 2, 4, 2, 128, 8, 4
    S_cap = 200
    ks = np.array([10, 0, 5, 3], np.int32)
    kl = np.array([50, 195, 60, 20], np.int32)  # sequence 1: tree rows past the cache
    cache = Cache(L, B, Hkv, S_cap, D)
    path, al = _random_paths(rng, B, M, md)
    path[3, 1] = 99  # out of the tree: commits nothing
    al[3] = max(al[3], 1)
    _step(orc, cache, M, md, path, al, np.zeros(B, np.int32), ks, kl, 1)


def test_no_mask_outputs(orc):
    rng = np.random.default_rng(2)
    L, B, Hkv, D, M, md = 1, 3, 1, 64, 6, 6
    P = np.array([5, 17, 9], np.int32)
    ks = (17 - P).astype(np.int32)
    cache = Cache(L, B, Hkv, 40, D)
    path, al = _random_paths(rng, B, M, md)
    _step(orc, cache, M, md, path, al, np.zeros(B, np.int32), ks, P.copy(), 1, with_mask=False)


@pytest.mark.parametrize("name", W.CONFIG_ORDER)
def test_config_commit(orc, name):
    cfg = W.CONFIGS[name]
    rng = np.random.default_rng(0)
    P = W.make_prefix_lengths(cfg, rng)
    ks, kl, S_cap = W.cache_geometry(cfg, P, extra_rows=cfg.max_depth + 1)
    L = min(cfg.L, {"stress": 2, "b32gqa": 3, "eqspec": 4}.get(name, cfg.L))
    cache = Cache(L, cfg.B, cfg.Hkv, S_cap, cfg.D)
    parent = W.make_parents(cfg, rng)
    path = np.zeros((cfg.B, cfg.max_depth + 1), np.int32)
    al = np.zeros(cfg.B, np.int32)
    for b in range(cfg.B):  # deepest node of each tree, as if everything were accepted
        dep = np.zeros(cfg.M + 1, np.int32)
        for i in range(1, cfg.M + 1):
            dep[i] = dep[parent[b, i]] + 1
        e = int(np.argmax(dep))
        x = e
        while True:
            path[b, dep[x]] = x
            if x == 0:
                break
            x = int(parent[b, x])
        al[b] = dep[e]
    _step(orc, cache, cfg.M, cfg.max_depth, path, al, np.zeros(cfg.B, np.int32), ks, kl,
          1 if cfg.left_padded else 0)
