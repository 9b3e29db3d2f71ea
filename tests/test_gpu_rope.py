"""GPU parity of the rotary position embedding fused into tree_kv_write (K rows)
and into tree_attention's query staging (TV_ATTN_ROPE), against the oracle.

Tree positions: node u of sequence b sits at kv_len[b] + depth[b][u] (position-ID
contiguity, "Batch Speculative Decoding Done Right", section 2).  The kernels
form each angle in double precision and rotate in single precision; the oracle
works in double throughout and rounds once to bf16.  V rows and every cell
outside the tree rows are compared bit for bit, attention at the usual
tolerance.  K rows: within half a bf16 unit of a value within the fp32 error
of the exact rotation (absolute near zero, where x cos - y sin cancels), and
nearly all equal to the oracle's own rounding.
"""
import numpy as np
import pytest
import torch

import tree_speculative_decoding_04_b200 as tv
import workloads as W
from gpu_helpers import dev, gpu_mask, i32
from helpers import assert_attn_close

pytestmark = pytest.mark.gpu

THETA = 10000.0


def _bits_to_f64(u16):
    return (np.asarray(u16, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _tree_rows(st, cfg):
    n = cfg.M + 1
    c0 = [int(a + b) for a, b in zip(st.kv_start, st.kv_len)]
    tk = torch.stack([st.k[b, :, c0[b]:c0[b] + n] for b in range(cfg.B)]).unsqueeze(0).contiguous()
    tvv = torch.stack([st.v[b, :, c0[b]:c0[b] + n] for b in range(cfg.B)]).unsqueeze(0).contiguous()
    return tk, tvv


@pytest.mark.parametrize("name", ["tiny", "mha7b", "eqspec", "stress"])
def test_kv_write_rotates_k_rows(orc, name):
    cfg = W.CONFIGS[name]
    st = W.make_step(cfg, seed=2, device=dev(), with_logits=False)
    _, anc, depth, status = gpu_mask(st.parent, cfg.max_depth)
    tk, tvv = _tree_rows(st, cfg)
    k0, v0 = W.bf16_bits(st.k).copy(), W.bf16_bits(st.v).copy()
    tv.tree_kv_write(tv.layer_pointers([st.k]), tv.layer_pointers([st.v]), tk, tvv, st.S_cap, i32(st.kv_start),
                     i32(st.kv_len), depth=depth, rope_theta=THETA)
    torch.cuda.synchronize()
    kh, vh = [k0.copy()], [v0.copy()]
    orc.tree_kv_write(kh, vh, W.bf16_bits(tk), W.bf16_bits(tvv), st.kv_start, st.kv_len,
                      depth=depth.cpu().numpy(), rope_base=THETA)
    gk, gv = W.bf16_bits(st.k), W.bf16_bits(st.v)
    np.testing.assert_array_equal(gv, vh[0])  # V rows copied, nothing else touched
    mask = np.ones(gk.shape[:3], bool)
    for b in range(cfg.B):
        c0 = int(st.kv_start[b] + st.kv_len[b])
        mask[b, :, c0:c0 + cfg.M + 1] = False
    np.testing.assert_array_equal(gk[mask], k0[mask])  # outside the tree rows: untouched
    # the rotated rows: within rounding of a value within the fp32 error of the
    # exact rotation (x cos - y sin cancels, so near zero the bound is absolute,
    # scaled by |x| + |y|), and nearly all equal to the oracle's own rounding
    n, D = cfg.M + 1, cfg.D
    raw = _bits_to_f64(W.bf16_bits(tk)[0])  # [B][Hkv][n][D]
    dep = depth.cpu().numpy()
    gpu_rows = np.stack([gk[b, :, int(st.kv_start[b] + st.kv_len[b]):int(st.kv_start[b] + st.kv_len[b]) + n]
                         for b in range(cfg.B)])
    for b in range(cfg.B):
        pos = (int(st.kv_len[b]) + dep[b]).astype(np.float64)
        for h in range(cfg.Hkv):
            exact = orc.rope_rows(raw[b, h], pos, THETA)
            mag = np.abs(raw[b, h]) + np.abs(np.roll(raw[b, h], D // 2, axis=1))
            err = np.abs(_bits_to_f64(gpu_rows[b, h]) - exact)
            bound = 2.0 ** -8 * np.abs(exact) + 2.0 ** -20 * mag
            assert (err <= bound).all(), f"K row rotation off by {float((err - bound).max()):.3e} (b={b}, h={h})"
    mismatch = (gpu_rows != np.stack([kh[0][b, :, int(st.kv_start[b] + st.kv_len[b]):
                                              int(st.kv_start[b] + st.kv_len[b]) + n] for b in range(cfg.B)]))
    assert mismatch.mean() < 1e-2, f"{mismatch.mean():.2e} of the K elements differ from the oracle's rounding"


@pytest.mark.parametrize("name,sampled", [("tiny", False), ("mha7b", False), ("eqspec", False),
                                          ("b32gqa", True), ("stress", True)])
def test_attention_with_rotation(orc, name, sampled):
    cfg = W.CONFIGS[name]
    if cfg.D != 128:
        pytest.skip("the rotation is fused into the head dim 128 kernel only")
    st = W.make_step(cfg, seed=4, device=dev(), with_logits=False)
    par, anc, depth, status = gpu_mask(st.parent, cfg.max_depth)
    tk, tvv = _tree_rows(st, cfg)
    ks, kl = i32(st.kv_start), i32(st.kv_len)
    tv.tree_kv_write(tv.layer_pointers([st.k]), tv.layer_pointers([st.v]), tk, tvv, st.S_cap, ks, kl,
                     depth=depth, rope_theta=THETA)
    out = torch.full_like(st.q, float("nan"))
    ws = tv.attention_workspace(cfg.B, cfg.M, cfg.Hq, cfg.Hkv, cfg.D, st.S_cap, dev())
    tv.tree_attention(st.q, st.k, st.v, ks, kl, anc, status, out, ws, flags=tv.ATTN_ROPE | tv.ATTN_PREFIX_READY,
                      depth=depth, rope_theta=THETA)
    torch.cuda.synchronize()
    assert int(status.abs().sum()) == 0
    # the oracle's own cache: its own rotation of the same raw tree rows
    k0 = W.bf16_bits(st.k).copy()
    v0 = W.bf16_bits(st.v).copy()
    kh, vh = [k0], [v0]
    orc.tree_kv_write(kh, vh, W.bf16_bits(tk), W.bf16_bits(tvv), st.kv_start, st.kv_len,
                      depth=depth.cpu().numpy(), rope_base=THETA)
    qb = W.bf16_bits(st.q)
    st_h = np.zeros(cfg.B, np.int32)
    got = out.float().cpu().numpy()
    if not sampled:
        ref = orc.tree_attention(qb, kh[0], vh[0], st.kv_start, st.kv_len, st.parent, st_h, cfg.Hkv,
                                 rope_base=THETA)
        assert_attn_close(got, ref, f"{name} with rotation")
    else:
        rng = np.random.default_rng(5)
        n = cfg.M + 1
        sel = [(0, u, h) for u in range(n) for h in range(0, cfg.Hq, max(1, cfg.Hq // 4))]
        sel += [(int(rng.integers(cfg.B)), int(rng.integers(n)), int(rng.integers(cfg.Hq))) for _ in range(64)]
        sel = np.array(sel, np.int32)
        ref = orc.tree_attention_rows(qb, kh[0], vh[0], st.kv_start, st.kv_len, st.parent, st_h, cfg.Hkv, sel,
                                      rope_base=THETA)
        assert_attn_close(np.stack([got[b, u, h] for b, u, h in sel]), ref, f"{name} sampled with rotation")


def test_rotation_changes_the_result(orc):
    """Guards against a flag that does nothing: with rotation (and a cache whose
    rows are used as they are) the output differs from the unrotated one and
    matches the oracle's attention with the query rows rotated."""
    cfg = W.CONFIGS["eqspec"]
    st = W.make_step(cfg, seed=6, device=dev(), with_logits=False)
    par, anc, depth, status = gpu_mask(st.parent, cfg.max_depth)
    ws = tv.attention_workspace(cfg.B, cfg.M, cfg.Hq, cfg.Hkv, cfg.D, st.S_cap, dev())
    ks, kl = i32(st.kv_start), i32(st.kv_len)
    a = torch.empty_like(st.q)
    b = torch.empty_like(st.q)
    tv.tree_attention(st.q, st.k, st.v, ks, kl, anc, status, a, ws)
    tv.tree_attention(st.q, st.k, st.v, ks, kl, anc, status, b, ws, flags=tv.ATTN_ROPE, depth=depth,
                      rope_theta=THETA)
    torch.cuda.synchronize()
    assert not torch.equal(a, b)
    ref = orc.tree_attention(W.bf16_bits(st.q), W.bf16_bits(st.k), W.bf16_bits(st.v), st.kv_start, st.kv_len,
                             st.parent, np.zeros(cfg.B, np.int32), cfg.Hkv, rope_base=THETA)
    assert_attn_close(b.float().cpu().numpy(), ref, "eqspec with rotation (cache not rotated)")
