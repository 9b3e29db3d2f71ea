"""GPU test of the timeout path of tree_attention, without a fault or a hang.

Every device wait of the tensor-core attention kernel is bounded.  The testing
hook tv_set_wait_limit_ns shortens the pipeline waits (scores, probabilities,
output, K/V tiles) to 1 ns for one launch, so they run out almost at once: the
kernel must give up on those sequences, OR TV_SEQ_TIMEOUT into their status,
give them zero rows, drain the copies and MMAs it has in flight (those waits
keep the full limit) and return promptly.  The next launch with the default
limit must compute the right result again (the context stays usable).
"""
import time

import numpy as np
import pytest
import torch

import tree_speculative_decoding_04_b200 as tv
import workloads as W
from gpu_helpers import dev, gpu_attention, gpu_mask
from helpers import assert_attn_close

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["eqspec", "mha7b"])
def test_short_wait_limit_times_out_cleanly_and_recovers(orc, name):
    cfg = W.CONFIGS[name]
    st = W.make_step(cfg, seed=9, device=dev(), with_logits=False)
    _, anc, _, status = gpu_mask(st.parent, cfg.max_depth)
    gpu_attention(st.q, st.k, st.v, st.kv_start, st.kv_len, anc, status)  # warm-up: module loaded, plan cached
    torch.cuda.synchronize()
    assert int(status.abs().sum()) == 0
    tv.set_wait_limit_ns(1)
    try:
        t0 = time.perf_counter()
        out = gpu_attention(st.q, st.k, st.v, st.kv_start, st.kv_len, anc, status)
        torch.cuda.synchronize()
        dt = time.perf_counter() - t0
    finally:
        tv.set_wait_limit_ns(0)
    st_h = status.cpu().numpy()
    timed = (st_h & tv.SEQ_TIMEOUT) != 0
    assert timed.any(), st_h
    assert ((st_h & ~tv.SEQ_TIMEOUT) == 0).all(), st_h  # no other bit
    got = out.float().cpu().numpy()
    for b in np.nonzero(timed)[0]:
        assert not got[b].any(), f"sequence {b} timed out but has non-zero rows"
    assert dt < 1.0, f"the launch with 1 ns pipeline waits took {dt:.3f} s"

    # the same inputs with the default limit: correct again
    _, anc2, _, status2 = gpu_mask(st.parent, cfg.max_depth)
    out2 = gpu_attention(st.q, st.k, st.v, st.kv_start, st.kv_len, anc2, status2)
    torch.cuda.synchronize()
    assert int(status2.abs().sum()) == 0
    rng = np.random.default_rng(3)
    n = cfg.M + 1
    sel = np.stack([rng.integers(cfg.B, size=48), rng.integers(n, size=48), rng.integers(cfg.Hq, size=48)],
                   axis=1).astype(np.int32)
    ref = orc.tree_attention_rows(W.bf16_bits(st.q), W.bf16_bits(st.k), W.bf16_bits(st.v), st.kv_start,
                                  st.kv_len, st.parent, np.zeros(cfg.B, np.int32), cfg.Hkv, sel)
    g2 = out2.float().cpu().numpy()
    assert_attn_close(np.stack([g2[b, u, h] for b, u, h in sel]), ref, f"{name} after a timed-out launch")
