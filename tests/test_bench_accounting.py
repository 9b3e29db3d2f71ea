"""The benchmark's algorithmic work counts, checked against their closed forms
on the workloads' own shapes (no GPU needed)."""
import dataclasses

import numpy as np

import bench
import workloads as W


def test_attention_bytes_mha7b():
    cfg = W.CONFIGS["mha7b"]
    kl = np.full(cfg.B, 2048)
    # K and V of 2048 prefix + 65 tree rows, 32 heads, 128 bf16 each; q in and out
    kv = 2 * 32 * (2048 + 65) * 128 * 2
    qo = 2 * 65 * 32 * 128 * 2
    assert bench.attention_bytes(cfg, kl) == kv + qo == 35_684_352


def test_attention_flops_counts_ancestors_only():
    cfg = W.CONFIGS["tiny"]  # B1, Hq4, D64, M16
    kl = np.array([128])
    chain_depth = np.arange(17)[None, :]  # a chain: node u has u+1 ancestors (itself included)
    star_depth = np.minimum(np.arange(17), 1)[None, :]  # a star: 1 (root) or 2 ancestors
    pre = 4 * 64 * 4 * 17 * 128
    assert bench.attention_flops(cfg, kl, chain_depth) == pre + 4 * 64 * 4 * sum(range(1, 18))
    assert bench.attention_flops(cfg, kl, star_depth) == pre + 4 * 64 * 4 * (1 + 16 * 2)


def test_commit_bytes_moves_only_rows_off_their_place():
    cfg = W.CONFIGS["tiny"]  # per-sequence lengths, L1, Hkv4, D64
    row = 64 * 2
    path = np.array([[0, 3, 7, 0, 0, 0, 0, 0, 0, 0, 0]])
    # j=0 takes row 0 (stays), j=1 takes row 3 and j=2 row 7 (both move)
    got = bench.commit_bytes(cfg, path, np.array([2]), np.array([128]), False, np.zeros(1, np.int64))
    assert got == 1 * 4 * 2 * 2 * row * 2
    chain = np.array([[0, 1, 2, 0, 0, 0, 0, 0, 0, 0, 0]])
    assert bench.commit_bytes(cfg, chain, np.array([2]), np.array([128]), False, np.zeros(1, np.int64)) == 0
    rejected = bench.commit_bytes(cfg, path, np.array([-1]), np.array([128]), False, np.zeros(1, np.int64))
    assert rejected == 0


def test_realign_bytes_move_the_whole_content_of_shifted_sequences():
    cfg = dataclasses.replace(W.CONFIGS["eqspec"], B=2)  # left-padded, L36, Hkv8, D128
    row = 128 * 2
    path = np.zeros((2, 6), np.int32)
    al = np.array([3, 0])
    kl = np.array([1000, 500])
    shift = np.array([0, 3])
    got = bench.commit_bytes(cfg, path, al, kl, True, shift)
    # sequence 0 stays in place; its path takes rows 1..3 from tree row 0, so 3 rows move
    seq0 = 36 * 8 * 2 * 3 * row * 2
    seq1 = 36 * 8 * 2 * (500 + 0 + 1) * row * 2
    assert got == seq0 + seq1
