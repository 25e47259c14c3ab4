"""The benchmark's algorithmic work counts, checked against closed forms on CPU: valid (row, key)
pairs of the causal, decode, varlen and compressed-key workloads, the key bytes of 16-bit and
fp8 caches, and the backward's flop count."""
import numpy as np
import pytest
import torch

import bench
from sparse_attention_token_lightning_b200 import synthetic


def test_causal_pairs_are_the_triangle():
    pb = synthetic.bsnd(1, 64, 64, 4, 8, 3, seed=1)
    assert bench.valid_pairs(pb) == 64 * 65 // 2
    assert bench.valid_pairs(synthetic.bsnd(2, 30, 50, 4, 8, 3, seed=2)) == 2 * sum(
        min(50, i + 1 + 20) for i in range(30))
    assert bench.valid_pairs(synthetic.bsnd(1, 30, 50, 4, 8, 0, seed=3)) == 30 * 50


def test_decode_pairs_and_key_bytes():
    lens = [700, 129, 1, 64]
    pb = synthetic.paged(lens, 1, 8, 32, block_size=64, seed=4)
    assert bench.valid_pairs(pb) == sum(lens)
    assert bench.key_bytes(pb) == sum(lens) * 128 * 2
    q8 = synthetic.quantized(pb)
    assert bench.key_bytes(q8) == sum(lens) * (128 + 4)


def test_varlen_pairs_sum_each_sequence():
    lens = [5, 200, 1, 77]
    pb = synthetic.tnd(lens, lens, 4, 16, 3, seed=5)
    assert bench.valid_pairs(pb) == sum(L * (L + 1) // 2 for L in lens)


def test_compressed_pairs_count_whole_blocks():
    pb = synthetic.compressed(synthetic.bsnd(1, 64, 16, 4, 8, 3, seed=6), 4, [0])
    # 64 original tokens, 16 keys of 4: row i sees floor((i + 1) / 4) keys
    assert bench.valid_pairs(pb) == sum((i + 1) // 4 for i in range(64))


def test_backward_flops():
    kp = synthetic.kl_bsnd(1, 20, 2, 16, 8, 3, 5, seed=7, Di=16)
    n = int((kp.sparse_indices >= 0).sum())
    assert n == sum(min(5, i + 1) for i in range(20))
    assert bench.kl_flops(kp) == n * (2 * 2 * (16 + 8) + 8 * 3 * 16)
