"""The seeded input generator: determinism, shapes, grid and bf16 rounding."""

import numpy as np
import torch

from block_sparse_attention_threshold_b200 import synthetic as syn


def test_deterministic_and_shaped():
    w = syn.workload("tiny_n1024")
    a = syn.generate_bf16(w)
    b = syn.generate_bf16(w)
    for x, y in zip(a, b):
        assert x.shape == (1, 2, 1024, 64) and x.dtype == np.uint16
        assert np.array_equal(x, y)
    # different seed -> different data
    c = syn.generate_bf16(w.replace(seed=w.seed + 1))
    assert not np.array_equal(a[0], c[0])


def test_grid_counts_match_the_workloads():
    for name, w in syn.WORKLOADS.items():
        T, Hg, Wg = w.grid
        assert w.N % 64 == 0 and w.prefix_len % 64 == 0
        assert T * Hg * Wg >= w.video_len, name
    pos = syn.video_positions((2, 3, 4), 24)
    assert pos[0].tolist() == [0, 0, 0] and pos[5].tolist() == [0, 1, 1] and pos[23].tolist() == [1, 2, 3]


def test_bf16_rounding_matches_torch_where_single_rounding_is_unambiguous():
    rng = np.random.default_rng(3)
    x = rng.standard_normal(100000) * 3
    ours = syn.fp64_to_bf16_bits(x)
    # values already exact in fp32 round identically through torch's fp32 -> bf16 path
    x32 = x.astype(np.float32).astype(np.float64)
    ref = torch.from_numpy(x32.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(syn.fp64_to_bf16_bits(x32), ref)
    # rounding error bounded by half an ulp of bf16
    back = syn.bf16_bits_to_fp64(ours)
    assert np.all(np.abs(back - x) <= np.abs(x) * 2.0 ** -8 + 1e-300)
    # ties go to even: 1 + 2^-8 lies halfway between 1 and 1 + 2^-7
    t = syn.fp64_to_bf16_bits(np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8]))
    assert syn.bf16_bits_to_fp64(t).tolist() == [1.0, 1 + 2 * 2.0 ** -7]


def test_prefix_is_unit_normal_and_video_is_local():
    w = syn.workload("tiny_n1024")
    q, k, v = syn.generate_fp64(w)
    L = w.prefix_len
    assert abs(q[0, 0, :L].std() - 1.0) < 0.05
    # neighbouring video tokens have correlated keys, far ones much less
    kv = k[0, 0, L:]
    near = np.mean(np.sum(kv[:-1] * kv[1:], axis=1))
    far = np.mean(np.sum(kv[:-700] * kv[700:], axis=1))
    assert near > far + 2.0


def test_sample_query_blocks():
    s = syn.sample_query_blocks(512, 16, 64, 5)
    assert len(s) == 64 and len(set(s.tolist())) == 64
    assert {0, 16, 511} <= set(s.tolist())
    assert np.array_equal(syn.sample_query_blocks(10, 2, 64, 5), np.arange(10))
