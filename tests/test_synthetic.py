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


# --------------------------------------------------------------------------- E4M3 inputs

def test_e4m3_hand_values():
    enc = syn.fp64_to_e4m3_bits
    cases = {
        1.0: 0x38, 2.0: 0x40, 0.5: 0x30, -1.0: 0xB8, 448.0: 0x7E, -448.0: 0xFE,
        1e6: 0x7E,                 # saturates at the largest finite value
        2.0 ** -6: 0x08,           # smallest normal
        2.0 ** -9: 0x01,           # smallest subnormal
        2.0 ** -10: 0x00,          # half of it: tie to even (zero)
        3 * 2.0 ** -10: 0x02,      # between 1 and 2 quanta of 2^-9: tie to even (2)
        1.0625: 0x38,              # between 1.0 and 1.125: tie to even (1.0)
        1.1875: 0x3A,              # between 1.125 and 1.25: tie to even (1.25)
        1.05: 0x38, 1.07: 0x39,    # ordinary rounding (1.07 is nearer 1.125)
        240.0: 0x77, 232.0: 0x76,  # 232 = 7.25 * 32 ties to 224 (even), 240 = 1.875 * 2^7
    }
    for x, b in cases.items():
        assert int(enc(np.array([x]))[0]) == b, (x, hex(int(enc(np.array([x]))[0])), hex(b))


def test_e4m3_decode_and_round_trip_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    vals = syn.e4m3_bits_to_fp64(codes)
    finite = ~np.isnan(vals)
    assert np.isnan(vals[0x7F]) and np.isnan(vals[0xFF]) and finite.sum() == 254
    assert vals[0x7E] == 448.0 and vals[0x01] == 2.0 ** -9 and vals[0x38] == 1.0
    # every finite code decodes and re-encodes to itself (0x80 is -0, which encodes back to 0x80)
    back = syn.fp64_to_e4m3_bits(vals[finite])
    assert np.array_equal(back, codes[finite])
    # positive codes are increasing
    pos = vals[0:0x7F]
    assert np.all(np.diff(pos) > 0)


def test_e4m3_rounding_is_nearest_on_random_values():
    rng = np.random.default_rng(3)
    x = rng.standard_normal(20000) * rng.choice([1e-3, 0.1, 1.0, 30.0], size=20000)
    got = syn.e4m3_bits_to_fp64(syn.fp64_to_e4m3_bits(x))
    grid = syn.e4m3_bits_to_fp64(np.arange(256, dtype=np.uint8))
    grid = np.unique(grid[~np.isnan(grid)])
    # brute force: the nearest representable value (saturation aside)
    idx = np.abs(x[:, None] - grid[None, :]).argmin(axis=1)
    best = np.abs(x - grid[idx])
    assert np.all(np.abs(x - got) <= best + 1e-300)
