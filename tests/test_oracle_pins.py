"""Pins of the CPU fp64 oracle to things other than itself.

Each test checks the oracle against a closed form, a library routine in a
special case, a hand-derived worked example, an invariant the definition
implies, or an independent brute force written here with plain loops.  The
cases are chosen so that a plausible slip (a dropped ln c term, a sample
instead of population std, statistics over the prefix, a flipped threshold
comparison, a transposed operand, a lost max shift) fails at least one.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import sol_attn_oracle as orc
from block_sparse_attention_threshold_b200 import synthetic as syn

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _blocky(values, block, D=1):
    """[len(values) * block, D] array whose block j rows all equal values[j]."""
    return np.repeat(np.asarray(values, np.float64)[:, None], block, axis=0).repeat(D, axis=1)


def _sdpa(q, k, v, scale, bias=None):
    """torch's fp64 CPU scaled-dot-product attention for one head [N, D]."""
    tq = torch.from_numpy(np.ascontiguousarray(q))[None, None]
    tk = torch.from_numpy(np.ascontiguousarray(k))[None, None]
    tv = torch.from_numpy(np.ascontiguousarray(v))[None, None]
    mask = None if bias is None else torch.from_numpy(np.ascontiguousarray(bias))[None, None]
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask, scale=scale)
    return o[0, 0].numpy()


def _tiny_inputs(rounded=True):
    w = syn.workload("tiny_n1024")
    if rounded:
        q, k, v = (syn.bf16_bits_to_fp64(a) for a in syn.generate_bf16(w))
    else:
        q, k, v = syn.generate_fp64(w)
    return w, q, k, v


# ----------------------------------------------------------------------------- pooling

def test_pool_constant_blocks_and_library_mean():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((64 * 5, 7))
    means, counts = orc.pool_blocks(x, 64)
    np.testing.assert_allclose(means, x.reshape(5, 64, 7).mean(axis=1), rtol=0, atol=1e-15)
    assert list(counts) == [64] * 5
    const = _blocky([1.5, -2.0, 0.25], 64, D=3)
    m2, _ = orc.pool_blocks(const, 64)
    assert np.array_equal(m2, np.array([[1.5] * 3, [-2.0] * 3, [0.25] * 3]))


def test_pool_ragged_tail_counts():
    x = np.arange(150 * 2, dtype=np.float64).reshape(150, 2)
    means, counts = orc.pool_blocks(x, 64)
    assert list(counts) == [64, 64, 22]
    # brute force mean of the 22-row tail
    tail = [sum(x[r, d] for r in range(128, 150)) / 22 for d in range(2)]
    np.testing.assert_allclose(means[2], tail, rtol=1e-15)


# ----------------------------------------------------------------------------- routing

def _golden():
    with open(os.path.join(GOLDEN, "route_worked_example.json")) as f:
        return json.load(f)


def _golden_head(g):
    s = g["setup"]
    block = s["block"]
    k = _blocky(s["k_block_values"], block)
    v = _blocky(s["v_block_values"], block)
    q = np.ones_like(k)
    return q, k, v, block, s["prefix_len"], s["scale"]


def test_route_worked_example():
    g = _golden()
    e = g["expect"]
    q, k, _, block, L, scale = _golden_head(g)
    r = orc.route(q, k, block, L, 1.2, scale)
    for i in range(1, 6):
        assert r.mu[i] == pytest.approx(e["mu"], abs=1e-15)
        assert r.sigma[i] == pytest.approx(e["sigma"], abs=1e-15)
        assert r.thr[i] == pytest.approx(e["thr_tau_1.2"], abs=1e-14)
        assert list(np.nonzero(r.keep[i, 1:])[0] + 1) == e["kept_video_tau_1.2"]
        assert r.keep[i, 0]
    assert r.keep[0].all()  # prefix query block dense
    for tau, key in ((0.5, "kept_video_tau_0.5"), (-1.0, "kept_video_tau_-1")):
        r = orc.route(q, k, block, L, tau, scale)
        assert list(np.nonzero(r.keep[3, 1:])[0] + 1) == e[key]


def test_route_tie_is_kept():
    block = 64
    k = _blocky([0.0, 2.0], block)
    q = np.ones_like(k)
    r = orc.route(q, k, block, 0, 1.0, 1.0)
    assert r.thr[0] == 2.0
    assert list(r.keep[0]) == [False, True]


def test_worked_example_output_and_count_weight():
    g = _golden()
    q, k, v, block, L, scale = _golden_head(g)
    out = orc.solattn_blocks(q, k, v, block, L, 1.2, scale, qblocks=[3])
    assert np.allclose(out, g["expect"]["out_video_row_tau_1.2"], rtol=0, atol=g["expect"]["out_tol"])


def test_route_special_taus_and_sigma_zero():
    w, q, k, _ = _tiny_inputs()
    for h in range(w.H):
        r_all = orc.route(q[0, h], k[0, h], 64, w.prefix_len, -math.inf)
        assert r_all.keep.all()
        r_none = orc.route(q[0, h], k[0, h], 64, w.prefix_len, math.inf)
        P = w.P
        assert r_none.keep[:, :P].all() and r_none.keep[:P].all()
        assert not r_none.keep[P:, P:].any()
    # identical pooled keys -> sigma = 0 -> every block kept for any tau
    kk = _blocky([0.7] * 8, 64, D=4)
    qq = np.random.default_rng(2).standard_normal(kk.shape)
    r = orc.route(qq, kk, 64, 64, 2.0)
    assert (r.sigma[1:] == 0).all() and r.keep.all()


def test_route_invariances():
    w, q, k, _ = _tiny_inputs()
    qh, kh = q[0, 0], k[0, 0]
    base = orc.route(qh, kh, 64, w.prefix_len, 1.0)
    # scaling queries by alpha > 0 leaves the mask unchanged
    for alpha in (0.1, 3.0):
        assert np.array_equal(orc.route(alpha * qh, kh, 64, w.prefix_len, 1.0).keep, base.keep)
    # kept count is non-increasing in tau
    counts = [orc.route(qh, kh, 64, w.prefix_len, t).keep.sum() for t in (-1, 0, 0.5, 1, 1.5, 2, 3)]
    assert all(a >= b for a, b in zip(counts, counts[1:]))
    # tau <= 0 keeps at least one video block per video query block (max >= mean)
    r0 = orc.route(qh, kh, 64, w.prefix_len, 0.0)
    assert r0.keep[w.P:, w.P:].any(axis=1).all()
    # mean and std are those of numpy over the video scores
    s = r0.score[w.P:, w.P:]
    np.testing.assert_allclose(r0.mu[w.P:], s.mean(axis=1), rtol=1e-13)
    np.testing.assert_allclose(r0.sigma[w.P:], s.std(axis=1, ddof=0), rtol=1e-12)


# ----------------------------------------------------------------------------- attention

def test_dense_rows_equal_library_sdpa():
    w, q, k, v = _tiny_inputs(rounded=False)
    scale = 1 / math.sqrt(w.D)
    for h in range(w.H):
        ref = _sdpa(q[0, h], k[0, h], v[0, h], scale)
        np.testing.assert_allclose(orc.dense_rows(q[0, h], k[0, h], v[0, h]), ref, rtol=0, atol=1e-12)


def test_tau_minus_inf_is_dense_attention():
    for rounded in (False, True):
        w, q, k, v = _tiny_inputs(rounded)
        out = orc.solattn(q, k, v, 64, w.prefix_len, -math.inf)
        for h in range(w.H):
            ref = _sdpa(q[0, h], k[0, h], v[0, h], 1 / math.sqrt(w.D))
            np.testing.assert_allclose(out[0, h], ref, rtol=0, atol=1e-12)


def test_tau_plus_inf_is_attention_over_prefix_and_pooled_keys():
    """tau = +inf: video rows attend to the prefix tokens plus one pooled key per
    video block with additive bias ln 64 -- textbook attention with a float bias."""
    w, q, k, v = _tiny_inputs()
    L, P = w.prefix_len, w.P
    scale = 1 / math.sqrt(w.D)
    for h in range(w.H):
        qh, kh, vh = q[0, h], k[0, h], v[0, h]
        kbar = kh[L:].reshape(-1, 64, w.D).mean(axis=1)
        vbar = vh[L:].reshape(-1, 64, w.D).mean(axis=1)
        keys = np.concatenate([kh[:L], kbar])
        vals = np.concatenate([vh[:L], vbar])
        bias = np.concatenate([np.zeros(L), np.full(kbar.shape[0], math.log(64))])
        ref = _sdpa(qh[L:], keys, vals, scale, np.broadcast_to(bias, (w.N - L, keys.shape[0])))
        out = orc.solattn_blocks(qh, kh, vh, 64, L, math.inf, qblocks=range(P, w.M))
        np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
        # prefix query rows stay dense
        out_p = orc.solattn_blocks(qh, kh, vh, 64, L, math.inf, qblocks=range(P))
        np.testing.assert_allclose(out_p, _sdpa(qh[:L], kh, vh, scale), rtol=0, atol=1e-12)


def test_identical_key_blocks_make_the_correction_exact():
    """If every key and value of a block is the same vector, sum_t e^{q.k_t} v_t =
    c e^{q.kbar} vbar, so Sol-Attn equals dense attention for every tau."""
    rng = np.random.default_rng(7)
    N, D, L = 64 * 10, 16, 128
    kb = rng.standard_normal((N // 64, D))
    vb = rng.standard_normal((N // 64, D))
    k = np.repeat(kb, 64, axis=0)
    v = np.repeat(vb, 64, axis=0)
    q = rng.standard_normal((N, D)) * 2.0
    ref = _sdpa(q, k, v, 1 / math.sqrt(D))
    for tau in (-0.5, 0.0, 0.75, 1.5, math.inf):
        r = orc.route(q, k, 64, L, tau)
        if tau > 0:
            assert not r.keep.all()  # some blocks really are skipped
        out = orc.solattn_blocks(q, k, v, 64, L, tau)
        np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_prefix_rows_are_dense_for_any_tau():
    w, q, k, v = _tiny_inputs()
    rows = range(w.prefix_len)
    for tau in (0.0, 1.0, 2.0, math.inf):
        out = orc.solattn(q, k, v, 64, w.prefix_len, tau, qblocks=range(w.P))
        ref = orc.dense(q, k, v, rows=rows)
        np.testing.assert_allclose(out, ref, rtol=0, atol=1e-13)


def test_value_shift_invariance():
    w, q, k, v = _tiny_inputs()
    c = np.linspace(-1, 1, w.D)
    a = orc.solattn(q, k, v, 64, w.prefix_len, 1.0)
    b = orc.solattn(q, k, v + c, 64, w.prefix_len, 1.0)
    np.testing.assert_allclose(b - a, np.broadcast_to(c, a.shape), rtol=0, atol=1e-12)


def _permute_blocks(x, order, block=64):
    """Rows of x regrouped so that block i of the result is block order[i] of x."""
    return np.concatenate([x[j * block:(j + 1) * block] for j in order], axis=0)


@pytest.mark.parametrize("tau", [0.5, 1.25])
def test_video_key_block_permutation_invariance(tau):
    """Every output row sums over key blocks, exact or pooled, and the keep
    rule uses the mean and std of the row's video scores: permuting the video
    key blocks (their K and V rows together) changes no output and permutes
    each row's keep mask with them.  A block-index slip anywhere in the
    routing or the correction breaks this."""
    w, q, k, v = _tiny_inputs()
    qh, kh, vh = q[0, 0], k[0, 0], v[0, 0]
    rng = np.random.default_rng(5)
    order = list(range(w.P)) + list(w.P + rng.permutation(w.M - w.P))
    kp, vp = _permute_blocks(kh, order), _permute_blocks(vh, order)
    a = orc.solattn_blocks(qh, kh, vh, 64, w.prefix_len, tau)
    b = orc.solattn_blocks(qh, kp, vp, 64, w.prefix_len, tau)
    np.testing.assert_allclose(b, a, rtol=0, atol=1e-12)
    ra = orc.route(qh, kh, 64, w.prefix_len, tau)
    rb = orc.route(qh, kp, 64, w.prefix_len, tau)
    assert np.array_equal(rb.keep, ra.keep[:, order])
    assert 0 < ra.keep[w.P:, w.P:].sum() < (w.M - w.P) ** 2


def test_query_block_permutation_moves_outputs():
    """Query blocks do not interact: permuting the video query blocks permutes
    their output blocks and keep rows, and nothing else."""
    w, q, k, v = _tiny_inputs()
    qh, kh, vh = q[0, 0], k[0, 0], v[0, 0]
    rng = np.random.default_rng(6)
    order = list(range(w.P)) + list(w.P + rng.permutation(w.M - w.P))
    a = orc.solattn_blocks(qh, kh, vh, 64, w.prefix_len, 1.0)
    b = orc.solattn_blocks(_permute_blocks(qh, order), kh, vh, 64, w.prefix_len, 1.0)
    np.testing.assert_allclose(b, _permute_blocks(a, order), rtol=0, atol=1e-12)
    ra = orc.route(qh, kh, 64, w.prefix_len, 1.0)
    rb = orc.route(_permute_blocks(qh, order), kh, 64, w.prefix_len, 1.0)
    assert np.array_equal(rb.keep, ra.keep[order, :])


def _brute_force_head(q, k, v, block, L, tau):
    """Independent plain-loop Sol-Attn for tiny inputs (lists and math only)."""
    N, D = len(q), len(q[0])
    M, P = N // block, L // block
    scale = 1.0 / math.sqrt(D)

    def mean_block(x, j):
        return [sum(x[t][d] for t in range(j * block, (j + 1) * block)) / block for d in range(D)]

    def dot(a, b):
        return sum(x * y for x, y in zip(a, b))

    qb = [mean_block(q, j) for j in range(M)]
    kb = [mean_block(k, j) for j in range(M)]
    vb = [mean_block(v, j) for j in range(M)]
    out = []
    for i in range(M):
        keep = [True] * M
        if i >= P and M > P:
            s = [scale * dot(qb[i], kb[j]) for j in range(P, M)]
            mu = sum(s) / len(s)
            sd = math.sqrt(sum((x - mu) ** 2 for x in s) / len(s))
            if tau != -math.inf and sd != 0:
                for j in range(P, M):
                    keep[j] = s[j - P] >= mu + tau * sd
        for r in range(i * block, (i + 1) * block):
            terms = []  # (logit, value)
            for j in range(M):
                if keep[j]:
                    for t in range(j * block, (j + 1) * block):
                        terms.append((scale * dot(q[r], k[t]), v[t]))
                else:
                    terms.append((scale * dot(q[r], kb[j]) + math.log(block), vb[j]))
            m = max(x for x, _ in terms)
            den = sum(math.exp(x - m) for x, _ in terms)
            out.append([sum(math.exp(x - m) * val[d] for x, val in terms) / den for d in range(D)])
    return out


@pytest.mark.parametrize("tau", [0.0, 0.8, 1.5])
def test_brute_force_tiny(tau):
    rng = np.random.default_rng(11)
    block, N, D, L = 8, 8 * 7, 3, 16
    base = np.repeat(rng.standard_normal((N // block, D)), block, axis=0)
    q = base + 0.5 * rng.standard_normal((N, D))
    k = base + 0.5 * rng.standard_normal((N, D))
    v = rng.standard_normal((N, D))
    ref = np.array(_brute_force_head(q.tolist(), k.tolist(), v.tolist(), block, L, tau))
    out = orc.solattn_blocks(q, k, v, block, L, tau)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    r = orc.route(q, k, block, L, tau)
    assert r.keep.sum() < r.keep.size or tau == 0.0


def test_dropping_the_count_weight_would_be_caught():
    """Plant the mistake in a copy of the oracle's correction: the worked example flags it."""
    g = _golden()
    q, k, v, block, L, scale = _golden_head(g)
    r = orc.route(q, k, block, L, 1.2, scale)
    # Recompute the row with weight 1 instead of c_j for skipped blocks.
    kept = np.nonzero(r.keep[3])[0]
    skipped = np.nonzero(~r.keep[3])[0]
    kv = np.array(g["setup"]["k_block_values"])
    vv = np.array(g["setup"]["v_block_values"])
    num = 64 * (np.exp(kv[kept]) * vv[kept]).sum() + (np.exp(kv[skipped]) * vv[skipped]).sum()
    den = 64 * np.exp(kv[kept]).sum() + np.exp(kv[skipped]).sum()
    wrong = num / den
    assert abs(wrong - g["expect"]["out_video_row_tau_1.2"]) > 1e-3


# ----------------------------------------------------------------------------- fixed budget (draft stage)

def test_budget_route_keeps_the_top_blocks_with_low_index_ties():
    block = 64
    # video scores 0.5, 2, 2, 1, 3 (prefix block 0 scores 9): budget 2 keeps
    # blocks 5 (3.0) and 2 (2.0, lower index than the tied block 3)
    k = _blocky([9.0, 0.5, 2.0, 2.0, 1.0, 3.0], block)
    q = np.ones_like(k)
    r = orc.route_budget(q, k, block, 64, 2, 1.0)
    for i in range(1, 6):
        assert list(np.nonzero(r.keep[i])[0]) == [0, 2, 5]
    assert r.keep[0].all()
    assert orc.route_budget(q, k, block, 64, 0, 1.0).keep[1:, 1:].sum() == 0
    assert orc.route_budget(q, k, block, 64, 99, 1.0).keep.all()


def test_budget_without_correction_is_attention_over_the_kept_keys():
    """No correction: each video row attends exactly to the prefix tokens plus
    its kept blocks' tokens -- textbook attention over that key subset."""
    w, q, k, v = _tiny_inputs()
    L, P = w.prefix_len, w.P
    scale = 1 / math.sqrt(w.D)
    qh, kh, vh = q[0, 1], k[0, 1], v[0, 1]
    r = orc.route_budget(qh, kh, 64, L, 3)
    assert (r.keep[P:, P:].sum(axis=1) == 3).all()
    for i in (P, P + 5, w.M - 1):
        tok = np.concatenate([np.arange(j * 64, (j + 1) * 64) for j in np.nonzero(r.keep[i])[0]])
        ref = _sdpa(qh[i * 64:(i + 1) * 64], kh[tok], vh[tok], scale)
        out = orc.solattn_blocks(qh, kh, vh, 64, L, 0.0, qblocks=[i], routing=r, correct=False)
        np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    # full budget = dense attention
    rf = orc.route_budget(qh, kh, 64, L, w.M)
    out = orc.solattn_blocks(qh, kh, vh, 64, L, 0.0, routing=rf, correct=False)
    np.testing.assert_allclose(out, _sdpa(qh, kh, vh, scale), rtol=0, atol=1e-12)


def test_budget_route_agrees_with_brute_force_ranking():
    rng = np.random.default_rng(21)
    N, D, L, kb = 64 * 12, 8, 128, 4
    q = rng.standard_normal((N, D))
    k = rng.standard_normal((N, D))
    r = orc.route_budget(q, k, 64, L, kb)
    M, P = N // 64, L // 64
    qb = [[sum(q[t, d] for t in range(i * 64, (i + 1) * 64)) / 64 for d in range(D)] for i in range(M)]
    kbar = [[sum(k[t, d] for t in range(j * 64, (j + 1) * 64)) / 64 for d in range(D)] for j in range(M)]
    for i in range(P, M):
        s = [(sum(a * b for a, b in zip(qb[i], kbar[j])), j) for j in range(P, M)]
        top = sorted(s, key=lambda x: (-x[0], x[1]))[:kb]
        assert sorted(j for _, j in top) == [j for j in range(P, M) if r.keep[i, j]]


# --------------------------------------------------------------------------- QKNorm + partial RoPE

def test_rms_norm_hand_values():
    # Row [3, 4]: mean square 12.5, so with eps = 0 the row becomes [3, 4] / 3.5355339...
    # = [0.8485281374238570, 1.1313708498984760] (computed by hand), times the weights.
    y = orc.rms_norm(np.array([[3.0, 4.0]]), np.array([1.0, 2.0]), 0.0)
    assert y[0, 0] == pytest.approx(0.8485281374238570, abs=1e-15)
    assert y[0, 1] == pytest.approx(2.0 * 1.1313708498984760, abs=1e-15)


def test_rms_norm_constant_row_closed_form():
    # A constant row c normalises to c / sqrt(c^2 + eps) in every dimension.
    c, eps = -3.0, 1e-6
    w = np.arange(1.0, 9.0)
    y = orc.rms_norm(np.full((1, 8), c), w, eps)
    assert np.allclose(y[0], w * (c / math.sqrt(c * c + eps)), rtol=0, atol=1e-15)


def test_rope_hand_values():
    # D = R = 4, base 10000: pair (0, 2) turns by pos * 1, pair (1, 3) by pos * 0.01.
    x = np.array([[1.0, 0, 0, 0], [0, 1.0, 0, 0], [0, 0, 0, 1.0]])
    y = orc.partial_rope(x, 4, 10000.0, positions=[1, 2, 3])
    # pos 1, e0: (cos 1, sin 1) on dims (0, 2)
    assert np.allclose(y[0], [0.5403023058681398, 0, 0.8414709848078965, 0], atol=1e-15)
    # pos 2, e1: angle 0.02 on dims (1, 3)
    assert np.allclose(y[1], [0, 0.9998000066665778, 0, 0.01999866669333308], atol=1e-15)
    # pos 3, e3 (second member of pair (1, 3)): (-sin 0.03, cos 0.03) on dims (1, 3)
    assert np.allclose(y[2], [0, -0.02999550020249566, 0, 0.9995500337489875], atol=1e-15)


def test_rope_invariants():
    rng = np.random.default_rng(7)
    N, D, R = 40, 16, 8
    x = rng.normal(size=(N, D))
    y = orc.partial_rope(x, R, 10000.0)
    assert np.array_equal(y[0], x[0])                    # position 0 is the identity
    assert np.array_equal(y[:, R:], x[:, R:])            # dimensions past R untouched
    for i in range(R // 2):                              # each rotated pair keeps its length
        assert np.allclose(np.hypot(y[:, i], y[:, i + R // 2]), np.hypot(x[:, i], x[:, i + R // 2]),
                           rtol=1e-13)
    # Relative position: <rope(a, m), rope(b, n)> depends on m - n only.
    a, b = rng.normal(size=D), rng.normal(size=D)
    m, n = 29, 11
    lhs = orc.partial_rope(a[None], D, positions=[m])[0] @ orc.partial_rope(b[None], D, positions=[n])[0]
    rhs = orc.partial_rope(a[None], D, positions=[m - n])[0] @ b
    assert lhs == pytest.approx(rhs, rel=1e-12)


def test_qknorm_rope_composition_order_hand_values():
    # The chain is RMSNorm (with its weight) first, then RoPE.  With D = R = 2,
    # w = [1, 2], eps = 0, the row [1, 0] at position 1 normalises to
    # [1, 0] / sqrt(1/2) * [1, 2] = [sqrt 2, 0] and then turns by 1 radian:
    # [sqrt 2 cos 1, sqrt 2 sin 1].  Applying the weight after the rotation
    # would give [sqrt 2 cos 1, 2 sqrt 2 sin 1]; rotating first and then
    # normalising with the weight gives the same wrong value, so this pins the
    # order.  Row 0 (position 0) is not rotated: [1, 0] -> [sqrt 2, 0] as well.
    x = np.array([[1.0, 0.0], [1.0, 0.0]])
    y = orc.qknorm_rope(x, np.array([1.0, 2.0]), 0.0, 2)
    r2 = math.sqrt(2.0)
    assert np.allclose(y[0], [r2, 0.0], rtol=0, atol=1e-15)
    assert np.allclose(y[1], [r2 * 0.5403023058681398, r2 * 0.8414709848078965], rtol=0, atol=1e-15)
    wrong = [r2 * 0.5403023058681398, 2 * r2 * 0.8414709848078965]
    assert not np.allclose(y[1], wrong, atol=1e-3)


def test_qknorm_rope_weight_inside_rotation_pair():
    # A non-uniform weight on a rotated pair separates "weight, then rotate"
    # from "rotate, then weight": for x = [0, 1] at position 1 with w = [3, 1],
    # the normalised row is [0, sqrt 2] (the weight meets a zero), so the
    # rotation gives [-sqrt 2 sin 1, sqrt 2 cos 1]; weighting after the
    # rotation would scale the first entry by 3.
    x = np.array([[0.0, 1.0], [0.0, 1.0]])
    y = orc.qknorm_rope(x, np.array([3.0, 1.0]), 0.0, 2)
    r2 = math.sqrt(2.0)
    assert np.allclose(y[1], [-r2 * 0.8414709848078965, r2 * 0.5403023058681398], rtol=0, atol=1e-15)


# --------------------------------------------------------------------------- first-order Taylor compensation

def test_taylor_first_order_hand_values():
    # Two keys k = kbar +- a u with kbar = 0, u = e0, a = 0.1; values e0 and e1;
    # q = e0, scale 1.  By hand: Cov = (1/2) sum_t d_t (v_t - vbar)^T
    # = (a/2) u (v1 - v2)^T = [[0.05, -0.05], [0, 0]], so Cov^T q = [0.05, -0.05];
    # weight c e^{q.kbar} = 2; order 0 gives num = 2 vbar = [1, 1], order 1
    # gives 2 ([0.5, 0.5] + [0.05, -0.05]) = [1.1, 0.9].  The exact sum is
    # e^{0.1} e0 + e^{-0.1} e1 = [1.1051709180756477, 0.9048374180359595].
    k = np.array([[0.1, 0.0], [-0.1, 0.0]])
    v = np.array([[1.0, 0.0], [0.0, 1.0]])
    q = np.array([[1.0, 0.0]])
    w0, n0 = orc.taylor_block_terms(q, k, v, 1.0, order=0)
    w1, n1 = orc.taylor_block_terms(q, k, v, 1.0, order=1)
    assert w0[0] == pytest.approx(2.0) and w1[0] == pytest.approx(2.0)
    assert np.allclose(n0[0], [1.0, 1.0], atol=1e-15)
    assert np.allclose(n1[0], [1.1, 0.9], atol=1e-15)
    # a transposed moment (Cov q instead of Cov^T q) would give [1.1, 1.0]
    assert not np.allclose(n1[0], [1.1, 1.0], atol=1e-3)
    exact = np.exp(k @ q[0]) @ v
    assert np.allclose(exact, [1.1051709180756477, 0.9048374180359595], atol=1e-15)
    assert np.abs(n1[0] - exact).max() < np.abs(n0[0] - exact).max() / 10


def test_taylor_error_orders_by_convergence():
    # Keys kbar + alpha * d_t: the numerator error of order 0 falls like
    # alpha, that of order 1 like alpha^2; the denominator error of both like
    # alpha^2 (its first-order term is zero).
    rng = np.random.default_rng(11)
    c, D = 64, 16
    kbar = rng.normal(size=D) * 0.3
    d = rng.normal(size=(c, D))
    d -= d.mean(axis=0)
    v = rng.normal(size=(c, D)) + 0.5 * d[:, :1]  # values correlated with the key offsets
    q = rng.normal(size=(3, D))
    s = 1.0 / math.sqrt(D)

    def errs(alpha, order):
        k = kbar + alpha * d
        den, num = orc.taylor_block_terms(q, k, v, s, order=order)
        e = np.exp(s * (q @ k.T))
        return np.abs(num - e @ v).max(), np.abs(den - e.sum(axis=1)).max()

    a = 0.02
    n0a, d0a = errs(a, 0)
    n0b, d0b = errs(a / 2, 0)
    n1a, d1a = errs(a, 1)
    n1b, d1b = errs(a / 2, 1)
    assert 1.8 < n0a / n0b < 2.2          # first order error of the zeroth-order term
    assert 3.6 < n1a / n1b < 4.4          # second order once the first-order term is in
    assert 3.6 < d0a / d0b < 4.4 and d1a == d0a


def test_taylor_first_order_reduces_to_zeroth_for_identical_keys():
    rng = np.random.default_rng(12)
    B, H, N, D, L = 1, 1, 64 * 10, 16, 128
    q = rng.normal(size=(N, D))
    k = np.repeat(rng.normal(size=(N // 64, D)), 64, axis=0)
    v = rng.normal(size=(N, D))
    k[:L] = rng.normal(size=(L, D))
    r = orc.route(q, k, 64, L, 1.0)
    assert not r.keep.all()
    o0 = orc.solattn_blocks(q, k, v, 64, L, 1.0, routing=r)
    o1 = orc.solattn_blocks(q, k, v, 64, L, 1.0, routing=r, order=1)
    assert np.allclose(o0, o1, rtol=0, atol=1e-14)
    # ... where identical values too make both exact
    v2 = np.repeat(rng.normal(size=(N // 64, D)), 64, axis=0)
    v2[:L] = rng.normal(size=(L, D))
    o1 = orc.solattn_blocks(q, k, v2, 64, L, 1.0, routing=r, order=1)
    assert np.allclose(o1, orc.dense_rows(q, k, v2), rtol=0, atol=1e-12)


def test_taylor_pooled_query_form_matches_per_row_form_on_constant_rows():
    # With every query row of a block equal, the pooled query is that row and
    # the cheaper per-block-pair form is the per-row form.
    rng = np.random.default_rng(13)
    N, D, L = 64 * 8, 8, 64
    q = np.repeat(rng.normal(size=(N // 64, D)), 64, axis=0)
    k, v = rng.normal(size=(N, D)), rng.normal(size=(N, D))
    r = orc.route(q, k, 64, L, 0.5)
    a = orc.solattn_blocks(q, k, v, 64, L, 0.5, routing=r, order=1)
    b = orc.solattn_blocks(q, k, v, 64, L, 0.5, routing=r, order=1, pooled_query_term=True)
    assert np.allclose(a, b, rtol=0, atol=1e-14)
    assert not np.allclose(a, orc.solattn_blocks(q, k, v, 64, L, 0.5, routing=r), atol=1e-6)


def test_taylor_first_order_matches_brute_force_expansion():
    # solattn_blocks(order=1) against a plain-loop evaluation of the expanded
    # terms, block by block and row by row.
    rng = np.random.default_rng(14)
    N, D, L, tau = 64 * 6, 4, 64, 0.7
    q, k, v = (rng.normal(size=(N, D)) for _ in range(3))
    s = 1.0 / math.sqrt(D)
    r = orc.route(q, k, 64, L, tau)
    got = orc.solattn_blocks(q, k, v, 64, L, tau, routing=r, order=1)
    M = N // 64
    for i in range(M):
        for rr in range(0, 64, 21):
            row = q[64 * i + rr]
            terms_w, terms_v = [], []
            for j in range(M):
                kb, vb = k[64 * j:64 * j + 64], v[64 * j:64 * j + 64]
                if r.keep[i, j]:
                    for t in range(64):
                        terms_w.append(math.exp(s * sum(row[d] * kb[t, d] for d in range(D))))
                        terms_v.append(vb[t])
                else:
                    km = [sum(kb[t, d] for t in range(64)) / 64 for d in range(D)]
                    vm = [sum(vb[t, d] for t in range(64)) / 64 for d in range(D)]
                    cov = [[sum((kb[t, a] - km[a]) * (vb[t, b] - vm[b]) for t in range(64)) / 64
                            for b in range(D)] for a in range(D)]
                    terms_w.append(64 * math.exp(s * sum(row[d] * km[d] for d in range(D))))
                    terms_v.append(np.array([vm[b] + s * sum(row[a] * cov[a][b] for a in range(D))
                                             for b in range(D)]))
            want = sum(w * x for w, x in zip(terms_w, terms_v)) / sum(terms_w)
            assert np.allclose(got[64 * i + rr], want, rtol=0, atol=1e-12)
