"""CPU fp64 oracle for Sol-Attn.  TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check of the entry module and the benchmark's
CPU-baseline / reference legs may import this module.  The CUDA library never
calls it and shares no code with it.

It is deliberately plain and slow: numpy fp64, one query block at a time, with
a library matmul as the only building block.  Every step follows the pages in
their own order; where the pages leave a step open the reading is stated in
the function's docstring.

Sources (the pages hold prose only; no formula, listing or worked example):

[S1] "NVIDIA 团队开源 Sol-H3 的 DGX Spark 版本" (arex-research 3d0ff631),
     section "119.68 GiB memory pool: how both models stay resident", the
     Sol-Attn bullet: blocks are picked while attention runs; each query block
     filters light query-key scores with its own threshold; selected blocks are
     computed exactly; skipped blocks get an approximate correction from
     pooled K/V summaries; routing, sparse compute and correction share one
     online softmax; no score map or routing index tensor is materialised.
[S2] "英伟达开源 Sol-H3，给 MiniMax-H3 加速" (yanziyuan 171844), the
     "sparse attention" paragraph: scoring is done in 64-token blocks and only
     high-scoring blocks are computed; the next paragraph gives tau = 1.0, 1.25,
     1.5 for the three refine steps; the "safety rail" paragraph: text | cond
     video | audio | target video are packed into one sequence and the whole
     prefix takes exact attention.
[S3] "MiniMax 官宣 NVIDIA Sol 团队 H3 加速" (arex-research 2a2a70ca), section
     "speed-up comes from stacking every stage of the pipeline", the Sol-Attn
     item: 64-token query blocks; a query-adaptive threshold "mean + tau x
     standard deviation" decides which blocks keep exact attention; skipped
     blocks are compensated approximately from pooled K/V; one shared
     online-softmax forward; no retraining.
[S4] "MiniMax 官推背书 Sol Engine" (arex-research 647c3193), section "another
     framing on the same project page: 3.95x near-lossless": rejected blocks get
     a "Taylor approximation" compensation.
[S5] Sol-H3 DGX Spark release (arex-research 3d0ff631), section "latent
     hand-off: 384p draft to 768p refine": the draft stage uses sparse attention
     at 90 % video sparsity in 64-token blocks on cuDNN block-sparse attention,
     i.e. a fixed budget of video key blocks per query block and no
     compensation for the dropped ones.

[S6] [S3]'s page, same section, the "fused operators" item: the residual +
     RMSNorm + modulation, QKNorm + partial RoPE and SwiGLU chains keep their
     intermediates in registers or on chip; and the kocpc.com.tw report of the
     same release (www.kocpc.com.tw/?p=668110), section "技術組成：Sol Engine ×
     Sol-Attn 完整堆疊": the lossless kernel work fuses QKNorm + RoPE among
     others to cut HBM round trips.  The pages name the chain only.

Readings where the pages are silent (each also listed in the design notes):
  * pooling is the arithmetic mean over the block's tokens (count c_j);
  * the block score uses pooled queries: s_ij = scale * <qbar_i, kbar_j>,
    scale = 1/sqrt(D) unless given;
  * mean and standard deviation are the population moments of s_i. over the
    video key blocks j >= P only (the prefix is forced exact and left out);
  * keep iff s_ij >= mu_i + tau * sigma_i; tau = -inf keeps all; when all
    video scores of a query block are equal (sigma_i = 0 exactly; tested as
    max == min, since a rounded mean of equal values can leave a spurious
    1e-17 spread) every block is kept; tau = +inf with sigma_i > 0 keeps no
    video block;
  * query blocks i < P (prefix queries) attend densely; key blocks j < P are
    always kept;
  * the correction is the zeroth-order term of the Taylor expansion around
    kbar_j: a skipped block j contributes weight c_j * exp(scale * <q_r, kbar_j>)
    (logit + ln c_j) with value vbar_j, inside the same softmax as the exact
    logits.  Per-row q_r is used here, since only K/V are named as pooled;
  * attention is bidirectional (no causal mask).

Functions taking a single head use arrays [N, D]; the batched wrappers take
[B, H, N, D].  All arithmetic is fp64.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

BLOCK = 64


def _check_head(x: np.ndarray) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    if x.ndim != 2:
        raise ValueError("expected a single head [N, D]")
    return x


def pool_blocks(x: np.ndarray, block: int = BLOCK):
    """Mean of each block of ``block`` consecutive rows [S1 "pooled K/V summaries"].

    Returns (means [M, D], counts [M]) with M = ceil(N / block); the last block
    may hold fewer than ``block`` rows, and its count says how many.
    """
    x = _check_head(x)
    N, D = x.shape
    M = -(-N // block)
    means = np.empty((M, D))
    counts = np.empty(M, dtype=np.int64)
    for j in range(M):
        rows = x[j * block:min(N, (j + 1) * block)]
        counts[j] = rows.shape[0]
        means[j] = rows.sum(axis=0) / counts[j]
    return means, counts


@dataclass
class Route:
    """Routing of one head: scores, per-query-block statistics and the keep set."""

    score: np.ndarray   # [M, M] scale * <qbar_i, kbar_j>; only i, j >= P enter the statistics
    mu: np.ndarray      # [M] mean over video key blocks (nan for prefix query blocks)
    sigma: np.ndarray   # [M] population std over video key blocks (nan for prefix query blocks)
    thr: np.ndarray     # [M] mu + tau * sigma (nan where not used)
    keep: np.ndarray    # [M, M] bool, forced entries included


def route(q: np.ndarray, k: np.ndarray, block: int, prefix_len: int, tau: float,
          scale: float | None = None) -> Route:
    """Score, threshold and keep set of every query block of one head.

    [S2] 64-token block scoring; [S1] light query-key scores filtered with a
    per-query-block threshold; [S3] threshold = mean + tau * std; [S2 safety
    rail] prefix exact.
    """
    q = _check_head(q)
    k = _check_head(k)
    N, D = q.shape
    if prefix_len % block:
        raise ValueError("prefix_len must be a whole number of blocks")
    if math.isnan(tau):
        raise ValueError("tau is NaN")
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    qbar, _ = pool_blocks(q, block)
    kbar, _ = pool_blocks(k, block)
    M = qbar.shape[0]
    P = prefix_len // block

    # 1. light scores from pooled queries and pooled keys
    score = scale * (qbar @ kbar.T)

    keep = np.ones((M, M), dtype=bool)
    mu = np.full(M, np.nan)
    sigma = np.full(M, np.nan)
    thr = np.full(M, np.nan)
    nv = M - P
    for i in range(P, M):
        if nv == 0:
            break
        s = score[i, P:]
        # 2. population mean and std over the video key blocks, two passes
        mu[i] = s.sum() / nv
        sigma[i] = math.sqrt(((s - mu[i]) ** 2).sum() / nv)
        if s.max() == s.min():
            sigma[i] = 0.0  # all scores equal: no spread, whatever the rounding of mu
        # 3. keep the blocks at or above mean + tau * std
        if tau == -math.inf or sigma[i] == 0.0:
            continue  # everything kept
        thr[i] = mu[i] + tau * sigma[i]
        keep[i, P:] = s >= thr[i]
    # prefix key blocks (j < P) and prefix query blocks (i < P) stay kept
    return Route(score=score, mu=mu, sigma=sigma, thr=thr, keep=keep)


def route_budget(q: np.ndarray, k: np.ndarray, block: int, prefix_len: int, keep_blocks: int,
                 scale: float | None = None) -> Route:
    """Fixed-budget routing of the draft stage [S5]: every video query block
    keeps its ``keep_blocks`` highest-scoring video key blocks (same pooled
    scores as ``route``; ties go to the lower block index), plus the prefix.
    Prefix query blocks stay dense.  mu/sigma/thr are not used (nan)."""
    q = _check_head(q)
    k = _check_head(k)
    N, D = q.shape
    if prefix_len % block:
        raise ValueError("prefix_len must be a whole number of blocks")
    if keep_blocks < 0:
        raise ValueError("keep_blocks must be >= 0")
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    qbar, _ = pool_blocks(q, block)
    kbar, _ = pool_blocks(k, block)
    M = qbar.shape[0]
    P = prefix_len // block
    score = scale * (qbar @ kbar.T)
    keep = np.ones((M, M), dtype=bool)
    for i in range(P, M):
        s = score[i, P:]
        order = np.argsort(-s, kind="stable")  # descending, lower index first on ties
        keep[i, P:] = False
        keep[i, P + order[:keep_blocks]] = True
    nan = np.full(M, np.nan)
    return Route(score=score, mu=nan, sigma=nan.copy(), thr=nan.copy(), keep=keep)


def block_cross_moment(k: np.ndarray, v: np.ndarray, block: int = BLOCK):
    """Centred key/value cross moments of every block, for the first-order
    term of the Taylor compensation [S4]:
        Cov_j = (1 / c_j) * sum_t (k_t - kbar_j) (v_t - vbar_j)^T   (D x D).
    Returns [M, D, D]."""
    k = _check_head(k)
    v = _check_head(v)
    N, D = k.shape
    kbar, counts = pool_blocks(k, block)
    vbar, _ = pool_blocks(v, block)
    out = np.empty((kbar.shape[0], D, v.shape[1]))
    for j in range(kbar.shape[0]):
        sl = slice(j * block, min(N, (j + 1) * block))
        out[j] = (k[sl] - kbar[j]).T @ (v[sl] - vbar[j]) / counts[j]
    return out


def taylor_block_terms(q_rows: np.ndarray, k_blk: np.ndarray, v_blk: np.ndarray, scale: float,
                       order: int = 0, q_expand=None):
    """Compensation of one skipped block for the given query rows [S4]: the
    Taylor expansion of its exact terms around the pooled key kbar.

    Exact:   den = sum_t e^{s q.k_t},   num = sum_t e^{s q.k_t} v_t.
    With k_t = kbar + d_t (sum_t d_t = 0) and e^{s q.d_t} ~ 1 + s q.d_t:
      order 0:  den = c e^{s q.kbar},  num = c e^{s q.kbar} vbar;
      order 1:  den unchanged (its first-order term is s q.sum_t d_t = 0),
                num = c e^{s q.kbar} (vbar + s Cov^T q),
                Cov = (1/c) sum_t d_t (v_t - vbar)^T.
    ``q_expand`` (rows x D, default the rows themselves) is the query used in
    the first-order term: passing the block's pooled query gives the cheaper
    per-block-pair form.  Returns (den [rows], num [rows, D]) without any
    max subtraction (small examples only).
    """
    q_rows = np.atleast_2d(np.asarray(q_rows, dtype=np.float64))
    k_blk = _check_head(k_blk)
    v_blk = _check_head(v_blk)
    c = k_blk.shape[0]
    kbar = k_blk.mean(axis=0)
    vbar = v_blk.mean(axis=0)
    w = c * np.exp(scale * (q_rows @ kbar))
    num = w[:, None] * vbar[None, :]
    if order >= 1:
        cov = (k_blk - kbar).T @ (v_blk - vbar) / c
        qe = q_rows if q_expand is None else np.atleast_2d(np.asarray(q_expand, dtype=np.float64))
        num = num + w[:, None] * (scale * (qe @ cov))
    if order > 1:
        raise ValueError("orders 0 and 1 only")
    return w, num


def solattn_blocks(q: np.ndarray, k: np.ndarray, v: np.ndarray, block: int, prefix_len: int,
                   tau: float, scale: float | None = None, qblocks=None,
                   routing: Route | None = None, correct: bool = True, order: int = 0,
                   pooled_query_term: bool = False) -> np.ndarray:
    """Sol-Attn output rows of the listed query blocks of one head.

    For each query row r of block i [S1, S3]:
      exact logits   l_rt = scale * <q_r, k_t> for every token t of a kept block;
      pooled logits  l_rj = scale * <q_r, kbar_j> + ln c_j for every skipped block j
                     (zeroth-order term of the compensation [S4]);
      out_r = (sum_t e^{l_rt - m} v_t + sum_j e^{l_rj - m} vbar_j)
              / (sum_t e^{l_rt - m} + sum_j e^{l_rj - m}),  m = max of all logits,
    i.e. one softmax over exact and pooled terms together.
    With ``correct=False`` skipped blocks are dropped instead (plain
    block-sparse attention, the draft stage of [S5]).
    ``order=1`` adds the first-order term of the compensation (see
    ``taylor_block_terms``): skipped block j's value becomes
    vbar_j + scale * Cov_j^T q_r, or with ``pooled_query_term`` the block's
    pooled query qbar_i in place of q_r; its weight is unchanged.
    Returns [len(qblocks) * block, D] (rows of a short last block are omitted).
    """
    q = _check_head(q)
    k = _check_head(k)
    v = _check_head(v)
    N, D = q.shape
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    r = routing if routing is not None else route(q, k, block, prefix_len, tau, scale)
    kbar, counts = pool_blocks(k, block)
    vbar, _ = pool_blocks(v, block)
    M = kbar.shape[0]
    if order not in (0, 1):
        raise ValueError("orders 0 and 1 only")
    cov = block_cross_moment(k, v, block) if (order == 1 and correct) else None
    qbar = pool_blocks(q, block)[0] if pooled_query_term else None
    if qblocks is None:
        qblocks = range(M)
    outs = []
    for i in qblocks:
        rows = q[i * block:min(N, (i + 1) * block)]
        kept = np.nonzero(r.keep[i])[0]
        skipped = np.nonzero(~r.keep[i])[0] if correct else np.zeros(0, dtype=np.int64)
        tok = np.concatenate([np.arange(j * block, min(N, (j + 1) * block)) for j in kept]) \
            if len(kept) else np.zeros(0, dtype=np.int64)
        l_exact = scale * (rows @ k[tok].T)
        l_pool = scale * (rows @ kbar[skipped].T) + np.log(counts[skipped].astype(np.float64))
        m = np.maximum(l_exact.max(axis=1, initial=-np.inf), l_pool.max(axis=1, initial=-np.inf))
        w_exact = np.exp(l_exact - m[:, None])
        w_pool = np.exp(l_pool - m[:, None])
        num = w_exact @ v[tok] + w_pool @ vbar[skipped]
        if cov is not None:
            qe = np.broadcast_to(qbar[i], rows.shape) if pooled_query_term else rows
            for col, j in enumerate(skipped):
                num += w_pool[:, col:col + 1] * (scale * (qe @ cov[j]))
        den = w_exact.sum(axis=1) + w_pool.sum(axis=1)
        outs.append(num / den[:, None])
    return np.concatenate(outs, axis=0) if outs else np.zeros((0, D))


def dense_rows(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float | None = None,
               rows=None) -> np.ndarray:
    """Textbook softmax attention softmax(scale * q k^T) v for the listed query rows.

    This is the comparator role FA4 plays on the pages [S1, Sol-Attn bullet]
    and the tau = -inf limit of Sol-Attn.
    """
    q = _check_head(q)
    k = _check_head(k)
    v = _check_head(v)
    D = q.shape[1]
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    qr = q if rows is None else q[np.asarray(rows)]
    logits = scale * (qr @ k.T)
    m = logits.max(axis=1, keepdims=True)
    w = np.exp(logits - m)
    return (w @ v) / w.sum(axis=1, keepdims=True)


def keep_masks(q: np.ndarray, k: np.ndarray, block: int, prefix_len: int, tau: float,
               scale: float | None = None) -> list:
    """Route of every (b, h) head of [B, H, N, D] inputs, in (b, h) order."""
    B, H = q.shape[:2]
    return [route(q[b, h], k[b, h], block, prefix_len, tau, scale)
            for b in range(B) for h in range(H)]


def solattn(q, k, v, block: int, prefix_len: int, tau: float, scale: float | None = None,
            qblocks=None) -> np.ndarray:
    """Sol-Attn over [B, H, N, D]; with ``qblocks`` only those query blocks' rows."""
    B, H, N, D = q.shape
    out = []
    for b in range(B):
        for h in range(H):
            out.append(solattn_blocks(q[b, h], k[b, h], v[b, h], block, prefix_len, tau,
                                      scale, qblocks))
    return np.stack(out).reshape(B, H, -1, D)


def dense(q, k, v, scale: float | None = None, rows=None) -> np.ndarray:
    """Dense attention over [B, H, N, D]; with ``rows`` only those query rows."""
    B, H, N, D = q.shape
    out = [dense_rows(q[b, h], k[b, h], v[b, h], scale, rows) for b in range(B) for h in range(H)]
    return np.stack(out).reshape(B, H, -1, D)


# ---------------------------------------------------------------------------
# QKNorm + partial RoPE in front of the pooling [S6].  The pages name the
# chain and nothing else; the readings:
#   * QKNorm is RMSNorm over the head dimension of each q (and k) row, with a
#     per-dimension weight: y = x / sqrt(mean(x^2) + eps) * w;
#   * "partial" RoPE rotates the first R (rope_dims) dimensions of the row and
#     leaves the rest, pairing dimension i with i + R/2 ("rotate half") for
#     i < R/2, by the angle pos * base^(-2 i / R);
#   * pos is the token's index in its (b, h) sequence, prefix included;
#   * the kernel writes the result as bf16, and the pooled summaries are the
#     block means of those bf16 values (what a separate pooling pass over the
#     written tensors would compute).


def rms_norm(x: np.ndarray, w: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm of each row over the last dimension [S6 "QKNorm"]: x / sqrt(mean(x^2) + eps) * w."""
    x = _check_head(x)
    w = np.asarray(w, dtype=np.float64)
    if w.shape != (x.shape[1],):
        raise ValueError("weight must have one entry per dimension")
    rms = np.sqrt(np.mean(x * x, axis=1, keepdims=True) + float(eps))
    return x / rms * w


def partial_rope(x: np.ndarray, rope_dims: int, base: float = 10000.0, positions=None) -> np.ndarray:
    """Rotary embedding of the first ``rope_dims`` dimensions of each row [S6 "partial RoPE"].

    Rows are positions 0..N-1 unless ``positions`` is given.  For i < R/2 the
    pair (x_i, x_{i+R/2}) is rotated by theta = pos * base^(-2 i / R):
    (a, b) -> (a cos theta - b sin theta, a sin theta + b cos theta).
    Dimensions R..D-1 are returned unchanged.
    """
    x = _check_head(x)
    N, D = x.shape
    R = int(rope_dims)
    if R < 0 or R > D or R % 2:
        raise ValueError("rope_dims must be even and within [0, D]")
    y = x.copy()
    if R == 0:
        return y
    pos = np.arange(N, dtype=np.float64) if positions is None else np.asarray(positions, dtype=np.float64)
    half = R // 2
    for i in range(half):
        theta = pos * float(base) ** (-2.0 * i / R)
        c, s_ = np.cos(theta), np.sin(theta)
        a, b = x[:, i], x[:, i + half]
        y[:, i] = a * c - b * s_
        y[:, i + half] = a * s_ + b * c
    return y


def qknorm_rope(x: np.ndarray, w: np.ndarray, eps: float, rope_dims: int, base: float = 10000.0):
    """The fused chain for one head: RMSNorm, then partial RoPE [S6]."""
    return partial_rope(rms_norm(x, w, eps), rope_dims, base)

