"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
and compare it with the CPU fp64 oracle on the same seeded inputs.

Tolerances (the operator's acceptance bar):
  * keep mask: >= 99.9 % of (query block, key block) pairs agree, and every
    disagreement lies within 1e-3 * sigma_i of its threshold (fp32 routing on
    the GPU vs fp64 in the oracle); a disagreement where the oracle's answer
    is forced (prefix rows or columns, tau = -inf, rows whose scores are all
    equal) fails outright;
  * output: relative L2 error <= 1e-2 and max abs error <= 2e-2 versus fp64
    on the bf16 inputs.
"""

from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

from block_sparse_attention_threshold_b200 import abi, synthetic as syn
from oracle import sol_attn_oracle as orc

REL_L2 = 1e-2
MAX_ABS = 2e-2
MASK_AGREE = 0.999
MASK_BAND = 1e-3


def to_device(*arrays):
    dev = torch.device("cuda", 0)
    return [torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
            for a in arrays]


def run_sol(w, tau, q, k, v, want_mask=True, budget=0, correct=True):
    """Sol-Attn on device tensors; returns (out bf16 tensor, keep [B,H,M,M] bool or None,
    kept_pairs, exact_pairs).  budget > 0 selects fixed-budget routing;
    correct=False drops skipped blocks."""
    M = w.M
    dev = q.device
    opts = abi.Opts()
    opts.budget_blocks = int(budget)
    opts.skip_correction = 0 if correct else 1
    cnt = torch.zeros(2, dtype=torch.int64, device=dev)
    opts.kept_pairs = cnt.data_ptr()
    opts.exact_pairs = cnt.data_ptr() + 8
    mask = None
    if want_mask:
        mask = torch.zeros(w.B * w.H * M * abi.mask_words(M), dtype=torch.int32, device=dev)
        opts.debug_mask = mask.data_ptr()
    out = abi.forward(q, k, v, tau, w.prefix_len, opts=opts)
    torch.cuda.synchronize()
    status = abi.device_status()
    assert status == abi.OK, abi.status_string(status)
    keep = None
    if want_mask:
        words = mask.cpu().numpy().view(np.uint32).reshape(w.B, w.H, M, -1)
        keep = abi.unpack_mask(words, M)
    c = cnt.cpu().tolist()
    return out, keep, int(c[0]), int(c[1])


def _blas_single_thread():
    try:
        from threadpoolctl import threadpool_limits
        return threadpool_limits(1)
    except Exception:  # pragma: no cover
        import contextlib
        return contextlib.nullcontext()


def oracle_compare(w, tau, qb, kb, vb, out, keep=None, qblocks=None, dense=False, workers=None,
                   budget=0, correct=True, decode=None):
    """Compare GPU `out` (and `keep`) with the oracle, head by head in threads.

    qblocks: query-block indices to check per head (None = all).
    budget > 0: fixed-budget routing; mask disagreements are then measured
    against the cut score (the budget-th highest) instead of the threshold.
    decode: (fq, fk, fv) turning one head's stored bits into fp64 values
    (default: bf16 bits widened exactly).
    Returns a dict of metrics; raises AssertionError on a violated bound.
    """
    fq, fk, fv = decode or (syn.bf16_bits_to_fp64,) * 3
    got_all = out.float().cpu().numpy()
    B, H = w.B, w.H
    jobs = [(b, h) for b in range(B) for h in range(H)]

    def one(bh):
        b, h = bh
        q64 = fq(qb[b, h])
        k64 = fk(kb[b, h])
        v64 = fv(vb[b, h])
        res = {}
        blocks = range(w.M) if qblocks is None else qblocks
        rows = np.concatenate([np.arange(i * 64, (i + 1) * 64) for i in blocks])
        if dense:
            ref = orc.dense_rows(q64, k64, v64, rows=rows)
        else:
            r = orc.route(q64, k64, 64, w.prefix_len, tau)
            cut = r.thr
            if budget > 0:
                rb = orc.route_budget(q64, k64, 64, w.prefix_len, budget)
                P = w.P
                cut = np.full(w.M, np.nan)
                for i in range(P, w.M):
                    sv = np.sort(r.score[i, P:])[::-1]
                    cut[i] = sv[min(budget, sv.size) - 1]
                r_use = orc.Route(score=r.score, mu=r.mu, sigma=r.sigma, thr=cut, keep=rb.keep)
            else:
                r_use = r
            ref = orc.solattn_blocks(q64, k64, v64, 64, w.prefix_len, tau, qblocks=blocks, routing=r_use,
                                     correct=correct)
            if keep is not None:
                g = keep[b, h]
                mism = g != r_use.keep
                res["pairs"] = r_use.keep.size
                res["mismatch"] = int(mism.sum())
                res["hard_mismatch"] = 0
                if res["mismatch"]:
                    ii, jj = np.nonzero(mism)
                    # A disagreement is only admissible at a routed pair
                    # (video query block, video key block) whose row has a
                    # finite cut and a positive spread.  Everywhere else the
                    # oracle's answer is forced (prefix rows and columns,
                    # tau = -inf, all scores equal), so any mismatch fails.
                    P = w.P
                    sig = r.sigma[ii]
                    ok = (ii >= P) & (jj >= P) & np.isfinite(cut[ii]) & np.isfinite(sig) & (sig > 0)
                    res["hard_mismatch"] = int((~ok).sum())
                    if ok.any():
                        dist = np.abs(r.score[ii[ok], jj[ok]] - cut[ii[ok]]) / sig[ok]
                        res["worst_band"] = float(dist.max())
                res["kept"] = int(r_use.keep.sum())
        got = got_all[b, h][rows].astype(np.float64)
        res["err2"] = float(np.sum((got - ref) ** 2))
        res["ref2"] = float(np.sum(ref ** 2))
        res["maxabs"] = float(np.abs(got - ref).max())
        return res

    with _blas_single_thread():
        with ThreadPoolExecutor(max_workers=workers or os.cpu_count()) as ex:
            results = list(ex.map(one, jobs))
    m = {
        "rel_l2": math.sqrt(sum(r["err2"] for r in results) / sum(r["ref2"] for r in results)),
        "max_abs": max(r["maxabs"] for r in results),
    }
    if keep is not None and not dense:
        pairs = sum(r["pairs"] for r in results)
        mism = sum(r["mismatch"] for r in results)
        m["mask_agree"] = 1.0 - mism / pairs
        m["mask_mismatch"] = mism
        m["worst_band"] = max((r.get("worst_band", 0.0) for r in results), default=0.0)
        m["hard_mismatch"] = sum(r["hard_mismatch"] for r in results)
        m["oracle_kept"] = sum(r["kept"] for r in results)
    return m


def assert_parity(m, rel_l2=REL_L2, max_abs=MAX_ABS):
    assert m["rel_l2"] <= rel_l2, m
    assert m["max_abs"] <= max_abs, m
    if "mask_agree" in m:
        assert m["mask_agree"] >= MASK_AGREE, m
        assert m["worst_band"] <= MASK_BAND, m
        assert m["hard_mismatch"] == 0, m


# ----------------------------------------------------------------------------- fp32 reference

def fp32_route(w, tau, qf, kf):
    """Keep bits of the video part ([B, H, M-P, M-P]) from the definition in
    fp32 PyTorch: pooled means, population std over the video key blocks,
    keep iff score >= mean + tau * std.  qf, kf: float32 [B, H, N, D] on any
    device.  A cross-check for full-length runs; the oracle stays the
    authority (tests/test_parity_harness.py pins this to it)."""
    B, H, N, D, M, P = w.B, w.H, w.N, w.D, w.M, w.P
    qbar, kbar = (x.view(B, H, M, 64, D).mean(3) for x in (qf, kf))
    s = (D ** -0.5) * qbar[:, :, P:] @ kbar[:, :, P:].transpose(-1, -2)
    mu = s.mean(-1, keepdim=True)
    sd = s.std(-1, unbiased=False, keepdim=True)
    return s >= mu + tau * sd


def fp32_rows(w, qf, kf, vf, keep, b, h, i0, i1):
    """Output rows of query blocks [i0, i1) of head (b, h) under the keep
    mask `keep` (bool [B, H, M, M], same device): exact logits over kept
    blocks, pooled logits + ln 64 with the pooled value over skipped ones, one
    softmax, in fp32 PyTorch."""
    import torch
    N, D, M = w.N, w.D, w.M
    scale = D ** -0.5
    kbar, vbar = (x[b, h].view(M, 64, D).mean(1) for x in (kf, vf))
    qc = qf[b, h, i0 * 64:i1 * 64]
    kb = keep[b, h, i0:i1].repeat_interleave(64, dim=0)                 # [rows, M]
    ex = (scale * qc @ kf[b, h].T).masked_fill(~kb.repeat_interleave(64, dim=1), float("-inf"))
    po = (scale * qc @ kbar.T + math.log(64.0)).masked_fill(kb, float("-inf"))
    p = torch.softmax(torch.cat([ex, po], dim=1), dim=1)
    return p[:, :N] @ vf[b, h] + p[:, N:] @ vbar
