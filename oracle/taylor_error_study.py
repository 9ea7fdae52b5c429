"""Accuracy of the zeroth- and first-order Taylor compensation of skipped
blocks, measured with the CPU oracle against dense attention.

TEST INFRASTRUCTURE: uses only the oracle and the seeded input generator.

The compensation of rejected blocks is called a "Taylor approximation" on
"MiniMax 官推背书 Sol Engine" (arex-research 647c3193, section "3.95x
near-lossless").  The operator as built uses the zeroth-order term; this
script measures what the first-order term (oracle ``order=1``) would add, in
its exact per-row form and in the cheaper form that uses the query block's
pooled query, on the five synthetic workloads.

For each workload: the first two heads (the workload with H = 2, same seed),
24 seeded query blocks per head (always blocks 0, P and M - 1), at the
workload's first tau (the sweep also at tau = 1.0 and 2.0).  Printed: relative
L2 error of each form against dense attention over the sampled rows, and the
same restricted to video query blocks.

    python -m oracle.taylor_error_study [workload ...]
    python -m oracle.taylor_error_study --ranks    # truncated cross moments on refine
"""

from __future__ import annotations

import math
import os
import sys
from concurrent.futures import ThreadPoolExecutor

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from block_sparse_attention_threshold_b200 import synthetic as syn  # noqa: E402
from oracle import sol_attn_oracle as orc  # noqa: E402

FORMS = (("zeroth", dict(order=0)), ("first_row", dict(order=1)),
         ("first_pooled_q", dict(order=1, pooled_query_term=True)))


def study(name: str, taus=None, heads: int = 2, blocks: int = 24):
    w = syn.workload(name).replace(H=heads)
    qb, kb, vb = syn.generate_bf16(w)
    taus = taus or [w.taus[0]]
    sample = syn.sample_query_blocks(w.M, w.P, blocks, w.seed + 3)
    video = [i for i in sample if i >= w.P]
    rows_all = np.concatenate([np.arange(64 * i, 64 * i + 64) for i in sample])
    rows_vid = np.concatenate([np.arange(64 * i, 64 * i + 64) for i in video])
    out = []

    def one(h):
        q, k, v = (syn.bf16_bits_to_fp64(a[0, h]) for a in (qb, kb, vb))
        ref = orc.dense_rows(q, k, v, rows=rows_all)
        res = {}
        for tau in taus:
            r = orc.route(q, k, 64, w.prefix_len, tau)
            for form, kw in FORMS:
                got = orc.solattn_blocks(q, k, v, 64, w.prefix_len, tau, qblocks=sample, routing=r, **kw)
                res[(tau, form)] = got
            res[(tau, "kept")] = r.keep[w.P:, w.P:].mean()
        return ref, res

    try:
        from threadpoolctl import threadpool_limits
        ctx = threadpool_limits(max(1, (os.cpu_count() or 2) // heads))
    except Exception:  # pragma: no cover
        import contextlib
        ctx = contextlib.nullcontext()
    with ctx, ThreadPoolExecutor(max_workers=heads) as ex:
        per_head = list(ex.map(one, range(heads)))
    vid_mask = np.isin(rows_all, rows_vid)
    for tau in taus:
        line = {"workload": name, "tau": tau,
                "video_kept_frac": float(np.mean([res[(tau, "kept")] for _, res in per_head]))}
        for form, _ in FORMS:
            e2 = sum(float(np.sum((res[(tau, form)] - ref) ** 2)) for ref, res in per_head)
            r2 = sum(float(np.sum(ref ** 2)) for ref, _ in per_head)
            ev = sum(float(np.sum((res[(tau, form)][vid_mask] - ref[vid_mask]) ** 2)) for ref, res in per_head)
            rv = sum(float(np.sum(ref[vid_mask] ** 2)) for ref, _ in per_head)
            line[form] = math.sqrt(e2 / r2)
            line[form + "_video_rows"] = math.sqrt(ev / rv)
        out.append(line)
    return out


def rank_study(name: str = "refine_n32768", ranks=(0, 1, 2, 4, 8, 16, 32, 128), blocks: int = 12):
    """Error against dense of the first-order form with each block's cross
    moment truncated to its top `rank` singular pairs (rank 0 = zeroth
    order), on the first head.  A rank-r moment costs 2 r D multiply-adds
    per (row, skipped block); exact attention on the block costs 128 D."""
    w = syn.workload(name).replace(H=1)
    qb, kb, vb = syn.generate_bf16(w)
    q, k, v = (syn.bf16_bits_to_fp64(a[0, 0]) for a in (qb, kb, vb))
    tau = w.taus[0]
    r = orc.route(q, k, 64, w.prefix_len, tau)
    sample = [i for i in syn.sample_query_blocks(w.M, w.P, blocks, 5) if i >= w.P]
    rows = np.concatenate([np.arange(64 * i, 64 * i + 64) for i in sample])
    ref = orc.dense_rows(q, k, v, rows=rows)
    cov = orc.block_cross_moment(k, v)
    kbar, _ = orc.pool_blocks(k)
    vbar, _ = orc.pool_blocks(v)
    U, S, Vt = np.linalg.svd(cov)
    s = 1.0 / math.sqrt(w.D)
    out = {"workload": name, "tau": tau,
           "top_singular_share": float(np.mean(S[:, 0] / S.sum(axis=1)))}
    for rank in ranks:
        res = []
        for i in sample:
            qr = q[64 * i:64 * i + 64]
            kept, sk = np.nonzero(r.keep[i])[0], np.nonzero(~r.keep[i])[0]
            tok = np.concatenate([np.arange(64 * j, 64 * j + 64) for j in kept])
            le = s * (qr @ k[tok].T)
            lp = s * (qr @ kbar[sk].T) + math.log(64)
            m = np.maximum(le.max(axis=1), lp.max(axis=1))
            we, wp = np.exp(le - m[:, None]), np.exp(lp - m[:, None])
            num = we @ v[tok] + wp @ vbar[sk]
            for col, j in enumerate(sk):
                if rank > 0:
                    cj = (U[j][:, :rank] * S[j][:rank]) @ Vt[j][:rank]
                    num += wp[:, col:col + 1] * (s * (qr @ cj))
            res.append(num / (we.sum(axis=1) + wp.sum(axis=1))[:, None])
        got = np.concatenate(res)
        out[f"rank_{rank}"] = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
    return out


def main(argv):
    if argv[:1] == ["--ranks"]:
        print({k: (round(v, 4) if isinstance(v, float) else v) for k, v in rank_study().items()})
        return
    names = argv or ["tiny_n1024", "draft_n16128", "refine_n32768", "long_n65536", "sweep_n131072"]
    for name in names:
        taus = [1.0, 1.25, 2.0] if name == "sweep_n131072" else None
        for line in study(name, taus):
            print({k: (round(v, 6) if isinstance(v, float) else v) for k, v in line.items()}, flush=True)


if __name__ == "__main__":
    main(sys.argv[1:])
