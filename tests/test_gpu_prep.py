"""QKNorm + partial RoPE with the pooling fused in (sol_attn_qknorm_rope_pool).

* q_out, k_out against the fp64 oracle chain (RMSNorm then rotate-half RoPE) on
  the same bf16 inputs: each element within one bf16 rounding step of the
  oracle value, plus a small fp32 allowance.
* The pooled workspace is bit-identical to sol_attn_pool run on the written
  q_out, k_out and the input v: the kernel sums the same bf16 values in the
  same order.
* Attention on top (sol_attn_attend with the fused workspace) is
  bit-identical to sol_attn_forward on q_out, k_out, v.
* Positions up to 131071 (the sweep workload's length) keep their angle
  precision.
"""

import numpy as np
import pytest
import torch

from block_sparse_attention_threshold_b200 import abi, synthetic as syn
from oracle import sol_attn_oracle as orc

from . import parity

pytestmark = pytest.mark.gpu


def _inputs(B, H, N, D, seed):
    rng = np.random.default_rng(seed)
    arrs = [syn.fp64_to_bf16_bits(rng.normal(size=(B, H, N, D)) * 1.5 + 0.3) for _ in range(3)]
    wq = (1.0 + 0.25 * rng.normal(size=D)).astype(np.float32)
    wk = (1.0 + 0.25 * rng.normal(size=D)).astype(np.float32)
    return arrs, wq, wk


def _check_chain(bits_in, w, got, R, eps, base, rows=None):
    """Every element of `got` (bf16 tensor [B,H,N,D]) within one bf16 step of the oracle."""
    x = syn.bf16_bits_to_fp64(bits_in)
    B, H, N, D = x.shape
    g = got.float().cpu().numpy().astype(np.float64)
    worst = 0.0
    for b in range(B):
        for h in range(H):
            xs = x[b, h] if rows is None else x[b, h]
            ref = orc.qknorm_rope(xs, w.astype(np.float64), eps, R, base)
            if rows is not None:
                ref, gg = ref[rows], g[b, h][rows]
            else:
                gg = g[b, h]
            err = np.abs(gg - ref) / (np.abs(ref) * 2.0 ** -8 + 1e-3)
            worst = max(worst, float(err.max()))
    assert worst <= 1.0, worst
    return worst


@pytest.mark.parametrize("D,R", [(128, 64), (128, 128), (128, 0), (64, 32), (64, 16)])
def test_chain_matches_oracle_and_pool_is_bit_identical(D, R):
    B, H, N = 1, 3, 1024
    (qb, kb, vb), wq, wk = _inputs(B, H, N, D, seed=20261201 + D + R)
    q, k, v = parity.to_device(qb, kb, vb)
    dev = q.device
    wq_t, wk_t = torch.from_numpy(wq).to(dev), torch.from_numpy(wk).to(dev)
    eps, base = 1e-6, 10000.0
    q_out, k_out, ws = abi.qknorm_rope_pool(q, k, v, wq_t, wk_t, R, eps, base)
    torch.cuda.synchronize()
    _check_chain(qb, wq, q_out, R, eps, base)
    _check_chain(kb, wk, k_out, R, eps, base)
    # pooled workspace == standalone pooling of the written tensors
    ref_ws = torch.empty_like(ws)
    abi.pool(q_out, k_out, v, ref_ws)
    torch.cuda.synchronize()
    assert torch.equal(ws, ref_ws)
    # the chain without pooling writes the same q_out, k_out
    q2, k2, none = abi.qknorm_rope_pool(q, k, v, wq_t, wk_t, R, eps, base, pool=False)
    torch.cuda.synchronize()
    assert none is None and torch.equal(q2, q_out) and torch.equal(k2, k_out)


def test_batched_odd_heads():
    B, H, N, D, R = 2, 3, 512, 128, 32
    (qb, kb, vb), wq, wk = _inputs(B, H, N, D, seed=20261231)
    q, k, v = parity.to_device(qb, kb, vb)
    dev = q.device
    q_out, k_out, ws = abi.qknorm_rope_pool(q, k, v, torch.from_numpy(wq).to(dev), torch.from_numpy(wk).to(dev),
                                            R, 1e-5, 500000.0)
    torch.cuda.synchronize()
    _check_chain(qb, wq, q_out, R, 1e-5, 500000.0)
    _check_chain(kb, wk, k_out, R, 1e-5, 500000.0)
    ref_ws = torch.empty_like(ws)
    abi.pool(q_out, k_out, v, ref_ws)
    torch.cuda.synchronize()
    assert torch.equal(ws, ref_ws)


def test_attention_on_fused_workspace_equals_forward():
    w = syn.workload("draft_n16128")
    B, H, N, D = 1, 4, 4096, 128
    (qb, kb, vb), wq, wk = _inputs(B, H, N, D, seed=20261211)
    q, k, v = parity.to_device(qb, kb, vb)
    dev = q.device
    q_out, k_out, ws = abi.qknorm_rope_pool(q, k, v, torch.from_numpy(wq).to(dev), torch.from_numpy(wk).to(dev),
                                            64, 1e-6, 10000.0)
    out_fused = torch.empty_like(q)
    abi.attend(q_out, k_out, v, ws, 1.0, 512, out=out_fused)
    out_ref = abi.forward(q_out, k_out, v, 1.0, 512)
    torch.cuda.synchronize()
    assert abi.device_status() == abi.OK
    assert torch.equal(out_fused, out_ref)


def test_long_positions_keep_angle_precision():
    # One head of 131072 tokens: rows near the end have angles up to ~1.3e5 rad.
    B, H, N, D, R = 1, 1, 131072, 64, 64
    (qb, kb, vb), wq, wk = _inputs(B, H, N, D, seed=20261221)
    q, k, v = parity.to_device(qb, kb, vb)
    dev = q.device
    q_out, k_out, _ = abi.qknorm_rope_pool(q, k, v, torch.from_numpy(wq).to(dev),
                                           torch.from_numpy(wk).to(dev), R, 1e-6, 10000.0, pool=False)
    torch.cuda.synchronize()
    rows = np.concatenate([np.arange(0, 64), np.arange(N - 256, N)])
    _check_chain(qb, wq, q_out, R, 1e-6, 10000.0, rows=rows)
