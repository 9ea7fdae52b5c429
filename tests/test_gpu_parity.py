"""Parity of the CUDA path (through the C ABI) with the CPU fp64 oracle.

Small cases are compared element by element in full; the large workloads
compare the full keep mask and 64 seeded sampled query blocks per head (always
including blocks 0, P and M-1), in the same launch configuration the
benchmark times.
"""

import math

import numpy as np
import pytest
import torch

from block_sparse_attention_threshold_b200 import abi, synthetic as syn
from oracle import sol_attn_oracle as orc

from . import parity

pytestmark = pytest.mark.gpu

_cache = {}


def inputs(w):
    if w.name not in _cache:
        _cache.clear()
        bits = syn.generate_bf16(w)
        _cache[w.name] = (bits, parity.to_device(*bits))
    return _cache[w.name]


def random_workload(name, B, H, N, D, prefix, seed, sigma=0.8, grid=None):
    grid = grid or (64, 24, 42)
    return syn.Workload(name, B, H, N, D, prefix, grid, sigma, (1.0,), seed)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from block_sparse_attention_threshold_b200 import build
    build.build()
    abi.lib()
    yield
    _cache.clear()
    torch.cuda.empty_cache()


# ------------------------------------------------------------------ pooling

@pytest.mark.parametrize("D", [64, 128])
def test_pool_matches_block_means(D):
    w = random_workload(f"pool{D}", 2, 3, 64 * 9, D, 128, 77 + D)
    bits, (q, k, v) = inputs(w)
    nbytes, off = abi.workspace_layout(w.B, w.H, w.N, D)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=q.device)
    abi.pool(q, k, v, ws)
    torch.cuda.synchronize()
    rows = w.B * w.H * w.M
    wsn = ws.cpu().numpy()
    sec = lambda i, dt, n: wsn[off[i]:off[i] + rows * D * n].view(dt).reshape(w.B, w.H, w.M, D)
    qbar, kbar = sec(0, np.float32, 4), sec(1, np.float32, 4)
    kbar16 = syn.bf16_bits_to_fp64(sec(2, np.uint16, 2))
    vbar16 = syn.bf16_bits_to_fp64(sec(3, np.uint16, 2))
    for b in range(w.B):
        for h in range(w.H):
            for arr, src in ((qbar, bits[0]), (kbar, bits[1])):
                ref, cnt = orc.pool_blocks(syn.bf16_bits_to_fp64(src[b, h]), 64)
                assert (cnt == 64).all()
                np.testing.assert_allclose(arr[b, h], ref, rtol=0, atol=2e-6 * np.abs(ref).max())
            for arr, src in ((kbar16, bits[1]), (vbar16, bits[2])):
                ref, _ = orc.pool_blocks(syn.bf16_bits_to_fp64(src[b, h]), 64)
                assert np.all(np.abs(arr[b, h] - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-6)


# ------------------------------------------------------------------ dense comparator

@pytest.mark.parametrize("B,H,N,D", [(1, 2, 1024, 64), (2, 2, 64 * 17, 128), (1, 1, 64, 128)])
def test_dense_kernel_matches_oracle(B, H, N, D):
    w = random_workload(f"dense{B}{H}{N}{D}", B, H, N, D, 0, 1234 + N + D)
    bits, (q, k, v) = inputs(w)
    out = abi.dense_forward(q, k, v)
    torch.cuda.synchronize()
    assert abi.device_status() == abi.OK
    m = parity.oracle_compare(w, -math.inf, *bits, out, dense=True)
    parity.assert_parity(m)


# ------------------------------------------------------------------ tiny workload, full check

@pytest.mark.parametrize("tau", [1.0, 0.5, 2.0, -math.inf, math.inf])
def test_tiny_workload_full(tau):
    w = syn.workload("tiny_n1024")
    bits, (q, k, v) = inputs(w)
    out, keep, kept, exact = parity.run_sol(w, tau, q, k, v)
    m = parity.oracle_compare(w, tau, *bits, out, keep)
    parity.assert_parity(m)
    assert kept == int(keep.sum())
    assert exact >= kept


def test_tau_minus_inf_equals_dense_kernel():
    w = syn.workload("tiny_n1024")
    bits, (q, k, v) = inputs(w)
    a, keep, _, _ = parity.run_sol(w, -math.inf, q, k, v)
    assert keep.all()
    d = abi.dense_forward(q, k, v)
    torch.cuda.synchronize()
    diff = (a.float() - d.float()).abs().max().item()
    assert diff <= 2e-2


# ------------------------------------------------------------------ edge cases

@pytest.mark.parametrize("case", [
    dict(B=1, H=2, N=640, D=64, prefix=0, tau=1.0),        # no prefix
    dict(B=1, H=2, N=640, D=64, prefix=640, tau=1.0),      # all prefix: dense
    dict(B=2, H=2, N=64 * 13, D=128, prefix=192, tau=0.8),  # odd M, B > 1, odd P
    dict(B=1, H=3, N=64, D=128, prefix=0, tau=1.0),        # a single block
    dict(B=1, H=2, N=64 * 5, D=64, prefix=64, tau=math.inf),  # only the prefix exact
    dict(B=1, H=2, N=64 * 40, D=128, prefix=128, tau=0.0),
])
def test_edge_cases(case):
    w = random_workload("edge%d%d%d%d%d" % (case["B"], case["H"], case["N"], case["D"], case["prefix"]),
                        case["B"], case["H"], case["N"], case["D"], case["prefix"],
                        99 + case["N"] + case["prefix"], grid=(8, 24, 42))
    bits, (q, k, v) = inputs(w)
    out, keep, kept, exact = parity.run_sol(w, case["tau"], q, k, v)
    m = parity.oracle_compare(w, case["tau"], *bits, out, keep)
    parity.assert_parity(m)
    assert kept == int(keep.sum()) and exact >= kept


def test_identical_key_blocks_give_dense_attention():
    """With every video key block made of 64 identical keys/values the pooled
    correction is exact, so the GPU Sol-Attn output must match dense attention."""
    rng = np.random.default_rng(5)
    B, H, N, D, L = 1, 2, 64 * 24, 128, 256
    q = rng.standard_normal((B, H, N, D))
    kb = np.repeat(rng.standard_normal((B, H, N // 64, D)), 64, axis=2)
    vb = np.repeat(rng.standard_normal((B, H, N // 64, D)), 64, axis=2)
    kb[:, :, :L] = rng.standard_normal((B, H, L, D))
    bits = [syn.fp64_to_bf16_bits(x) for x in (q, kb, vb)]
    qd, kd, vd = parity.to_device(*bits)
    w = syn.Workload("ident", B, H, N, D, L, (1, 1, N - L), 1.0, (1.0,), 0)
    out, keep, _, _ = parity.run_sol(w, 1.0, qd, kd, vd)
    assert not keep.all()
    m = parity.oracle_compare(w, -math.inf, *bits, out, dense=True)
    parity.assert_parity(m)


# ------------------------------------------------------------------ the named workloads

@pytest.mark.parametrize("name", ["draft_n16128", "refine_n32768", "long_n65536"])
def test_workload_parity(name):
    w = syn.workload(name)
    bits, (q, k, v) = inputs(w)
    tau = w.taus[0]
    out, keep, kept, exact = parity.run_sol(w, tau, q, k, v)
    blocks = syn.sample_query_blocks(w.M, w.P, 64, w.seed)
    m = parity.oracle_compare(w, tau, *bits, out, keep, qblocks=blocks)
    print(name, m, "kept", kept, "exact", exact)
    parity.assert_parity(m)
    assert kept == int(keep.sum())
    assert abs(kept - m["oracle_kept"]) <= m["mask_mismatch"]


def test_sparsity_sweep_parity():
    w = syn.workload("sweep_n131072")
    bits, (q, k, v) = inputs(w)
    blocks = syn.sample_query_blocks(w.M, w.P, 64, w.seed + 1)
    for tau in w.taus:
        out, keep, kept, _ = parity.run_sol(w, tau, q, k, v)
        m = parity.oracle_compare(w, tau, *bits, out, keep, qblocks=blocks)
        print("sweep tau", tau, m, "kept frac", kept / keep.size)
        parity.assert_parity(m)
        del out
