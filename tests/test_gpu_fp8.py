"""Parity of the 8-bit (E4M3) entry point, sol_attn_forward_fp8, with the CPU
fp64 oracle run on the decoded E4M3 inputs (times their scales).

Routing is computed in fp32 from the decoded values, so the keep mask is held
to the same bar as the bf16 path (>= 99.9 % agreement, every disagreement
within 1e-3 sigma of its threshold, none at a forced position).  The output
bar is the 8-bit one derived from the arithmetic: the kernel rounds the
probabilities P and the pooled means used by the correction to E4M3 (3
mantissa bits, relative rounding error at most 2^-4, about 2^-4/sqrt(3) RMS),
while the row sums are accumulated from the unrounded fp32 P.  The output's
relative error is then of the order of that RMS (~3.6 %, less where many keys
share the weight); the bar is rel-L2 <= 5e-2 and max-abs <= 1e-1.
"""

import math

import numpy as np
import pytest
import torch

from block_sparse_attention_threshold_b200 import abi, build, synthetic as syn

from . import parity

pytestmark = pytest.mark.gpu

REL_L2_FP8 = 5e-2
MAX_ABS_FP8 = 1e-1


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    abi.lib()


def _decoders(scales):
    return tuple((lambda b, s=s: syn.e4m3_bits_to_fp64(b) * s) for s in scales)


def _run(w, tau, bits, scales=(1.0, 1.0, 1.0), budget=0, correct=True):
    dev = torch.device("cuda", 0)
    q8, k8, v8 = (torch.from_numpy(np.ascontiguousarray(a)).to(dev) for a in bits)
    opts = abi.Opts()
    opts.budget_blocks = int(budget)
    opts.skip_correction = 0 if correct else 1
    cnt = torch.zeros(2, dtype=torch.int64, device=dev)
    opts.kept_pairs = cnt.data_ptr()
    opts.exact_pairs = cnt.data_ptr() + 8
    mask = torch.zeros(w.B * w.H * w.M * abi.mask_words(w.M), dtype=torch.int32, device=dev)
    opts.debug_mask = mask.data_ptr()
    out = abi.forward_fp8(q8, k8, v8, tau, w.prefix_len, *scales, opts=opts)
    torch.cuda.synchronize()
    st = abi.device_status()
    assert st == abi.OK, abi.status_string(st)
    keep = abi.unpack_mask(mask.cpu().numpy().view(np.uint32).reshape(w.B, w.H, w.M, -1), w.M)
    kept, exact = (int(x) for x in cnt.cpu().tolist())
    return out, keep, kept, exact


def _workload(B, H, N, prefix, seed):
    return syn.Workload("fp8", B, H, N, 128, prefix, (16, 24, 42), 0.8, (1.0,), seed)


@pytest.mark.parametrize("tau", [1.0, 0.5, -math.inf, math.inf])
def test_fp8_small_full(tau):
    w = _workload(1, 2, 64 * 16, 128, 8101)
    bits = syn.generate_e4m3(w)
    out, keep, kept, exact = _run(w, tau, bits)
    m = parity.oracle_compare(w, tau, *bits, out, keep, decode=_decoders((1.0, 1.0, 1.0)))
    print("fp8 small tau", tau, m)
    parity.assert_parity(m, REL_L2_FP8, MAX_ABS_FP8)
    assert kept == int(keep.sum()) and exact >= kept


def test_fp8_odd_blocks_batch_and_scales():
    w = _workload(2, 2, 64 * 13, 192, 8102)
    scales = (0.5, 2.0, 0.25)
    bits = syn.generate_e4m3(w, scales)
    out, keep, _, _ = _run(w, 0.8, bits, scales)
    m = parity.oracle_compare(w, 0.8, *bits, out, keep, decode=_decoders(scales))
    print("fp8 odd/scales", m)
    parity.assert_parity(m, REL_L2_FP8, MAX_ABS_FP8)


def test_fp8_budget_routing_without_correction():
    w = _workload(1, 2, 64 * 24, 128, 8103)
    bits = syn.generate_e4m3(w)
    out, keep, _, _ = _run(w, 0.0, bits, budget=5, correct=False)
    m = parity.oracle_compare(w, 0.0, *bits, out, keep, budget=5, correct=False,
                              decode=_decoders((1.0, 1.0, 1.0)))
    print("fp8 budget", m)
    parity.assert_parity(m, REL_L2_FP8, MAX_ABS_FP8)


def test_fp8_refine_workload():
    w = syn.workload("refine_n32768")
    bits = syn.generate_e4m3(w)
    tau = w.taus[0]
    out, keep, kept, _ = _run(w, tau, bits)
    blocks = syn.sample_query_blocks(w.M, w.P, 64, w.seed)
    m = parity.oracle_compare(w, tau, *bits, out, keep, qblocks=blocks, decode=_decoders((1.0, 1.0, 1.0)))
    print("fp8 refine", m, "kept", kept)
    parity.assert_parity(m, REL_L2_FP8, MAX_ABS_FP8)


def test_fp8_pool_then_attend_equals_forward():
    w = _workload(1, 3, 64 * 10, 64, 8104)
    bits = syn.generate_e4m3(w, (0.5, 0.5, 2.0))
    dev = torch.device("cuda", 0)
    q8, k8, v8 = (torch.from_numpy(np.ascontiguousarray(a)).to(dev) for a in bits)
    nbytes, _ = abi.workspace_layout(w.B, w.H, w.N, w.D)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    abi.pool_fp8(q8, k8, v8, ws, 0.5, 0.5)
    a = abi.attend_fp8(q8, k8, v8, ws, 1.0, w.prefix_len, 0.5, 0.5, 2.0)
    b = abi.forward_fp8(q8, k8, v8, 1.0, w.prefix_len, 0.5, 0.5, 2.0)
    torch.cuda.synchronize()
    assert abi.device_status() == abi.OK
    assert torch.equal(a, b)
