"""Guard bands: the kernels write nothing outside the buffers they are given.

compute-sanitizer is closed on this machine, so every output buffer here sits
inside a larger allocation whose margins hold a sentinel pattern, and the
margins are checked after the call.  The inputs are checked to be unchanged.
Shapes cover odd block counts (a last 128-row tile holding one block), B > 1
and odd prefixes; the host-buffer entry point runs
with uneven head chunks; the debug keep-mask export and the pooled
workspace are guarded the same way, and so is the 8-bit entry point.  Each
result is also compared with the same call on plain buffers, so the guards
cannot hide a wrong answer.
"""

import math

import numpy as np
import pytest
import torch

from block_sparse_attention_threshold_b200 import abi, build, synthetic as syn

from . import parity

pytestmark = pytest.mark.gpu

GUARD = 4096            # elements of margin on each side (multiple of 128 bytes)
SENTINEL_BF16 = 0x7FA5  # a NaN payload no kernel produces
SENTINEL_U8 = 0xA5


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    abi.lib()


def _guarded_bf16(shape, device):
    n = int(np.prod(shape))
    big = torch.full((GUARD + n + GUARD,), SENTINEL_BF16, dtype=torch.int16, device=device)
    return big, big[GUARD:GUARD + n].view(torch.bfloat16).view(*shape)


def _margins_intact_bf16(big, n):
    h = big.cpu().numpy().view(np.uint16)
    return bool((h[:GUARD] == SENTINEL_BF16).all() and (h[GUARD + n:] == SENTINEL_BF16).all())


def _inputs(B, H, N, D, prefix, seed):
    w = syn.Workload("guard", B, H, N, D, prefix, (16, 24, 42), 0.8, (1.0,), seed)
    bits = syn.generate_bf16(w)
    return w, bits, parity.to_device(*bits)


CASES = [
    dict(B=2, H=3, N=64 * 13, D=128, prefix=192, tau=0.8),   # M = 13: the last tile holds one block
    dict(B=1, H=2, N=64 * 14, D=128, prefix=0, tau=1.0),     # M = 14: every tile holds two blocks
    dict(B=3, H=1, N=64 * 7, D=64, prefix=64, tau=0.5),      # D = 64, M = 7
    dict(B=1, H=2, N=64, D=128, prefix=0, tau=1.0),          # one block
    dict(B=1, H=2, N=64 * 9, D=128, prefix=64 * 9, tau=1.0), # all prefix
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dH%dM%dD%dP%d" % (
    c["B"], c["H"], c["N"] // 64, c["D"], c["prefix"] // 64))
def test_forward_writes_only_out_and_mask(case):
    B, H, N, D, L, tau = (case[k] for k in ("B", "H", "N", "D", "prefix", "tau"))
    w, bits, (q, k, v) = _inputs(B, H, N, D, L, 4242 + N + D + L)
    q0, k0, v0 = q.clone(), k.clone(), v.clone()
    big, out = _guarded_bf16((B, H, N, D), q.device)
    M = N // 64
    nwords = B * H * M * abi.mask_words(M)
    mbig = torch.full((GUARD + nwords + GUARD,), -0x5A5A5A5B, dtype=torch.int32, device=q.device)
    opts = abi.Opts()
    opts.debug_mask = mbig[GUARD:GUARD + nwords].data_ptr()
    abi.forward(q, k, v, tau, L, out=out, opts=opts)
    torch.cuda.synchronize()
    assert abi.device_status() == abi.OK
    assert _margins_intact_bf16(big, out.numel())
    mh = mbig.cpu().numpy()
    assert (mh[:GUARD] == -0x5A5A5A5B).all() and (mh[GUARD + nwords:] == -0x5A5A5A5B).all()
    assert torch.equal(q, q0) and torch.equal(k, k0) and torch.equal(v, v0)
    ref = abi.forward(q, k, v, tau, L)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    # and the dense comparator
    big_d, out_d = _guarded_bf16((B, H, N, D), q.device)
    abi.dense_forward(q, k, v, out=out_d)
    torch.cuda.synchronize()
    assert _margins_intact_bf16(big_d, out_d.numel())
    m = parity.oracle_compare(w, -math.inf, *bits, out_d, dense=True)
    parity.assert_parity(m)


@pytest.mark.parametrize("case", CASES[:3], ids=lambda c: "B%dH%dM%dD%d" % (c["B"], c["H"], c["N"] // 64, c["D"]))
def test_pool_and_attend_stay_inside_the_workspace(case):
    B, H, N, D, L, tau = (case[k] for k in ("B", "H", "N", "D", "prefix", "tau"))
    _, _, (q, k, v) = _inputs(B, H, N, D, L, 777 + N + D)
    nbytes, _ = abi.workspace_layout(B, H, N, D)
    gb = 4096
    wbig = torch.full((gb + nbytes + gb,), SENTINEL_U8, dtype=torch.uint8, device=q.device)
    ws = wbig[gb:gb + nbytes]
    assert ws.data_ptr() % 256 == 0
    abi.pool(q, k, v, ws)
    big, out = _guarded_bf16((B, H, N, D), q.device)
    abi.attend(q, k, v, ws, tau, L, out=out)
    torch.cuda.synchronize()
    assert abi.device_status() == abi.OK
    h = wbig.cpu().numpy()
    assert (h[:gb] == SENTINEL_U8).all() and (h[gb + nbytes:] == SENTINEL_U8).all()
    assert _margins_intact_bf16(big, out.numel())
    assert torch.equal(out, abi.forward(q, k, v, tau, L))


def test_host_entry_point_with_uneven_chunks_writes_only_out():
    B, H, N, D, L, tau = 1, 7, 64 * 13, 128, 128, 1.0
    w, bits, (q, k, v) = _inputs(B, H, N, D, L, 9090)
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    n = B * H * N * D
    hbig = torch.full((GUARD + n + GUARD,), SENTINEL_BF16, dtype=torch.int16).pin_memory()
    hout = hbig[GUARD:GUARD + n].view(torch.bfloat16).view(B, H, N, D)
    abi.forward_host(hq, hk, hv, tau, L, out=hout, heads_per_chunk=3)   # chunks of 3, 3, 1 heads
    torch.cuda.synchronize()
    assert abi.device_status() == abi.OK
    hh = hbig.numpy().view(np.uint16)
    assert (hh[:GUARD] == SENTINEL_BF16).all() and (hh[GUARD + n:] == SENTINEL_BF16).all()
    ref = abi.forward(q, k, v, tau, L)
    torch.cuda.synchronize()
    assert torch.equal(hout, ref.cpu())


def test_fp8_forward_writes_only_out():
    B, H, N, D, L, tau = 2, 2, 64 * 13, 128, 192, 0.8
    w = syn.Workload("guard8", B, H, N, D, L, (16, 24, 42), 0.8, (1.0,), 5151)
    bits = syn.generate_e4m3(w)
    dev = torch.device("cuda", 0)
    q8, k8, v8 = (torch.from_numpy(np.ascontiguousarray(a)).to(dev) for a in bits)
    q0, k0, v0 = q8.clone(), k8.clone(), v8.clone()
    big, out = _guarded_bf16((B, H, N, D), dev)
    abi.forward_fp8(q8, k8, v8, tau, L, out=out)
    torch.cuda.synchronize()
    assert abi.device_status() == abi.OK
    assert _margins_intact_bf16(big, out.numel())
    assert torch.equal(q8, q0) and torch.equal(k8, k0) and torch.equal(v8, v0)
    ref = abi.forward_fp8(q8, k8, v8, tau, L)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
