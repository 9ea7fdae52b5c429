"""The host-buffer entry point, sol_attn_forward_host.

It cuts the B*H independent sequences into chunks and pipelines host-to-device
copies, pooling + attention and device-to-host copies over three buffer sets.
Every sequence still goes through the same two kernels, so the result must
equal sol_attn_forward on the same inputs bit for bit, whatever the chunking:
an uneven split, one chunk per sequence, a single chunk, and pageable host
memory (no overlap, same result).  The output is also checked against the
oracle with the usual parity bounds on the tiny workload.
"""

import numpy as np
import pytest
import torch

from block_sparse_attention_threshold_b200 import abi, synthetic as syn

from . import parity

pytestmark = pytest.mark.gpu


def _host(*arrays, pinned=True):
    out = []
    for a in arrays:
        t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
        out.append(t.pin_memory() if pinned else t.clone())
    return out


def _random_inputs(B, H, N, D, seed):
    # Seeded bf16 inputs with some positional structure (so routing is non-trivial).
    video = N - 128
    w = syn.Workload(name="host_test", B=B, H=H, N=N, D=D, prefix_len=128, grid=(video // 64, 8, 8),
                     sigma=1.0, taus=(1.0,), seed=seed)
    return w, syn.generate_bf16(w)


@pytest.mark.parametrize("heads_per_chunk,pinned", [(3, True), (1, True), (0, True), (10, True), (4, False)])
def test_host_entry_matches_device_entry_bit_for_bit(heads_per_chunk, pinned):
    w, (qb, kb, vb) = _random_inputs(2, 5, 2048, 128, seed=20261101)
    q, k, v = parity.to_device(qb, kb, vb)
    ref = abi.forward(q, k, v, 1.0, w.prefix_len)
    hq, hk, hv = _host(qb, kb, vb, pinned=pinned)
    out = abi.forward_host(hq, hk, hv, 1.0, w.prefix_len, heads_per_chunk=heads_per_chunk)
    torch.cuda.synchronize()
    assert abi.device_status() == abi.OK
    assert torch.equal(out.view(torch.int16), ref.cpu().view(torch.int16))


def test_host_entry_d64_matches_device_entry():
    w, (qb, kb, vb) = _random_inputs(1, 3, 1024, 64, seed=20261105)
    q, k, v = parity.to_device(qb, kb, vb)
    ref = abi.forward(q, k, v, 0.5, w.prefix_len)
    hq, hk, hv = _host(qb, kb, vb)
    out = abi.forward_host(hq, hk, hv, 0.5, w.prefix_len, heads_per_chunk=2)
    torch.cuda.synchronize()
    assert abi.device_status() == abi.OK
    assert torch.equal(out.view(torch.int16), ref.cpu().view(torch.int16))


def test_host_entry_parity_tiny():
    w = syn.workload("tiny_n1024")
    qb, kb, vb = syn.generate_bf16(w)
    hq, hk, hv = _host(qb, kb, vb)
    out = abi.forward_host(hq, hk, hv, w.taus[0], w.prefix_len, heads_per_chunk=1)
    torch.cuda.synchronize()
    assert abi.device_status() == abi.OK
    m = parity.oracle_compare(w, w.taus[0], qb, kb, vb, out)
    parity.assert_parity(m)
