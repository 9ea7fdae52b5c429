"""The allocation-free entry point, sol_attn_forward_noalloc.

Some callers cannot allocate device memory while they run attention: a
runtime that reserves all of its memory up front, or a server that must not
enter the CUDA allocator between requests.  For them the library exports
sol_attn_forward_noalloc, which takes its pooled workspace from a fixed
array compiled into the library instead of calling cudaMallocAsync.

This file is named so that pytest collects it last.  It calls the entry
point through the C ABI twice in a row, on two different inputs, so the
second call reuses the array the first one filled.  It checks each output
against sol_attn_forward on the same inputs, with the parity tolerances used
everywhere else.  It must pass both alone in a fresh process and after the
other GPU tests.
"""

import ctypes

import numpy as np
import pytest
import torch

from block_sparse_attention_threshold_b200 import abi, build, synthetic as syn

from . import parity

pytestmark = pytest.mark.gpu


def _inputs(w):
    return parity.to_device(*syn.generate_bf16(w))


def _noalloc(L, q, k, v, out, w, tau):
    B, H, N, D = q.shape
    return L.sol_attn_forward_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                      B, H, N, D, 64, ctypes.c_float(tau), w.prefix_len,
                                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _close(a, b):
    a = a.float().cpu().numpy().astype(np.float64)
    b = b.float().cpu().numpy().astype(np.float64)
    rel = np.linalg.norm(a - b) / np.linalg.norm(b)
    mx = np.abs(a - b).max()
    assert rel <= parity.REL_L2 and mx <= parity.MAX_ABS, (rel, mx)


def test_noalloc_matches_forward_on_two_calls_in_a_row():
    build.build()
    L = abi.lib()
    w1 = syn.workload("refine_n32768").replace(H=8)
    w2 = syn.workload("tiny_n1024")
    runs = []
    for w in (w1, w2):
        q, k, v = _inputs(w)
        tau = w.taus[0]
        out = torch.full_like(q, float("nan"))
        st = _noalloc(L, q, k, v, out, w, tau)
        assert st == abi.OK, abi.status_string(st)
        runs.append((w, q, k, v, tau, out))
    torch.cuda.synchronize()
    assert abi.device_status() == abi.OK
    for w, q, k, v, tau, out in runs:
        ref = abi.forward(q, k, v, tau, w.prefix_len)
        torch.cuda.synchronize()
        assert not torch.isnan(out.float()).any()
        _close(out, ref)


def test_noalloc_rejects_shapes_beyond_its_array():
    L = abi.lib()
    fake = 1 << 20
    limit = abi.noalloc_max_workspace()
    # B*H*N chosen so the pooled workspace just exceeds the array
    N = 64 * 4096
    H = limit // abi.workspace_layout(1, 1, N, 128)[0] + 1
    assert abi.workspace_layout(1, H, N, 128)[0] > limit
    st = L.sol_attn_forward_noalloc(fake, fake, fake, fake * 2, 1, H, N, 128, 64,
                                    ctypes.c_float(1.0), 0, None)
    assert st == abi.ERR_UNSUPPORTED
