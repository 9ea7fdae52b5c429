"""The allocation-free entry point, sol_attn_forward_noalloc.

Some callers cannot allocate device memory while they run attention: a
runtime that reserves all of its memory up front, or a server that must not
enter the CUDA allocator between requests.  For them the library exports
sol_attn_forward_noalloc, which takes its pooled workspace from a fixed
array compiled into the library instead of calling cudaMallocAsync.

This file is named so that pytest collects it last.  It calls the entry
point through the C ABI three times in a row, on inputs whose workspaces
grow (the last one fills the array exactly), so each call reuses the array
the previous one filled and reaches past the bytes it left.  It checks each output
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


def _close(a, b):
    a = a.float().cpu().numpy().astype(np.float64)
    b = b.float().cpu().numpy().astype(np.float64)
    rel = np.linalg.norm(a - b) / np.linalg.norm(b)
    mx = np.abs(a - b).max()
    assert rel <= parity.REL_L2 and mx <= parity.MAX_ABS, (rel, mx)


def _random_case(B, H, N, D, prefix_len, seed):
    """Seeded random bf16 inputs on the device (no locality; the comparison is
    between two entry points on the same inputs)."""
    g = torch.Generator(device="cuda").manual_seed(seed)
    shape = (B, H, N, D)
    q, k, v = (torch.randn(shape, generator=g, device="cuda").to(torch.bfloat16) for _ in range(3))
    return q, k, v, prefix_len


def test_noalloc_matches_forward_on_calls_in_a_row():
    """Small, then large, then a shape whose workspace fills the array exactly:
    each later call's workspace reaches past the bytes the earlier one left."""
    build.build()
    L = abi.lib()
    limit = abi.noalloc_max_workspace()
    cases = []
    for w in (syn.workload("tiny_n1024"), syn.workload("refine_n32768").replace(H=8)):
        q, k, v = _inputs(w)
        cases.append((q, k, v, w.prefix_len, w.taus[0]))
    # D = 64, B*H*(N/64) = 63 * 1387 = 87,381 blocks: 64 MiB of workspace exactly.
    big = _random_case(1, 63, 64 * 1387, 64, 64 * 3, 20261202)
    assert abi.workspace_layout(1, 63, 64 * 1387, 64)[0] == limit
    cases.append(big + (1.0,))
    sizes = [abi.workspace_layout(*c[0].shape)[0] for c in cases]
    assert sizes == sorted(sizes) and sizes[0] < sizes[1] < sizes[2]
    outs = []
    for q, k, v, prefix_len, tau in cases:
        out = torch.full_like(q, float("nan"))
        B, H, N, D = q.shape
        st = L.sol_attn_forward_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                        B, H, N, D, 64, ctypes.c_float(tau), prefix_len,
                                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == abi.OK, abi.status_string(st)
        outs.append(out)
    torch.cuda.synchronize()
    assert abi.device_status() == abi.OK
    for (q, k, v, prefix_len, tau), out in zip(cases, outs):
        ref = abi.forward(q, k, v, tau, prefix_len)
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
