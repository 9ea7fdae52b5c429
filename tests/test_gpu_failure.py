"""Failure detection without a GPU fault.

Every wait inside the attention kernel has a time limit.  The test hook
`test_skip_first_k_load` makes the loader skip the first key tile, so the
tensor-core issuer's bounded wait on it runs out.  The kernel must then raise
its abort flag, drain, free its tensor memory and record the site, the host
must read SOL_ATTN_ERR_DEVICE_TIMEOUT from sol_attn_device_status, and the
context must stay usable: the next call succeeds and matches the oracle.
No fault, trap or endless loop is involved.
"""

import pytest
import torch

from block_sparse_attention_threshold_b200 import abi, build, synthetic as syn

from . import parity

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    build.build()
    abi.lib()
    w = syn.workload("tiny_n1024")
    bits = syn.generate_bf16(w)
    q, k, v = parity.to_device(*bits)
    tau = w.taus[0]
    assert abi.device_status() == abi.OK  # start clean
    opts = abi.Opts()
    opts.timeout_ms = 50
    opts.test_skip_first_k_load = 1
    abi.forward(q, k, v, tau, w.prefix_len, opts=opts)
    assert abi.device_status() == abi.ERR_DEVICE_TIMEOUT
    assert abi.device_status() == abi.OK  # the word was cleared
    out, keep, _, _ = parity.run_sol(w, tau, q, k, v)
    parity.assert_parity(parity.oracle_compare(w, tau, *bits, out, keep))
    torch.cuda.synchronize()
