"""The C-ABI library without a GPU: it loads, exports every declared symbol,
and rejects bad arguments before touching the device."""

import ctypes
import math
import os
import subprocess

import pytest

from block_sparse_attention_threshold_b200 import abi, build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "sol_attn.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return abi.lib()


def test_every_declared_symbol_is_exported(L):
    names = abi.declared_symbols(HEADER)
    assert len(names) == 14
    out = subprocess.run(["nm", "-D", "--defined-only", abi.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for n in names:
        assert n in exported, n
        assert hasattr(L, n)


def test_status_strings(L):
    for code, name in [(0, "SOL_ATTN_OK"), (1, "SOL_ATTN_ERR_INVALID_ARG"),
                       (2, "SOL_ATTN_ERR_UNSUPPORTED"), (3, "SOL_ATTN_ERR_ARCH"),
                       (4, "SOL_ATTN_ERR_CUDA"), (5, "SOL_ATTN_ERR_DEVICE_TIMEOUT")]:
        assert abi.status_string(code) == name
    assert abi.status_string(99) == "SOL_ATTN_ERR_UNKNOWN"


def test_workspace_layout(L):
    n, off = abi.workspace_layout(1, 40, 32768, 128)
    rows = 40 * 512
    assert off == [0, rows * 128 * 4, 2 * rows * 128 * 4, 2 * rows * 128 * 4 + rows * 128 * 2]
    assert n == 2 * rows * 128 * 4 + 2 * rows * 128 * 2
    assert all(o % 256 == 0 for o in off)
    # ragged sizes are rounded up per section
    n2, off2 = abi.workspace_layout(1, 1, 64, 64)
    assert off2 == [0, 256, 512, 768] and n2 == 1024
    assert abi.workspace_layout(1, 1, 100, 64)[0] == 0   # N not a multiple of 64
    assert abi.workspace_layout(1, 1, 64, 96)[0] == 0    # unsupported D
    assert abi.workspace_layout(0, 1, 64, 64)[0] == 0    # empty


FAKE = 1 << 20  # a 16-byte aligned non-null address; never dereferenced by these calls


def _fwd(L, B=1, H=1, N=128, D=64, block=64, tau=1.0, prefix=0, q=FAKE, out=FAKE * 2, opts=None):
    return L.sol_attn_forward_ex(q, FAKE, FAKE, out, B, H, N, D, block, tau, prefix,
                                 ctypes.byref(opts) if opts is not None else None, None)


def test_argument_validation_happens_before_any_device_call(L):
    E = abi
    assert _fwd(L, D=96) == E.ERR_UNSUPPORTED
    assert _fwd(L, D=256) == E.ERR_UNSUPPORTED
    assert _fwd(L, block=32) == E.ERR_UNSUPPORTED
    assert _fwd(L, N=100) == E.ERR_INVALID_ARG                 # ragged N
    assert _fwd(L, N=64 * 4097) == E.ERR_UNSUPPORTED           # more than 4096 blocks
    assert _fwd(L, B=-1) == E.ERR_INVALID_ARG
    assert _fwd(L, prefix=32) == E.ERR_INVALID_ARG             # prefix not whole blocks
    assert _fwd(L, prefix=192) == E.ERR_INVALID_ARG            # prefix > N
    assert _fwd(L, prefix=-64) == E.ERR_INVALID_ARG
    assert _fwd(L, tau=math.nan) == E.ERR_INVALID_ARG
    assert _fwd(L, q=0) == E.ERR_INVALID_ARG                   # null pointer
    assert _fwd(L, q=FAKE + 8) == E.ERR_INVALID_ARG            # misaligned
    o = abi.Opts()
    o.softmax_scale = -1.0
    assert _fwd(L, opts=o) == E.ERR_INVALID_ARG
    o.softmax_scale = math.inf
    assert _fwd(L, opts=o) == E.ERR_INVALID_ARG
    o.softmax_scale = 0.0
    o.budget_blocks = -1
    assert _fwd(L, opts=o) == E.ERR_INVALID_ARG
    # empty problems succeed without doing anything
    assert _fwd(L, B=0) == E.OK
    assert _fwd(L, N=0) == E.OK
    assert L.sol_attn_dense_forward(FAKE, FAKE, FAKE, FAKE, 1, 0, 64, 64, None) == E.OK
    assert L.sol_attn_dense_forward(FAKE, FAKE, FAKE, FAKE, 1, 1, 64, 80, None) == E.ERR_UNSUPPORTED
    assert L.sol_attn_pool(FAKE, FAKE, FAKE, FAKE + 16, 1, 1, 64, 64, None) == E.ERR_INVALID_ARG
    assert L.sol_attn_attend(FAKE, FAKE, FAKE, FAKE, None, 1, 1, 64, 64, 64, 1.0, 0, None,
                             None) == E.ERR_INVALID_ARG
    # host-buffer entry point: same checks, plus the chunk size
    def host(hq=FAKE, heads=0, D=64, tau=1.0, B=1):
        return L.sol_attn_forward_host(hq, FAKE, FAKE, FAKE, B, 2, 128, D, 64, tau, 0, heads, None)
    assert host(heads=-1) == E.ERR_INVALID_ARG
    assert host(hq=0) == E.ERR_INVALID_ARG
    assert host(hq=FAKE + 8) == E.ERR_INVALID_ARG
    assert host(D=96) == E.ERR_UNSUPPORTED
    assert host(tau=math.nan) == E.ERR_INVALID_ARG
    assert host(B=0) == E.OK
    # QKNorm + RoPE + pooling: rope_dims, eps, base and pointer checks
    def prep(R=64, eps=1e-6, base=1e4, ws=None, v=FAKE, w=FAKE, D=128, N=128):
        return L.sol_attn_qknorm_rope_pool(FAKE, FAKE, v, w, FAKE, FAKE, FAKE, ws, 1, 2, N, D, R, eps, base, None)
    assert prep(R=48) == E.ERR_INVALID_ARG         # 48 / 16 = 3 is not a power of two
    assert prep(R=8) == E.ERR_INVALID_ARG          # not a multiple of 16
    assert prep(R=256) == E.ERR_INVALID_ARG        # more than D
    assert prep(R=-16) == E.ERR_INVALID_ARG
    assert prep(eps=0.0) == E.ERR_INVALID_ARG
    assert prep(eps=math.nan) == E.ERR_INVALID_ARG
    assert prep(base=1.0) == E.ERR_INVALID_ARG
    assert prep(base=math.inf) == E.ERR_INVALID_ARG
    assert prep(w=0) == E.ERR_INVALID_ARG          # null weight
    assert prep(ws=FAKE + 16) == E.ERR_INVALID_ARG  # workspace not 256-byte aligned
    assert prep(ws=FAKE, v=0) == E.ERR_INVALID_ARG  # pooling needs v
    assert prep(D=96) == E.ERR_UNSUPPORTED
    assert prep(N=0) == E.OK
    # 8-bit entry point: D = 128 only, positive finite scales
    def fp8(D=128, qs=1.0, ks=1.0, vs=1.0, q=FAKE, tau=1.0, B=1):
        return L.sol_attn_forward_fp8(q, FAKE, FAKE, FAKE * 2, B, 2, 128, D, 64, tau, 0, qs, ks, vs, None, None)
    assert fp8(D=64) == E.ERR_UNSUPPORTED
    assert fp8(D=96) == E.ERR_UNSUPPORTED
    assert fp8(qs=0.0) == E.ERR_INVALID_ARG
    assert fp8(ks=-1.0) == E.ERR_INVALID_ARG
    assert fp8(vs=math.inf) == E.ERR_INVALID_ARG
    assert fp8(qs=math.nan) == E.ERR_INVALID_ARG
    assert fp8(q=FAKE + 8) == E.ERR_INVALID_ARG
    assert fp8(tau=math.nan) == E.ERR_INVALID_ARG
    assert fp8(B=0) == E.OK
    assert L.sol_attn_pool_fp8(FAKE, FAKE, FAKE, FAKE + 16, 1, 1, 64, 128, 1.0, 1.0, None) == E.ERR_INVALID_ARG
    assert L.sol_attn_pool_fp8(FAKE, FAKE, FAKE, FAKE, 1, 1, 64, 64, 1.0, 1.0, None) == E.ERR_UNSUPPORTED
    assert L.sol_attn_pool_fp8(FAKE, FAKE, FAKE, FAKE, 1, 1, 64, 128, 0.0, 1.0, None) == E.ERR_INVALID_ARG
    assert L.sol_attn_attend_fp8(FAKE, FAKE, FAKE, FAKE * 2, None, 1, 1, 64, 128, 64, 1.0, 0, 1.0, 1.0, 1.0,
                                 None, None) == E.ERR_INVALID_ARG


def test_python_binding_rejects_non_cuda_tensors(L):
    import torch
    x = torch.zeros(1, 1, 64, 64, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        abi.forward(x, x, x, 1.0)
    with pytest.raises(TypeError):  # the host entry point wants bf16 CPU tensors
        abi.forward_host(x.float(), x, x, 1.0)


def test_unpack_mask_bit_order():
    import numpy as np
    words = np.array([[0b101, 0x80000000]], dtype=np.uint32)
    bits = abi.unpack_mask(words, 40)
    assert bits.shape == (1, 40)
    assert list(np.nonzero(bits[0])[0]) == [0, 2]
    bits64 = abi.unpack_mask(words, 64)
    assert list(np.nonzero(bits64[0])[0]) == [0, 2, 63]
