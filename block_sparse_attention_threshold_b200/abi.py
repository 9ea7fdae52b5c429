"""ctypes binding of libsolattn.so (the C ABI in include/sol_attn.h).

Argument marshalling only: tensors are passed as raw device pointers and the
current CUDA stream as a handle.  Every step of the computation runs in the
library's kernels; there is no fallback path.  If the library is missing the
first call raises.
"""

from __future__ import annotations

import ctypes
import math
import os
import re

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsolattn.so")

OK = 0
ERR_INVALID_ARG = 1
ERR_UNSUPPORTED = 2
ERR_ARCH = 3
ERR_CUDA = 4
ERR_DEVICE_TIMEOUT = 5

BLOCK = 64


class SolAttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


class Opts(ctypes.Structure):
    """Mirror of sol_attn_opts."""

    _fields_ = [
        ("kept_pairs", ctypes.c_void_p),
        ("exact_pairs", ctypes.c_void_p),
        ("debug_mask", ctypes.c_void_p),
        ("softmax_scale", ctypes.c_float),
        ("timeout_ms", ctypes.c_uint),
        ("test_skip_first_k_load", ctypes.c_int),
        ("budget_blocks", ctypes.c_int),
        ("skip_correction", ctypes.c_int),
    ]


_lib = None

_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_SIGS = {
    "sol_attn_forward": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _P]),
    "sol_attn_forward_ex": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, ctypes.POINTER(Opts), _P]),
    "sol_attn_dense_forward": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _P]),
    "sol_attn_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I, _I, ctypes.POINTER(ctypes.c_size_t)]),
    "sol_attn_pool": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _P]),
    "sol_attn_attend": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, ctypes.POINTER(Opts), _P]),
    "sol_attn_forward_noalloc": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _P]),
    "sol_attn_forward_fp8": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _F, _F, _F, ctypes.POINTER(Opts), _P]),
    "sol_attn_pool_fp8": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _F, _F, _P]),
    "sol_attn_attend_fp8": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _F, _F, _F, ctypes.POINTER(Opts), _P]),
    "sol_attn_forward_host": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _I, _P]),
    "sol_attn_qknorm_rope_pool": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _F, _P]),
    "sol_attn_device_status": (_I, [_P]),
    "sol_attn_status_string": (ctypes.c_char_p, [_I]),
}


def lib() -> ctypes.CDLL:
    """Load libsolattn.so once; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -c 'import __graft_entry__ as g; g.build()'`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def declared_symbols(header: str) -> list:
    """Function names declared in a C header (for export checks)."""
    with open(header) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sol_attn_\w+)\s*\(", text)))


def status_string(status: int) -> str:
    return lib().sol_attn_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != OK:
        raise SolAttnError(status, where)


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _shape(q, k, v):
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or not t.is_cuda:
            raise TypeError(f"{name} must be a CUDA bf16 tensor")
        if t.dim() != 4 or not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous [B, H, N, D]")
    if not (q.shape == k.shape == v.shape):
        raise ValueError("q, k, v must have the same shape")
    return tuple(int(x) for x in q.shape)


def _out_like(q, out):
    import torch
    if out is None:
        return torch.empty_like(q)
    if out.shape != q.shape or out.dtype != torch.bfloat16 or not out.is_contiguous():
        raise ValueError("out must be a contiguous bf16 tensor shaped like q")
    return out


def forward(q, k, v, tau: float, prefix_len: int = 0, out=None, opts: Opts | None = None,
            stream=None, block: int = BLOCK):
    """Sol-Attn forward through sol_attn_forward_ex; returns `out`."""
    B, H, N, D = _shape(q, k, v)
    out = _out_like(q, out)
    st = lib().sol_attn_forward_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                   B, H, N, D, block, float(tau), int(prefix_len),
                                   ctypes.byref(opts) if opts is not None else None,
                                   _stream(stream))
    _check(st, "sol_attn_forward_ex")
    return out


def forward_noalloc(q, k, v, tau: float, prefix_len: int = 0, out=None, stream=None,
                    block: int = BLOCK):
    """Sol-Attn through sol_attn_forward_noalloc: the pooled workspace comes from
    a fixed array inside the library, for callers that cannot allocate device
    memory while they run.  Calls whose kernels overlap on the GPU race on that
    array; the first call on a device must come before any stream capture."""
    B, H, N, D = _shape(q, k, v)
    out = _out_like(q, out)
    st = lib().sol_attn_forward_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                        B, H, N, D, block, float(tau), int(prefix_len),
                                        _stream(stream))
    _check(st, "sol_attn_forward_noalloc")
    return out


def forward_fp8(q8, k8, v8, tau: float, prefix_len: int = 0, q_scale: float = 1.0, k_scale: float = 1.0,
                v_scale: float = 1.0, out=None, opts: Opts | None = None, stream=None, block: int = BLOCK):
    """Sol-Attn on E4M3 inputs through sol_attn_forward_fp8.  q8, k8, v8 are
    CUDA uint8 tensors [B, H, N, D] holding E4M3 bytes (real value = decoded
    byte times the tensor's scale); returns the bf16 output."""
    import torch
    for name, t in (("q8", q8), ("k8", k8), ("v8", v8)):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.uint8 or not t.is_cuda:
            raise TypeError(f"{name} must be a CUDA uint8 tensor of E4M3 bytes")
        if t.dim() != 4 or not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous [B, H, N, D]")
    if not (q8.shape == k8.shape == v8.shape):
        raise ValueError("q8, k8, v8 must have the same shape")
    B, H, N, D = (int(x) for x in q8.shape)
    if out is None:
        out = torch.empty(q8.shape, dtype=torch.bfloat16, device=q8.device)
    elif out.shape != q8.shape or out.dtype != torch.bfloat16 or not out.is_contiguous():
        raise ValueError("out must be a contiguous bf16 tensor shaped like q8")
    st = lib().sol_attn_forward_fp8(q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), out.data_ptr(),
                                    B, H, N, D, block, float(tau), int(prefix_len), float(q_scale),
                                    float(k_scale), float(v_scale),
                                    ctypes.byref(opts) if opts is not None else None, _stream(stream))
    _check(st, "sol_attn_forward_fp8")
    return out


def pool_fp8(q8, k8, v8, workspace, q_scale: float = 1.0, k_scale: float = 1.0, stream=None) -> None:
    """Pooling of E4M3 inputs into `workspace` (CUDA uint8) via sol_attn_pool_fp8."""
    B, H, N, D = (int(x) for x in q8.shape)
    st = lib().sol_attn_pool_fp8(q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), workspace.data_ptr(),
                                 B, H, N, D, float(q_scale), float(k_scale), _stream(stream))
    _check(st, "sol_attn_pool_fp8")


def attend_fp8(q8, k8, v8, workspace, tau: float, prefix_len: int = 0, q_scale: float = 1.0,
               k_scale: float = 1.0, v_scale: float = 1.0, out=None, opts: Opts | None = None, stream=None,
               block: int = BLOCK):
    """Routing + attention on a pool_fp8 workspace via sol_attn_attend_fp8."""
    import torch
    B, H, N, D = (int(x) for x in q8.shape)
    if out is None:
        out = torch.empty(q8.shape, dtype=torch.bfloat16, device=q8.device)
    st = lib().sol_attn_attend_fp8(q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), out.data_ptr(),
                                   workspace.data_ptr(), B, H, N, D, block, float(tau), int(prefix_len),
                                   float(q_scale), float(k_scale), float(v_scale),
                                   ctypes.byref(opts) if opts is not None else None, _stream(stream))
    _check(st, "sol_attn_attend_fp8")
    return out


def forward_host(q, k, v, tau: float, prefix_len: int = 0, out=None, heads_per_chunk: int = 0,
                 stream=None, block: int = BLOCK):
    """Sol-Attn through sol_attn_forward_host: q, k, v and out are CPU bf16
    tensors (page-locked for copy/compute overlap), contiguous [B, H, N, D].
    The library copies head chunks in, computes and copies them back on its
    own pipeline; `out` is complete once `stream` (the current CUDA stream by
    default) has finished."""
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or t.is_cuda:
            raise TypeError(f"{name} must be a CPU bf16 tensor")
        if t.dim() != 4 or not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous [B, H, N, D]")
    if not (q.shape == k.shape == v.shape):
        raise ValueError("q, k, v must have the same shape")
    B, H, N, D = (int(x) for x in q.shape)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, pin_memory=q.is_pinned())
    elif out.shape != q.shape or out.dtype != torch.bfloat16 or out.is_cuda or not out.is_contiguous():
        raise ValueError("out must be a contiguous CPU bf16 tensor shaped like q")
    st = lib().sol_attn_forward_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                     B, H, N, D, block, float(tau), int(prefix_len),
                                     int(heads_per_chunk), _stream(stream))
    _check(st, "sol_attn_forward_host")
    return out


def qknorm_rope_pool(q_in, k_in, v, q_weight, k_weight, rope_dims: int, eps: float = 1e-6,
                     rope_base: float = 10000.0, q_out=None, k_out=None, workspace=None, pool: bool = True,
                     stream=None):
    """QKNorm + partial RoPE of q and k through sol_attn_qknorm_rope_pool, with the
    pooled workspace for sol_attn_attend filled in the same pass (pool=True).
    q_weight, k_weight: CUDA fp32 [D].  Returns (q_out, k_out, workspace or None)."""
    import torch
    B, H, N, D = _shape(q_in, k_in, v)
    for name, t in (("q_weight", q_weight), ("k_weight", k_weight)):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.float32 or not t.is_cuda or t.shape != (D,):
            raise TypeError(f"{name} must be a CUDA fp32 tensor of shape [D]")
    q_out = _out_like(q_in, q_out)
    k_out = _out_like(k_in, k_out)
    ws_ptr = None
    if pool:
        if workspace is None:
            nbytes, _ = workspace_layout(B, H, N, D)
            workspace = torch.empty(nbytes, dtype=torch.uint8, device=q_in.device)
        ws_ptr = workspace.data_ptr()
    else:
        workspace = None
    st = lib().sol_attn_qknorm_rope_pool(q_in.data_ptr(), k_in.data_ptr(), v.data_ptr(), q_weight.data_ptr(),
                                         k_weight.data_ptr(), q_out.data_ptr(), k_out.data_ptr(), ws_ptr,
                                         B, H, N, D, int(rope_dims), float(eps), float(rope_base),
                                         _stream(stream))
    _check(st, "sol_attn_qknorm_rope_pool")
    return q_out, k_out, workspace


def noalloc_max_workspace() -> int:
    """SOL_ATTN_NOALLOC_MAX_WORKSPACE from the header: bytes of the fixed array."""
    header = os.path.join(os.path.dirname(_HERE), "include", "sol_attn.h")
    with open(header) as f:
        m = re.search(r"#define\s+SOL_ATTN_NOALLOC_MAX_WORKSPACE\s+\((\d+)u\s*<<\s*(\d+)\)", f.read())
    return int(m.group(1)) << int(m.group(2))


def dense_forward(q, k, v, out=None, stream=None):
    """Dense attention through sol_attn_dense_forward; returns `out`."""
    B, H, N, D = _shape(q, k, v)
    out = _out_like(q, out)
    st = lib().sol_attn_dense_forward(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                      B, H, N, D, _stream(stream))
    _check(st, "sol_attn_dense_forward")
    return out


def workspace_layout(B: int, H: int, N: int, D: int):
    """(bytes, [4 section offsets]) of the pooled-summary workspace."""
    offs = (ctypes.c_size_t * 4)()
    n = lib().sol_attn_workspace_bytes(B, H, N, D, offs)
    return int(n), [int(x) for x in offs]


def pool(q, k, v, workspace, stream=None) -> None:
    """Block means into `workspace` (a CUDA uint8 tensor) via sol_attn_pool."""
    B, H, N, D = _shape(q, k, v)
    st = lib().sol_attn_pool(q.data_ptr(), k.data_ptr(), v.data_ptr(), workspace.data_ptr(),
                             B, H, N, D, _stream(stream))
    _check(st, "sol_attn_pool")


def attend(q, k, v, workspace, tau: float, prefix_len: int = 0, out=None,
           opts: Opts | None = None, stream=None, block: int = BLOCK):
    """Routing + attention on a pooled workspace via sol_attn_attend."""
    B, H, N, D = _shape(q, k, v)
    out = _out_like(q, out)
    st = lib().sol_attn_attend(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                               workspace.data_ptr(), B, H, N, D, block, float(tau),
                               int(prefix_len), ctypes.byref(opts) if opts is not None else None,
                               _stream(stream))
    _check(st, "sol_attn_attend")
    return out


def device_status(stream=None) -> int:
    """Synchronise the stream and read/clear the kernels' timeout word."""
    return int(lib().sol_attn_device_status(_stream(stream)))


def mask_words(M: int) -> int:
    return (M + 31) // 32


def unpack_mask(words, M: int):
    """[..., ceil(M/32)] uint32 words (numpy) -> [..., M] bool."""
    import numpy as np
    w = np.ascontiguousarray(words).astype(np.uint32)
    bits = ((w[..., :, None] >> np.arange(32, dtype=np.uint32)) & 1).astype(bool)
    return bits.reshape(*w.shape[:-1], -1)[..., :M]


def default_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)
