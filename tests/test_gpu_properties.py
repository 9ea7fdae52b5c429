"""Properties of the CUDA path that hold at any size, checked at full sequence
length (refine, N = 32768, four or eight of its heads; the 131072-token sweep
workload, one head), where the oracle can only sample rows: a block permutation, agreement of the
dense paths with a library dense kernel, and every output row against the
definition written out in fp32 PyTorch (bf16 and E4M3 entry points).

Permuting the video key blocks (their K and V rows together) permutes every
row's keep mask with them and changes no output beyond summation order: the
router's scores are the same dot products of the same pooled vectors, and the
output sums the same exact and pooled terms in another order.  The kernel
visits a tile's blocks in ascending index order, so a permutation changes its
work list, its online-softmax rescale points and its correction tiles; an
index slip anywhere in that path shows up here at full size, where the oracle
can only sample.
"""

import numpy as np
import pytest
import torch

from block_sparse_attention_threshold_b200 import abi, build, synthetic as syn

from . import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    abi.lib()


def _permute_key_blocks(x, order, M, D):
    B, H, N, _ = x.shape
    return x.view(B, H, M, 64, D)[:, :, order].reshape(B, H, N, D).contiguous()


def test_video_key_block_permutation_full_size():
    w = syn.workload("refine_n32768").replace(H=4)
    tau = 1.25
    q, k, v = parity.to_device(*syn.generate_bf16(w))
    rng = np.random.default_rng(17)
    order = list(range(w.P)) + list(w.P + rng.permutation(w.M - w.P))
    idx = torch.tensor(order, device=q.device)
    kp, vp = (_permute_key_blocks(t, idx, w.M, w.D) for t in (k, v))
    out_a, keep_a, kept_a, _ = parity.run_sol(w, tau, q, k, v)
    out_b, keep_b, kept_b, _ = parity.run_sol(w, tau, q, kp, vp)
    # The scores are bit-identical; the mean and std differ at most by fp32
    # summation order, so a block flips only where it sits on its threshold.
    agree = (keep_b == keep_a[:, :, :, order]).mean()
    assert agree >= 1.0 - 1e-5, agree
    assert abs(kept_a - kept_b) <= 16
    a = out_a.float()
    b = out_b.float()
    rel = ((a - b).norm() / a.norm()).item()
    assert rel <= 2e-3, rel
    assert (a - b).abs().max().item() <= 2e-2


def test_dense_paths_agree_with_a_library_kernel_on_every_row():
    """A cross-check, not parity (parity is against the CPU oracle, which can
    only sample rows at this length): on every row of refine's full length,
    the in-repo dense kernel and Sol-Attn at tau = -inf (which keeps every
    block) agree with cuDNN's dense attention through PyTorch's SDPA, up to
    the rounding of two fp32-accumulating bf16 kernels."""
    from torch.nn.attention import SDPBackend, sdpa_kernel
    import torch.nn.functional as F
    w = syn.workload("refine_n32768").replace(H=8)
    q, k, v = parity.to_device(*syn.generate_bf16(w))
    try:
        with sdpa_kernel([SDPBackend.CUDNN_ATTENTION]):
            ref = F.scaled_dot_product_attention(q, k, v).float()
    except RuntimeError as e:  # the backend is not built for this device
        pytest.skip(f"cuDNN SDPA unavailable: {e}")
    dense = abi.dense_forward(q, k, v)
    sol = abi.forward(q, k, v, float("-inf"), w.prefix_len)
    torch.cuda.synchronize()
    assert abi.device_status() == abi.OK
    for out in (dense, sol):
        d = out.float() - ref
        assert (d.norm() / ref.norm()).item() <= 5e-3
        assert d.abs().max().item() <= 2e-2


def _check_against_fp32_reference(w, tau, qf, kf, vf, out, keep, rel_bar, abs_bar):
    """Routing and output of one run against the Sol-Attn definition in fp32
    PyTorch (parity.fp32_route / fp32_rows, themselves pinned to the oracle
    on the CPU): the mask against fp32 routing, every output row under the
    kernel's own mask."""
    torch.backends.cuda.matmul.allow_tf32 = False
    keep = torch.from_numpy(keep).to(qf.device)
    P = w.P
    mine = parity.fp32_route(w, tau, qf, kf)
    agree = (mine == keep[:, :, P:, P:]).float().mean().item()
    assert agree >= 0.999, agree
    assert keep[:, :, :P].all() and keep[:, :, :, :P].all()
    worst_rel, worst_abs = 0.0, 0.0
    for b in range(w.B):
        for h in range(w.H):
            num = den = 0.0
            for i0 in range(0, w.M, 8):               # eight query blocks at a time
                i1 = min(w.M, i0 + 8)
                ref = parity.fp32_rows(w, qf, kf, vf, keep, b, h, i0, i1)
                d = out[b, h, i0 * 64:i1 * 64].float() - ref
                num += d.square().sum().item()
                den += ref.square().sum().item()
                worst_abs = max(worst_abs, d.abs().max().item())
            worst_rel = max(worst_rel, (num / den) ** 0.5)
    assert worst_rel <= rel_bar, worst_rel
    assert worst_abs <= abs_bar, worst_abs


@pytest.mark.parametrize("name,heads,tau", [("refine_n32768", 4, 1.25), ("sweep_n131072", 1, 1.25)])
def test_every_row_matches_an_fp32_reference_at_full_length(name, heads, tau):
    """Every output row at full length against the Sol-Attn definition
    written out here in fp32 PyTorch (library matmuls and softmax, no TF32).
    The output is compared under the kernel's own keep mask (the debug
    export), so threshold ties cannot blur it; the mask itself is checked
    against fp32 routing done here (pooled means, population std over the
    video key blocks, keep iff score >= mean + tau * std).  Parity with the
    fp64 oracle stays the sampled test; this covers the rows it skips."""
    w = syn.workload(name).replace(H=heads)
    q, k, v = parity.to_device(*syn.generate_bf16(w))
    out, keep, _, _ = parity.run_sol(w, tau, q, k, v)
    _check_against_fp32_reference(w, tau, q.float(), k.float(), v.float(), out, keep,
                                  parity.REL_L2, parity.MAX_ABS)


def test_every_row_of_the_8bit_path_matches_an_fp32_reference():
    """The E4M3 entry point, refine at full length (four heads, scales 0.5,
    2 and 0.25), against the same fp32 reference on the decoded inputs times
    their scales, at the 8-bit bar (rel-L2 <= 5e-2, max-abs <= 1e-1)."""
    w = syn.workload("refine_n32768").replace(H=4)
    tau, scales = 1.25, (0.5, 2.0, 0.25)
    dev = torch.device("cuda", 0)
    q8, k8, v8 = (torch.from_numpy(np.ascontiguousarray(a)).to(dev) for a in syn.generate_e4m3(w, scales))
    M = w.M
    mask = torch.zeros(w.B * w.H * M * abi.mask_words(M), dtype=torch.int32, device=dev)
    opts = abi.Opts()
    opts.debug_mask = mask.data_ptr()
    out = abi.forward_fp8(q8, k8, v8, tau, w.prefix_len, *scales, opts=opts)
    torch.cuda.synchronize()
    assert abi.device_status() == abi.OK
    keep = abi.unpack_mask(mask.cpu().numpy().view(np.uint32).reshape(w.B, w.H, M, -1), M)
    qf, kf, vf = (x.view(torch.float8_e4m3fn).float() * sc for x, sc in zip((q8, k8, v8), scales))
    _check_against_fp32_reference(w, tau, qf, kf, vf, out, keep, 5e-2, 1e-1)
