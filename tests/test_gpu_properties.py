"""Properties of the CUDA path that hold at any size, checked at full sequence
length (refine: N = 32768, D = 128, prefix 1024; four or eight of its heads),
where the oracle can only sample rows.

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
