"""The parity harness itself, on the CPU: a keep mask that disagrees with the
oracle where the oracle's answer is forced must fail, whatever the distance
of the score to the threshold.

The "device" output here is the oracle's own result, so only the mask check
is exercised.  Mistakes are planted in the mask handed to the harness.
"""

import math

import numpy as np
import pytest
import torch

from block_sparse_attention_threshold_b200 import synthetic as syn
from oracle import sol_attn_oracle as orc

from . import parity


def _case(tau):
    w = syn.workload("tiny_n1024")
    bits = syn.generate_bf16(w)
    q, k, v = (syn.bf16_bits_to_fp64(b) for b in bits)
    out = orc.solattn(q, k, v, 64, w.prefix_len, tau)
    out_t = torch.from_numpy(out.astype(np.float32)).to(torch.bfloat16)
    keep = np.stack([np.stack([orc.route(q[b, h], k[b, h], 64, w.prefix_len, tau).keep
                               for h in range(w.H)]) for b in range(w.B)])
    return w, bits, out_t, keep


def test_harness_accepts_the_oracle_itself():
    w, bits, out, keep = _case(1.0)
    m = parity.oracle_compare(w, 1.0, *bits, out, keep, workers=2)
    parity.assert_parity(m)
    assert m["mask_mismatch"] == 0 and m["hard_mismatch"] == 0


@pytest.mark.parametrize("where", ["prefix_column", "prefix_row", "tau_minus_inf"])
def test_harness_fails_on_forced_mismatch(where):
    tau = -math.inf if where == "tau_minus_inf" else 1.0
    w, bits, out, keep = _case(tau)
    bad = keep.copy()
    P = w.P
    if where == "prefix_column":
        bad[0, 0, P + 1, 0] = False          # a video query block dropping a prefix key block
    elif where == "prefix_row":
        bad[0, 1, 0, P + 3] = False          # a prefix query block dropping a video key block
    else:
        bad[0, 0, P + 2, P + 5] = False      # tau = -inf keeps everything
    m = parity.oracle_compare(w, tau, *bits, out, bad, workers=2)
    assert m["hard_mismatch"] == 1
    with pytest.raises(AssertionError):
        parity.assert_parity(m)
    # the forced-position check fails on its own, even where the agreement
    # rate and the band would pass (as on a large workload)
    m.update(mask_agree=1.0, worst_band=0.0)
    with pytest.raises(AssertionError, match="hard_mismatch"):
        parity.assert_parity(m)


def test_harness_measures_routed_mismatch_against_sigma():
    w, bits, out, keep = _case(1.0)
    q = syn.bf16_bits_to_fp64(bits[0][0, 0])
    k = syn.bf16_bits_to_fp64(bits[1][0, 0])
    r = orc.route(q, k, 64, w.prefix_len, 1.0)
    P = w.P
    # flip the routed pair whose score is closest to its row's threshold
    i, j = min(((i, j) for i in range(P, w.M) for j in range(P, w.M)),
               key=lambda ij: abs(r.score[ij] - r.thr[ij[0]]) / r.sigma[ij[0]])
    bad = keep.copy()
    bad[0, 0, i, j] = ~bad[0, 0, i, j]
    m = parity.oracle_compare(w, 1.0, *bits, out, bad, workers=2)
    assert m["hard_mismatch"] == 0 and m["mask_mismatch"] == 1
    assert m["worst_band"] == pytest.approx(abs(r.score[i, j] - r.thr[i]) / r.sigma[i])


@pytest.mark.parametrize("tau", [0.5, 1.0, 1.5])
def test_fp32_reference_matches_the_oracle(tau):
    """The fp32 PyTorch reference that the full-length GPU checks use, pinned
    to the oracle on the tiny workload: the same keep mask and the same rows."""
    import torch
    w = syn.workload("tiny_n1024")
    q, k, v = (syn.bf16_bits_to_fp64(a) for a in syn.generate_bf16(w))
    qf, kf, vf = (torch.from_numpy(x).float() for x in (q, k, v))
    mine = parity.fp32_route(w, tau, qf, kf).numpy()
    keep = np.stack([np.stack([orc.route(q[b, h], k[b, h], 64, w.prefix_len, tau).keep
                               for h in range(w.H)]) for b in range(w.B)])
    assert np.array_equal(mine, keep[:, :, w.P:, w.P:])
    ref = orc.solattn(q, k, v, 64, w.prefix_len, tau)
    kt = torch.from_numpy(keep)
    for b in range(w.B):
        for h in range(w.H):
            rows = parity.fp32_rows(w, qf, kf, vf, kt, b, h, 0, w.M).double().numpy()
            np.testing.assert_allclose(rows, ref[b, h], rtol=0, atol=2e-5)
