"""Fixed-budget routing (the draft stage's block-sparse attention) through the
C ABI against the oracle: every video query block keeps its budget of
highest-scoring video key blocks, skipped blocks dropped or corrected."""

import math

import numpy as np
import pytest
import torch

from block_sparse_attention_threshold_b200 import abi, synthetic as syn

from . import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from block_sparse_attention_threshold_b200 import build
    build.build()
    abi.lib()


def draft_budget(w, video_sparsity=0.9):
    return max(1, round((1.0 - video_sparsity) * (w.M - w.P)))


@pytest.mark.parametrize("budget,correct", [(3, False), (3, True), (1, False), (64, False)])
def test_tiny_budget(budget, correct):
    w = syn.workload("tiny_n1024")
    bits = syn.generate_bf16(w)
    q, k, v = parity.to_device(*bits)
    out, keep, kept, _ = parity.run_sol(w, 0.0, q, k, v, budget=budget, correct=correct)
    nv = w.M - w.P
    assert (keep[0, :, w.P:, w.P:].sum(axis=-1) == min(budget, nv)).all()
    m = parity.oracle_compare(w, 0.0, *bits, out, keep, budget=budget, correct=correct)
    parity.assert_parity(m)


def test_budget_edge_shapes():
    w = syn.Workload("bedge", 2, 2, 64 * 13, 128, 192, (8, 24, 42), 0.8, (1.0,), 4242)
    bits = syn.generate_bf16(w)
    q, k, v = parity.to_device(*bits)
    for budget, correct in ((2, False), (5, True)):
        out, keep, _, _ = parity.run_sol(w, 0.0, q, k, v, budget=budget, correct=correct)
        m = parity.oracle_compare(w, 0.0, *bits, out, keep, budget=budget, correct=correct)
        parity.assert_parity(m)


def test_draft_workload_at_90_percent_video_sparsity():
    w = syn.workload("draft_n16128")
    bits = syn.generate_bf16(w)
    q, k, v = parity.to_device(*bits)
    budget = draft_budget(w)
    out, keep, kept, exact = parity.run_sol(w, 0.0, q, k, v, budget=budget, correct=False)
    assert (keep[0, :, w.P:, w.P:].sum(axis=-1) == budget).all()
    blocks = syn.sample_query_blocks(w.M, w.P, 64, w.seed + 7)
    m = parity.oracle_compare(w, 0.0, *bits, out, keep, qblocks=blocks, budget=budget, correct=False)
    print("draft budget", budget, m, "kept", kept, "exact", exact)
    parity.assert_parity(m)


def test_full_budget_equals_dense():
    w = syn.workload("tiny_n1024")
    bits = syn.generate_bf16(w)
    q, k, v = parity.to_device(*bits)
    out, keep, _, _ = parity.run_sol(w, 0.0, q, k, v, budget=10_000, correct=False)
    assert keep.all()
    d = abi.dense_forward(q, k, v)
    torch.cuda.synchronize()
    assert (out.float() - d.float()).abs().max().item() <= 2e-2
