"""GPU parity of the online chunking step (dhsa_segment) against the oracle.

The rule (oracle ``segment``): with the current chunk starting at b, token t
starts a chunk when t - b >= max_len, or t - b >= min_len and the mean over KV
heads of cos(k[t-1], k[t]) is below the threshold.  The GPU takes each
decision on an fp32 similarity; where no similarity on the path lies within
the fp32 band of the threshold, its chunks must equal the oracle's exactly,
and otherwise every chunk must be a legal step of the rule.
"""

from types import SimpleNamespace

import numpy as np
import pytest
import torch

from dynamic_hierarchical_sparse_b200 import api, workloads as W
from oracle import dhsa_oracle as O
from tests.helpers import (attention_gate, check_segmentation, compare_plans, gpu_rows, segment_tie_band,
                           segmentations_agree_until_latitude)

pytestmark = pytest.mark.gpu


def _run(k, cu, rule):
    dev = torch.device("cuda")
    bounds, ptr = api.segment(k.to(dev), cu, rule, check=True)
    torch.cuda.synchronize()
    return bounds, ptr


def _check(k, cu, rule, exact=True):
    bounds, ptr = _run(k, cu, rule)
    want_b, want_p = O.segment(k, cu, rule.threshold, rule.min_len, rule.max_len)
    sim = O.adjacent_key_similarity(k)
    first_loose = check_segmentation(bounds, ptr, sim, cu, rule, segment_tie_band(k.shape[2]))
    segmentations_agree_until_latitude(bounds, ptr, want_b, want_p, first_loose)
    if exact:
        assert all(f is None for f in first_loose), "a decision within the fp32 band on an input built to have none"
    return bounds, ptr, first_loose


@pytest.mark.parametrize("d,hkv,dtype", [(64, 1, "bf16"), (128, 8, "bf16"), (256, 4, "bf16"),
                                         (64, 2, "f32"), (128, 3, "f32"), (256, 1, "f32")])
def test_planted_segments(d, hkv, dtype):
    """Planted segments U[100, 300] in ragged sequences (one empty, one
    shorter than min_len, lengths not multiples of 32): recovered exactly."""
    k, cu, bounds, ptr = W.planted_segment_keys(d + hkv, [2000, 0, 37, 5003, 1], hkv, d, 100, 300, dtype)
    rule = W.SegmentRule(0.5, 100, 300)
    got_b, got_p, _ = _check(k, cu, rule)
    assert np.array_equal(got_b, bounds) and np.array_equal(got_p, ptr)


@pytest.mark.parametrize("seed,rho,thr,lo,hi", [(0, 0.9, 0.9, 8, 64), (1, 0.95, 0.95, 1, 40),
                                                (2, 0.8, 0.78, 32, 32), (3, 0.9, 0.9, 100, 1000)])
def test_drifting_keys_near_the_threshold(seed, rho, thr, lo, hi):
    """Similarities packed around the threshold: every GPU chunk is a legal
    step, and equal to the oracle's wherever no decision fell in the band."""
    k = W.drifting_keys(seed, 12000, 8, 128, rho=rho)
    cu = [0, 5000, 5001, 5001, 12000]
    _check(k, cu, W.SegmentRule(thr, lo, hi), exact=False)


@pytest.mark.parametrize("thr", [float("-inf"), -2.0, 2.0, float("inf")])
def test_thresholds_that_no_or_every_cosine_passes(thr):
    k = torch.randn(70001, 2, 64, generator=torch.Generator().manual_seed(7)).to(torch.bfloat16)
    cu = [0, 33, 33, 40000, 70001]
    rule = W.SegmentRule(thr, 7, 1000)
    bounds, ptr = _run(k, cu, rule)
    step = rule.max_len if thr < 0 else rule.min_len
    want, wptr = [], [0]
    for s0, s1 in zip(cu[:-1], cu[1:]):
        want += list(range(s0, s1, step))
        wptr.append(len(want))
    assert bounds.tolist() == want + [cu[-1]]
    assert ptr.tolist() == wptr


def test_every_token_its_own_chunk_and_longest_chunks():
    """min_len = max_len = 1 (capacity = T), and max_len = 65536 on a
    sequence long enough to move the walk's shared-memory window."""
    k = torch.randn(3000, 1, 64, generator=torch.Generator().manual_seed(8)).to(torch.bfloat16)
    b, p = _run(k, [0, 1000, 3000], W.SegmentRule(0.0, 1, 1))
    assert b.tolist() == list(range(3001)) and p.tolist() == [0, 1000, 3000]
    k = torch.randn(300000, 1, 64, generator=torch.Generator().manual_seed(9)).to(torch.bfloat16)
    cu = [0, 5, 300000]
    b, p = _run(k, cu, W.SegmentRule(-2.0, 65536, 65536))
    assert b.tolist() == [0, 5, 5 + 65536, 5 + 2 * 65536, 5 + 3 * 65536, 5 + 4 * 65536, 300000]
    assert p.tolist() == [0, 1, 6]
    # breaks far apart: drops only every 40000 tokens, max_len 65536
    k = torch.ones(300000, 1, 64)
    k[::40000] *= -1.0
    k = k.to(torch.bfloat16)
    b, p = _run(k, cu, W.SegmentRule(0.0, 100, 65536))
    want_b, want_p = O.segment(k, cu, 0.0, 100, 65536)
    assert np.array_equal(b, want_b) and np.array_equal(p, want_p)


def test_zero_keys_never_break():
    k = W.drifting_keys(4, 4000, 2, 128, rho=0.5)
    k[1000:1100] = 0
    k[2000:2100, 0] = 0  # one head only: that head counts as cosine 1
    _check(k, [0, 4000], W.SegmentRule(0.45, 4, 300), exact=False)


def test_empty_batch_and_empty_sequences():
    k = torch.zeros(0, 2, 64, dtype=torch.bfloat16)
    b, p = _run(k, [0, 0, 0], W.SegmentRule(0.5, 4, 8))
    assert b.tolist() == [0] and p.tolist() == [0, 0, 0]


def test_full_size_128k_planted_then_plan_and_attention():
    """The 128K LLaMA shape (Hkv = 8, d = 128), segments planted as the
    workload's chunks U[256, 1024]: recovered exactly; the resulting problem
    then plans and attends like any other (sampled rows against the oracle)."""
    k, cu, bounds, ptr = W.planted_segment_keys(11, [131072], 8, 128, 256, 1024)
    rule = W.SegmentRule(0.5, 256, 1024)
    got_b, got_p = _run(k, cu, rule)
    assert np.array_equal(got_b, bounds) and np.array_equal(got_p, ptr)
    # a short pipeline on the GPU's own boundaries
    k2, cu2, _, _ = W.planted_segment_keys(12, [3000, 1500], 2, 128, 64, 256)
    b2, p2 = _run(k2, cu2, W.SegmentRule(0.5, 64, 256))
    dev = torch.device("cuda")
    gen = torch.Generator().manual_seed(13)
    q = torch.randn(k2.shape[0], 4, 128, generator=gen).to(torch.bfloat16)
    v = torch.randn(k2.shape[0], 2, 128, generator=gen).to(torch.bfloat16)
    prob = api.Problem(cu2, b2, p2, 4, 2, 128, torch.bfloat16, device=dev)
    budget = W.Budget.topk(3)
    plan = api.plan(q.to(dev), k2.to(dev), prob, budget, check=True)
    out = api.attention(q.to(dev), k2.to(dev), v.to(dev), prob, plan, check=True)
    torch.cuda.synchronize()
    ref = O.build_plan(q, k2, b2, p2, budget.kind, budget.k)
    rows = gpu_rows(plan, 4 * (b2.shape[0] - 1))
    tolerated = compare_plans(rows, ref, SimpleNamespace(num_chunks=b2.shape[0] - 1, seq_chunk_ptr=p2), budget)
    assert len(tolerated) <= 2
    want = O.attention_gather(q, k2, v, b2, plan.row_ptr.cpu().numpy(), plan.col.cpu().numpy())
    attention_gate(out, want, q.dtype)
