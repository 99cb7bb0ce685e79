"""GPU parity: every step of the CUDA path against the fp64 oracle, through the C ABI.

Sizes are small enough for the oracle to finish in seconds, yet span several
tiles and ragged tails (chunk lengths 1, 2, 17, 127..129, 255..300).
"""

import math

import numpy as np
import pytest
import torch

from dynamic_hierarchical_sparse_b200 import api, workloads as W
from oracle import dhsa_oracle as O
from tests.helpers import (attention_gate, compare_plans, gpu_rows, reduce_bound, to_device)

pytestmark = pytest.mark.gpu

RAGGED_LENS = [[1, 2, 17, 127, 128, 129, 60, 255, 3, 300], [64, 1, 190, 45], [7]]


def _case(name):
    if name == "ragged_d128_top2":
        return W.explicit_problem(0, RAGGED_LENS, 4, 2, 128, "bf16", W.Budget.topk(2))
    if name == "ragged_d64_frac":
        return W.explicit_problem(1, RAGGED_LENS, 2, 1, 64, "bf16", W.Budget.fraction(1, 3))
    if name == "d256_structured_top3":
        return W.random_problem(2, [1500], 4, 2, 256, "bf16", 64, 256, W.Budget.topk(3), "structured")
    if name == "d128_dense":
        return W.random_problem(3, [900, 400], 4, 1, 128, "bf16", 30, 200, W.Budget.topk(10 ** 6))
    if name == "d128_diag_only":
        return W.random_problem(4, [1000], 2, 2, 128, "bf16", 50, 300, W.Budget.topk(0))
    if name == "d128_long_runs":
        return W.random_problem(5, [3000], 2, 1, 128, "bf16", 128, 512, W.Budget.fraction(1, 2), "structured")
    if name == "d128_many_runs":
        # ~600 chunks of 3-7 tokens, half of each row kept: late rows hold more
        # than a hundred separate runs of chunks
        return W.random_problem(8, [3000], 2, 1, 128, "bf16", 3, 7, W.Budget.fraction(1, 2))
    if name == "d64_many_runs":
        return W.random_problem(9, [2500], 2, 2, 64, "bf16", 2, 5, W.Budget.fraction(1, 2))
    if name == "d128_fixed96":
        # equal chunks of 96 tokens (not a tile multiple) and a shorter last chunk
        return W.random_problem(10, [2000], 4, 2, 128, "bf16", 96, 96, W.Budget.topk(3), "structured")
    if name == "d64_fixed256":
        return W.random_problem(11, [2048, 1024], 2, 1, 64, "bf16", 256, 256, W.Budget.fraction(1, 4))
    if name == "d128_group3":
        # three query heads per KV head: a per-KV-head plan cannot pair heads
        return W.random_problem(12, [1700, 900], 6, 2, 128, "bf16", 60, 300, W.Budget.fraction(1, 4), "structured")
    if name == "d64_group3":
        return W.random_problem(13, [1300], 3, 1, 64, "bf16", 40, 200, W.Budget.topk(3))
    if name == "d256_group3":
        return W.random_problem(14, [1200], 3, 1, 256, "bf16", 64, 256, W.Budget.topk(2), "structured")
    if name == "tiny_f32":
        return W.generate(W.TINY_1K_F32, 0)
    if name == "f32_d128_ragged":
        return W.explicit_problem(6, RAGGED_LENS, 2, 1, 128, "f32", W.Budget.topk(3))
    raise KeyError(name)


CASES = ["ragged_d128_top2", "ragged_d64_frac", "d256_structured_top3", "d128_dense", "d128_diag_only",
         "d128_long_runs", "d128_many_runs", "d64_many_runs", "d128_fixed96", "d64_fixed256", "tiny_f32",
         "f32_d128_ragged", "d128_group3"]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    api.lib()


@pytest.mark.parametrize("name", CASES)
def test_chunk_reduce(name):
    inp = _case(name)
    q, k, v, prob = to_device(inp)
    for x in (inp.q, inp.k):
        got = api.chunk_reduce(x.cuda(), prob).double().cpu().numpy()
        want = O.chunk_representations(x, inp.chunk_bounds)
        bound = reduce_bound(x, inp.chunk_bounds)
        assert np.all(np.abs(got - want) <= bound), float(np.max(np.abs(got - want) - bound))


@pytest.mark.parametrize("name", CASES)
def test_chunk_similarity(name):
    """Same fp32 representations in; fp32 dot products out, within the fp32 bound."""
    inp = _case(name)
    _, _, _, prob = to_device(inp)
    qc = O.chunk_representations(inp.q, inp.chunk_bounds).astype(np.float32)
    kc = O.chunk_representations(inp.k, inp.chunk_bounds).astype(np.float32)
    got = api.chunk_similarity(torch.from_numpy(qc).cuda(), torch.from_numpy(kc).cuda(), prob).double().cpu().numpy()
    want = O.chunk_scores(qc.astype(np.float64), kc.astype(np.float64), inp.seq_chunk_ptr)
    d = qc.shape[2]
    group = qc.shape[0] // kc.shape[0]
    absdot = np.einsum("hid,hjd->hij", np.abs(qc.astype(np.float64)),
                       np.abs(np.repeat(kc.astype(np.float64), group, axis=0)))
    mask = ~np.isnan(want)
    err = np.abs(got - np.nan_to_num(want))[mask]
    assert np.all(err <= (d + 2) * 2.0 ** -24 * absdot[mask] + 1e-30)


@pytest.mark.parametrize("name", CASES)
def test_topk_select_bit_exact_on_same_scores(name):
    """Selection from identical fp32 scores is integer work: bit-exact."""
    inp = _case(name)
    _, _, _, prob = to_device(inp)
    qc = O.chunk_representations(inp.q, inp.chunk_bounds).astype(np.float32)
    kc = O.chunk_representations(inp.k, inp.chunk_bounds).astype(np.float32)
    S32 = api.chunk_similarity(torch.from_numpy(qc).cuda(), torch.from_numpy(kc).cuda(), prob)
    # plant exact ties: copy a score onto its neighbour in a few rows
    S32 = S32.clone()
    n = inp.num_chunks
    for i in range(2, n, 3):
        S32[:, i, i - 1] = S32[:, i, i - 2]
    plan = api.topk_select(S32, prob, inp.budget, check=True)
    S = S32.double().cpu().numpy()
    b = inp.budget
    ptr = inp.seq_chunk_ptr
    rows = gpu_rows(plan, inp.spec.num_q_heads * n)
    for h in range(inp.spec.num_q_heads):
        for bb in range(len(ptr) - 1):
            for i in range(int(ptr[bb]), int(ptr[bb + 1])):
                cand = list(range(int(ptr[bb]), i))
                keep = O.row_budget(i - int(ptr[bb]), b.kind, b.k, b.num, b.den)
                want = sorted(O.select_row([S[h, i, j] for j in cand], cand, keep)) + [i]
                assert rows[h * n + i] == want, (h, i)


def _long_row_scores(n, hq, seed):
    """Score patterns for rows of hundreds to ~1300 candidates: Gaussian, heavy
    ties with signed zeros, constant, monotone up and down, rounded Gaussian."""
    rng = np.random.default_rng(seed)
    S = np.empty((hq, n, n), dtype=np.float32)
    S[0] = rng.standard_normal((n, n))
    S[1] = rng.choice(np.array([-0.0, 0.0, 1.0, 2.0], dtype=np.float32), size=(n, n))
    S[2] = 0.5
    S[3] = np.arange(n, dtype=np.float32)[None, :]
    S[4] = -np.arange(n, dtype=np.float32)[None, :]
    S[5] = np.round(rng.standard_normal((n, n)), 1)
    return S


@pytest.mark.parametrize("budget", [W.Budget.fraction(1, 20), W.Budget.topk(7), W.Budget.fraction(1, 8),
                                    W.Budget.topk(1)], ids=["frac5", "top7", "frac12.5", "top1"])
def test_topk_select_long_rows(budget):
    """Rows long enough for the sampled-threshold filter, with score patterns
    that make it succeed (Gaussian, ties inside the survivors, monotone rows)
    and fail (constant rows overflow the survivor space): every row equals the
    oracle's selection, bit for bit."""
    lens = [[1] * 1300, [1] * 600]
    cu, bounds, sptr = W.make_bounds([1300, 600], lens)
    hq = 6
    prob = api.Problem(cu, bounds, sptr, hq, 1, 128, torch.bfloat16, torch.device("cuda"))
    n = prob.num_chunks
    S = _long_row_scores(n, hq, 11)
    plan = api.topk_select(torch.from_numpy(S).cuda(), prob, budget, check=True)
    rows = gpu_rows(plan, hq * n)
    for h in range(hq):
        for bb in range(len(sptr) - 1):
            c0 = int(sptr[bb])
            for i in range(c0, int(sptr[bb + 1])):
                cand = list(range(c0, i))
                keep = O.row_budget(i - c0, budget.kind, budget.k, budget.num, budget.den)
                want = sorted(O.select_row([float(S[h, i, j]) for j in cand], cand, keep)) + [i]
                assert rows[h * n + i] == want, (h, i)


def _very_long_row_scores(n, hq, seed):
    """Rows of up to ~3300 candidates (the select micro-benchmark's length):
    Gaussian, a narrow band where every score shares its sign, exponent and
    high mantissa bits (the radix must start low), a range over 60 decades,
    heavy ties with signed zeros, constant, and spikes placed exactly where
    a sampler with 64 evenly spaced samples looks, so that a sampled threshold
    keeps too few scores."""
    rng = np.random.default_rng(seed)
    S = np.empty((hq, n, n), dtype=np.float32)
    S[0] = rng.standard_normal((n, n))
    S[1] = 1000.0 + 1e-3 * rng.standard_normal((n, n))
    S[2] = rng.standard_normal((n, n)) * 10.0 ** rng.integers(-30, 30, size=(n, n))
    S[3] = rng.choice(np.array([-0.0, 0.0, 1.0, 2.0], dtype=np.float32), size=(n, n))
    S[4] = -0.25
    S[5] = 0.1 * rng.standard_normal((n, n))
    for i in range(1, n):
        S[5, i, ((2 * np.arange(64) + 1) * i) // 128] = 10.0
    return S


@pytest.mark.parametrize("budget", [W.Budget.fraction(1, 20), W.Budget.topk(40), W.Budget.fraction(1, 8)],
                         ids=["frac5", "top40", "frac12.5"])
def test_topk_select_very_long_rows(budget):
    """One sequence of 3300 single-token chunks: rows from 0 to 3299
    candidates through every route (staged, filter, staged after a failed
    filter, global-memory fallback).  Every 5th row and the last 40 rows of
    each head are checked against the oracle's selection, bit for bit; every
    row's length and diagonal are checked."""
    n_tok = 3300
    cu, bounds, sptr = W.make_bounds([n_tok], [[1] * n_tok])
    hq = 6
    prob = api.Problem(cu, bounds, sptr, hq, 1, 128, torch.bfloat16, torch.device("cuda"))
    n = prob.num_chunks
    S = _very_long_row_scores(n, hq, 5)
    plan = api.topk_select(torch.from_numpy(S).cuda(), prob, budget, check=True)
    rows = gpu_rows(plan, hq * n)
    for h in range(hq):
        for i in range(n):
            keep = O.row_budget(i, budget.kind, budget.k, budget.num, budget.den)
            assert len(rows[h * n + i]) == keep + 1 and rows[h * n + i][-1] == i, (h, i)
            if i % 5 and i < n - 40:
                continue
            cand = list(range(i))
            want = sorted(O.select_row([float(S[h, i, j]) for j in cand], cand, keep)) + [i]
            assert rows[h * n + i] == want, (h, i)


@pytest.mark.parametrize("name", CASES)
def test_plan_and_attention(name):
    inp = _case(name)
    q, k, v, prob = to_device(inp)
    b = inp.budget
    plan = api.plan(q, k, prob, b, check=True)
    ref = O.build_plan(inp.q, inp.k, inp.chunk_bounds, inp.seq_chunk_ptr, b.kind, b.k, b.num, b.den)
    rows = gpu_rows(plan, inp.spec.num_q_heads * inp.num_chunks)
    tolerated = compare_plans(rows, ref, inp, b)
    assert len(tolerated) <= max(2, len(rows) // 100)
    out = api.attention(q, k, v, prob, plan, check=True)
    torch.cuda.synchronize()
    want = O.attention_gather(inp.q, inp.k, inp.v, inp.chunk_bounds, plan.row_ptr.cpu().numpy(),
                              plan.col.cpu().numpy())
    stats = attention_gate(out, want, inp.q.dtype)
    print(name, "max_err=%.3g max|O|=%.3g median|O|=%.3g rel_fro=%.3g" % stats)


@pytest.mark.parametrize("name", ["ragged_d128_top2", "ragged_d64_frac", "d256_structured_top3", "d128_many_runs",
                                  "d128_fixed96", "f32_d128_ragged", "d128_group3", "d64_group3", "d256_group3"])
def test_per_kv_head_plan_and_attention(name):
    """Grouped-query mode: one plan row per KV head, scored by the group's
    summed query chunks, equals the oracle's per-KV-head plan (near-tie rule),
    and every query head attends over its group's row."""
    inp = _case(name)
    q, k, v, prob = to_device(inp)
    b = inp.budget.kv()
    plan = api.plan(q, k, prob, b, check=True)
    assert plan.per_kv_head and plan.row_ptr.numel() == inp.spec.num_kv_heads * inp.num_chunks + 1
    ref = O.build_plan(inp.q, inp.k, inp.chunk_bounds, inp.seq_chunk_ptr, b.kind, b.k, b.num, b.den,
                       per_kv_head=True)
    rows = gpu_rows(plan, inp.spec.num_kv_heads * inp.num_chunks)
    tolerated = compare_plans(rows, ref, inp, b)
    assert len(tolerated) <= max(2, len(rows) // 100)
    out = api.attention(q, k, v, prob, plan, check=True)
    torch.cuda.synchronize()
    want = O.attention_gather(inp.q, inp.k, inp.v, inp.chunk_bounds, plan.row_ptr.cpu().numpy(),
                              plan.col.cpu().numpy(), per_kv_head=True)
    stats = attention_gate(out, want, inp.q.dtype)
    print(name, "kv plan: max_err=%.3g max|O|=%.3g" % stats[:2])


def test_dense_budget_matches_sdpa():
    inp = _case("d128_dense")
    q, k, v, prob = to_device(inp)
    plan = api.plan(q, k, prob, inp.budget)
    out = api.attention(q, k, v, prob, plan, check=True).float()
    ref = torch.empty_like(out)
    cu = inp.cu_seqlens
    for bb in range(len(cu) - 1):
        s, e = int(cu[bb]), int(cu[bb + 1])
        qq = q[s:e].float().transpose(0, 1)[None]
        kk = k[s:e].float().transpose(0, 1).repeat_interleave(4, 0)[None]
        vv = v[s:e].float().transpose(0, 1).repeat_interleave(4, 0)[None]
        ref[s:e] = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, is_causal=True)[0].transpose(0, 1)
    assert float((out - ref).abs().max()) <= 2e-2


def test_custom_scale_and_repeat_calls_are_deterministic():
    inp = _case("ragged_d128_top2")
    q, k, v, prob = to_device(inp)
    plan = api.plan(q, k, prob, inp.budget)
    plan2 = api.plan(q, k, prob, inp.budget)
    assert torch.equal(plan.col, plan2.col) and torch.equal(plan.row_ptr, plan2.row_ptr)
    o1 = api.attention(q, k, v, prob, plan, scale=0.05)
    o2 = api.attention(q, k, v, prob, plan, scale=0.05)
    assert torch.equal(o1, o2)
    want = O.attention_gather(inp.q, inp.k, inp.v, inp.chunk_bounds, plan.row_ptr.cpu().numpy(),
                              plan.col.cpu().numpy(), scale=0.05)
    attention_gate(o1, want, torch.bfloat16)


def test_concurrent_calls_on_two_streams():
    """Attention calls overlapping on two streams, each with its own workspace
    (status word and work-item counter of the persistent kernel), give the
    outputs of the same calls run one after the other."""
    cases = [_case("d128_long_runs"), _case("ragged_d128_top2")]
    dev = torch.device("cuda")
    runs = []
    for inp in cases:
        q, k, v, prob = to_device(inp)
        plan = api.plan(q, k, prob, inp.budget, check=True)
        runs.append((q, k, v, prob, plan, api.Attention(prob, dev)))
    serial = []
    for q, k, v, prob, plan, attn in runs:
        out = torch.empty_like(q)
        attn(q, k, v, plan, out)
        serial.append(out)
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = [torch.empty_like(r[0]) for r in runs]
    for rep in range(3):
        for (q, k, v, prob, plan, attn), out, st in zip(runs, outs, streams):
            st.wait_stream(torch.cuda.current_stream())
            attn(q, k, v, plan, out, stream=st)
        torch.cuda.synchronize()
        for (q, k, v, prob, plan, attn), out, ref, st in zip(runs, outs, serial, streams):
            assert attn.status(st) == 0
            assert torch.equal(out, ref), rep


def test_one_shot_calls_on_a_side_stream():
    """The one-shot functions given a side stream order themselves against the
    current stream (inputs, zeroed outputs, and the result's use there) and give
    the same results as on the current stream."""
    inp = _case("d128_long_runs")
    q, k, v, prob = to_device(inp)
    ref_plan = api.plan(q, k, prob, inp.budget, check=True)
    ref_out = api.attention(q, k, v, prob, ref_plan, check=True)
    ref_qc = api.chunk_reduce(q, prob)
    ref_kc = api.chunk_reduce(k, prob)
    ref_s = api.chunk_similarity(ref_qc, ref_kc, prob)
    torch.cuda.synchronize()
    st = torch.cuda.Stream()
    for rep in range(2):
        plan = api.plan(q, k, prob, inp.budget, stream=st, check=True)
        out = api.attention(q, k, v, prob, plan, stream=st, check=True)
        qc = api.chunk_reduce(q, prob, stream=st)
        kc = api.chunk_reduce(k, prob, stream=st)
        sc = api.chunk_similarity(qc, kc, prob, stream=st)
        sel = api.topk_select(sc, prob, inp.budget, stream=st, check=True)
        # used on the current stream without any explicit synchronisation
        assert torch.equal(plan.row_ptr, ref_plan.row_ptr) and torch.equal(plan.col, ref_plan.col), rep
        assert torch.equal(sel.row_ptr, ref_plan.row_ptr) and torch.equal(sel.col, ref_plan.col), rep
        assert torch.equal(out, ref_out), rep
        assert torch.equal(qc, ref_qc) and torch.equal(kc, ref_kc) and torch.equal(sc, ref_s), rep


def test_empty_sequence_in_batch():
    inp = W.random_problem(7, [500, 0, 300], 2, 1, 64, "bf16", 40, 120, W.Budget.topk(2))
    q, k, v, prob = to_device(inp)
    plan = api.plan(q, k, prob, inp.budget, check=True)
    ref = O.build_plan(inp.q, inp.k, inp.chunk_bounds, inp.seq_chunk_ptr, O.TOPK, 2)
    compare_plans(gpu_rows(plan, 2 * inp.num_chunks), ref, inp, inp.budget)
    out = api.attention(q, k, v, prob, plan, check=True)
    want = O.attention_gather(inp.q, inp.k, inp.v, inp.chunk_bounds, plan.row_ptr.cpu().numpy(),
                              plan.col.cpu().numpy())
    attention_gate(out, want, torch.bfloat16)


@pytest.mark.parametrize("d", [128, 256])
def test_v_outside_f16_range_is_reported(d):
    """The bf16 kernels read an f16 copy of V (P V in f16): a V magnitude above
    65504 has no f16 counterpart and is reported (DHSA_ERR_DEVICE_CHECK); the
    next call with a V in range runs clean and correct."""
    inp = W.random_problem(11, [600], 2, 1, d, "bf16", 40, 160, W.Budget.topk(2))
    q, k, v, prob = to_device(inp)
    plan = api.plan(q, k, prob, inp.budget, check=True)
    attn = api.Attention(prob, q.device)
    out = torch.empty_like(q)
    bad = v.clone()
    bad[123, 0, 7] = 1.0e5
    attn(q, k, bad, plan, out)
    torch.cuda.synchronize()
    assert attn.status() == 6
    attn(q, k, v, plan, out)
    torch.cuda.synchronize()
    assert attn.status() == 0
    want = O.attention_gather(inp.q, inp.k, inp.v, inp.chunk_bounds, plan.row_ptr.cpu().numpy(),
                              plan.col.cpu().numpy())
    attention_gate(out, want, torch.bfloat16)


def test_timeout_path_reports_and_context_survives():
    assert api.selftest_timeout(20000) == 5  # DHSA_ERR_TIMEOUT
    inp = _case("d128_diag_only")
    q, k, v, prob = to_device(inp)
    plan = api.plan(q, k, prob, inp.budget, check=True)
    api.attention(q, k, v, prob, plan, check=True)
    torch.cuda.synchronize()
