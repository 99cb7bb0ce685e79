"""Pins for the fp64 oracle: checks against things other than the oracle itself.

Each test fixes the oracle to a fact the pages or the mathematics fix: a worked
example derived by hand, closed forms of the length-normalised aggregation,
brute-force enumeration of the selection, dense causal attention from a library
routine, and metamorphic invariants.  A plausible slip in the oracle (a dropped
sqrt, a wrong sign, a flipped tie rule, a transposed operand, a missing causal
mask) fails at least one of them; ``test_planted_mistakes_are_caught`` checks
that on planted copies of such slips.
"""

import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import dhsa_oracle as O
from dynamic_hierarchical_sparse_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _hand():
    with open(os.path.join(GOLDEN, "hand_example_4chunks.json")) as f:
        ex = json.load(f)
    q = np.asarray(ex["q"], dtype=np.float64)[:, None, :]
    k = np.asarray(ex["k"], dtype=np.float64)[:, None, :]
    v = np.asarray(ex["v"], dtype=np.float64)[:, None, :]
    return ex, q, k, v, np.asarray(ex["chunk_bounds"]), np.asarray([0, 4])


# ------------------------------------------------------------ worked example
def test_hand_example_representations_and_scores():
    ex, q, k, v, bounds, sptr = _hand()
    qc = O.chunk_representations(q, bounds)
    kc = O.chunk_representations(k, bounds)
    np.testing.assert_allclose(qc[0], np.asarray(ex["qc"]), rtol=0, atol=1e-15)
    np.testing.assert_allclose(kc[0], np.asarray(ex["kc"]), rtol=0, atol=1e-15)
    S = O.chunk_scores(qc, kc, sptr)
    for key, val in ex["scores_lower"].items():
        i, j = map(int, key.split(","))
        assert abs(S[0, i, j] - val) < 1e-14, (i, j)
    # never-scored (future) entries stay NaN
    assert np.isnan(S[0, 0, 1]) and np.isnan(S[0, 2, 3])


def test_hand_example_plans():
    ex, q, k, v, bounds, sptr = _hand()
    p = O.build_plan(q, k, bounds, sptr, O.TOPK, 1)
    assert O.plan_rows(p["row_ptr"], p["col"]) == ex["plan_top1"]
    p = O.build_plan(q, k, bounds, sptr, O.FRACTION, num=1, den=2)
    assert O.plan_rows(p["row_ptr"], p["col"]) == ex["plan_fraction_1_2"]


def test_hand_example_attention_closed_form():
    ex, q, k, v, bounds, sptr = _hand()
    p = O.build_plan(q, k, bounds, sptr, O.TOPK, 1)
    out = O.attention_gather(q, k, v, bounds, p["row_ptr"], p["col"], scale=1.0)[:, 0, :]
    e = math.e
    want = np.array([
        [1.0, 0.0],
        np.array([e, e ** 4]) / (e + e ** 4),
        np.array([e + e ** 2, e ** 4 + e ** 2]) / (e + e ** 4 + e ** 2),
        np.array([e ** 2 + 2 / e, 2 * e ** 2]) / (2 * e ** 2 + 1 / e),
        np.array([1.0, e ** 4 + 1 + 2 * e ** 2]) / (e ** 4 + 1 + e ** 2),
        np.array([e ** 4 - e ** -2, 2 * e ** 4 + 2 * e ** 2 + e ** -2]) / (2 * e ** 4 + e ** 2 + e ** -2),
    ])
    np.testing.assert_allclose(out, want, rtol=0, atol=1e-14)
    lit, keep, _ = O.attention_literal(q, k, v, [0, 6], bounds, sptr, p["S"], O.TOPK, 1, scale=1.0)
    np.testing.assert_allclose(lit[:, 0, :], want, rtol=0, atol=1e-14)


# ------------------------------------------------------------- closed forms
def test_equal_length_closed_form():
    """Equal chunk length L: Qc.Kc = L * (mean q . mean k)."""
    rng = np.random.default_rng(3)
    L, n, d = 7, 6, 5
    q = rng.standard_normal((L * n, 2, d))
    k = rng.standard_normal((L * n, 1, d))
    bounds = np.arange(0, L * n + 1, L)
    qc = O.chunk_representations(q, bounds)
    kc = O.chunk_representations(k, bounds)
    S = O.chunk_scores(qc, kc, [0, n])
    for h in range(2):
        for i in range(n):
            for j in range(i + 1):
                mq = q[i * L:(i + 1) * L, h].mean(axis=0)
                mk = k[j * L:(j + 1) * L, 0].mean(axis=0)
                assert abs(S[h, i, j] - L * float(mq @ mk)) < 1e-12


def test_single_token_and_constant_chunks():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((5, 3, 4))
    np.testing.assert_array_equal(O.chunk_representations(x, np.arange(6)).transpose(1, 0, 2), x)
    c = rng.standard_normal(4)
    xs = np.broadcast_to(c, (9, 1, 4)).copy()
    rep = O.chunk_representations(xs, [0, 9])
    np.testing.assert_allclose(rep[0, 0], 3.0 * c, rtol=1e-15, atol=1e-15)  # sqrt(9) * c


def test_row_budget_values():
    assert [O.row_budget(i, O.TOPK, 4) for i in range(7)] == [0, 1, 2, 3, 4, 4, 4]
    # keep 10 %: ceil(i/10) capped at i
    assert [O.row_budget(i, O.FRACTION, num=1, den=10) for i in [0, 1, 9, 10, 11, 20, 21]] == [0, 1, 1, 1, 2, 2, 3]
    assert [O.row_budget(i, O.FRACTION, num=1, den=20) for i in [0, 1, 20, 21, 40, 41]] == [0, 1, 1, 2, 2, 3]
    assert O.row_budget(5, O.FRACTION, num=3, den=2) == 5  # above 100 % caps at i


# --------------------------------------------------------------- brute force
def _brute_select(scores, cands, keep):
    """The unique keep-subset whose every member beats every non-member."""
    def beats(a, b):  # candidate position a ranks before b
        return scores[a] > scores[b] or (scores[a] == scores[b] and cands[a] < cands[b])
    winners = []
    for sub in itertools.combinations(range(len(cands)), keep):
        rest = [t for t in range(len(cands)) if t not in sub]
        if all(beats(a, b) for a in sub for b in rest):
            winners.append(sorted(cands[t] for t in sub))
    assert len(winners) == 1
    return winners[0]


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
@pytest.mark.parametrize("kk", [1, 2, 3, 5])
def test_selection_matches_brute_force(seed, kk):
    rng = np.random.default_rng(seed)
    lens = [3, 1, 4, 2, 5, 1, 3, 2, 4, 2]
    inp = W.explicit_problem(seed, [lens], 2, 1, 8, "f32", W.Budget.topk(kk))
    # force exact ties: chunk 3 and chunk 6 get identical K rows as chunk 1
    k = inp.k.clone()
    b = inp.chunk_bounds
    for dst in (3, 6):
        k[b[dst]:b[dst + 1]] = 0
        k[b[dst]] = k[b[1]] * math.sqrt(b[dst + 1] - b[dst])  # same rep as chunk 1 (length 1)
    p = O.build_plan(inp.q, k, b, inp.seq_chunk_ptr, O.TOPK, kk)
    rows = O.plan_rows(p["row_ptr"], p["col"])
    n = len(lens)
    for h in range(2):
        for i in range(n):
            cands = list(range(i))
            sc = [p["S"][h, i, j] for j in cands]
            keep = min(kk, i)
            want = _brute_select(sc, cands, keep) + [i]
            assert rows[h * n + i] == want


def test_tie_goes_to_lower_index():
    # three identical key chunks, budget 1: the earliest must win
    lens = [2, 2, 2, 2]
    inp = W.explicit_problem(0, [lens], 1, 1, 4, "f32", W.Budget.topk(1))
    k = inp.k.clone()
    k[2:4] = k[0:2]
    k[4:6] = k[0:2]
    q = inp.q.clone()
    q[6:8] = k[0:2].sum(0, keepdim=True) * 5.0  # query aligned with those chunks
    p = O.build_plan(q, k, inp.chunk_bounds, inp.seq_chunk_ptr, O.TOPK, 1)
    assert O.plan_rows(p["row_ptr"], p["col"])[3] == [0, 3]


# ------------------------------------------------- dense-attention reduction
def _sdpa_dense(q, k, v, cu, scale):
    out = torch.zeros(q.shape, dtype=torch.float64)
    Hq, Hkv = q.shape[1], k.shape[1]
    for b in range(len(cu) - 1):
        s, e = int(cu[b]), int(cu[b + 1])
        qq = torch.from_numpy(q[s:e]).transpose(0, 1)[None]
        kk = torch.from_numpy(k[s:e]).transpose(0, 1).repeat_interleave(Hq // Hkv, 0)[None]
        vv = torch.from_numpy(v[s:e]).transpose(0, 1).repeat_interleave(Hq // Hkv, 0)[None]
        o = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, is_causal=True, scale=scale)
        out[s:e] = o[0].transpose(0, 1)
    return out.numpy()


@pytest.mark.parametrize("seed", [0, 1])
def test_full_budget_equals_dense_causal(seed):
    inp = W.random_problem(seed, [97, 160, 33], 4, 2, 16, "f32", 5, 40, W.Budget.topk(10 ** 6))
    q, k, v = (O.as_f64(t) for t in (inp.q, inp.k, inp.v))
    p = O.build_plan(q, k, inp.chunk_bounds, inp.seq_chunk_ptr, O.TOPK, 10 ** 6)
    scale = 1.0 / math.sqrt(16)
    got = O.attention_gather(q, k, v, inp.chunk_bounds, p["row_ptr"], p["col"])
    want = _sdpa_dense(q, k, v, inp.cu_seqlens, scale)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)
    # a fraction of 1/1 keeps everything too
    p2 = O.build_plan(q, k, inp.chunk_bounds, inp.seq_chunk_ptr, O.FRACTION, num=1, den=1)
    assert np.array_equal(p2["col"], p["col"])


def test_single_chunk_sequences_are_causal_attention():
    inp = W.explicit_problem(5, [[40], [25], [63]], 2, 2, 8, "f32", W.Budget.topk(0))
    q, k, v = (O.as_f64(t) for t in (inp.q, inp.k, inp.v))
    p = O.build_plan(q, k, inp.chunk_bounds, inp.seq_chunk_ptr, O.TOPK, 0)
    got = O.attention_gather(q, k, v, inp.chunk_bounds, p["row_ptr"], p["col"])
    np.testing.assert_allclose(got, _sdpa_dense(q, k, v, inp.cu_seqlens, 1 / math.sqrt(8)), atol=1e-12)


# ------------------------------------------------- literal vs chunk-gather
@pytest.mark.parametrize("budget", [W.Budget.topk(2), W.Budget.fraction(1, 3)])
def test_literal_upsampling_equals_gather(budget):
    inp = W.random_problem(7, [150, 90], 2, 1, 8, "f32", 3, 25, budget)
    q, k, v = (O.as_f64(t) for t in (inp.q, inp.k, inp.v))
    p = O.build_plan(q, k, inp.chunk_bounds, inp.seq_chunk_ptr, budget.kind, budget.k, budget.num, budget.den)
    lit, keep, stok = O.attention_literal(q, k, v, inp.cu_seqlens, inp.chunk_bounds, inp.seq_chunk_ptr,
                                          p["S"], budget.kind, budget.k, budget.num, budget.den)
    gat = O.attention_gather(q, k, v, inp.chunk_bounds, p["row_ptr"], p["col"])
    np.testing.assert_allclose(lit, gat, rtol=0, atol=1e-12)
    # the mask is constant on every off-diagonal chunk block and causal on the diagonal
    b = inp.chunk_bounds
    n = len(b) - 1
    for h in range(2):
        for i in range(n):
            for j in range(n):
                blk = keep[h, b[i]:b[i + 1], b[j]:b[j + 1]]
                if j < i:
                    assert blk.all() or (~blk).all()
                elif j == i:
                    assert np.array_equal(blk, np.tril(np.ones_like(blk)))
                else:
                    assert not blk.any()
        # kept pair count agrees with the mask
    assert O.kept_pairs(inp.chunk_bounds, p["row_ptr"], p["col"], 2) == int(keep.sum())


def test_rows_mode_equals_gather():
    inp = W.random_problem(8, [300], 4, 2, 16, "bf16", 20, 60, W.Budget.topk(3), values="structured")
    p = O.build_plan(inp.q, inp.k, inp.chunk_bounds, inp.seq_chunk_ptr, O.TOPK, 3)
    gat = O.attention_gather(inp.q, inp.k, inp.v, inp.chunk_bounds, p["row_ptr"], p["col"])
    rows = [(0, 0), (17, 1), (150, 2), (299, 3), (123, 0)]
    got = O.attention_rows(inp.q, inp.k, inp.v, inp.chunk_bounds, p["row_ptr"], p["col"], rows)
    for idx, (t, h) in enumerate(rows):
        np.testing.assert_allclose(got[idx], gat[t, h], rtol=0, atol=1e-12)


# ---------------------------------------------------------------- metamorphic
def test_permuting_an_offdiagonal_key_chunk():
    inp = W.random_problem(9, [400], 2, 1, 16, "f32", 20, 70, W.Budget.topk(2))
    b = inp.chunk_bounds
    c = 2
    perm = np.arange(inp.q.shape[0])
    perm[b[c]:b[c + 1]] = perm[b[c]:b[c + 1]][::-1]
    k2, v2 = inp.k[perm], inp.v[perm]
    p1 = O.build_plan(inp.q, inp.k, b, inp.seq_chunk_ptr, O.TOPK, 2)
    p2 = O.build_plan(inp.q, k2, b, inp.seq_chunk_ptr, O.TOPK, 2)
    assert np.array_equal(p1["col"], p2["col"])
    o1 = O.attention_gather(inp.q, inp.k, inp.v, b, p1["row_ptr"], p1["col"])
    o2 = O.attention_gather(inp.q, k2, v2, b, p2["row_ptr"], p2["col"])
    later = slice(int(b[c + 1]), None)
    np.testing.assert_allclose(o1[later], o2[later], rtol=0, atol=1e-12)
    assert not np.allclose(o1[b[c]:b[c + 1]], o2[b[c]:b[c + 1]])  # causal order matters inside


def test_scaling_v_scales_output():
    inp = W.random_problem(10, [200], 2, 2, 8, "f32", 10, 40, W.Budget.topk(2))
    p = O.build_plan(inp.q, inp.k, inp.chunk_bounds, inp.seq_chunk_ptr, O.TOPK, 2)
    o1 = O.attention_gather(inp.q, inp.k, inp.v, inp.chunk_bounds, p["row_ptr"], p["col"])
    o2 = O.attention_gather(inp.q, inp.k, 2.5 * O.as_f64(inp.v), inp.chunk_bounds, p["row_ptr"], p["col"])
    np.testing.assert_allclose(o2, 2.5 * o1, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("budget", [W.Budget.topk(3), W.Budget.fraction(1, 4)])
def test_plan_structure(budget):
    inp = W.random_problem(11, [300, 120, 77], 4, 2, 8, "f32", 8, 30, budget)
    p = O.build_plan(inp.q, inp.k, inp.chunk_bounds, inp.seq_chunk_ptr, budget.kind, budget.k,
                     budget.num, budget.den)
    rows = O.plan_rows(p["row_ptr"], p["col"])
    n = inp.num_chunks
    ptr = inp.seq_chunk_ptr
    for r, row in enumerate(rows):
        i = r % n
        b = int(np.searchsorted(ptr, i, side="right") - 1)
        il = i - int(ptr[b])
        assert len(row) == O.row_budget(il, budget.kind, budget.k, budget.num, budget.den) + 1
        assert row == sorted(row) and len(set(row)) == len(row)
        assert row[-1] == i
        assert all(ptr[b] <= j <= i for j in row)


def test_needle_is_selected():
    spec = W.RAGGED_NEEDLE
    inp = W.generate(spec, 0, seq_lens=[1024, 1536])
    p = O.build_plan(inp.q, inp.k, inp.chunk_bounds, inp.seq_chunk_ptr, O.TOPK, 8)
    rows = O.plan_rows(p["row_ptr"], p["col"])
    n = inp.num_chunks
    group = spec.num_q_heads // spec.num_kv_heads
    for b, jstar in enumerate(inp.needle_chunks):
        last = int(inp.seq_chunk_ptr[b + 1]) - 1
        for g in range(spec.num_kv_heads):
            assert jstar in rows[(g * group) * n + last]


# --------------------------------------- grouped-query (per-KV-head) plans
def _kv_problem(seed, hq=4, hkv=2, d=8):
    return W.random_problem(seed, [60, 90], hq, hkv, d, "f32", 4, 14, W.Budget.topk(3))


@pytest.mark.parametrize("seed", [0, 1])
def test_kv_plan_equals_head_plan_without_grouping(seed):
    """With one query head per KV head the group score is the head's score."""
    inp = _kv_problem(seed, hq=2, hkv=2)
    b = inp.chunk_bounds
    p_head = O.build_plan(inp.q, inp.k, b, inp.seq_chunk_ptr, O.TOPK, 3)
    p_kv = O.build_plan(inp.q, inp.k, b, inp.seq_chunk_ptr, O.TOPK, 3, per_kv_head=True)
    assert np.array_equal(p_head["row_ptr"], p_kv["row_ptr"]) and np.array_equal(p_head["col"], p_kv["col"])


@pytest.mark.parametrize("seed", [0, 1])
def test_kv_plan_with_identical_heads_in_a_group(seed):
    """When every query head of a group carries the same Q, the group score is
    the head score times the group size (exact in fp64 for a power of two), so
    the group's row equals each of its heads' rows."""
    inp = _kv_problem(seed, hq=4, hkv=2)
    q = inp.q.clone()
    q[:, 1] = q[:, 0]
    q[:, 3] = q[:, 2]
    b = inp.chunk_bounds
    n = inp.num_chunks
    rows_h = O.plan_rows(**{k: v for k, v in O.build_plan(q, inp.k, b, inp.seq_chunk_ptr, O.TOPK, 3).items()
                            if k in ("row_ptr", "col")})
    rows_g = O.plan_rows(**{k: v for k, v in O.build_plan(q, inp.k, b, inp.seq_chunk_ptr, O.TOPK, 3,
                                                          per_kv_head=True).items() if k in ("row_ptr", "col")})
    assert len(rows_g) == 2 * n
    for h in range(4):
        for i in range(n):
            assert rows_g[(h // 2) * n + i] == rows_h[h * n + i], (h, i)


def test_group_scores_are_the_dot_of_summed_query_chunks():
    """Linearity: the sum over a group's heads of qc[h,i].kc[g,j] equals
    (sum_h qc[h,i]).kc[g,j]; a wrong head-to-group map breaks it."""
    inp = _kv_problem(3, hq=6, hkv=2)
    qc = O.chunk_representations(inp.q, inp.chunk_bounds)
    kc = O.chunk_representations(inp.k, inp.chunk_bounds)
    Sg = O.group_chunk_scores(qc, kc, inp.seq_chunk_ptr)
    summed = qc.reshape(2, 3, qc.shape[1], qc.shape[2]).sum(axis=1)
    want = np.einsum("gid,gjd->gij", summed, kc)
    mask = ~np.isnan(Sg)
    assert mask.sum() > 0 and np.array_equal(mask, ~np.isnan(O.chunk_scores(summed, kc, inp.seq_chunk_ptr)))
    np.testing.assert_allclose(Sg[mask], want[mask], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("kk", [1, 2, 4])
def test_kv_plan_matches_brute_force(kk):
    lens = [3, 1, 4, 2, 5, 1, 3, 2, 4, 2]
    inp = W.explicit_problem(7, [lens], 4, 2, 8, "f32", W.Budget.topk(kk))
    p = O.build_plan(inp.q, inp.k, inp.chunk_bounds, inp.seq_chunk_ptr, O.TOPK, kk, per_kv_head=True)
    rows = O.plan_rows(p["row_ptr"], p["col"])
    qc = O.chunk_representations(inp.q, inp.chunk_bounds)
    kc = O.chunk_representations(inp.k, inp.chunk_bounds)
    n = len(lens)
    for g in range(2):
        for i in range(n):
            cands = list(range(i))
            sc = [float(np.dot(qc[2 * g, i], kc[g, j]) + np.dot(qc[2 * g + 1, i], kc[g, j])) for j in cands]
            assert rows[g * n + i] == _brute_select(sc, cands, min(kk, i)) + [i]


def test_kv_plan_full_budget_equals_dense_causal():
    """Every query head reads its group's row: with all chunks kept this is
    dense causal GQA attention (a wrong row lookup reads another group's or a
    missing row)."""
    inp = W.random_problem(4, [97, 160], 4, 2, 16, "f32", 5, 40, W.Budget.topk(10 ** 6))
    q, k, v = (O.as_f64(t) for t in (inp.q, inp.k, inp.v))
    p = O.build_plan(q, k, inp.chunk_bounds, inp.seq_chunk_ptr, O.TOPK, 10 ** 6, per_kv_head=True)
    assert p["row_ptr"].shape[0] == 2 * inp.num_chunks + 1
    got = O.attention_gather(q, k, v, inp.chunk_bounds, p["row_ptr"], p["col"], per_kv_head=True)
    np.testing.assert_allclose(got, _sdpa_dense(q, k, v, inp.cu_seqlens, 1 / 4.0), rtol=0, atol=1e-12)
    rows = [(int(t), h) for t in (0, 50, 96, 150, 256) for h in range(4)]
    np.testing.assert_allclose(O.attention_rows(q, k, v, inp.chunk_bounds, p["row_ptr"], p["col"], rows,
                                                per_kv_head=True),
                               np.stack([got[t, h] for t, h in rows]), atol=1e-12)
    assert O.kept_pairs(inp.chunk_bounds, p["row_ptr"], p["col"], 4, group=2) == 4 * (97 * 98 + 160 * 161) // 2


def test_kv_plan_sparse_attention_uses_the_group_row():
    """With a sparse per-KV-head plan, head h's output equals per-head
    attention over a plan whose row (h, i) is a copy of row (h // group, i)."""
    inp = _kv_problem(5, hq=4, hkv=2, d=8)
    q, k, v = (O.as_f64(t) for t in (inp.q, inp.k, inp.v))
    b = inp.chunk_bounds
    n = inp.num_chunks
    p = O.build_plan(q, k, b, inp.seq_chunk_ptr, O.TOPK, 2, per_kv_head=True)
    rows = O.plan_rows(p["row_ptr"], p["col"])
    expanded = [rows[(h // 2) * n + i] for h in range(4) for i in range(n)]
    rp = np.cumsum([0] + [len(r) for r in expanded])
    cl = np.asarray([c for r in expanded for c in r])
    got = O.attention_gather(q, k, v, b, p["row_ptr"], p["col"], per_kv_head=True)
    want = O.attention_gather(q, k, v, b, rp, cl)
    np.testing.assert_allclose(got, want, rtol=0, atol=0)


# ------------------------------------------------------ planted-mistake check
def test_planted_mistakes_are_caught(monkeypatch):
    """Each planted slip in the oracle must break at least one pin above."""
    ex, q, k, v, bounds, sptr = _hand()

    def hand_pins_pass():
        try:
            test_hand_example_representations_and_scores()
            test_hand_example_plans()
            test_hand_example_attention_closed_form()
            test_equal_length_closed_form()
            test_tie_goes_to_lower_index()
            test_single_chunk_sequences_are_causal_attention()
            return True
        except AssertionError:
            return False

    assert hand_pins_pass()
    real_reps = O.chunk_representations
    real_select = O.select_row
    real_softmax = O._softmax_rows

    # 1) mean instead of mean*sqrt(L)
    def reps_mean(x, b):
        r = real_reps(x, b)
        lens = np.diff(np.asarray(b))
        return r / np.sqrt(lens)[None, :, None]
    monkeypatch.setattr(O, "chunk_representations", reps_mean)
    assert not hand_pins_pass()
    monkeypatch.setattr(O, "chunk_representations", real_reps)

    # 2) tie to the higher index
    def select_hi(scores, cands, keep):
        order = sorted(range(len(cands)), key=lambda t: (-scores[t], -cands[t]))
        return [int(cands[t]) for t in order[:keep]]
    monkeypatch.setattr(O, "select_row", select_hi)
    assert not hand_pins_pass()
    monkeypatch.setattr(O, "select_row", real_select)

    # 3) ascending scores (wrong sign)
    def select_low(scores, cands, keep):
        order = sorted(range(len(cands)), key=lambda t: (scores[t], cands[t]))
        return [int(cands[t]) for t in order[:keep]]
    monkeypatch.setattr(O, "select_row", select_low)
    assert not hand_pins_pass()
    monkeypatch.setattr(O, "select_row", real_select)

    # 5) group scores summing the wrong heads (h % Hkv instead of h // group)
    real_group = O.group_chunk_scores

    def group_wrong(qc, kc, ptr):
        S = O.chunk_scores(qc, kc, ptr)
        Hkv = kc.shape[0]
        out = np.zeros((Hkv,) + S.shape[1:])
        for h in range(qc.shape[0]):
            out[h % Hkv] += S[h]
        return out
    monkeypatch.setattr(O, "group_chunk_scores", group_wrong)
    with pytest.raises(AssertionError):
        test_group_scores_are_the_dot_of_summed_query_chunks()
    monkeypatch.setattr(O, "group_chunk_scores", real_group)

    # 4) softmax without the max shift AND a dropped normaliser
    monkeypatch.setattr(O, "_softmax_rows", lambda lg: np.exp(lg))
    assert not hand_pins_pass()
    monkeypatch.setattr(O, "_softmax_rows", real_softmax)
    assert hand_pins_pass()
