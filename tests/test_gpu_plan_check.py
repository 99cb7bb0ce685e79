"""Device-side plan validation (dhsa_plan_check) through the C ABI.

Plans from dhsa_plan pass.  Malformed plans, built on the host from a valid
one, are handed only to the check kernel (never to an attention kernel), and
each kind is reported as DHSA_ERR_DEVICE_CHECK: an entry outside the chunk
range, a row out of order, a row whose last entry is not its diagonal chunk,
a later chunk (not causally admissible), a chunk of another sequence, and row
offsets that decrease, do not start at 0 or do not end at nnz."""

import numpy as np
import pytest
import torch

from dynamic_hierarchical_sparse_b200 import api, workloads as W

pytestmark = pytest.mark.gpu

DEVICE_CHECK = 6


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    api.lib()


@pytest.fixture(scope="module")
def case():
    inp = W.random_problem(21, [1200, 900], 4, 2, 64, "bf16", 30, 120, W.Budget.topk(3))
    dev = torch.device("cuda")
    q, k = inp.q.to(dev), inp.k.to(dev)
    prob = api.Problem.from_inputs(inp, dev)
    plan = api.plan(q, k, prob, inp.budget, check=True)
    kv_plan = api.plan(q, k, prob, inp.budget.kv(), check=True)
    return inp, prob, plan, kv_plan


def _rows(plan):
    return plan.row_ptr.cpu().numpy().astype(np.int64), plan.col.cpu().numpy().astype(np.int64)


def _check(prob, rp, cl, per_kv_head=False):
    dev = torch.device("cuda")
    return api.check_plan(prob, torch.from_numpy(np.asarray(rp, dtype=np.int32)).to(dev),
                          torch.from_numpy(np.asarray(cl, dtype=np.int32)).to(dev), per_kv_head)


def _row_with(rp, cl, n, pred):
    """First row r (and its entries) whose entries satisfy pred(i, entries)."""
    for r in range(rp.shape[0] - 1):
        e = cl[rp[r]:rp[r + 1]]
        if pred(r % n, e):
            return r, int(rp[r])
    raise AssertionError("no such row")


def test_valid_plans_pass(case):
    inp, prob, plan, kv_plan = case
    assert _check(prob, *_rows(plan)) == 0
    assert _check(prob, *_rows(kv_plan), per_kv_head=True) == 0


def test_each_kind_of_malformed_plan_is_reported(case):
    inp, prob, plan, _ = case
    n = prob.num_chunks
    ptr = inp.seq_chunk_ptr
    rp, cl = _rows(plan)
    bad = {}
    # an entry past the last chunk, and a negative one
    c = cl.copy()
    r, p0 = _row_with(rp, cl, n, lambda i, e: len(e) >= 2)
    c[p0] = n
    bad["index_past_range"] = (rp, c)
    c = cl.copy()
    c[p0] = -1
    bad["negative_index"] = (rp, c)
    # two entries swapped: not ascending
    c = cl.copy()
    r, p0 = _row_with(rp, cl, n, lambda i, e: len(e) >= 3)
    c[p0], c[p0 + 1] = cl[p0 + 1], cl[p0]
    bad["not_ascending"] = (rp, c)
    # last entry is not the diagonal (still ascending)
    c = cl.copy()
    r, p0 = _row_with(rp, cl, n, lambda i, e: len(e) >= 2 and e[-2] + 1 < e[-1])
    c[rp[r + 1] - 1] = cl[rp[r + 1] - 2] + 1
    bad["diagonal_missing"] = (rp, c)
    # a later chunk of the same sequence
    c = cl.copy()
    last_of_seq0 = int(ptr[1]) - 1
    r, p0 = _row_with(rp, cl, n, lambda i, e: len(e) >= 2 and i + 1 <= last_of_seq0)
    c[rp[r + 1] - 1] = r % n + 1
    bad["later_chunk"] = (rp, c)
    # a chunk of the previous sequence in a row of the second sequence
    c = cl.copy()
    r, p0 = _row_with(rp, cl, n, lambda i, e: i >= int(ptr[1]) and len(e) >= 2 and e[0] > 0)
    c[p0] = int(ptr[1]) - 1
    bad["other_sequence"] = (rp, c)
    # row offsets: a decrease, a non-zero start, an end short of nnz
    q = rp.copy()
    q[5] = q[4] - 1
    bad["row_ptr_decreasing"] = (q, cl)
    q = rp.copy()
    q[0] = 1
    bad["row_ptr_start"] = (q, cl)
    q = rp.copy()
    q[-1] = q[-1] - 1
    bad["row_ptr_end"] = (q, cl)
    q = rp.copy()
    q[7] = q[6]  # an empty row: no diagonal
    bad["empty_row"] = (q, cl)
    for name, (q, c) in bad.items():
        assert _check(prob, q, c) == DEVICE_CHECK, name
    # the check leaves nothing behind: a valid plan passes again afterwards
    assert _check(prob, rp, cl) == 0
