"""dhsa_plan_noalloc: the planning step for callers that cannot allocate device
memory (for instance code handed only its input and output buffers, or running
where allocations belong to a pool it does not own).  Its scratch is a fixed
array inside the library, so these tests check, through the C ABI, that it
returns exactly what dhsa_plan returns with a caller workspace, on two calls in
a row that reuse that array, and that a problem too large for it is refused.

This file is collected last on purpose: it also passes when run on its own in a
fresh process."""

import ctypes

import numpy as np
import pytest
import torch

from dynamic_hierarchical_sparse_b200 import api, workloads as W

pytestmark = pytest.mark.gpu

MAX_SCRATCH = 16 << 20  # DHSA_PLAN_NOALLOC_MAX_SCRATCH


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    api.lib()


def _noalloc(q, k, prob, budget, nnz):
    dev = q.device
    heads = prob.num_kv_heads if budget.per_kv_head else prob.num_q_heads
    row_ptr = torch.full((heads * prob.num_chunks + 1,), -1, dtype=torch.int32, device=dev)
    col = torch.full((max(nnz, 1),), -1, dtype=torch.int32, device=dev)
    rc = api.lib().dhsa_plan_noalloc(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), prob.ref(),
                                     api._budget(budget), ctypes.c_void_p(row_ptr.data_ptr()),
                                     ctypes.c_void_p(col.data_ptr()), nnz,
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, api.STATUS_NAMES.get(rc, rc)
    return row_ptr, col[:nnz]


def _case(i):
    if i == 0:
        return W.random_problem(11, [3000, 700], 8, 2, 128, "bf16", 40, 200, W.Budget.topk(4), "structured")
    return W.random_problem(12, [2048], 4, 4, 64, "f32", 16, 96, W.Budget.fraction(1, 5))


def test_noalloc_matches_workspace_plan_on_consecutive_calls():
    dev = torch.device("cuda")
    inputs = [_case(0), _case(1)]
    for rep in range(2):  # second pass reuses the scratch the first pass left behind
        for inp in inputs:
            q, k = inp.q.to(dev), inp.k.to(dev)
            prob = api.Problem.from_inputs(inp, dev)
            ws_bytes = prob.plan_workspace_bytes(inp.budget)
            assert ws_bytes <= MAX_SCRATCH
            want = api.plan(q, k, prob, inp.budget, check=True)
            row_ptr, col = _noalloc(q, k, prob, inp.budget, want.nnz)
            torch.cuda.synchronize()
            assert torch.equal(row_ptr, want.row_ptr), (rep, inp.spec.dtype)
            assert torch.equal(col, want.col), (rep, inp.spec.dtype)


def test_noalloc_per_kv_head_plan_on_consecutive_calls():
    """The per-KV-head layout of the fixed scratch (it adds the summed query
    chunks and moves the score matrix) gives dhsa_plan's per-KV-head plan, bit
    for bit, on consecutive calls, also after a per-query-head call has left
    the differently laid out scratch behind."""
    dev = torch.device("cuda")
    inp = _case(0)
    q, k = inp.q.to(dev), inp.k.to(dev)
    prob = api.Problem.from_inputs(inp, dev)
    per_q, per_kv = inp.budget, inp.budget.kv()
    assert prob.plan_workspace_bytes(per_kv) <= MAX_SCRATCH
    want_kv = api.plan(q, k, prob, per_kv, check=True)
    want_q = api.plan(q, k, prob, per_q, check=True)
    assert want_kv.row_ptr.numel() == prob.num_kv_heads * prob.num_chunks + 1
    for rep in range(2):
        row_ptr, col = _noalloc(q, k, prob, per_kv, want_kv.nnz)
        torch.cuda.synchronize()
        assert torch.equal(row_ptr, want_kv.row_ptr), rep
        assert torch.equal(col, want_kv.col), rep
        row_ptr, col = _noalloc(q, k, prob, per_q, want_q.nnz)
        torch.cuda.synchronize()
        assert torch.equal(row_ptr, want_q.row_ptr) and torch.equal(col, want_q.col), rep


def test_noalloc_rejects_problems_beyond_its_scratch():
    # 32 heads x 1100 chunks: the score matrix alone is 155 MB > 16 MiB
    lens = [[16] * 1100]
    inp = W.explicit_problem(0, lens, 32, 8, 128, "bf16", W.Budget.topk(2))
    prob = api.Problem.from_inputs(inp, torch.device("cuda"))
    assert prob.plan_workspace_bytes(inp.budget) > MAX_SCRATCH
    nnz = prob.nnz(inp.budget)
    null = ctypes.c_void_p(16)
    rc = api.lib().dhsa_plan_noalloc(null, null, prob.ref(), api._budget(inp.budget), null, null, nnz,
                                     ctypes.c_void_p(0))
    assert rc == 3  # DHSA_ERR_WORKSPACE, returned before any launch
