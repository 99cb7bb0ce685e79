"""Selection margins of a plan (dhsa_plan_margins) through the C ABI.

For every plan row the library reports the smallest kept score (the k-th
largest admissible one) and the largest score left out (the (k+1)-th).  They
are min / max over the GPU's own fp32 scores, so they must equal, bit for bit,
the same min / max taken on the host over the scores that the library's
similarity kernel gives for the same inputs; they must agree with the oracle's
k-th and (k+1)-th scores within the fp32 score error; the first must never be
below the second (the selection keeps the largest); and NaN marks exactly the
rows that keep nothing or leave nothing out."""

import numpy as np
import pytest
import torch

from dynamic_hierarchical_sparse_b200 import api
from oracle import dhsa_oracle as O
from tests import test_gpu_parity as TP

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    api.lib()


@pytest.mark.parametrize("name", ["ragged_d128_top2", "d128_long_runs", "d128_dense", "d128_diag_only",
                                  "d64_many_runs", "d128_group3"])
def test_margins_match_the_scores(name):
    inp = TP._case(name)
    q, k, v, prob = TP.to_device(inp)
    b = inp.budget
    planner = api.Planner(prob, b)
    plan = planner(q, k)
    m = planner.margins()
    torch.cuda.synchronize()
    assert planner.status() == 0
    m = m.double().cpu().numpy()
    # the same fp32 scores through the library's own steps 1-2
    S = api.chunk_similarity(api.chunk_reduce(q, prob), api.chunk_reduce(k, prob), prob).double().cpu().numpy()
    rp, cl = plan.row_ptr.cpu().numpy(), plan.col.cpu().numpy()
    n = prob.num_chunks
    ptr = inp.seq_chunk_ptr
    ref = O.build_plan(inp.q, inp.k, inp.chunk_bounds, inp.seq_chunk_ptr, b.kind, b.k, b.num, b.den)
    for r in range(rp.shape[0] - 1):
        h, i = r // n, r % n
        c0 = int(ptr[np.searchsorted(ptr, i, side="right") - 1])
        kept = [int(j) for j in cl[rp[r]:rp[r + 1] - 1]]
        left = [j for j in range(c0, i) if j not in set(kept)]
        want0 = min(S[h, i, j] for j in kept) if kept else np.nan
        want1 = max(S[h, i, j] for j in left) if left else np.nan
        assert (np.isnan(m[r, 0]) and np.isnan(want0)) or m[r, 0] == want0, (r, m[r], want0)
        assert (np.isnan(m[r, 1]) and np.isnan(want1)) or m[r, 1] == want1, (r, m[r], want1)
        if kept and left:
            assert m[r, 0] >= m[r, 1], r
        # the oracle's k-th and (k+1)-th scores (fp64), within the fp32 score error
        scale = max(ref["rowmax"][r], 1e-30)
        for c in (0, 1):
            o = ref["kth"][r, c]
            assert np.isnan(o) == np.isnan(m[r, c]), (r, c)
            if not np.isnan(o):
                assert abs(m[r, c] - o) <= 1e-4 * scale, (r, c, m[r, c], o)


def test_margins_of_a_per_kv_head_plan():
    inp = TP._case("d128_group3")
    q, k, v, prob = TP.to_device(inp)
    b = inp.budget.kv()
    planner = api.Planner(prob, b)
    planner(q, k)
    m = planner.margins().double().cpu().numpy()
    torch.cuda.synchronize()
    ref = O.build_plan(inp.q, inp.k, inp.chunk_bounds, inp.seq_chunk_ptr, b.kind, b.k, b.num, b.den,
                       per_kv_head=True)
    assert m.shape == ref["kth"].shape
    assert np.array_equal(np.isnan(m), np.isnan(ref["kth"]))
    ok = ~np.isnan(m)
    scale = np.maximum(ref["rowmax"], 1e-30)[:, None].repeat(2, axis=1)
    assert np.all(np.abs(m[ok] - ref["kth"][ok]) <= 1e-4 * scale[ok])
    both = ok.all(axis=1)
    assert np.all(m[both, 0] >= m[both, 1])
