"""The near-tie rule that the GPU plan comparisons apply (tests/helpers.py::
compare_plans), on a hand-built plan on the CPU: a differing row passes only
at a near tie of the k-th and (k+1)-th scores, and only as a valid selection."""

from types import SimpleNamespace

import numpy as np
import pytest

from oracle import dhsa_oracle as O
from tests.helpers import compare_plans

# One head, one sequence of five chunks, top-2 + diagonal.  Rows 0-2 keep every
# earlier chunk.  Row 3 scores chunks 0..2 at (3, 2, 1): keeps {0, 1}, no tie.
# Row 4 scores chunks 0..3 at (10, 5, 5 + 1e-7, 1): keeps {0, 2}; its 2nd and
# 3rd scores are within 1e-5 of the row's largest |score| (10), a near tie.
ROWS = [[0], [0, 1], [0, 1, 2], [0, 1, 3], [0, 2, 4]]
S = np.full((1, 5, 5), np.nan)
S[0, 3, :3] = [3.0, 2.0, 1.0]
S[0, 4, :4] = [10.0, 5.0, 5.0 + 1e-7, 1.0]
S[0, 1, 0] = 0.5
S[0, 2, :2] = [0.25, 0.75]
KTH = np.array([[np.nan, np.nan], [np.nan, np.nan], [np.nan, np.nan], [2.0, 1.0], [5.0 + 1e-7, 5.0]])
REF = {"row_ptr": np.cumsum([0] + [len(r) for r in ROWS]), "col": np.concatenate(ROWS), "S": S, "kth": KTH,
       "rowmax": np.array([0.0, 0.5, 0.75, 3.0, 10.0])}
INP = SimpleNamespace(num_chunks=5, seq_chunk_ptr=np.array([0, 5]))
BUDGET = SimpleNamespace(kind=O.TOPK, k=2, num=0, den=1)


def test_the_hand_built_plan_is_the_oracle_rule():
    for i in range(3, 5):
        keep = O.row_budget(i, O.TOPK, 2)
        assert sorted(O.select_row(list(S[0, i, :i]), list(range(i)), keep)) == ROWS[i][:-1]


def test_identical_plans_and_the_other_tied_chunk_pass():
    assert compare_plans([list(r) for r in ROWS], REF, INP, BUDGET) == []
    swapped = [list(r) for r in ROWS]
    swapped[4] = [0, 1, 4]  # chunk 1 for chunk 2: the near tie
    assert compare_plans(swapped, REF, INP, BUDGET) == [4]


@pytest.mark.parametrize("row,bad", [
    (3, [0, 2, 3]),     # no near tie in row 3
    (4, [1, 2, 4]),     # the tied pair kept, the clear top chunk 0 dropped
    (4, [0, 3, 4]),     # chunk 3 scores far below the threshold
    (4, [0, 2, 4, 4]),  # not a set
    (4, [0, 2]),        # diagonal missing
])
def test_invalid_rows_fail(row, bad):
    rows = [list(r) for r in ROWS]
    rows[row] = bad
    with pytest.raises(AssertionError):
        compare_plans(rows, REF, INP, BUDGET)
