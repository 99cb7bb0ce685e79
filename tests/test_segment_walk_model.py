"""The online-chunking walk's algorithm (tests/segment_walk_model.py, a
restatement of segment_walk_kernel) against the oracle's rule, on the CPU:
random drop patterns, shrunken windows (so that the walk leaves them), small
node caps (the step-by-step route) and small start buffers."""

import os
import random
import re

import numpy as np
import pytest

import segment_walk_model as M
from oracle import dhsa_oracle as O


def _oracle_starts(drops, s0, s1, min_len, max_len):
    sim = np.full(s1, 1.0)
    sim[list(drops)] = 0.0
    return O.segment_sequence(sim, s0, s1, 0.5, min_len, max_len)


def test_random_patterns_match_the_rule():
    rng = random.Random(5)
    for trial in range(500):
        T = rng.choice([1, 2, 31, 33, 100, 1000, 5000])
        s0 = rng.choice([0, 0, 5, 37]) if T > 40 else 0
        if T <= s0:
            continue
        min_len = rng.choice([1, 2, 3, 8, 16, 50, 256])
        max_len = min_len + rng.choice([0, 0, 1, 5, 31, 100, 1000])
        dens = rng.choice([0.0, 0.001, 0.01, 0.1, 0.5, 1.0])
        drops = [t for t in range(s0 + 1, T) if rng.random() < dens]
        win = rng.choice([64, 128, 4096])
        if (max_len + 29) // 32 + 1 + 4 > win:  # the kernel's window always holds one rule interval
            win = 4096
        got = M.run(drops, s0, T, min_len, max_len, win_words=win, node_cap=rng.choice([8, 64, 8192]),
                    start_buf=rng.choice([1, 3, 1024]), rng=rng)
        assert got == _oracle_starts(drops, s0, T, min_len, max_len), (trial, T, s0, min_len, max_len, dens, win)


@pytest.mark.parametrize("case", ["no_drops", "every_token", "equal_lengths", "long_forced_run_across_windows"])
def test_edge_patterns(case):
    rng = random.Random(1)
    if case == "no_drops":
        args = ([], 0, 20000, 256, 1000)
    elif case == "every_token":
        args = (list(range(1, 3000)), 0, 3000, 7, 40)
    elif case == "equal_lengths":
        args = ([t for t in range(1, 4000) if t % 13 == 0], 0, 4000, 64, 64)
    else:
        args = ([5, 6, 7] + list(range(15000, 15010)), 0, 20000, 32, 96)
    drops, s0, s1, min_len, max_len = args
    for win in (64, 4096):
        got = M.run(drops, s0, s1, min_len, max_len, win_words=win, rng=rng)
        assert got == _oracle_starts(drops, s0, s1, min_len, max_len)


def test_model_matches_the_kernel_source():
    src = open(os.path.join(os.path.dirname(__file__), "..", "dynamic_hierarchical_sparse_b200", "csrc",
                            "segment.cu")).read()
    assert re.search(r"constexpr int kWinWords = 4096;", src)
    assert re.search(r"constexpr int kNodeCap = 8192;", src)
    assert re.search(r"constexpr int kStartBuf = 1024;", src)
    # the closed forms of forced runs and the empty interval of min_len == max_len
    assert "const int k = (f - x) / max_len;" in src
    assert "const int k = max(1, static_cast<int>(room / max_len) - 1);" in src
    assert "(static_cast<long long>(s1) - 1 - x) / max_len" in src
    assert src.count("if (clo < chi) {") == 2
    # pointer jumping runs while the span is at most the number of drops
    assert "for (int span = 1; span <= nodes; span <<= 1) {" in src
