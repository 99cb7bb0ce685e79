"""Pins for the oracle's online chunking step (``segment``).

The pages say that DHSA segments each sequence into variable-length chunks
adaptively and online, but give no rule.  The oracle states one: with the
current chunk starting at token b, token t starts a new chunk when
t - b >= max_len, or when t - b >= min_len and the mean over KV heads of
cos(k[t-1], k[t]) is below the threshold (a zero key has cosine 1).

These tests fix that rule from outside the oracle: a worked example whose
cosines are exact ratios of small integers, closed forms at thresholds that
every or no cosine passes, planted segments that the rule must recover, the
cosine of a library routine, and invariants of the walk.  Planted slips (an
off-by-one pairing, a non-strict comparison, max instead of mean over heads,
zero keys counted as orthogonal, an off-by-one length test) each fail one.
"""

import numpy as np
import pytest
import torch

from oracle import dhsa_oracle as O
from dynamic_hierarchical_sparse_b200 import workloads as W

# Worked example, Hkv = 2, d = 2, threshold 0.6, min_len 2, max_len 4.
# Sequence A (tokens 0..11) has the same key in both heads; the comment on each
# token gives cos(k[t-1], k[t]) and the decision with the current chunk start b.
_A = [
    (1, 0),     # t0   sequence start
    (0, 1),     # t1   cos 0 < 0.6, but t - b = 1 < min_len: no break
    (0, 1),     # t2   cos 1
    (1, 0),     # t3   cos 0, t - b = 3: break (b = 3)
    (1, 0),     # t4   cos 1
    (3, 4),     # t5   cos 3/5 = 0.6, equal to the threshold: no break (strict)
    (4, 3),     # t6   cos 24/25
    (4, 3),     # t7   cos 1, t - b = 4 = max_len: forced break (b = 7)
    (-4, -3),   # t8   cos -1, t - b = 1: no break
    (-4, -3),   # t9   cos 1
    (-4, -3),   # t10  cos 1
    (-4, -3),   # t11  cos 1, t - b = 4: forced break (b = 11)
]
# Sequence B (tokens 12..21), heads differ: (head 0, head 1), mean of the cosines.
_B = [
    ((1, 0), (1, 0)),     # t12  sequence start
    ((1, 0), (1, 0)),     # t13  mean 1
    ((1, 0), (0, 1)),     # t14  (1 + 0)/2 = 0.5, t - b = 2: break (b = 14)
    ((1, 0), (0, 1)),     # t15  mean 1
    ((1, 0), (24, 7)),    # t16  (1 + 7/25)/2 = 0.64: no break (the minimum, 0.28, would break)
    ((-1, 0), (24, 7)),   # t17  (-1 + 1)/2 = 0, t - b = 3: break (b = 17)
    ((0, 0), (-24, -7)),  # t18  (1 + -1)/2 = 0 (zero key: cosine 1), t - b = 1: no break
    ((0, 0), (0, -1)),    # t19  (1 + 7/25)/2 = 0.64: no break (a zero key at cosine 0 would give 0.14)
    ((1, 0), (0, 1)),     # t20  (1 + -1)/2 = 0, t - b = 3: break (b = 20); NaN for zero keys would not
    ((1, 0), (0, 1)),     # t21  mean 1
]
# Sequence C is empty; sequence D is the single token 22.
_D = [((2, 0), (0, 2))]
HAND_BOUNDS = [0, 3, 7, 11, 12, 14, 17, 20, 22, 23]
HAND_SEQ_PTR = [0, 4, 8, 8, 9]
HAND_CU = [0, 12, 22, 22, 23]
HAND_RULE = (0.6, 2, 4)


def _hand_keys():
    rows = [(a, a) for a in _A] + _B + _D
    return np.asarray(rows, dtype=np.float64)  # [T, 2, 2]


def test_hand_example():
    b, p = O.segment(_hand_keys(), HAND_CU, *HAND_RULE)
    assert b.tolist() == HAND_BOUNDS
    assert p.tolist() == HAND_SEQ_PTR


def test_hand_example_similarities():
    sim = O.adjacent_key_similarity(_hand_keys())
    assert np.isnan(sim[0])
    want = {1: 0.0, 2: 1.0, 3: 0.0, 5: 0.6, 6: 0.96, 8: -1.0, 14: 0.5, 16: 0.64, 17: 0.0, 18: 0.0,
            19: 0.64, 20: 0.0}
    for t, v in want.items():
        assert sim[t] == pytest.approx(v, abs=1e-15), t
    assert sim[5] == 0.6  # 15/25 rounds to the same double as the literal


@pytest.mark.parametrize("seed", [0, 1])
def test_thresholds_that_no_or_every_cosine_passes(seed):
    """Threshold below -1: only max_len breaks (fixed-length chunks, the
    block-sparse special case).  Threshold above 1: every chunk is min_len."""
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((900, 3, 16))
    cu = [0, 1, 400, 400, 900]
    for thr, step in ((-2.0, 37), (2.0, 11)):
        b, p = O.segment(k, cu, thr, 11, 37)
        want, ptr = [], [0]
        for s0, s1 in zip(cu[:-1], cu[1:]):
            want += list(range(s0, s1, step))
            ptr.append(len(want))
        assert b.tolist() == want + [900]
        assert p.tolist() == ptr


@pytest.mark.parametrize("d,hkv", [(64, 1), (128, 8)])
def test_planted_segments_are_recovered(d, hkv):
    k, cu, bounds, ptr = W.planted_segment_keys(3, [3000, 17, 0, 5000], hkv, d, 128, 512)
    b, p = O.segment(k, cu, 0.5, 128, 512)
    assert np.array_equal(b, bounds)
    assert np.array_equal(p, ptr)


def test_similarity_is_the_library_cosine():
    k = torch.randn(300, 4, 32, generator=torch.Generator().manual_seed(5), dtype=torch.float64)
    lib = torch.nn.functional.cosine_similarity(k[:-1], k[1:], dim=-1, eps=0.0).mean(dim=1).numpy()
    sim = O.adjacent_key_similarity(k)
    np.testing.assert_allclose(sim[1:], lib, rtol=0, atol=1e-14)


def test_walk_invariants_on_drifting_keys():
    k = W.drifting_keys(2, 6000, 4, 64, rho=0.9)
    cu = [0, 2500, 2501, 6000]
    thr, lo, hi = 0.9, 16, 96
    sim = O.adjacent_key_similarity(k)
    b, p = O.segment(k, cu, thr, lo, hi)
    assert p[0] == 0 and p[-1] == len(b) - 1 and b[-1] == cu[-1]
    for s in range(len(cu) - 1):
        starts = b[p[s]:p[s + 1]].tolist()
        ends = starts[1:] + [cu[s + 1]]
        assert starts[0] == cu[s]
        for c0, c1 in zip(starts, ends):
            assert c1 - c0 <= hi
            # no break was due strictly inside the chunk
            assert not any(sim[t] < thr for t in range(c0 + lo, c1))
            if c1 < cu[s + 1]:
                assert c1 - c0 >= lo
                assert c1 - c0 == hi or sim[c1] < thr
    # the stress input really does decide close to the threshold
    assert np.nanmin(np.abs(sim - thr)) < 1e-3


def test_planted_mistakes_are_caught(monkeypatch):
    real_sim = O.adjacent_key_similarity
    real_seq = O.segment_sequence

    def fails():
        try:
            test_hand_example()
            return False
        except AssertionError:
            return True

    assert not fails()

    # 1) pairing t with t + 1 instead of t - 1
    monkeypatch.setattr(O, "adjacent_key_similarity", lambda k: np.roll(real_sim(k), -1))
    assert fails()
    # 2) max over heads instead of the mean
    def sim_max(k):
        K = O.as_f64(k)
        out = np.full(K.shape[0], np.nan)
        for t in range(1, K.shape[0]):
            c = []
            for g in range(K.shape[1]):
                den = np.linalg.norm(K[t - 1, g]) * np.linalg.norm(K[t, g])
                c.append(1.0 if den == 0 else float(K[t - 1, g] @ K[t, g]) / den)
            out[t] = max(c)
        return out
    monkeypatch.setattr(O, "adjacent_key_similarity", sim_max)
    assert fails()
    # 3) zero keys counted as orthogonal (cosine 0)
    def sim_zero_orth(k):
        K = O.as_f64(k)
        s = real_sim(k)
        n = np.linalg.norm(K, axis=-1)
        for t in range(1, K.shape[0]):
            zero = (n[t - 1] == 0) | (n[t] == 0)
            if zero.any():
                c = [0.0 if zero[g] else float(K[t - 1, g] @ K[t, g]) / (n[t - 1, g] * n[t, g])
                     for g in range(K.shape[1])]
                s[t] = np.mean(c)
        return s
    monkeypatch.setattr(O, "adjacent_key_similarity", sim_zero_orth)
    assert fails()
    monkeypatch.setattr(O, "adjacent_key_similarity", real_sim)

    # 4) non-strict comparison with the threshold
    def seq_le(sim, start, end, thr, lo, hi):
        return real_seq(sim, start, end, np.nextafter(thr, np.inf), lo, hi)
    monkeypatch.setattr(O, "segment_sequence", seq_le)
    assert fails()
    # 5) the minimum length tested with > instead of >=
    monkeypatch.setattr(O, "segment_sequence", lambda sim, s, e, thr, lo, hi: real_seq(sim, s, e, thr, lo + 1, hi))
    assert fails()
    monkeypatch.setattr(O, "segment_sequence", real_seq)
    assert not fails()
