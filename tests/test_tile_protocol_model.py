"""Model check of the d = 256 attention kernel's synchronisation protocol
(csrc/attention_bf16.cu) on the CPU; see tests/tile_protocol_model.py."""

import dataclasses
import os
import random
import re

import pytest

import tile_protocol_model as TM


def test_random_tile_counts_and_schedules():
    for seed in range(400):
        rng = random.Random(seed)
        TM.TileModel(rng.randint(1, 14), rng=rng, rescale_prob=rng.random()).run()


@pytest.mark.parametrize("nt", [1, 2, 3, 4, 17])
def test_edge_tile_counts(nt):
    for seed in range(40):
        for p in (0.0, 1.0):
            TM.TileModel(nt, rng=random.Random(seed), rescale_prob=p).run()


@pytest.mark.parametrize("slip", [f.name for f in dataclasses.fields(TM.TileMutation)])
def test_planted_protocol_slips_are_caught(slip):
    mut = TM.TileMutation(**{slip: True})
    for seed in range(300):
        rng = random.Random(seed)
        try:
            TM.TileModel(rng.randint(3, 10), mut=mut, rng=rng).run()
        except TM.ProtocolViolation:
            return
    pytest.fail("slip %s not caught in 300 schedules" % slip)


def test_s_free_barrier_is_implied_by_p_full():
    """The issuing thread waits for P(j) (written by every warp after it read
    S(j)) before PV(j) and S(j+2), so the S-free wait never decides anything:
    the protocol stays correct without it."""
    for seed in range(300):
        rng = random.Random(seed)
        TM.TileModel(rng.randint(1, 12), rng=rng, variant=TM.TileVariant(no_sfree_wait=True)).run()


def test_model_matches_the_kernel_source():
    src = open(os.path.join(os.path.dirname(__file__), "..", "dynamic_hierarchical_sparse_b200", "csrc",
                            "attention_bf16.cu")).read()
    counts = dict(re.findall(r"mbar_init\(bar\((kBar\w+)(?: \+ s)?\), (\w+)\)", src))
    assert counts["kBarSFree"] == "kBM" and counts["kBarPFull"] == "kBM"  # one arrival per softmax thread
    for name in ("kBarQ", "kBarKFull", "kBarKEmpty", "kBarVFull", "kBarVEmpty", "kBarSFull", "kBarOReady"):
        assert counts[name] == "1", name
    assert "kOffV = kOffK + 2 * kKVBytes" in src and "kOffP = kOffV + 2 * kKVBytes" in src  # 2-stage rings
