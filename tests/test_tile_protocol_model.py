"""Model check of the d = 256 attention kernel's synchronisation protocol
(csrc/attention_bf16_d256.cu) on the CPU; see tests/tile_protocol_model.py."""

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
    for seed in range(400):
        rng = random.Random(seed)
        try:
            TM.TileModel(rng.randint(3, 10), mut=mut, rng=rng, rescale_prob=0.3).run()
        except TM.ProtocolViolation:
            return
    pytest.fail("slip %s not caught in 400 schedules" % slip)


def test_model_matches_the_kernel_source():
    src = open(os.path.join(os.path.dirname(__file__), "..", "dynamic_hierarchical_sparse_b200", "csrc",
                            "attention_bf16_d256.cu")).read()
    counts = dict(re.findall(r"mbar_init\(bar\((kBar\w+)(?: \+ \w+)?\), (\w+)\)", src))
    assert counts["kBarPFull"] == "4"  # one arrival per softmax warp
    for name in ("kBarQ", "kBarKFull", "kBarVFull", "kBarSFull", "kBarOReady"):
        assert counts[name] == "1", name
    assert "kBarKEmpty" not in src and "kBarVEmpty" not in src
    assert "constexpr int kKSlots = %d;" % TM.K_SLOTS in src
    assert "kSlices = kD / 64" in src and TM.K_SLICES == 256 // 64
    # slot of slice s of key tile t, and the release the producer waits for
    assert src.count("((kSlices * t + s) % kKSlots)") == 1 and "((kSlices * j + s) % kKSlots)" in src
    assert "if (t >= 1 && !wait_qk(t - 1)) return false;" in src
    assert "!mbar_wait(bar(kBarOReady), (j - 1) & 1, abort_flag, status)) break;" in src
    # the O-ready wait guards every release of P(j), j > 0, not only a rescale
    body = src[src.index("P(j) is released only once PV(j-1) is done"):]
    assert body.index("if (j > 0) {") < body.index("kBarOReady") < body.index("if (any && j > 0)")
