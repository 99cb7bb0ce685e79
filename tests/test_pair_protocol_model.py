"""Model check of the persistent bf16 attention kernel's synchronisation
protocol (csrc/attention_bf16_pair.cu), on the CPU: random interleavings of its
roles, asynchronous TMA landings and in-order tcgen05 queues, over work-item
mixes the kernel's scheduler produces.  See tests/pair_protocol_model.py for
what is modelled and checked."""

import dataclasses
import random

import pytest

import pair_protocol_model as M


def _run(items, seed, mut=M.Mutation(), rescale_prob=0.5):
    return M.Model(items, mut=mut, rng=random.Random(seed), rescale_prob=rescale_prob).run()


def test_random_item_mixes_and_schedules():
    for seed in range(300):
        rng = random.Random(seed)
        items = M.random_items(rng, rng.randint(1, 8), max_nt=7, head_pair=(seed % 4 == 0))
        assert _run(items, seed) > 0


I = M.ItemSpec
EDGE_MIXES = {
    "one_item_one_tile": [I(1, 1, False)],
    "single_query_tile_items": [I(nt, nt, False) for nt in (3, 1, 5, 2, 4, 1)],
    "one_key_tile_items": [I(1, 1, True)] * 7,
    "long_items_wrap_every_ring": [I(13, 5, True), I(14, 14, False), I(13, 1, True)],
    "tile0_one_key_tile": [I(8, 1, True), I(6, 1, True), I(1, 1, True)],
    "alternating_one_and_two_tiles": [I(4, 2, True), I(3, 3, False)] * 4,
    "head_pair_items": [I(nt, nt, True) for nt in (5, 2, 7, 1, 3)],
}


@pytest.mark.parametrize("mix", sorted(EDGE_MIXES))
def test_edge_item_mixes(mix):
    for seed in range(40):
        for p in (0.0, 1.0):  # O rescaled never / on every tile after the first
            _run(EDGE_MIXES[mix], seed, rescale_prob=p)


@pytest.mark.parametrize("slip", [f.name for f in dataclasses.fields(M.Mutation)])
def test_planted_protocol_slips_are_caught(slip):
    mut = M.Mutation(**{slip: True})
    for seed in range(400):
        rng = random.Random(seed)
        items = M.random_items(rng, rng.randint(2, 6))
        try:
            _run(items, seed, mut=mut)
        except M.ProtocolViolation:
            return
    pytest.fail("slip %s not caught in 400 schedules" % slip)


class _Waiters:
    def __init__(self, waiters=()):
        self.w = list(waiters)

    def blocked_on(self, bar):
        return self.w


def test_barrier_rejects_arrival_in_another_phase_and_double_arrival():
    b = M._Barrier("B", 2)
    m = _Waiters()
    b.arrive("x", 0, m)
    with pytest.raises(M.ProtocolViolation):
        b.arrive("x", 0, m)  # same arriver twice in one phase
    with pytest.raises(M.ProtocolViolation):
        b.arrive("y", 1, m)  # counts a phase that is not open
    b.arrive("y", 0, m)
    assert b.phase == 1


def test_barrier_flags_a_waiter_two_phases_behind():
    b = M._Barrier("B", 1)
    b.arrive("x", 0, _Waiters())
    with pytest.raises(M.ProtocolViolation):
        b.arrive("x", 1, _Waiters([("late", 0)]))  # phase 1 completes while a waiter still waits for phase 0


def test_model_constants_match_the_kernel_source():
    """The barrier arrival counts and ring depths the model assumes are the ones
    the kernel initialises (guards the model against drifting from the source)."""
    import os
    import re
    src = open(os.path.join(os.path.dirname(__file__), "..", "dynamic_hierarchical_sparse_b200", "csrc",
                            "attention_bf16_pair.cu")).read()
    consts = dict(re.findall(r"constexpr int (k\w+) = (\d+);", src))
    assert int(consts["kVStages"]) == M.V_STAGES
    assert int(consts["kItemUsers"]) == M.ITEM_USERS
    counts = {}
    for name, count in re.findall(r"mbar_init\(bar\((kBar\w+)(?: \+ s)?\), (\w+)\)", src):
        counts[name] = int(consts.get(count, count))
    model = M.Model([M.ItemSpec(1, 1, False)])
    want = {"kBarQ": "Q", "kBarKFull": "KFull0", "kBarVFull": "VFull0", "kBarRel": "Rel0", "kBarSFull": "SFull0",
            "kBarPFull": "PFull0", "kBarPHalf": "PHalf0", "kBarOReady": "OReady0", "kBarTurn": "Turn0",
            "kBarQFree": "QFree", "kBarItemReady": "ItemReady0", "kBarItemFree": "ItemFree0"}
    for kname, mname in want.items():
        assert counts[kname] == model.bars[mname].count, kname
    assert re.search(r"for \(int s = 0; s < %d; \+\+s\) mbar_init\(bar\(kBarRel \+ s\)" % M.REL_SLOTS, src)
    assert "kOffV = kOffK + %d * kKVBytes" % M.K_STAGES in src
