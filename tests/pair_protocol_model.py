"""Executable model of the synchronisation protocol of the persistent bf16
attention kernel (dynamic_hierarchical_sparse_b200/csrc/attention_bf16_pair.cu).

The kernel's roles are restated here as sequential programs of the waits,
arrivals, commits, loads and tensor-memory accesses they make, in the kernel's
order; an interleaving driver runs them under random schedules.  What the
hardware does asynchronously is modelled as such:

* a TMA load lands at any time after it is issued; its barrier phase completes
  when the producer's expect-tx arrival is in and every load of the phase has
  landed;
* each MMA-issuing thread has its own queue of tcgen05 operations, executed in
  issue order (a thread's tcgen05.mma and tcgen05.commit complete in order);
  the queues of the two threads run independently of each other;
* an mbarrier wait on parity passes once the awaited phase has completed.

Checked on every run:

* no deadlock: every role finishes;
* phase integrity: every arrival lands in the phase its arriver counts, at most
  once per arriver and phase; no waiter is ever two phases behind a barrier
  (a parity wait would then alias) or ahead of it (it would pass at once);
* shared memory: an MMA reads Q, K and V buffers only after the load of the
  expected tile has landed and while no other load to them is in flight;
* tensor memory: S is read by all four warps of its softmax warpgroup before
  the next QK^T overwrites it; each half of P is written by all four warps
  before the PV product that reads it runs, and is not overwritten before;
  the O accumulator is rescaled only between PV(t-1) and PV(t), read by the
  epilogue only after the item's last PV and before the next item's first PV
  (which overwrites it);
* item slots: the scheduler rewrites a slot only after all eleven users are
  done with its previous item.

The model is of the protocol, not of the arithmetic; it holds the kernel's
constants: two K stages, three V stages, four release barriers, two item
slots, four softmax warps per query tile.  `Mutation` plants one slip in the
protocol so that tests can show the checks catch it.
"""

from __future__ import annotations

import dataclasses
import random
from typing import Dict, List, Optional, Set, Tuple

K_STAGES = 2
V_STAGES = 3
REL_SLOTS = 4
ITEM_USERS = 11  # producer + 2 MMA threads + 8 softmax warps


class ProtocolViolation(AssertionError):
    pass


@dataclasses.dataclass(frozen=True)
class ItemSpec:
    """One work item: nt key tiles; tile 0 walks the first nt0 of them; the
    second query tile exists when valid1 (and then walks all nt)."""
    nt: int
    nt0: int
    valid1: bool


@dataclasses.dataclass(frozen=True)
class Mutation:
    """Protocol slips (each off by default)."""
    producer_skips_qfree: bool = False        # Q reloaded without waiting for the last QK^T
    producer_rel_lag3: bool = False           # K/V(t) loaded once S(t-3) is done instead of S(t-2)
    rel_commit_before_first_s: bool = False   # first release commit issued ahead of the first QK^T
    s_before_second_pv_half: bool = False     # S(t+1) issued between the two PV halves
    oready_one_tile_early: bool = False       # O declared ready after PV(nta-2)
    scheduler_skips_itemfree: bool = False    # slot rewritten without waiting for its users
    phalf_before_rescale: bool = False        # first P half released before O is rescaled
    qfree_from_thread0_only: bool = False     # Q-free barrier gets one commit instead of two


class _Barrier:
    def __init__(self, name: str, count: int):
        self.name, self.count = name, count
        self.phase = 0           # completed phases
        self.arrived: Set[str] = set()
        self.tx = 0              # loads of the current phase not yet landed
        self.expecting = False

    def _maybe_complete(self, model: "Model") -> None:
        if len(self.arrived) == self.count and self.tx == 0:
            self.phase += 1
            self.arrived = set()
            self.expecting = False
            for (role, n) in model.blocked_on(self):
                if self.phase >= n + 2:
                    raise ProtocolViolation("%s: %s waits for phase %d but the barrier completed phase %d "
                                            "(parity alias)" % (self.name, role, n, self.phase - 1))

    def arrive(self, who: str, n: int, model: "Model") -> None:
        if n != self.phase:
            raise ProtocolViolation("%s: %s arrives for phase %d while phase %d is open"
                                    % (self.name, who, n, self.phase))
        if who in self.arrived:
            raise ProtocolViolation("%s: %s arrives twice in phase %d" % (self.name, who, n))
        self.arrived.add(who)
        self._maybe_complete(model)


class Model:
    def __init__(self, items: List[ItemSpec], mut: Mutation = Mutation(), rescale_prob: float = 0.5,
                 rng: Optional[random.Random] = None):
        self.items = items
        self.mut = mut
        self.rng = rng or random.Random(0)
        self.rescale_prob = rescale_prob
        B = self.bars = {}

        def mk(name, count):
            B[name] = _Barrier(name, count)
        mk("Q", 1)
        for s in range(K_STAGES):
            mk("KFull%d" % s, 1)
        for s in range(V_STAGES):
            mk("VFull%d" % s, 1)
        for s in range(REL_SLOTS):
            mk("Rel%d" % s, 2)
        for a in (0, 1):
            mk("SFull%d" % a, 1)
            mk("PHalf%d" % a, 4)
            mk("PFull%d" % a, 4)
            mk("OReady%d" % a, 1)
            mk("Turn%d" % a, 1)
        mk("QFree", 2)
        for s in (0, 1):
            mk("ItemReady%d" % s, 1)
            mk("ItemFree%d" % s, ITEM_USERS)

        # shared-memory buffers: tag of the landed tile, loads in flight
        self.smem: Dict[str, list] = {}
        for name in ["Q0", "Q1"] + ["K%d" % s for s in range(K_STAGES)] + ["V%d" % s for s in range(V_STAGES)]:
            self.smem[name] = [None, 0]
        self.tma: List[Tuple[str, object, str]] = []  # (buffer, tag, barrier)
        self.queues: Dict[int, List[tuple]] = {0: [], 1: []}
        # tensor memory per query tile
        self.S = {a: {"tag": None, "readers": set(), "P": [[None] * 2 for _ in range(4)]} for a in (0, 1)}
        self.pv_done: Dict[Tuple[int, tuple], Set[int]] = {}
        self.O = {a: {"item": None, "done": set(), "nta": 0, "epi": set()} for a in (0, 1)}
        # item slots: item index held, users done with it
        self.slot = {s: {"item": None, "released": set()} for s in (0, 1)}
        self.waiting: Dict[str, Tuple[_Barrier, int]] = {}
        self.roles = {}
        self.roles["sched"] = self._scheduler()
        self.roles["prod"] = self._producer()
        for a in (0, 1):
            self.roles["mma%d" % a] = self._mma(a)
            for w in range(4):
                self.roles["smx%d.%d" % (a, w)] = self._softmax(a, w)
        self.pending_op: Dict[str, Optional[tuple]] = {r: None for r in self.roles}
        self.finished: Set[str] = set()

    # ------------------------------------------------------------- helpers
    def blocked_on(self, bar: _Barrier):
        return [(r, n) for r, (b, n) in self.waiting.items() if b is bar]

    def _item(self, k: int) -> Optional[ItemSpec]:
        return self.items[k] if k < len(self.items) else None

    @staticmethod
    def _nta(it: ItemSpec, a: int) -> int:
        return it.nt0 if a == 0 else (it.nt if it.valid1 else 0)

    def _slot_read(self, s: int, k: int, who: str) -> None:
        if self.slot[s]["item"] != k:
            raise ProtocolViolation("%s reads slot %d expecting item %d, holds %s" % (who, s, k, self.slot[s]["item"]))

    # --------------------------------------------------------------- roles
    def _scheduler(self):
        k = 0
        while True:
            s = k & 1
            if k >= 2 and not self.mut.scheduler_skips_itemfree:
                yield ("wait", "ItemFree%d" % s, (k - 2) >> 1)
            yield ("slot_write", s, k)
            yield ("arrive", "ItemReady%d" % s, k >> 1, "sched")
            if self._item(k) is None:
                return
            k += 1

    def _producer(self):
        T = 0
        k = 0
        while True:
            s = k & 1
            yield ("wait", "ItemReady%d" % s, k >> 1)
            yield ("slot_read", s, k, "prod")
            it = self._item(k)
            if it is None:
                return
            if k >= 1 and not self.mut.producer_skips_qfree:
                yield ("wait", "QFree", k - 1)
            yield ("expect", "Q", k, "prod", 2 if it.valid1 else 1)
            yield ("tma", "Q0", k, "Q")
            if it.valid1:
                yield ("tma", "Q1", k, "Q")
            for t in range(it.nt):
                tg = T + t
                lag = 3 if self.mut.producer_rel_lag3 else 2
                if tg >= lag:
                    j = tg - lag
                    yield ("wait", "Rel%d" % (j % REL_SLOTS), j // REL_SLOTS)
                yield ("expect", "KFull%d" % (tg % K_STAGES), tg // K_STAGES, "prod", 1)
                yield ("tma", "K%d" % (tg % K_STAGES), tg, "KFull%d" % (tg % K_STAGES))
                yield ("expect", "VFull%d" % (tg % V_STAGES), tg // V_STAGES, "prod", 1)
                yield ("tma", "V%d" % (tg % V_STAGES), tg, "VFull%d" % (tg % V_STAGES))
            T += it.nt
            yield ("slot_release", s, k, "prod")
            yield ("arrive", "ItemFree%d" % s, k >> 1, "prod")
            k += 1

    def _mma(self, a: int):
        me = "mma%d" % a
        T = kt = np_ = 0
        k = 0
        issued = {"S": 0, "O": 0}  # phases of this thread's S-ready and O-ready commits

        def wait_turn(kt):
            if a == 1:
                return [("wait", "Turn0", kt)]
            return [] if kt == 0 else [("wait", "Turn1", kt - 1)]

        def issue_s(k, t, tg):
            ops = [("mma", a, "S", k, t, tg), ("commit", a, "SFull%d" % a, issued["S"])]
            issued["S"] += 1
            return ops

        def rel(j):
            return ("commit", a, "Rel%d" % (j % REL_SLOTS), j // REL_SLOTS)

        def qfree(k):
            if self.mut.qfree_from_thread0_only and a == 1:
                return []
            return [("commit", a, "QFree", k)]

        while True:
            s = k & 1
            yield ("wait", "ItemReady%d" % s, k >> 1)
            yield ("slot_read", s, k, me)
            it = self._item(k)
            if it is None:
                return
            nt, nta = it.nt, self._nta(it, a)
            yield ("wait", "Q", k)
            yield ("wait", "KFull%d" % (T % K_STAGES), T // K_STAGES)
            for op in wait_turn(kt):
                yield op
            first = [rel(T)] if self.mut.rel_commit_before_first_s else []
            for op in first:
                yield op
            if nta > 0:
                for op in issue_s(k, 0, T):
                    yield op
            yield ("arrive", "Turn%d" % a, kt, me)
            kt += 1
            if nta <= 1:
                for op in qfree(k):
                    yield op
            if not self.mut.rel_commit_before_first_s:
                yield rel(T)
            for t in range(nt):
                tg = T + t
                if t < nta:
                    yield ("wait", "VFull%d" % (tg % V_STAGES), tg // V_STAGES)
                    yield ("wait", "PHalf%d" % a, np_)
                    if t + 1 < nta:
                        yield ("wait", "KFull%d" % ((tg + 1) % K_STAGES), (tg + 1) // K_STAGES)
                    for op in wait_turn(kt):
                        yield op
                    yield ("mma", a, "PV", k, t, tg, 0)
                    if self.mut.s_before_second_pv_half and t + 1 < nta:
                        for op in issue_s(k, t + 1, tg + 1):
                            yield op
                    yield ("wait", "PFull%d" % a, np_)
                    yield ("mma", a, "PV", k, t, tg, 1)
                    np_ += 1
                    if t + 1 < nta and not self.mut.s_before_second_pv_half:
                        for op in issue_s(k, t + 1, tg + 1):
                            yield op
                    yield ("arrive", "Turn%d" % a, kt, me)
                    kt += 1
                    last = nta - 2 if self.mut.oready_one_tile_early and nta >= 2 else nta - 1
                    if t == last:
                        yield ("commit", a, "OReady%d" % a, issued["O"])
                        issued["O"] += 1
                    if t + 2 == nta:
                        for op in qfree(k):
                            yield op
                else:
                    for op in wait_turn(kt):
                        yield op
                    yield ("arrive", "Turn%d" % a, kt, me)
                    kt += 1
                if t + 1 < nt:
                    yield rel(tg + 1)
            T += nt
            yield ("slot_release", s, k, me)
            yield ("arrive", "ItemFree%d" % s, k >> 1, me)
            k += 1

    def _softmax(self, a: int, w: int):
        me = "smx%d.%d" % (a, w)
        ns = no = 0
        k = 0
        while True:
            s = k & 1
            yield ("wait", "ItemReady%d" % s, k >> 1)
            yield ("slot_read", s, k, me)
            it = self._item(k)
            if it is None:
                return
            nta = self._nta(it, a)
            for t in range(nta):
                yield ("wait", "SFull%d" % a, ns)
                ns += 1
                yield ("read_S", a, w, k, t)
                yield ("write_P", a, w, 0, k, t)
                rescale = t > 0 and self.rng.random() < self.rescale_prob
                if self.mut.phalf_before_rescale:
                    yield ("arrive", "PHalf%d" % a, ns - 1, me)
                    if rescale:
                        yield ("rescale", a, w, k, t)
                else:
                    if rescale:
                        yield ("rescale", a, w, k, t)
                    yield ("arrive", "PHalf%d" % a, ns - 1, me)
                yield ("write_P", a, w, 1, k, t)
                yield ("arrive", "PFull%d" % a, ns - 1, me)
            yield ("slot_release", s, k, me)
            yield ("arrive", "ItemFree%d" % s, k >> 1, me)
            if nta > 0:
                yield ("wait", "OReady%d" % a, no)
                no += 1
                yield ("epilogue", a, w, k, nta)
            k += 1

    # ------------------------------------------------------ op execution
    def _run_sync(self, role: str, op: tuple) -> bool:
        """Executes a synchronous op of a role; False if it has to wait."""
        kind = op[0]
        if kind == "wait":
            bar, n = self.bars[op[1]], op[2]
            if bar.phase < n:
                raise ProtocolViolation("%s: %s waits for phase %d while phase %d is open (would pass at once)"
                                        % (bar.name, role, n, bar.phase))
            if role not in self.waiting and bar.phase >= n + 2:
                raise ProtocolViolation("%s: %s starts waiting for phase %d after phase %d completed "
                                        "(parity alias)" % (bar.name, role, n, bar.phase - 1))
            if bar.phase >= n + 1:
                self.waiting.pop(role, None)
                return True
            self.waiting[role] = (bar, n)
            return False
        if kind == "arrive":
            self.bars[op[1]].arrive(op[3], op[2], self)
            return True
        if kind == "expect":
            bar = self.bars[op[1]]
            if bar.expecting:
                raise ProtocolViolation("%s: second expect-tx in phase %d" % (bar.name, bar.phase))
            bar.expecting = True
            bar.tx += op[4]
            bar.arrive(op[3], op[2], self)
            return True
        if kind == "tma":
            buf = self.smem[op[1]]
            if buf[1]:
                raise ProtocolViolation("two loads in flight to %s" % op[1])
            buf[1] = 1
            self.tma.append((op[1], op[2], op[3]))
            return True
        if kind in ("mma", "commit"):
            self.queues[op[1]].append(op)
            return True
        if kind == "slot_write":
            s, k = op[1], op[2]
            if k >= 2 and len(self.slot[s]["released"]) != ITEM_USERS:
                raise ProtocolViolation("slot %d rewritten with item %d while %d of %d users hold item %d"
                                        % (s, k, ITEM_USERS - len(self.slot[s]["released"]), ITEM_USERS, k - 2))
            self.slot[s] = {"item": k, "released": set()}
            return True
        if kind == "slot_read":
            self._slot_read(op[1], op[2], op[3])
            return True
        if kind == "slot_release":
            self._slot_read(op[1], op[2], op[3])
            self.slot[op[1]]["released"].add(op[3])
            return True
        if kind == "read_S":
            _, a, w, k, t = op
            S = self.S[a]
            if S["tag"] != (k, t):
                raise ProtocolViolation("warp %d.%d reads S expecting %s, holds %s" % (a, w, (k, t), S["tag"]))
            S["readers"].add(w)
            return True
        if kind == "write_P":
            _, a, w, h, k, t = op
            S = self.S[a]
            if S["tag"] != (k, t) or w not in S["readers"]:
                raise ProtocolViolation("warp %d.%d writes P%d of %s over S %s" % (a, w, h, (k, t), S["tag"]))
            S["P"][w][h] = (k, t)
            return True
        if kind == "rescale":
            _, a, w, k, t = op
            O = self.O[a]
            want = {(tt, h) for tt in range(t) for h in (0, 1)}
            if O["item"] != k or O["done"] != want:
                raise ProtocolViolation("warp %d.%d rescales O for %s with PV done %s of item %s"
                                        % (a, w, (k, t), sorted(O["done"]), O["item"]))
            return True
        if kind == "epilogue":
            _, a, w, k, nta = op
            O = self.O[a]
            want = {(tt, h) for tt in range(nta) for h in (0, 1)}
            if O["item"] != k or O["done"] != want:
                raise ProtocolViolation("warp %d.%d reads O of item %d with PV done %s of item %s"
                                        % (a, w, k, sorted(O["done"]), O["item"]))
            O["epi"].add(w)
            return True
        raise ValueError(op)

    def _land_tma(self, i: int) -> None:
        buf, tag, barname = self.tma.pop(i)
        self.smem[buf] = [tag, 0]
        bar = self.bars[barname]
        bar.tx -= 1
        bar._maybe_complete(self)

    def _read_smem(self, name: str, tag) -> None:
        cur, inflight = self.smem[name]
        if inflight or cur != tag:
            raise ProtocolViolation("MMA reads %s expecting tile %s: holds %s%s"
                                    % (name, tag, cur, " with a load in flight" if inflight else ""))

    def _exec_mma(self, a: int) -> None:
        op = self.queues[a].pop(0)
        if op[0] == "commit":
            self.bars[op[2]].arrive("mma%d" % a, op[3], self)
            return
        if op[2] == "S":
            _, _, _, k, t, tg = op
            self._read_smem("Q%d" % a, k)
            self._read_smem("K%d" % (tg % K_STAGES), tg)
            S = self.S[a]
            if S["tag"] is not None:
                if len(S["readers"]) != 4:
                    raise ProtocolViolation("S%d(%s) overwrites S%s read by warps %s only"
                                            % (a, (k, t), S["tag"], sorted(S["readers"])))
                if self.pv_done.get((a, S["tag"]), set()) != {0, 1}:
                    raise ProtocolViolation("S%d(%s) overwrites P%s before its PV ran" % (a, (k, t), S["tag"]))
            self.S[a] = {"tag": (k, t), "readers": set(), "P": [[None] * 2 for _ in range(4)]}
            return
        _, _, _, k, t, tg, h = op
        self._read_smem("V%d" % (tg % V_STAGES), tg)
        S = self.S[a]
        for w in range(4):
            if S["P"][w][h] != (k, t):
                raise ProtocolViolation("PV%d(%s) half %d reads P of warp %d holding %s"
                                        % (a, (k, t), h, w, S["P"][w][h]))
        O = self.O[a]
        if t == 0 and h == 0:
            if O["item"] is not None and O["nta"] > 0 and len(O["epi"]) != 4:
                raise ProtocolViolation("PV%d of item %d overwrites O before the epilogue of item %d (warps %s)"
                                        % (a, k, O["item"], sorted(O["epi"])))
            it = self.items[k]
            self.O[a] = O = {"item": k, "done": set(), "nta": self._nta(it, a), "epi": set()}
        elif O["item"] != k or (t, h) in O["done"]:
            raise ProtocolViolation("PV%d(%s) half %d out of order" % (a, (k, t), h))
        O["done"].add((t, h))
        self.pv_done.setdefault((a, (k, t)), set()).add(h)

    # ---------------------------------------------------------- driver
    def run(self, max_steps: int = 1_000_000) -> int:
        """Runs to completion under a random schedule; returns the step count.
        Raises ProtocolViolation on a broken invariant or a deadlock."""
        rng = self.rng
        # each actor runs at its own random speed (log-uniform over four decades),
        # so that schedules where one role lags far behind the others are common
        weight: Dict[tuple, float] = {}

        def wt(key):
            if key not in weight:
                weight[key] = 10.0 ** rng.uniform(-4.0, 0.0)
            return weight[key]
        for step in range(max_steps):
            choices = []
            for r in self.roles:
                if r in self.finished:
                    continue
                op = self.pending_op[r]
                if op is not None and op[0] == "wait":
                    bar, n = self.bars[op[1]], op[2]
                    if bar.phase < n + 1:
                        continue
                choices.append(("role", r))
            for i in range(len(self.tma)):
                choices.append(("tma", i))
            for a in (0, 1):
                if self.queues[a]:
                    choices.append(("mma", a))
            if not choices:
                if len(self.finished) == len(self.roles) and not self.tma and not any(self.queues.values()):
                    return step
                stuck = {r: self.pending_op[r] for r in self.roles if r not in self.finished}
                raise ProtocolViolation("deadlock: %s" % stuck)
            keys = [(c[0], c[1] if c[0] != "tma" else self.tma[c[1]][0]) for c in choices]
            kind, x = rng.choices(choices, weights=[wt(key) for key in keys])[0]
            if kind == "tma":
                self._land_tma(x)
            elif kind == "mma":
                self._exec_mma(x)
            else:
                self._step_role(x)
        raise RuntimeError("model did not finish in %d steps" % max_steps)

    def _step_role(self, r: str) -> None:
        op = self.pending_op[r]
        if op is None:
            try:
                op = next(self.roles[r])
            except StopIteration:
                self.finished.add(r)
                return
        if self._run_sync(r, op):
            self.pending_op[r] = None
        else:
            self.pending_op[r] = op


def random_items(rng: random.Random, n_items: int, max_nt: int = 6, head_pair: bool = False) -> List[ItemSpec]:
    """Work items as the kernel's scheduler forms them: nt >= 1 key tiles;
    tile 0 walks a prefix nt0 >= 1 of them (all of them with head pairing or
    when the item has one query tile)."""
    items = []
    for _ in range(n_items):
        nt = rng.randint(1, max_nt)
        valid1 = True if head_pair else rng.random() < 0.7
        nt0 = nt if (head_pair or not valid1) else rng.randint(1, nt)
        items.append(ItemSpec(nt, nt0, valid1))
    return items
