"""Executable model of the synchronisation protocol of the per-tile bf16
attention kernel for d = 256 (dynamic_hierarchical_sparse_b200/csrc/attention_bf16.cu).

One CTA handles one 128-row query tile over `nt` key tiles. Its roles are
restated as sequential programs, in the kernel's order: the TMA producer (Q
once, then K and V tiles into 2-stage rings guarded by empty/full barrier
pairs), the single MMA-issuing thread (S = QK^T two tiles ahead into a TMEM
double buffer, O += P V with P from shared memory), and the four softmax warps
(read S, release its buffer, exponentiate, rescale O when needed, write P to
shared memory). The driver and the phase checks are those of
pair_protocol_model.Model: loads land asynchronously, the issuing thread's
tcgen05 operations complete in issue order, and parity waits must neither
alias nor pass early.

Barriers whose expected count is the 128 softmax threads are modelled with one
arrival per warp (4). A fresh barrier waited on with the "previous phase"
parity passes at once in the kernel; the model omits those first waits.

Checked: no deadlock; phase integrity; K/V/Q read only once landed and with no
load in flight; S(t+2) overwrites S(t) only after all four warps read it; P(j)
written only after PV(j-1) has read P(j-1), and read by PV(j) only when all
four warps wrote it; O rescaled only between PV(j-1) and PV(j); the epilogue
reads O after the last PV.
"""

from __future__ import annotations

import dataclasses
import random
from typing import Optional

from pair_protocol_model import Model, ProtocolViolation, _Barrier


@dataclasses.dataclass(frozen=True)
class TileMutation:
    """Protocol slips (each off by default)."""
    producer_skips_kempty: bool = False       # K(t) loaded over K(t-2) without waiting for S(t-2)
    kempty_before_s: bool = False             # K stage released before its QK^T is issued
    s_before_pfull: bool = False              # S(j+2) issued before P(j) is written, without the buffer wait
    p_before_oready: bool = False             # P(j) written before PV(j-1) is done
    oready_before_pv: bool = False            # O declared ready (and P free) before PV(j) is issued
    vempty_before_pv: bool = False            # V stage released before its PV is issued


@dataclasses.dataclass(frozen=True)
class TileVariant:
    """Protocol changes that are not slips."""
    no_sfree_wait: bool = False  # S(j+2) issued after PV(j) without the S-free wait


class TileModel(Model):
    def __init__(self, nt: int, mut: TileMutation = TileMutation(), rescale_prob: float = 0.5,
                 rng: Optional[random.Random] = None, variant: TileVariant = TileVariant()):
        # the pair model's driver, with this kernel's roles and state
        self.nt = nt
        self.tmut = mut
        self.variant = variant
        self.rng = rng or random.Random(0)
        self.rescale_prob = rescale_prob
        B = self.bars = {}
        for name, count in [("Q", 1), ("PFull", 4), ("OReady", 1)] + \
                [("%s%d" % (n, s), c) for s in (0, 1) for n, c in
                 (("KFull", 1), ("KEmpty", 1), ("VFull", 1), ("VEmpty", 1), ("SFull", 1), ("SFree", 4))]:
            B[name] = _Barrier(name, count)
        self.smem = {name: [None, 0] for name in ("Q0", "K0", "K1", "V0", "V1")}
        self.tma = []
        self.queues = {0: [], 1: []}
        self.waiting = {}
        self.Sbuf = {b: {"tag": None, "readers": set()} for b in (0, 1)}
        self.P = {"tag": [None] * 4, "read": None}  # P rows per warp; last tile a PV has read
        self.Odone = set()
        self.roles = {"prod": self._tile_producer(), "mma0": self._tile_mma()}
        for w in range(4):
            self.roles["smx%d" % w] = self._tile_softmax(w)
        self.pending_op = {r: None for r in self.roles}
        self.finished = set()

    # --------------------------------------------------------------- roles
    def _tile_producer(self):
        nt = self.nt
        yield ("expect", "Q", 0, "prod", 1)
        yield ("tma", "Q0", 0, "Q")
        for t in range(nt):
            s = t & 1
            if t >= 2 and not self.tmut.producer_skips_kempty:
                yield ("wait", "KEmpty%d" % s, (t >> 1) - 1)
            yield ("expect", "KFull%d" % s, t >> 1, "prod", 1)
            yield ("tma", "K%d" % s, t, "KFull%d" % s)
            if t >= 2:
                yield ("wait", "VEmpty%d" % s, (t >> 1) - 1)
            yield ("expect", "VFull%d" % s, t >> 1, "prod", 1)
            yield ("tma", "V%d" % s, t, "VFull%d" % s)

    def _tile_mma(self):
        nt = self.nt

        def issue_s(t):
            s = t & 1
            ops = [("wait", "KFull%d" % s, t >> 1)]
            if self.tmut.kempty_before_s:
                ops.append(("commit", 0, "KEmpty%d" % s, t >> 1))
            ops.append(("mma", 0, "S", t))
            ops.append(("commit", 0, "SFull%d" % s, t >> 1))
            if not self.tmut.kempty_before_s:
                ops.append(("commit", 0, "KEmpty%d" % s, t >> 1))
            return ops

        yield ("wait", "Q", 0)
        for op in issue_s(0):
            yield op
        if nt > 1:
            for op in issue_s(1):
                yield op
        for j in range(nt):
            s = j & 1
            if self.tmut.s_before_pfull and j + 2 < nt:
                for op in issue_s(j + 2):
                    yield op
            yield ("wait", "PFull", j)
            yield ("wait", "VFull%d" % s, j >> 1)
            if self.tmut.vempty_before_pv:
                yield ("commit", 0, "VEmpty%d" % s, j >> 1)
            if self.tmut.oready_before_pv:
                yield ("commit", 0, "OReady", j)
            yield ("mma", 0, "PV", j)
            if not self.tmut.oready_before_pv:
                yield ("commit", 0, "OReady", j)
            if not self.tmut.vempty_before_pv:
                yield ("commit", 0, "VEmpty%d" % s, j >> 1)
            if j + 2 < nt and not self.tmut.s_before_pfull:
                if not self.variant.no_sfree_wait:
                    yield ("wait", "SFree%d" % s, j >> 1)
                for op in issue_s(j + 2):
                    yield op

    def _tile_softmax(self, w: int):
        me = "smx%d" % w
        nt = self.nt
        for j in range(nt):
            b = j & 1
            yield ("wait", "SFull%d" % b, j >> 1)
            yield ("t_read_S", w, j)
            yield ("arrive", "SFree%d" % b, j >> 1, me)
            if self.tmut.p_before_oready:
                yield ("t_write_P", w, j)
            if j > 0:
                yield ("wait", "OReady", j - 1)
                if self.rng.random() < self.rescale_prob:
                    yield ("t_rescale", w, j)
            if not self.tmut.p_before_oready:
                yield ("t_write_P", w, j)
            yield ("arrive", "PFull", j, me)
        yield ("wait", "OReady", nt - 1)
        yield ("t_epilogue", w)

    # -------------------------------------------------------------- ops
    def _run_sync(self, role, op):
        kind = op[0]
        if kind == "t_read_S":
            _, w, j = op
            S = self.Sbuf[j & 1]
            if S["tag"] != j:
                raise ProtocolViolation("warp %d reads S buffer %d expecting tile %d, holds %s" % (w, j & 1, j, S["tag"]))
            S["readers"].add(w)
            return True
        if kind == "t_write_P":
            _, w, j = op
            prev = self.P["tag"][w]
            if prev is not None and not (prev == j - 1 and self.P["read"] == prev):
                raise ProtocolViolation("warp %d writes P(%d) over P(%s) not yet read by its PV" % (w, j, prev))
            if j > 0 and self.P["read"] != j - 1:
                raise ProtocolViolation("warp %d writes P(%d) before PV(%d) read P" % (w, j, j - 1))
            self.P["tag"][w] = j
            return True
        if kind == "t_rescale":
            _, w, j = op
            if self.Odone != set(range(j)):
                raise ProtocolViolation("warp %d rescales O before PV(%d) with PV done %s" % (w, j, sorted(self.Odone)))
            return True
        if kind == "t_epilogue":
            if self.Odone != set(range(self.nt)):
                raise ProtocolViolation("epilogue reads O with PV done %s of %d" % (sorted(self.Odone), self.nt))
            return True
        return super()._run_sync(role, op)

    def _exec_mma(self, a: int) -> None:
        op = self.queues[a][0]
        if op[0] == "commit":
            return super()._exec_mma(a)
        self.queues[a].pop(0)
        if op[2] == "S":
            t = op[3]
            self._read_smem("Q0", 0)
            self._read_smem("K%d" % (t & 1), t)
            S = self.Sbuf[t & 1]
            if S["tag"] is not None and len(S["readers"]) != 4:
                raise ProtocolViolation("S(%d) overwrites S(%d) read by warps %s only" % (t, S["tag"], sorted(S["readers"])))
            self.Sbuf[t & 1] = {"tag": t, "readers": set()}
            return
        j = op[3]
        self._read_smem("V%d" % (j & 1), j)
        if any(tag != j for tag in self.P["tag"]):
            raise ProtocolViolation("PV(%d) reads P holding %s" % (j, self.P["tag"]))
        if self.Odone != set(range(j)):
            raise ProtocolViolation("PV(%d) out of order (done %s)" % (j, sorted(self.Odone)))
        self.P["read"] = j
        self.Odone.add(j)
