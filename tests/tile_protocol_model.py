"""Executable model of the synchronisation protocol of the per-tile bf16
attention kernel for d = 256 (dynamic_hierarchical_sparse_b200/csrc/attention_bf16_d256.cu).

One CTA handles one 128-row query tile over `nt` key tiles. Its roles are
restated as sequential programs, in the kernel's order:

* the TMA producer: Q once; K as 16 KB slices, slice s of key tile t into
  ring slot (4t + s) % K_SLOTS, the tile's four slices behind one K-full
  barrier per tile parity, loaded once QK(t-1) is done (its S-full commit:
  the slots hold slices of tiles t-2 and t-1); K(j+1) ahead of V(j); V as one
  tile-sized buffer, reloaded once PV(j-1) is done (its O-ready commit);
* the single MMA-issuing thread: QK(0), QK(1), then per tile j the PV(j)
  product (after P-full(j) and V-full(j)) and QK(j+2) (after K-full); it
  commits S-full(b) after a whole QK^T and O-ready after each PV, nothing
  else;
* the four softmax warps: read S(j) from its TMEM buffer j % 2, write P(j)
  over that buffer, wait for O-ready(j-1) (then maybe rescale O), release P(j)
  with one arrival per warp.

The driver and the phase checks are those of pair_protocol_model.Model: loads
land asynchronously, the issuing thread's tcgen05 operations complete in issue
order, and parity waits must neither alias nor pass early.

Checked: no deadlock; phase integrity (among it, that no warp arrives on P-full
for tile j+1 while tile j's phase is still open, which S double-buffering would
allow without the O-ready wait); K slices and V read only once landed and
with no load in flight; QK(j+2) overwrites S buffer j % 2 only after every warp
read S(j) and PV(j) read P(j); PV(j) reads P(j) only after every warp wrote it;
O rescaled only between PV(j-1) and PV(j); the epilogue reads O after the last
PV.
"""

from __future__ import annotations

import dataclasses
import random
from typing import Optional

from pair_protocol_model import Model, ProtocolViolation, _Barrier

K_SLOTS = 6    # K ring slots (16 KB slices)
K_SLICES = 4   # 64-column slices of a 256-column K tile


@dataclasses.dataclass(frozen=True)
class TileMutation:
    """Protocol slips (each off by default)."""
    producer_skips_qk_wait: bool = False  # K(t) loaded without waiting for QK(t-1)
    producer_waits_qk_two_back: bool = False  # K(t) loaded after QK(t-2) only (tile t-1's slots)
    producer_skips_oready: bool = False   # V(j) loaded over V(j-1) without waiting for PV(j-1)
    s_before_pv: bool = False             # QK(j+2) issued before PV(j) (over P(j))
    oready_before_pv: bool = False        # O declared ready (and V free) before PV(j) is issued
    pfull_without_oready: bool = False    # P(j) released without waiting for PV(j-1) unless rescaling


class TileModel(Model):
    def __init__(self, nt: int, mut: TileMutation = TileMutation(), rescale_prob: float = 0.5,
                 rng: Optional[random.Random] = None):
        # the pair model's driver, with this kernel's roles and state
        self.nt = nt
        self.tmut = mut
        self.rng = rng or random.Random(0)
        self.rescale_prob = rescale_prob
        B = self.bars = {}
        names = [("Q", 1), ("PFull", 4), ("OReady", 1), ("VFull", 1), ("SFull0", 1), ("SFull1", 1), ("KFull0", 1),
                 ("KFull1", 1)]
        for name, count in names:
            B[name] = _Barrier(name, count)
        self.smem = {name: [None, 0] for name in ["Q", "V"] + ["K%d" % s for s in range(K_SLOTS)]}
        self.tma = []
        self.queues = {0: [], 1: []}
        self.waiting = {}
        # TMEM buffers: S(j) with the warps that read it, P(j) rows per warp, PV(j) done
        self.Sbuf = {b: {"tag": None, "readers": set(), "P": [None] * 4, "pv": False} for b in (0, 1)}
        self.Odone = set()
        self.roles = {"prod": self._producer(), "mma0": self._issuer()}
        for w in range(4):
            self.roles["smx%d" % w] = self._softmax(w)
        self.pending_op = {r: None for r in self.roles}
        self.finished = set()

    # --------------------------------------------------------------- roles
    def _kfull(self, t: int):
        """(barrier, phase) of key tile t's K-full barrier."""
        return "KFull%d" % (t & 1), t >> 1

    def _producer(self):
        nt = self.nt
        yield ("expect", "Q", 0, "prod", 1)
        yield ("tma", "Q", 0, "Q")
        seen = [-1]

        def wait_qk(t):
            if t < 0 or t <= seen[0]:
                return
            yield ("wait", "SFull%d" % (t & 1), t >> 1)
            seen[0] = t

        def load_k(t):
            if not self.tmut.producer_skips_qk_wait:
                yield from wait_qk(t - 2 if self.tmut.producer_waits_qk_two_back else t - 1)
            bar, n = self._kfull(t)
            yield ("expect", bar, n, "prod", K_SLICES)
            for s in range(K_SLICES):
                yield ("tma", "K%d" % ((K_SLICES * t + s) % K_SLOTS), (t, s), bar)

        yield from load_k(0)
        for j in range(nt):
            if j + 1 < nt:
                yield from load_k(j + 1)
            if j >= 1 and not self.tmut.producer_skips_oready:
                yield ("wait", "OReady", j - 1)
            yield ("expect", "VFull", j, "prod", 1)
            yield ("tma", "V", j, "VFull")

    def _issuer(self):
        nt = self.nt

        def issue_s(j):
            bar, n = self._kfull(j)
            yield ("wait", bar, n)
            yield ("mma", 0, "S", j)
            yield ("commit", 0, "SFull%d" % (j & 1), j >> 1)

        yield ("wait", "Q", 0)
        yield from issue_s(0)
        if nt > 1:
            yield from issue_s(1)
        for j in range(nt):
            if self.tmut.s_before_pv and j + 2 < nt:
                yield from issue_s(j + 2)
            yield ("wait", "PFull", j)
            yield ("wait", "VFull", j)
            if self.tmut.oready_before_pv:
                yield ("commit", 0, "OReady", j)
            yield ("mma", 0, "PV", j)
            if not self.tmut.oready_before_pv:
                yield ("commit", 0, "OReady", j)
            if j + 2 < nt and not self.tmut.s_before_pv:
                yield from issue_s(j + 2)

    def _softmax(self, w: int):
        me = "smx%d" % w
        nt = self.nt
        for j in range(nt):
            yield ("wait", "SFull%d" % (j & 1), j >> 1)
            yield ("t_read_S", w, j)
            yield ("t_write_P", w, j)
            rescale = j > 0 and self.rng.random() < self.rescale_prob
            if j > 0 and (rescale or not self.tmut.pfull_without_oready):
                yield ("wait", "OReady", j - 1)
            if rescale:
                yield ("t_rescale", w, j)
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
            S = self.Sbuf[j & 1]
            if S["tag"] != j or w not in S["readers"]:
                raise ProtocolViolation("warp %d writes P(%d) over S buffer %d holding %s" % (w, j, j & 1, S["tag"]))
            S["P"][w] = j
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
            j = op[3]
            self._read_smem("Q", 0)
            for s in range(K_SLICES):
                self._read_smem("K%d" % ((K_SLICES * j + s) % K_SLOTS), (j, s))
            S = self.Sbuf[j & 1]
            if S["tag"] is not None:
                if len(S["readers"]) != 4:
                    raise ProtocolViolation("S(%d) overwrites S(%d) read by warps %s only"
                                            % (j, S["tag"], sorted(S["readers"])))
                if not S["pv"]:
                    raise ProtocolViolation("S(%d) overwrites P(%d) before PV(%d) read it" % (j, S["tag"], S["tag"]))
            self.Sbuf[j & 1] = {"tag": j, "readers": set(), "P": [None] * 4, "pv": False}
            return
        j = op[3]
        self._read_smem("V", j)
        S = self.Sbuf[j & 1]
        if S["tag"] != j or any(p != j for p in S["P"]):
            raise ProtocolViolation("PV(%d) reads P rows %s of S buffer holding %s" % (j, S["P"], S["tag"]))
        if self.Odone != set(range(j)):
            raise ProtocolViolation("PV(%d) out of order (done %s)" % (j, sorted(self.Odone)))
        S["pv"] = True
        self.Odone.add(j)
