"""Executable model of the online-chunking walk of segment_walk_kernel
(dynamic_hierarchical_sparse_b200/csrc/segment.cu), restated as sequential
Python so that its algorithm can be checked against the oracle's rule on the
CPU.

The rule (oracle.segment_sequence): from a chunk start b, the next start is the
first drop in [b + min_len, b + max_len), else b + max_len while that is inside
the sequence.  The kernel takes it window by window (`win_words` bitmap words
at a time):

* every drop of the window is a possible chunk start ("node"); the rule's step
  from each node is taken independently (`walk_from`): the first drop that
  becomes a start, after a run of forced starts x + max_len, x + 2 max_len, ...
  counted in closed form, or the end of the sequence, or "out" (the step needs
  bits past the window);
* the nodes reached from the window's first start are found by pointer jumping
  (round r marks the nodes 2^r .. 2^(r+1) - 1 steps on); the kernel's in-round
  reads and writes race, modelled here by a random order of the updates;
* a window with more drops than `node_cap` is walked step by step, at most
  `start_buf` starts per round.

`run` returns the set of chunk starts and checks on the way that the marked
set is exactly the reachable one and that one node ends the chain.
"""

from __future__ import annotations

import bisect
import random
from typing import List, Sequence

K_NONE = 0x7FFFFFFF
K_END = -1
K_OUT = -2


def walk_from(pos: List[int], x: int, wb: int, n: int, full: bool, s1: int, min_len: int, max_len: int):
    """The rule's step from a start x within the window [32 wb, 32 (wb + n)):
    (next drop start's index | K_END | K_OUT, forced starts on the way, last start)."""
    forced = 0
    while True:
        clo = x + min_len
        if clo >= s1:
            return K_END, forced, x
        xm = x + max_len
        chi = min(xm, s1)
        if ((chi - 1) >> 5) >= wb + n:
            return K_OUT, forced, x
        idx, f = len(pos), K_NONE
        if clo < chi:  # an empty interval (min_len == max_len) needs no lookup
            idx = bisect.bisect_left(pos, clo)
            if idx < len(pos):
                f = pos[idx]
        if f < chi:
            return idx, forced, x
        if xm >= s1:
            return K_END, forced, x
        if f == K_NONE:
            if full:  # no drop up to the end: forced starts while below s1
                k = (s1 - 1 - x) // max_len
                return K_END, forced + k, x + k * max_len
            room = ((wb + n) << 5) - x  # forced starts while their rule window stays inside
            k = max(1, room // max_len - 1)
            x += k * max_len
            forced += k
            continue
        k = (f - x) // max_len  # f >= x + max_len: starts up to f are forced
        assert k >= 1
        x += k * max_len
        forced += k


def run(drops: Sequence[int], s0: int, s1: int, min_len: int, max_len: int, win_words: int = 4096,
        node_cap: int = 8192, start_buf: int = 1024, rng: random.Random = None) -> List[int]:
    """Chunk starts of tokens [s0, s1) with drops at `drops` (ascending)."""
    rng = rng or random.Random(0)
    words = (s1 + 31) // 32
    bits = [0] * (words + 4)
    for p in drops:
        bits[p >> 5] |= 1 << (p & 31)
    last_word = (s1 - 1) >> 5
    starts = {s0}
    b, wb, n, full = s0, -1, 0, False
    pos: List[int] = []
    nxt: List[int] = []
    kk: List[int] = []
    nd: List[int] = []
    win: List[int] = []
    for _ in range(1_000_000):
        lo = b + min_len
        if lo >= s1:
            break
        hi = min(b + max_len, s1)
        if wb < 0 or ((hi - 1) >> 5) >= wb + win_words:
            wb = (lo >> 5) & ~3
            n = min(win_words, last_word + 1 - wb)
            full = wb + n > last_word
            win = [bits[wb + i] for i in range(n)]
            pos = []
            for i in range(n):
                m = win[i]
                while m:
                    pos.append(((wb + i) << 5) + ((m & -m).bit_length() - 1))
                    m &= m - 1
            if len(pos) <= node_cap:
                steps = [walk_from(pos, x, wb, n, full, s1, min_len, max_len) for x in pos]
                nxt = [st[0] for st in steps]
                kk = [st[1] for st in steps]
            else:
                nd = [K_NONE] * (n + 1)
                run_ = K_NONE
                for i in range(n - 1, -1, -1):
                    if win[i]:
                        run_ = ((wb + i) << 5) + ((win[i] & -win[i]).bit_length() - 1)
                    nd[i] = run_
        if len(pos) <= node_cap:
            nodes = len(pos)
            f, forced, last = walk_from(pos, b, wb, n, full, s1, min_len, max_len)
            for k in range(1, forced + 1):
                starts.add(b + k * max_len)
            new_b, done = last, f == K_END
            if f >= 0:
                on = [j == f for j in range(nodes)]
                jump = list(nxt)
                span = 1
                while span <= nodes:
                    order = list(range(nodes))
                    rng.shuffle(order)
                    new = [0] * nodes
                    for j in order:
                        t = jump[j]
                        if t >= 0:
                            if on[j]:
                                on[t] = True
                            new[j] = jump[t]
                        else:
                            new[j] = t
                    jump = new
                    span <<= 1
                reach, j = set(), f
                while j >= 0:
                    reach.add(j)
                    j = nxt[j]
                assert {j for j in range(nodes) if on[j]} == reach, "pointer jumping missed or added a node"
                ends = 0
                for j in range(nodes):
                    if not on[j]:
                        continue
                    for q in range(kk[j] + 1):
                        starts.add(pos[j] + q * max_len)
                    if nxt[j] < 0:
                        ends += 1
                        new_b, done = pos[j] + kk[j] * max_len, nxt[j] == K_END
                assert ends == 1, "the chain must end at exactly one node"
            assert done or new_b > b, "a round that leaves the window must move the walk on"
            b = new_b
            if done:
                break
            continue
        ne, done, cb = 0, False, b
        while ne < start_buf:
            clo = cb + min_len
            if clo >= s1:
                done = True
                break
            chi = min(cb + max_len, s1)
            if ((chi - 1) >> 5) >= wb + n:
                break
            f = K_NONE
            if clo < chi:
                wl = clo >> 5
                assert 0 <= wl - wb < n, "the step-by-step walk reads inside the window"
                m = win[wl - wb] & ((0xFFFFFFFF << (clo & 31)) & 0xFFFFFFFF)
                f = (wl << 5) + ((m & -m).bit_length() - 1) if m else nd[wl - wb + 1]
            if f < chi:
                nx = f
            elif cb + max_len < s1:
                nx = cb + max_len
            else:
                done = True
                break
            starts.add(nx)
            ne += 1
            cb = nx
        b = cb
        if done:
            break
    else:
        raise AssertionError("the walk made no progress")
    assert all(s0 <= q < s1 for q in starts)
    return sorted(starts)
