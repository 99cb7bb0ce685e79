"""fp64 CPU oracle for the DHSA prefill path.  TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  The product path (the CUDA library and its
Python binding) never calls it, and it shares no code with that path.

What it computes, step by step, in the order the method's pages give them
("Long-Context Modeling with Dynamic Hierarchical Sparse Attention for
On-Device LLMs", Abstract and AI Summary; "Long-Context Modeling with Dynamic
Hierarchical Sparse Attention for Memory-Constrained LLM Inference",
abstract):

1. ``chunk_representations``: each variable-length chunk is aggregated into one
   vector: the mean of its tokens' vectors times sqrt(L), L the chunk length
   (length-normalised aggregation; On-Device page, Abstract).  Mean times
   sqrt(L) equals sum divided by sqrt(L).
2. ``chunk_scores``: chunk-level similarity is the dot product of a query-chunk
   representation and a key-chunk representation (On-Device page, Abstract:
   similarity is scored between chunks).
3. ``build_plan``: the chunk score is upsampled to token level (every token pair
   of chunks (i, j) inherits score(i, j)); for each query chunk the top-k
   causally admissible key chunks (earlier chunks of the same sequence) are kept
   by (score descending, chunk index ascending), and the diagonal chunk is kept
   in addition (On-Device page, Abstract: the chunk scores are carried down to
   token level, where they act as the importance of each token interaction;
   Memory-Constrained page, abstract: importance is judged per chunk, handed on
   to the token interactions, and the causal dependencies that matter are
   kept).  Because every token of a chunk pair inherits one score,
   selecting the best tokens by upsampled score keeps whole chunks;
   ``attention_literal`` re-derives the keep set from the materialised
   token-level score matrix to check that equivalence.
4. ``attention_query_chunk`` / ``attention_gather`` / ``attention_literal`` /
   ``attention_rows``: causal
   softmax attention of each query token over the kept key tokens only.

Readings taken where the pages are silent (each listed in the design notes):
per-head Q/K as the per-token vectors that are aggregated; plain dot product without 1/sqrt(d);
admissible key chunks are j < i in the same sequence, the diagonal is added on
top of k; k above the admissible count keeps all; a fractional budget keeps
ceil(i_local * num / den) chunks (integer arithmetic) capped at i_local; ties go
to the lower chunk index; plans are per query head (GQA head h reads KV head
h // (Hq/Hkv)); softmax scale 1/sqrt(d) unless given.

Grouped-query variant (the pages never mention GQA; this is an added mode):
``per_kv_head=True`` builds one plan row per (KV head g, query chunk i), scored
by the sum of the chunk scores of g's query heads; every query head of the
group then attends over that row.  ``group_chunk_scores`` writes the sum out
head by head.

Online segmentation (step 0; the pages say the sequence is segmented into
variable-length chunks adaptively and online, but give no rule):
``segment`` applies this library's stated rule.  Tokens are taken left to
right within each sequence; with the current chunk starting at token b, token t
starts a new chunk when t - b >= max_len, or when t - b >= min_len and the
similarity of t to its predecessor, the mean over KV heads of the cosine of
k[t-1] and k[t] (``adjacent_key_similarity``), is below the threshold.  A
zero key has cosine 1 with anything (it never breaks a chunk).

All arithmetic is numpy float64.  Inputs may be bf16/fp32 torch tensors or
numpy arrays; they are upcast exactly.
"""

from __future__ import annotations

import math
from typing import Dict, Iterable, List, Optional, Sequence, Tuple

import numpy as np

TOPK = 0
FRACTION = 1


def as_f64(x) -> np.ndarray:
    """Exact upcast of a torch tensor (bf16/fp32) or array to numpy float64."""
    if hasattr(x, "detach"):
        import torch  # only for the upcast of the caller's tensors
        return x.detach().to(torch.float64).cpu().numpy()
    return np.asarray(x, dtype=np.float64)


def chunk_of_token(chunk_bounds: np.ndarray) -> np.ndarray:
    """c(t): the chunk index of every token."""
    bounds = np.asarray(chunk_bounds, dtype=np.int64)
    lens = np.diff(bounds)
    return np.repeat(np.arange(lens.shape[0]), lens)


def sequence_of_chunk(seq_chunk_ptr: np.ndarray, num_chunks: int) -> np.ndarray:
    ptr = np.asarray(seq_chunk_ptr, dtype=np.int64)
    out = np.empty(num_chunks, dtype=np.int64)
    for b in range(ptr.shape[0] - 1):
        out[ptr[b]:ptr[b + 1]] = b
    return out


# ---------------------------------------------------------------- step 1 ---
def chunk_representations(x, chunk_bounds) -> np.ndarray:
    """Length-normalised chunk aggregation (On-Device page, Abstract).

    ``x``: [T, H, d].  Returns [H, n, d] with rep[h, c] = mean(x[c]) * sqrt(L_c),
    computed as sum(x[c]) / sqrt(L_c) (the same number, fewer roundings).
    """
    bounds = np.asarray(chunk_bounds, dtype=np.int64)
    n = bounds.shape[0] - 1
    T, H, d = x.shape
    reps = np.zeros((H, n, d), dtype=np.float64)
    for c in range(n):
        s, e = int(bounds[c]), int(bounds[c + 1])
        reps[:, c, :] = as_f64(x[s:e]).sum(axis=0) / math.sqrt(e - s)
    return reps


# ---------------------------------------------------------------- step 2 ---
def chunk_scores(qc: np.ndarray, kc: np.ndarray, seq_chunk_ptr) -> np.ndarray:
    """Chunk-chunk dot-product similarity (On-Device page, Abstract).

    Returns S [Hq, n, n] with S[h, i, j] = qc[h, i] . kc[g(h), j] for j <= i in
    the same sequence and NaN elsewhere (never scored: future or other sequence).
    """
    Hq, n, d = qc.shape
    Hkv = kc.shape[0]
    group = Hq // Hkv
    seq_of = sequence_of_chunk(seq_chunk_ptr, n)
    S = np.full((Hq, n, n), np.nan, dtype=np.float64)
    for h in range(Hq):
        g = h // group
        for i in range(n):
            for j in range(i + 1):
                if seq_of[j] == seq_of[i]:
                    S[h, i, j] = float(np.dot(qc[h, i], kc[g, j]))
    return S


def group_chunk_scores(qc: np.ndarray, kc: np.ndarray, seq_chunk_ptr) -> np.ndarray:
    """Chunk scores of a KV group: S_g[g, i, j] = sum over the query heads h of
    group g of qc[h, i] . kc[g, j] (same support as ``chunk_scores``)."""
    S = chunk_scores(qc, kc, seq_chunk_ptr)
    Hq = qc.shape[0]
    Hkv = kc.shape[0]
    group = Hq // Hkv
    out = np.zeros((Hkv,) + S.shape[1:], dtype=np.float64)
    for g in range(Hkv):
        for r in range(group):
            out[g] += S[g * group + r]
    return out


# ---------------------------------------------------------------- step 3 ---
def row_budget(i_local: int, kind: int, k: int = 0, num: int = 0, den: int = 1) -> int:
    """How many admissible key chunks a query chunk keeps (diagonal not counted).

    TOPK: min(k, i_local).  FRACTION: min(i_local, ceil(i_local * num / den)) in
    integer arithmetic.  i_local = number of earlier chunks in the sequence.
    """
    if kind == TOPK:
        return min(int(k), int(i_local))
    if kind == FRACTION:
        want = -((-int(i_local) * int(num)) // int(den))  # ceil division
        return min(int(i_local), want)
    raise ValueError("unknown budget kind")


def select_row(scores: Sequence[float], candidates: Sequence[int], keep: int) -> List[int]:
    """Top-``keep`` candidates ordered by (score descending, index ascending)."""
    order = sorted(range(len(candidates)), key=lambda t: (-scores[t], candidates[t]))
    return [int(candidates[t]) for t in order[:keep]]


def build_plan(q, k, chunk_bounds, seq_chunk_ptr, budget_kind: int, k_top: int = 0,
               num: int = 0, den: int = 1, per_kv_head: bool = False):
    """The full planning step: representations, scores, per-row selection.

    Returns a dict with
      ``row_ptr`` int64 [Hq*n+1] and ``col`` int64 [nnz]: CSR over rows r = h*n+i,
        each row ascending global chunk ids with the diagonal i last (with
        ``per_kv_head``: [Hkv*n+1] over rows r = g*n+i, scored by
        ``group_chunk_scores``);
      ``qc``, ``kc``, ``S``: the intermediate fp64 quantities;
      ``kth`` float64 [Hq*n, 2]: the k-th and (k+1)-th best admissible scores of
        the row (NaN where they do not exist), for tie analysis;
      ``rowmax`` float64 [Hq*n]: max |S| over the row's admissible candidates.
    """
    qc = chunk_representations(q, chunk_bounds)
    kc = chunk_representations(k, chunk_bounds)
    S = group_chunk_scores(qc, kc, seq_chunk_ptr) if per_kv_head else chunk_scores(qc, kc, seq_chunk_ptr)
    Hq, n = S.shape[0], S.shape[1]
    ptr = np.asarray(seq_chunk_ptr, dtype=np.int64)
    row_ptr = np.zeros(Hq * n + 1, dtype=np.int64)
    cols: List[int] = []
    kth = np.full((Hq * n, 2), np.nan)
    rowmax = np.zeros(Hq * n)
    for h in range(Hq):
        for b in range(ptr.shape[0] - 1):
            c0, c1 = int(ptr[b]), int(ptr[b + 1])
            for i in range(c0, c1):
                r = h * n + i
                cand = list(range(c0, i))
                sc = [float(S[h, i, j]) for j in cand]
                keep = row_budget(i - c0, budget_kind, k_top, num, den)
                chosen = select_row(sc, cand, keep)
                ordered = sorted(sc, reverse=True)
                if keep >= 1 and keep <= len(ordered):
                    kth[r, 0] = ordered[keep - 1]
                if keep < len(ordered):
                    kth[r, 1] = ordered[keep]
                if sc:
                    rowmax[r] = max(abs(s) for s in sc)
                row = sorted(chosen) + [i]
                cols.extend(row)
                row_ptr[r + 1] = row_ptr[r] + len(row)
    # rows are emitted in (h, b, i) order == (h, i) order since sequences are consecutive
    return {"row_ptr": row_ptr, "col": np.asarray(cols, dtype=np.int64), "qc": qc,
            "kc": kc, "S": S, "kth": kth, "rowmax": rowmax}


def plan_rows(row_ptr, col) -> List[List[int]]:
    rp = np.asarray(row_ptr, dtype=np.int64)
    cl = np.asarray(col, dtype=np.int64)
    return [[int(x) for x in cl[rp[r]:rp[r + 1]]] for r in range(rp.shape[0] - 1)]


# ---------------------------------------------------------------- step 4 ---
def _softmax_rows(logits: np.ndarray) -> np.ndarray:
    m = np.max(logits, axis=-1, keepdims=True)
    e = np.exp(logits - m)
    return e / e.sum(axis=-1, keepdims=True)


def attention_query_chunk(q, k, v, chunk_bounds, row_ptr, col, h: int, i: int,
                          scale: Optional[float] = None, per_kv_head: bool = False) -> np.ndarray:
    """Sparse causal attention of the tokens of query chunk i, head h.

    The kept key chunks' tokens (plan row h*n+i, or g*n+i for a per-KV-head
    plan) are concatenated; each query token t attends to the kept tokens
    s <= t with softmax weights of q_t . k_s * scale and averages v_s.
    Returns [L_i, d] float64.
    """
    Hq, d = q.shape[1], q.shape[2]
    group = Hq // k.shape[1]
    g = h // group
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    bounds = np.asarray(chunk_bounds, dtype=np.int64)
    n = bounds.shape[0] - 1
    rp = np.asarray(row_ptr, dtype=np.int64)
    cl = np.asarray(col, dtype=np.int64)
    r = (g if per_kv_head else h) * n + i
    kept = cl[rp[r]:rp[r + 1]]
    key_tok = np.concatenate([np.arange(bounds[j], bounds[j + 1]) for j in kept])
    qs = np.arange(bounds[i], bounds[i + 1])
    qq = as_f64(q[int(bounds[i]):int(bounds[i + 1]), h, :])
    kk = as_f64(k[:, g, :][key_tok])
    vv = as_f64(v[:, g, :][key_tok])
    logits = (qq @ kk.T) * scale
    logits = np.where(key_tok[None, :] <= qs[:, None], logits, -np.inf)
    return _softmax_rows(logits) @ vv


def attention_gather(q, k, v, chunk_bounds, row_ptr, col, scale: Optional[float] = None,
                     heads: Optional[Iterable[int]] = None, per_kv_head: bool = False) -> np.ndarray:
    """Sparse causal attention, chunk-gather form, for every query chunk.

    Returns O [T, Hq, d] float64 (rows of heads not in ``heads`` stay zero).
    """
    T, Hq, d = q.shape
    bounds = np.asarray(chunk_bounds, dtype=np.int64)
    n = bounds.shape[0] - 1
    out = np.zeros((T, Hq, d), dtype=np.float64)
    for h in (range(Hq) if heads is None else heads):
        for i in range(n):
            out[bounds[i]:bounds[i + 1], h, :] = attention_query_chunk(q, k, v, bounds, row_ptr, col, h, i,
                                                                       scale, per_kv_head)
    return out


def attention_rows(q, k, v, chunk_bounds, row_ptr, col, rows: Sequence[Tuple[int, int]],
                   scale: Optional[float] = None, per_kv_head: bool = False) -> np.ndarray:
    """Output of single (token t, head h) rows, one at a time (for large inputs)."""
    d = q.shape[2]
    Hq, Hkv = q.shape[1], k.shape[1]
    group = Hq // Hkv
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    bounds = np.asarray(chunk_bounds, dtype=np.int64)
    n = bounds.shape[0] - 1
    rp = np.asarray(row_ptr, dtype=np.int64)
    cl = np.asarray(col, dtype=np.int64)
    out = np.zeros((len(rows), d), dtype=np.float64)
    for idx, (t, h) in enumerate(rows):
        i = int(np.searchsorted(bounds, t, side="right") - 1)
        g = h // group
        r = (g if per_kv_head else h) * n + i
        kept = cl[rp[r]:rp[r + 1]]
        key_tok = np.concatenate([np.arange(bounds[j], bounds[j + 1]) for j in kept])
        key_tok = key_tok[key_tok <= t]
        qt = as_f64(q[t, h, :])
        kk = as_f64(k[key_tok, g, :])
        vv = as_f64(v[key_tok, g, :])
        logits = (kk @ qt) * scale
        p = np.exp(logits - logits.max())
        out[idx] = (p / p.sum()) @ vv
    return out


def attention_literal(q, k, v, cu_seqlens, chunk_bounds, seq_chunk_ptr, S: np.ndarray,
                      budget_kind: int, k_top: int = 0, num: int = 0, den: int = 1,
                      scale: Optional[float] = None):
    """Sparse attention through the materialised token-level score matrix.

    Upsamples S to token level, ``score_tok[h, t, s] = S[h, c(t), c(s)]``, and
    derives the keep mask token by token: key token s is kept for query token t
    when s <= t in the same sequence and either s lies in t's own chunk or the
    pair (score_tok[t, s], c(s)) ranks among the row's best ``k_t`` distinct
    (score, chunk) keys of earlier chunks.  Meant for tiny inputs (T <= 8192).
    Returns (O [T, Hq, d], keep mask [Hq, T, T] bool, score_tok [Hq, T, T]).
    """
    q64, k64, v64 = as_f64(q), as_f64(k), as_f64(v)
    T, Hq, d = q64.shape
    Hkv = k64.shape[1]
    group = Hq // Hkv
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    cot = chunk_of_token(chunk_bounds)
    n = np.asarray(chunk_bounds).shape[0] - 1
    seq_of_chunk = sequence_of_chunk(seq_chunk_ptr, n)
    seq_of_tok = seq_of_chunk[cot]
    ptr = np.asarray(seq_chunk_ptr, dtype=np.int64)
    score_tok = np.full((Hq, T, T), np.nan)
    keep = np.zeros((Hq, T, T), dtype=bool)
    out = np.zeros((T, Hq, d))
    tt = np.arange(T)
    for h in range(Hq):
        score_tok[h] = S[h][cot[:, None], cot[None, :]]
        g = h // group
        for t in range(T):
            ci = cot[t]
            b = seq_of_tok[t]
            same = (seq_of_tok == b) & (tt <= t)
            earlier = same & (cot < ci)
            # distinct (score, chunk) keys present in the upsampled row
            keys = sorted({(-score_tok[h, t, s], int(cot[s])) for s in np.nonzero(earlier)[0]})
            kt = row_budget(ci - ptr[b], budget_kind, k_top, num, den)
            best = {c for (_, c) in keys[:kt]}
            row_keep = same & ((cot == ci) | np.isin(cot, list(best)))
            keep[h, t] = row_keep
            logits = (k64[row_keep, g, :] @ q64[t, h, :]) * scale
            p = np.exp(logits - logits.max())
            out[t, h] = (p / p.sum()) @ v64[row_keep, g, :]
    return out, keep, score_tok


def kept_pairs(chunk_bounds, row_ptr, col, num_q_heads: int, group: int = 1) -> int:
    """Exact number of (query token, key token, head) pairs the plan keeps.

    ``group`` > 1: a per-KV-head plan whose rows serve ``group`` query heads."""
    bounds = np.asarray(chunk_bounds, dtype=np.int64)
    lens = np.diff(bounds)
    n = lens.shape[0]
    rp = np.asarray(row_ptr, dtype=np.int64)
    cl = np.asarray(col, dtype=np.int64)
    total = 0
    for r in range((num_q_heads // group) * n):
        i = r % n
        Li = int(lens[i])
        for j in cl[rp[r]:rp[r + 1]]:
            total += (Li * (Li + 1) // 2 if j == i else Li * int(lens[j])) * group
    return total


# ------------------------------------------------- step 0 (added mode) ---
def adjacent_key_similarity(k) -> np.ndarray:
    """sim[t] = (1/Hkv) sum_g cos(k[t-1, g], k[t, g]) for t >= 1; sim[0] = NaN.

    cos(x, y) = x.y / (|x| |y|), and 1 when either vector is zero.  Sequence
    edges are not looked at here; ``segment`` never reads sim at a sequence's
    first token.
    """
    K = as_f64(k)
    T = K.shape[0]
    sim = np.full(T, np.nan)
    if T < 2:
        return sim
    dot = np.einsum("thd,thd->th", K[:-1], K[1:])
    norm = np.sqrt(np.einsum("thd,thd->th", K, K))
    den = norm[:-1] * norm[1:]
    cos = np.ones_like(dot)
    nz = den > 0
    cos[nz] = dot[nz] / den[nz]
    sim[1:] = cos.mean(axis=1)
    return sim


def segment_sequence(sim: np.ndarray, start: int, end: int, threshold: float, min_len: int,
                     max_len: int) -> List[int]:
    """Chunk starts of tokens [start, end) under the greedy online rule."""
    if end <= start:
        return []
    starts = [start]
    b = start
    for t in range(start + 1, end):
        if t - b >= max_len or (t - b >= min_len and sim[t] < threshold):
            starts.append(t)
            b = t
    return starts


def segment(k, cu_seqlens, threshold: float, min_len: int, max_len: int):
    """Online variable-length chunking of every sequence of a packed batch.

    Returns (chunk_bounds int32 [n+1], seq_chunk_ptr int32 [B+1]) in the
    layout the rest of the path takes.
    """
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    sim = adjacent_key_similarity(k)
    bounds: List[int] = []
    ptr = [0]
    for b in range(cu.shape[0] - 1):
        bounds += segment_sequence(sim, int(cu[b]), int(cu[b + 1]), threshold, min_len, max_len)
        ptr.append(len(bounds))
    bounds.append(int(cu[-1]))
    return np.asarray(bounds, dtype=np.int32), np.asarray(ptr, dtype=np.int32)
