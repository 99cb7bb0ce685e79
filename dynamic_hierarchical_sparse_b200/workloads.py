"""Seeded synthetic workloads for the DHSA prefill path.

This module only *makes inputs*: token tensors, sequence offsets, chunk
boundaries and budgets.  It holds none of the method's arithmetic (no chunk
aggregation, scoring, selection or attention), so both the CUDA path and the
fp64 oracle can consume what it produces without sharing any method code.

The five named workloads mirror the shapes the DHSA pages measure on
("Long-Context Modeling with Dynamic Hierarchical Sparse Attention for
On-Device LLMs", Abstract: Gemma2; "... for Memory-Constrained LLM Inference",
abstract: LLaMA-3.1-8B at up to 128K context).  The pages use NIAH, LongBench
and RULER; those suites are not available here, so seeded synthetic tensors of
the same attention shapes stand in for them.

Recipe (one generator per quantity, all seeded):

* chunk lengths come from ``numpy.random.default_rng(seed)``;
* token values come from ``torch.Generator('cpu').manual_seed(seed)``, drawn in
  fp32 and cast to the workload dtype;
* the "structured" value mix is ``X = Z + 2 * A @ B`` with ``Z, A, B ~ N(0,1)``,
  ``A`` of shape ``[T, 4]`` drawn per tensor and per head, ``B`` of shape
  ``[4, d]`` shared by the query heads of a KV group and that group's K head
  (V draws its own ``B`` and is divided by sqrt(17), its standard deviation,
  so outputs are O(1)).  The shared rank-4 part gives hub ("sink-like") keys
  and peaky attention rows;
* the ragged workload plants one "needle" key chunk per sequence: every K token
  of a seeded chunk ``j*`` is set, per KV head ``g``, to ``4 * m / |m|`` where
  ``m`` is the mean query (head ``g * Hq/Hkv``) over the sequence's last chunk.
"""

from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence

import numpy as np
import torch

BUDGET_TOPK = 0
BUDGET_FRACTION = 1


@dataclasses.dataclass(frozen=True)
class Budget:
    """Per-query-chunk key-chunk budget.

    ``kind == BUDGET_TOPK``: keep ``k`` admissible key chunks.
    ``kind == BUDGET_FRACTION``: keep ``num/den`` of the admissible key chunks
    (rounded up).  The diagonal chunk is kept in addition in both cases.
    ``per_kv_head``: one plan row per KV head instead of per query head.
    """

    kind: int
    k: int = 0
    num: int = 0
    den: int = 1
    per_kv_head: bool = False  # one plan row per KV head (grouped-query mode)

    @staticmethod
    def topk(k: int) -> "Budget":
        return Budget(BUDGET_TOPK, k=int(k))

    @staticmethod
    def fraction(num: int, den: int) -> "Budget":
        return Budget(BUDGET_FRACTION, num=int(num), den=int(den))

    def kv(self) -> "Budget":
        """The same budget for a per-KV-head plan."""
        return dataclasses.replace(self, per_kv_head=True)


@dataclasses.dataclass(frozen=True)
class SegmentRule:
    """Parameters of the online chunking rule.

    Within a sequence, with the current chunk starting at token b, token t
    starts a new chunk when ``t - b >= max_len``, or when ``t - b >= min_len``
    and t's adjacent-key similarity (mean over KV heads of cos(k[t-1], k[t]))
    is below ``threshold``.
    """

    threshold: float
    min_len: int
    max_len: int


@dataclasses.dataclass(frozen=True)
class WorkloadSpec:
    name: str
    seq_lens: Sequence[int]
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    dtype: str  # "bf16" or "f32"
    chunk_lo: int
    chunk_hi: int
    budget: Budget
    values: str  # "normal" or "structured"
    needle: bool = False
    fixed_num_chunks: Optional[int] = None  # rescaled-lengths recipe

    @property
    def total_tokens(self) -> int:
        return int(sum(self.seq_lens))


# The five workloads.  Names say what they are; sizes are in the fields.
TINY_1K_F32 = WorkloadSpec(
    "tiny_1k_h1_d64_f32_top4", [1024], 1, 1, 64, "f32", 32, 128,
    Budget.topk(4), "normal", fixed_num_chunks=16)
GEMMA2_8K = WorkloadSpec(
    "gemma2_2b_8k_h8kv4_d256_bf16_top16", [8192], 8, 4, 256, "bf16", 64, 256,
    Budget.topk(16), "structured")
LLAMA_32K = WorkloadSpec(
    "llama31_8b_32k_h32kv8_d128_bf16_frac10", [32768], 32, 8, 128, "bf16", 128,
    512, Budget.fraction(1, 10), "structured")
LLAMA_128K = WorkloadSpec(
    "llama31_8b_128k_h32kv8_d128_bf16_frac5", [131072], 32, 8, 128, "bf16", 256,
    1024, Budget.fraction(1, 20), "structured")
RAGGED_NEEDLE = WorkloadSpec(
    "ragged4_4k8k12k16k_h32kv8_d128_bf16_top8_needle", [4096, 8192, 12288, 16384],
    32, 8, 128, "bf16", 64, 512, Budget.topk(8), "normal", needle=True)

WORKLOADS = [TINY_1K_F32, GEMMA2_8K, LLAMA_32K, LLAMA_128K, RAGGED_NEEDLE]

# Fixed-length chunks: DHSA with every chunk 512 tokens long is plain
# block-sparse attention with 512-token blocks (the comparison baseline the
# pages name), run through the same kernels, on the 128K shape.
BLOCKSPARSE_128K = WorkloadSpec(
    "blocksparse512_128k_h32kv8_d128_bf16_frac5", [131072], 32, 8, 128, "bf16", 512,
    512, Budget.fraction(1, 20), "structured")
EXTRA_WORKLOADS = [BLOCKSPARSE_128K]
BY_NAME = {w.name: w for w in WORKLOADS + EXTRA_WORKLOADS}


@dataclasses.dataclass
class Inputs:
    spec: WorkloadSpec
    seed: int
    q: torch.Tensor  # [T, Hq, d] (workload dtype, CPU)
    k: torch.Tensor  # [T, Hkv, d]
    v: torch.Tensor  # [T, Hkv, d]
    cu_seqlens: np.ndarray  # int32 [B+1]
    chunk_bounds: np.ndarray  # int32 [n+1] global token offsets
    seq_chunk_ptr: np.ndarray  # int32 [B+1]
    budget: Budget
    needle_chunks: Optional[List[int]] = None  # global chunk id of j* per sequence

    @property
    def num_chunks(self) -> int:
        return int(self.chunk_bounds.shape[0] - 1)


def chunk_lengths_fixed_count(rng: np.random.Generator, total: int, count: int,
                              lo: int, hi: int) -> List[int]:
    """``count`` lengths U[lo,hi], rescaled so they sum to ``total`` exactly."""
    raw = rng.integers(lo, hi + 1, size=count).astype(np.float64)
    cum = np.round(total * np.cumsum(raw) / raw.sum()).astype(np.int64)
    cum[-1] = total
    edges = np.concatenate([[0], cum])
    lens = np.diff(edges)
    if (lens <= 0).any():
        raise ValueError("rescaled chunk length fell to zero")
    return [int(x) for x in lens]


def chunk_lengths_until(rng: np.random.Generator, total: int, lo: int,
                        hi: int) -> List[int]:
    """Draw U[lo,hi] lengths until they cover ``total``; the last is truncated."""
    lens: List[int] = []
    acc = 0
    while acc < total:
        L = int(rng.integers(lo, hi + 1))
        L = min(L, total - acc)
        lens.append(L)
        acc += L
    return lens


def make_bounds(seq_lens: Sequence[int], per_seq_chunk_lens: Sequence[Sequence[int]]):
    cu = np.zeros(len(seq_lens) + 1, dtype=np.int64)
    cu[1:] = np.cumsum(seq_lens)
    bounds = [0]
    seq_ptr = [0]
    for b, lens in enumerate(per_seq_chunk_lens):
        if sum(lens) != seq_lens[b]:
            raise ValueError("chunk lengths do not cover the sequence")
        for L in lens:
            if L <= 0:
                raise ValueError("chunk length must be positive")
            bounds.append(bounds[-1] + int(L))
        seq_ptr.append(len(bounds) - 1)
    return (cu.astype(np.int32), np.asarray(bounds, dtype=np.int32),
            np.asarray(seq_ptr, dtype=np.int32))


def _structured(gen: torch.Generator, T: int, H: int, d: int,
                Bmats: torch.Tensor, head_to_b: Sequence[int]) -> torch.Tensor:
    z = torch.randn(T, H, d, generator=gen, dtype=torch.float32)
    for h in range(H):
        a = torch.randn(T, 4, generator=gen, dtype=torch.float32)
        z[:, h, :] += 2.0 * (a @ Bmats[head_to_b[h]])
    return z


def generate(spec: WorkloadSpec, seed: int = 0, seq_lens: Optional[Sequence[int]] = None,
             budget: Optional[Budget] = None) -> Inputs:
    """Build the seeded inputs of ``spec`` (optionally with other sequence lengths)."""
    seq_lens = list(spec.seq_lens if seq_lens is None else seq_lens)
    budget = spec.budget if budget is None else budget
    rng = np.random.default_rng(seed)
    per_seq = []
    for L in seq_lens:
        if spec.fixed_num_chunks is not None:
            per_seq.append(chunk_lengths_fixed_count(rng, L, spec.fixed_num_chunks,
                                                     spec.chunk_lo, spec.chunk_hi))
        else:
            per_seq.append(chunk_lengths_until(rng, L, spec.chunk_lo, spec.chunk_hi))
    cu, bounds, seq_ptr = make_bounds(seq_lens, per_seq)
    T = int(cu[-1])
    Hq, Hkv, d = spec.num_q_heads, spec.num_kv_heads, spec.head_dim
    gen = torch.Generator("cpu").manual_seed(seed)
    if spec.values == "structured":
        group = Hq // Hkv
        bq = torch.randn(Hkv, 4, d, generator=gen, dtype=torch.float32)
        bv = torch.randn(Hkv, 4, d, generator=gen, dtype=torch.float32)
        q = _structured(gen, T, Hq, d, bq, [h // group for h in range(Hq)])
        k = _structured(gen, T, Hkv, d, bq, list(range(Hkv)))
        # V at unit per-element variance (Z + 2AB has variance 1 + 16) so that
        # attention outputs stay O(1), the regime the absolute error gate is for
        v = _structured(gen, T, Hkv, d, bv, list(range(Hkv))) / math.sqrt(17.0)
    else:
        q = torch.randn(T, Hq, d, generator=gen, dtype=torch.float32)
        k = torch.randn(T, Hkv, d, generator=gen, dtype=torch.float32)
        v = torch.randn(T, Hkv, d, generator=gen, dtype=torch.float32)
    tdtype = torch.bfloat16 if spec.dtype == "bf16" else torch.float32
    q = q.to(tdtype).contiguous()
    k = k.to(tdtype)
    v = v.to(tdtype).contiguous()
    needles = None
    if spec.needle:
        needles = []
        group = Hq // Hkv
        for b in range(len(seq_lens)):
            c0, c1 = int(seq_ptr[b]), int(seq_ptr[b + 1])
            nb = c1 - c0
            if nb < 2:
                needles.append(-1)
                continue
            jstar = c0 + int(rng.integers(0, nb - 1))  # uniform in [0, nb-2]
            last0, last1 = int(bounds[c1 - 1]), int(bounds[c1])
            s0, s1 = int(bounds[jstar]), int(bounds[jstar + 1])
            for g in range(Hkv):
                m = q[last0:last1, g * group, :].float().mean(dim=0)
                planted = (4.0 * m / m.norm()).to(tdtype)
                k[s0:s1, g, :] = planted
            needles.append(jstar)
    k = k.contiguous()
    return Inputs(spec, seed, q, k, v, cu, bounds, seq_ptr, budget, needles)


def random_problem(seed: int, seq_lens: Sequence[int], hq: int, hkv: int, d: int,
                   dtype: str, chunk_lo: int, chunk_hi: int, budget: Budget,
                   values: str = "normal") -> Inputs:
    """Small ad-hoc problems for parity and edge-case tests."""
    spec = WorkloadSpec("adhoc", list(seq_lens), hq, hkv, d, dtype, chunk_lo,
                        chunk_hi, budget, values)
    return generate(spec, seed)


def explicit_problem(seed: int, per_seq_chunk_lens: Sequence[Sequence[int]], hq: int,
                     hkv: int, d: int, dtype: str, budget: Budget,
                     values: str = "normal") -> Inputs:
    """A problem with caller-chosen chunk lengths (edge cases: length 1, ragged tails)."""
    seq_lens = [int(sum(x)) for x in per_seq_chunk_lens]
    cu, bounds, seq_ptr = make_bounds(seq_lens, per_seq_chunk_lens)
    T = int(cu[-1])
    gen = torch.Generator("cpu").manual_seed(seed)
    tdtype = torch.bfloat16 if dtype == "bf16" else torch.float32
    q = torch.randn(T, hq, d, generator=gen).to(tdtype).contiguous()
    k = torch.randn(T, hkv, d, generator=gen).to(tdtype).contiguous()
    v = torch.randn(T, hkv, d, generator=gen).to(tdtype).contiguous()
    spec = WorkloadSpec("explicit", seq_lens, hq, hkv, d, dtype, 1, 1, budget, values)
    return Inputs(spec, seed, q, k, v, cu, bounds, seq_ptr, budget, None)


def planted_segment_keys(seed: int, seq_lens: Sequence[int], hkv: int, d: int, lo: int, hi: int,
                         dtype: str = "bf16", scale: float = 2.0, noise: float = 0.05):
    """Keys with planted topic segments, for the online chunking step.

    Segment lengths are drawn U[lo, hi] per sequence (the last one truncated),
    as for the workloads' chunks.  Every token of a segment has, per KV head,
    ``scale * u + noise * z``: ``u`` a seeded random unit direction of the
    segment and head, ``z ~ N(0, 1)`` per token.  Adjacent keys of one segment
    then have cosine about ``scale^2 / (scale^2 + noise^2 d)`` (0.93 for the
    defaults at d = 128) and keys of different segments about 0, so a rule
    with threshold 0.5, min_len = lo and max_len = hi recovers the planted
    segments.  Returns (k [T, hkv, d], cu_seqlens, chunk_bounds, seq_chunk_ptr)
    of the planted segments.
    """
    rng = np.random.default_rng(seed)
    per_seq = [chunk_lengths_until(rng, int(L), lo, hi) for L in seq_lens]
    cu, bounds, seq_ptr = make_bounds(list(seq_lens), per_seq)
    T = int(cu[-1])
    n = int(bounds.shape[0] - 1)
    gen = torch.Generator("cpu").manual_seed(seed)
    u = torch.randn(n, hkv, d, generator=gen, dtype=torch.float32)
    u = u / u.norm(dim=-1, keepdim=True)
    lens = torch.from_numpy(np.diff(bounds).astype(np.int64))
    k = scale * u.repeat_interleave(lens, dim=0) + noise * torch.randn(T, hkv, d, generator=gen)
    tdtype = torch.bfloat16 if dtype == "bf16" else torch.float32
    return k.to(tdtype).contiguous(), cu, bounds, seq_ptr


def drifting_keys(seed: int, T: int, hkv: int, d: int, rho: float = 0.9, dtype: str = "bf16"):
    """Keys that drift: k[t] = rho * k[t-1] + sqrt(1 - rho^2) * z[t], z ~ N(0, 1).

    Adjacent cosines cluster near ``rho`` with a spread of a few percent, so a
    threshold near ``rho`` makes many break decisions close to it (the stress
    case for decisions taken in different precisions)."""
    gen = torch.Generator("cpu").manual_seed(seed)
    z = torch.randn(T, hkv, d, generator=gen, dtype=torch.float32)
    k = torch.empty_like(z)
    if T:
        k[0] = z[0]
    c = math.sqrt(1.0 - rho * rho)
    for t in range(1, T):
        k[t] = rho * k[t - 1] + c * z[t]
    tdtype = torch.bfloat16 if dtype == "bf16" else torch.float32
    return k.to(tdtype).contiguous()
