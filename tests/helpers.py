"""Shared helpers for the GPU parity tests (test code only)."""

import math

import numpy as np
import torch

from dynamic_hierarchical_sparse_b200 import api
from oracle import dhsa_oracle as O

TIE_REL = 1e-5      # near-tie rule on the oracle's k-th / (k+1)-th scores
ATOL_BF16 = 2e-2    # max-abs gate on bf16 outputs
ATOL_F32 = 1e-4     # max-abs gate on fp32 outputs
# Relative Frobenius gates, beside the absolute ones.  bf16: the kernel adds
# two roundings to the exact computation, the bf16 output (2^-8 relative at
# most, the unit roundoff of an 8-bit significand; about 0.17 % RMS) and the
# 16-bit attention weights P before the PV product (bf16 when this gate was
# set, the same per weight and independent across keys; f16 now, 2^-11 at
# most), about 0.2 % RMS together; 1e-2 leaves about five times that.  The ratio does not depend on the
# output's scale, so it binds on diffuse rows (N(0,1) inputs, |O| ~ 0.02)
# where a 2e-2 absolute gate alone would allow a 100 % error.  fp32: the FFMA
# kernel's error is ~1e-6 relative; 1e-4 is the absolute gate's own figure.
REL_FRO_BF16 = 1e-2
REL_FRO_F32 = 1e-4
# Below this |O_ref| the bf16 gate is the flat ATOL_BF16; from it up, half a
# bf16 ulp of the reference (2^-5 at [8, 16)) exceeds ATOL_BF16 by itself.
BF16_ROUNDING_FLOOR = 8.0


def to_device(inp):
    dev = torch.device("cuda")
    return inp.q.to(dev), inp.k.to(dev), inp.v.to(dev), api.Problem.from_inputs(inp, dev)


def gpu_rows(plan, num_rows):
    rp = plan.row_ptr.cpu().numpy().astype(np.int64)
    cl = plan.col.cpu().numpy().astype(np.int64)
    assert rp.shape[0] == num_rows + 1 and rp[-1] == cl.shape[0]
    return [list(map(int, cl[rp[r]:rp[r + 1]])) for r in range(num_rows)]


def compare_plans(rows_gpu, ref, inp, budget):
    """Bit-exact comparison under the near-tie rule.

    A row may differ from the oracle only when the oracle's k-th and (k+1)-th
    best admissible scores are within TIE_REL of the larger of |s_k|, |s_k+1|
    and the row's largest |score| (fp32 score error scales with the row, not
    with one score); even then the GPU row must
    be a valid selection: its members all score at least the threshold less
    that margin, and it holds every candidate that scores more than the
    threshold plus the margin.  Returns the list of tolerated near-tie rows.
    """
    rows_ref = O.plan_rows(ref["row_ptr"], ref["col"])
    assert len(rows_gpu) == len(rows_ref)
    n = inp.num_chunks
    ptr = inp.seq_chunk_ptr
    tolerated = []
    for r, (g, o) in enumerate(zip(rows_gpu, rows_ref)):
        if g == o:
            continue
        i = r % n
        h = r // n
        b = int(np.searchsorted(ptr, i, side="right") - 1)
        il = i - int(ptr[b])
        keep = O.row_budget(il, budget.kind, budget.k, budget.num, budget.den)
        assert len(g) == keep + 1 and g[-1] == i and g == sorted(set(g)), (r, g)
        assert all(ptr[b] <= j < i for j in g[:-1]), (r, g)
        sk, sk1 = ref["kth"][r]
        margin = TIE_REL * max(abs(sk), abs(sk1), ref["rowmax"][r])
        assert abs(sk - sk1) < margin, ("plan mismatch outside the tie rule", r, g, o, sk, sk1)
        S = ref["S"][h, i]
        for j in g[:-1]:
            assert S[j] >= sk - margin, (r, j)
        # and every candidate clearly above the threshold is kept
        clear = [j for j in range(int(ptr[b]), i) if S[j] > sk + margin]
        assert set(clear) <= set(g), ("a candidate clearly above the threshold is missing", r, g, clear)
        tolerated.append(r)
    return tolerated


def reduce_bound(x, bounds):
    """Per-(h, c, :) error bound of an fp32 chunk sum / sqrt(L) of x (test-side)."""
    x64 = O.as_f64(x)
    lens = np.diff(np.asarray(bounds, dtype=np.int64))
    out = np.zeros((x64.shape[1], lens.shape[0], x64.shape[2]))
    eps = 2.0 ** -24
    for c in range(lens.shape[0]):
        s, e = int(bounds[c]), int(bounds[c + 1])
        L = e - s
        gamma = (L / 8 + 10) * eps
        out[:, c, :] = (gamma * np.abs(x64[s:e]).sum(axis=0) + 4 * eps) / math.sqrt(L)
    return out


def half_ulp_bf16(x):
    """Half a bf16 ulp at |x| (8 significand bits): the rounding error any
    bf16 output of value x carries, whatever computed it."""
    a = np.maximum(np.abs(np.asarray(x, dtype=np.float64)), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(a)) - 8)


def gate_tolerance(want, dtype):
    """Per-element max-abs gate.  bf16: the flat 2e-2 wherever |O_ref| < 8.
    From |O_ref| = 8 up, the output's own bf16 rounding (half an ulp of the
    reference, 2^-5 = 0.031 at [8, 16)) exceeds 2e-2, so even the exactly
    rounded result could miss it; there the gate is 2e-2 plus that half ulp.
    fp32: 1e-4."""
    if dtype == torch.bfloat16:
        w = np.asarray(want, dtype=np.float64)
        return np.where(np.abs(w) >= BF16_ROUNDING_FLOOR, ATOL_BF16 + half_ulp_bf16(w), ATOL_BF16)
    return np.full(np.shape(want), ATOL_F32)


def rel_fro_gate(dtype):
    return REL_FRO_BF16 if dtype == torch.bfloat16 else REL_FRO_F32


def attention_gate(got, want, dtype):
    """Max-abs gate per element and relative Frobenius gate over the whole
    comparison; returns (max_err, max|ref|, median|ref|, rel_fro)."""
    g = got.double().cpu().numpy() if hasattr(got, "cpu") else np.asarray(got)
    err = np.abs(g - want)
    tol = gate_tolerance(want, dtype)
    stats = (float(err.max()), float(np.abs(want).max()), float(np.median(np.abs(want))),
             float(np.linalg.norm(g - want) / max(np.linalg.norm(want), 1e-30)))
    assert np.all(err <= tol), ("attention error above gate", stats, float((err - tol).max()))
    assert stats[3] <= rel_fro_gate(dtype), ("relative Frobenius error above gate", stats)
    return stats


def oracle_head(inp, row_ptr, col, h, per_kv_head=False):
    """The oracle's attention output of one whole query head, [T, d] fp64,
    chunk by chunk on the given plan."""
    b = np.asarray(inp.chunk_bounds, dtype=np.int64)
    out = np.zeros((int(b[-1]), inp.q.shape[2]))
    for i in range(b.shape[0] - 1):
        out[b[i]:b[i + 1]] = O.attention_query_chunk(inp.q, inp.k, inp.v, b, row_ptr, col, h, i,
                                                     per_kv_head=per_kv_head)
    return out


def segment_tie_band(head_dim):
    """Half-width of the band around the threshold inside which an fp32
    adjacent-key similarity may decide differently from the exact one.  The
    kernel forms each dot product and squared norm of a head as 8 or 16 fused
    multiply-adds per lane and at most 5 shuffle additions (log2 of the lanes
    per head), so at most 21 roundings of 2^-24 relative to |x||y|.  The
    square roots halve the norms' share.  The two rsqrtf (2 ulp each), the two
    products, the mean over heads and the division add about 16 more.  The
    computed similarity is thus within about 60 * 2^-24 of the exact one, for
    every head size and dtype built.  The band, (2d + 16) * 2^-24 (144 at
    d = 64), is more than twice that."""
    return (2 * head_dim + 16) * 2.0 ** -24


def check_segmentation(bounds, seq_ptr, sim, cu_seqlens, rule, band):
    """Checks a segmentation (from the GPU) against the exact similarities.

    Every chunk must be a legal step of the rule, where a similarity within
    ``band`` of the threshold may be taken either way.  Returns, per sequence,
    the start of the first chunk whose step needed that latitude (None when no
    step did): up to there the segmentation must be the exact rule's."""
    bounds = np.asarray(bounds, dtype=np.int64)
    ptr = np.asarray(seq_ptr, dtype=np.int64)
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    thr, lo, hi = float(rule.threshold), int(rule.min_len), int(rule.max_len)
    sure = sim < thr - band     # a break is due
    maybe = np.abs(sim - thr) <= band
    assert ptr.shape[0] == cu.shape[0] and ptr[0] == 0 and ptr[-1] == bounds.shape[0] - 1
    assert bounds[-1] == cu[-1]
    first_loose = []
    for s in range(cu.shape[0] - 1):
        s0, s1 = int(cu[s]), int(cu[s + 1])
        starts = bounds[ptr[s]:ptr[s + 1]].tolist()
        first_loose.append(None)
        if s1 == s0:
            assert starts == []
            continue
        assert starts and starts[0] == s0, (s, starts[:3])
        ends = starts[1:] + [s1]
        for b, e in zip(starts, ends):
            assert b < e <= s1 and e - b <= hi, (b, e)
            inner = range(b + lo, min(e, b + hi))
            assert not any(sure[t] for t in inner), ("missed break", b, e)
            used = any(maybe[t] for t in inner)
            if e < s1:
                assert e - b >= lo, (b, e)
                if e - b != hi:
                    assert sure[e] or maybe[e], ("break without cause", b, e, sim[e])
                    used = used or bool(maybe[e])
            if used and first_loose[-1] is None:
                first_loose[-1] = b
    return first_loose


def segmentations_agree_until_latitude(got_bounds, got_ptr, want_bounds, want_ptr, first_loose):
    """Per sequence, the chunk starts of both segmentations up to and including
    the first step that had latitude (where both chose from the same start)."""
    for s, fl in enumerate(first_loose):
        g = list(got_bounds[got_ptr[s]:got_ptr[s + 1]])
        w = list(want_bounds[want_ptr[s]:want_ptr[s + 1]])
        if fl is None:
            assert g == w, s
        else:
            cut = g.index(fl) + 1
            assert g[:cut] == w[:cut], s
