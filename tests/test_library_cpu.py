"""CPU-only checks of the C-ABI library: it builds, loads, exports every symbol
the header declares, and validates arguments on the host (no kernel runs)."""

import ctypes
import os
import re

import numpy as np
import pytest
import torch

from dynamic_hierarchical_sparse_b200 import api, build, workloads as W
from oracle import dhsa_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CPU = torch.device("cpu")


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()


def _declared_symbols():
    with open(os.path.join(ROOT, "include", "dhsa.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"DHSA_API\s+[\w\s\*]+?\b(dhsa_\w+)\s*\(", text)))


def test_header_declares_the_binding_names():
    assert _declared_symbols() == sorted(api.EXPORTED)


def test_library_exports_every_declared_symbol():
    L = ctypes.CDLL(api.library_path())
    for name in _declared_symbols():
        assert hasattr(L, name), name
    # nothing else with C linkage leaks out under the dhsa_ prefix
    out = os.popen("nm -D --defined-only %s" % api.library_path()).read()
    exported = sorted(set(re.findall(r"\bT (dhsa_\w+)", out)))
    assert exported == _declared_symbols()


def test_binding_signatures_match_the_header():
    """Every entry point takes as many arguments in the binding as the header
    declares (a dropped or extra argument would shift every later one)."""
    hdr = open(os.path.join(ROOT, "include", "dhsa.h")).read()
    hdr = re.sub(r"/\*.*?\*/", "", hdr, flags=re.S)
    hdr = re.sub(r"//[^\n]*", "", hdr)
    L = api.lib()
    for name in api.EXPORTED:
        m = re.search(r"\b%s\s*\(([^;{]*)\)\s*;" % name, hdr, re.S)
        assert m, name
        params = [q for q in m.group(1).split(",") if q.strip() and q.strip() != "void"]
        assert len(params) == len(getattr(L, name).argtypes), name


def test_status_strings():
    L = api.lib()
    for code, name in api.STATUS_NAMES.items():
        assert L.dhsa_status_string(code).decode() == name


def _problem(inp, **over):
    s = inp.spec
    kw = dict(num_q_heads=s.num_q_heads, num_kv_heads=s.num_kv_heads, head_dim=s.head_dim,
              dtype=inp.q.dtype)
    kw.update(over)
    return api.Problem(inp.cu_seqlens, inp.chunk_bounds, inp.seq_chunk_ptr, device=CPU, **kw)


@pytest.mark.parametrize("budget", [W.Budget.topk(0), W.Budget.topk(3), W.Budget.topk(10 ** 6),
                                    W.Budget.fraction(1, 10), W.Budget.fraction(1, 20),
                                    W.Budget.fraction(3, 2)])
def test_plan_nnz_matches_oracle_row_budget(budget):
    inp = W.random_problem(0, [700, 33, 1500], 4, 2, 64, "bf16", 16, 80, budget)
    p = _problem(inp)
    ptr = inp.seq_chunk_ptr
    per_head = 0
    for b in range(len(ptr) - 1):
        for il in range(ptr[b + 1] - ptr[b]):
            per_head += O.row_budget(il, budget.kind, budget.k, budget.num, budget.den) + 1
    assert p.nnz(budget) == 4 * per_head


def test_workspace_sizes():
    inp = W.random_problem(0, [2048], 8, 2, 128, "bf16", 64, 256, W.Budget.topk(4))
    p = _problem(inp)
    n = inp.num_chunks
    ws = p.plan_workspace_bytes(W.Budget.topk(4))
    need = 256 + (8 * n * 128 + 2 * n * 128 + 8 * n * n) * 4
    assert need <= ws <= need + 4 * 256
    # bf16: the status words, then an f16 copy of V (T * Hkv * d * 2 bytes, 256-byte aligned)
    v16 = 2048 * 2 * 128 * 2
    assert p.attention_workspace_bytes() == 256 + v16
    # fp32 needs no copy
    inp32 = W.random_problem(0, [2048], 8, 2, 128, "f32", 64, 256, W.Budget.topk(4))
    assert _problem(inp32).attention_workspace_bytes() == 256


def test_per_kv_head_plan_sizes():
    """A per-KV-head plan has Hkv*n rows (nnz scales with Hkv, not Hq); its
    workspace adds the summed query chunks and holds an [Hkv, n, n] score
    matrix; unknown flag bits are rejected."""
    inp = W.random_problem(0, [2048, 700], 8, 2, 128, "bf16", 64, 256, W.Budget.topk(4))
    p = _problem(inp)
    n = inp.num_chunks
    for budget in (W.Budget.topk(4), W.Budget.fraction(1, 10)):
        assert p.nnz(budget.kv()) * 4 == p.nnz(budget)
    ws = p.plan_workspace_bytes(W.Budget.topk(4).kv())
    need = 256 + (8 * n * 128 + 2 * n * 128 + 2 * n * 128 + 2 * n * n) * 4
    assert need <= ws <= need + 5 * 256
    assert _code(p, W.Budget.topk(4).kv()) == 0
    bad = W.Budget(W.BUDGET_TOPK | 0x200, k=4)
    assert _code(p, bad) == 1


def _code(problem, budget=None):
    return problem.validate(budget)


def test_validation_accepts_good_problems():
    for spec in [W.TINY_1K_F32, W.RAGGED_NEEDLE]:
        inp = W.generate(spec, 0, seq_lens=[256, 512] if spec.needle else None)
        assert _code(_problem(inp), spec.budget) == 0


@pytest.mark.parametrize("case", ["gqa", "head_dim", "head_dim_neg", "budget_k", "budget_den",
                                  "bounds_order", "bounds_cover", "cross_seq", "seqptr"])
def test_validation_rejects(case):
    inp = W.random_problem(1, [300, 200], 4, 2, 64, "bf16", 20, 60, W.Budget.topk(2))
    budget = W.Budget.topk(2)
    bounds = inp.chunk_bounds.copy()
    sptr = inp.seq_chunk_ptr.copy()
    cu = inp.cu_seqlens.copy()
    kw = {}
    want = 1
    if case == "gqa":
        kw = dict(num_q_heads=6, num_kv_heads=4)
    elif case == "head_dim":
        kw = dict(head_dim=96)
        want = 2
    elif case == "head_dim_neg":
        kw = dict(head_dim=0)
    elif case == "budget_k":
        budget = W.Budget.topk(-1)
    elif case == "budget_den":
        budget = W.Budget.fraction(1, 0)
    elif case == "bounds_order":
        bounds[2], bounds[3] = bounds[3], bounds[2]
    elif case == "bounds_cover":
        bounds[-1] -= 1
    elif case == "cross_seq":
        # move the sequence edge inside a chunk
        cu[1] += 1
    elif case == "seqptr":
        sptr[1] = sptr[1] + 1
    s = inp.spec
    args = dict(num_q_heads=s.num_q_heads, num_kv_heads=s.num_kv_heads, head_dim=s.head_dim,
                dtype=inp.q.dtype)
    args.update(kw)
    p = api.Problem(cu, bounds, sptr, device=CPU, **args)
    assert _code(p, budget) == want


def test_entry_points_reject_before_launch():
    """Invalid calls return their error code without touching the (absent) GPU."""
    inp = W.random_problem(2, [300], 2, 1, 64, "bf16", 20, 60, W.Budget.topk(2))
    p = _problem(inp)
    L = api.lib()
    b = api._budget(W.Budget.topk(2))
    nnz = p.nnz(W.Budget.topk(2))
    null = ctypes.c_void_p(0)
    ws = ctypes.c_void_p(256)
    # wrong nnz
    assert L.dhsa_plan(ctypes.c_void_p(16), ctypes.c_void_p(16), p.ref(), b, ctypes.c_void_p(16),
                       ctypes.c_void_p(16), nnz + 1, ws, 1 << 30, null) == 1
    # too little workspace
    assert L.dhsa_plan(ctypes.c_void_p(16), ctypes.c_void_p(16), p.ref(), b, ctypes.c_void_p(16),
                       ctypes.c_void_p(16), nnz, ws, 16, null) == 3
    # misaligned q
    assert L.dhsa_attention(ctypes.c_void_p(17), ctypes.c_void_p(16), ctypes.c_void_p(16), p.ref(),
                            ctypes.c_void_p(16), ctypes.c_void_p(16), nnz, ctypes.c_float(0.0),
                            ctypes.c_void_p(16), ws, 1 << 30, null) == 1
    # a workspace without room for the f16 copy of V, or not 256-byte aligned
    assert L.dhsa_attention(ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.c_void_p(16), p.ref(),
                            ctypes.c_void_p(16), ctypes.c_void_p(16), nnz, ctypes.c_float(0.0),
                            ctypes.c_void_p(16), ws, p.attention_workspace_bytes() - 1, null) == 3
    assert L.dhsa_attention(ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.c_void_p(16), p.ref(),
                            ctypes.c_void_p(16), ctypes.c_void_p(16), nnz, ctypes.c_float(0.0),
                            ctypes.c_void_p(16), ctypes.c_void_p(272), 1 << 30, null) == 3
    # missing workspace
    assert L.dhsa_attention(ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.c_void_p(16), p.ref(),
                            ctypes.c_void_p(16), ctypes.c_void_p(16), nnz, ctypes.c_float(0.0),
                            ctypes.c_void_p(16), null, 0, null) == 3
    # timeout self-test limits
    assert L.dhsa_selftest_timeout(ws, 0, null) == 1
    assert L.dhsa_selftest_timeout(null, 100, null) == 3
    # plan check: fewer entries than rows (every row holds its diagonal), a
    # missing workspace, a missing plan
    rows = 2 * p.num_chunks
    assert L.dhsa_plan_check(p.ref(), ctypes.c_void_p(16), ctypes.c_void_p(16), rows - 1, 0, ws, 256, null) == 1
    assert L.dhsa_plan_check(p.ref(), ctypes.c_void_p(16), ctypes.c_void_p(16), nnz, 0, null, 0, null) == 3
    assert L.dhsa_plan_check(p.ref(), ctypes.c_void_p(16), ctypes.c_void_p(16), nnz, 0, ws, 16, null) == 3
    assert L.dhsa_plan_check(p.ref(), null, ctypes.c_void_p(16), nnz, 0, ws, 256, null) == 1
    # plan margins: another nnz, a workspace smaller than the plan's
    assert L.dhsa_plan_margins(p.ref(), b, ctypes.c_void_p(16), ctypes.c_void_p(16), nnz + 1, ws, 1 << 30,
                               ctypes.c_void_p(16), null) == 1
    assert L.dhsa_plan_margins(p.ref(), b, ctypes.c_void_p(16), ctypes.c_void_p(16), nnz, ws, 16,
                               ctypes.c_void_p(16), null) == 3
    # per-KV-head rows (Hkv * n) accept fewer entries than per-query-head ones
    assert L.dhsa_plan_check(p.ref(), ctypes.c_void_p(16), ctypes.c_void_p(16), p.num_chunks - 1, 1, ws, 256,
                             null) == 1


def test_empty_problem_is_a_no_op():
    p = api.Problem([0], [0], [0], 4, 2, 128, torch.bfloat16, device=CPU)
    assert p.validate(W.Budget.topk(3)) == 0
    assert p.nnz(W.Budget.topk(3)) == 0
    L = api.lib()
    null = ctypes.c_void_p(0)
    ws = ctypes.c_void_p(256)
    assert L.dhsa_plan(null, null, p.ref(), api._budget(W.Budget.topk(3)), null, null, 0, ws,
                       p.plan_workspace_bytes(W.Budget.topk(3)), null) == 0
    assert L.dhsa_attention(null, null, null, p.ref(), null, null, 0, ctypes.c_float(0.0), null, ws, 256,
                            null) == 0


def test_product_path_has_no_cpu_fallback(monkeypatch):
    """Without the library the binding raises instead of computing anything."""
    monkeypatch.setattr(api, "_lib", None)
    monkeypatch.setattr(api, "_LIB_PATH", "/nonexistent/libdhsa.so")
    with pytest.raises(RuntimeError):
        api.lib()


def test_library_loads_once_under_concurrent_first_calls(monkeypatch):
    """Threads racing on the first call all get the one loaded library, with
    every signature set."""
    import threading
    monkeypatch.setattr(api, "_lib", None)
    got, barrier = [], threading.Barrier(8)

    def first_call():
        barrier.wait()
        got.append(api.lib())
    threads = [threading.Thread(target=first_call) for _ in range(8)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert len(got) == 8 and all(g is got[0] for g in got)
    assert got[0].dhsa_plan.argtypes is not None and got[0].dhsa_segment.restype is ctypes.c_int


def test_product_package_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "dynamic_hierarchical_sparse_b200")
    pat = re.compile(r"^\s*(from\s+oracle|import\s+oracle)|dhsa_oracle", re.M)
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                with open(os.path.join(dirpath, fn)) as f:
                    assert not pat.search(f.read()), fn


def _floor_sum(n, m, a, c):
    """The select kernel's lattice-point recursion, restated (Python ints)."""
    total = 0
    while n > 0:
        if a >= m:
            total += (n * (n - 1) // 2) * (a // m)
            a %= m
        if c >= m:
            total += n * (c // m)
            c %= m
        y = a * n + c
        if y < m:
            break
        n, c, m, a = y // m, y % m, a, m
    return total


def _plan_entries(L, budget):
    if L <= 0:
        return 0
    if budget.kind == W.BUDGET_TOPK:
        k = budget.k
        s = L * (L - 1) // 2 if L <= k else k * (k - 1) // 2 + k * (L - k)
    elif budget.num >= budget.den:
        s = L * (L - 1) // 2
    else:
        s = _floor_sum(L, budget.den, budget.num, budget.den - 1)
    return s + L


@pytest.mark.parametrize("budget", [W.Budget.topk(0), W.Budget.topk(1), W.Budget.topk(7),
                                    W.Budget.fraction(1, 20), W.Budget.fraction(1, 10),
                                    W.Budget.fraction(3, 7), W.Budget.fraction(5, 4), W.Budget.fraction(0, 3)])
def test_closed_form_plan_offsets(budget):
    """Closed form of the per-chunk plan offsets used by the select kernel
    equals the running sum of (row budget + 1) from the oracle's rule."""
    running = 0
    for L in range(0, 3000):
        assert _plan_entries(L, budget) == running, L
        running += O.row_budget(L, budget.kind, budget.k, budget.num, budget.den) + 1


def test_gate_rounding_allowance_is_half_a_bf16_ulp():
    """The bf16 gate adds the output's own rounding: for any value, rounding
    to bf16 moves it by at most the allowance, and the allowance is the
    smallest power of two that always does (a full ulp would be twice it)."""
    from tests.helpers import half_ulp_bf16
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-3, 3, 20000), [1.0, 4.0, 7.99, 8.0]])
    r = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    assert np.all(np.abs(r - x) <= half_ulp_bf16(x))
    assert np.abs(r - x).max() > 0.5 * half_ulp_bf16(x[np.argmax(np.abs(r - x))])
    assert half_ulp_bf16(8.0) == 2.0 ** -5 and half_ulp_bf16(7.99) == 2.0 ** -6


def test_bf16_gate_is_flat_below_the_rounding_floor():
    """The bf16 max-abs gate is the flat 2e-2 wherever |O_ref| < 8 (there the
    exactly rounded output is within 2^-6 < 2e-2 of the reference), and adds
    half a bf16 ulp only from |O_ref| = 8 up, where that half ulp (2^-5) alone
    exceeds 2e-2."""
    from tests.helpers import ATOL_BF16, gate_tolerance, half_ulp_bf16
    want = np.array([0.0, -0.02, 0.5, 3.99, -4.0, 7.999, -8.0, 8.25, 15.9, 16.0, -100.0])
    tol = gate_tolerance(want, torch.bfloat16)
    below = np.abs(want) < 8
    assert np.all(tol[below] == ATOL_BF16)
    assert np.all(tol[~below] == ATOL_BF16 + half_ulp_bf16(want[~below]))
    assert np.all(half_ulp_bf16(want[below]) < ATOL_BF16)
    assert np.all(half_ulp_bf16(want[~below]) > ATOL_BF16)
    assert np.all(gate_tolerance(want, torch.float32) == 1e-4)


def test_attention_gate_rejects_a_relative_error_the_absolute_gate_misses():
    """On diffuse outputs (|O| ~ 0.01) a 50 % error stays under the 2e-2
    absolute gate; the relative Frobenius gate rejects it, and passes the
    output's own bf16 rounding."""
    from tests.helpers import attention_gate
    rng = np.random.default_rng(1)
    want = 0.008 * rng.standard_normal((512, 128))
    rounded = torch.from_numpy(want).to(torch.bfloat16)
    stats = attention_gate(rounded, want, torch.bfloat16)
    assert stats[3] < 3e-3
    wrong = torch.from_numpy(want * 1.5)
    assert np.abs(want * 0.5).max() < 2e-2
    with pytest.raises(AssertionError, match="relative Frobenius"):
        attention_gate(wrong, want, torch.bfloat16)


def test_segment_capacity_and_workspace():
    """Chunk capacity of the online chunking step is sum ceil(L_b / min_len);
    its workspace holds the status word and two bitmaps of ceil(T/32) words."""
    L = api.lib()
    cu = np.array([0, 0, 1, 100, 356], dtype=np.int32)
    cap = ctypes.c_int64(-1)
    assert L.dhsa_segment_capacity(cu.ctypes.data_as(ctypes.c_void_p), 4, 16, ctypes.byref(cap)) == 0
    assert cap.value == 0 + 1 + 7 + 16
    assert L.dhsa_segment_capacity(cu.ctypes.data_as(ctypes.c_void_p), 4, 0, ctypes.byref(cap)) == 1
    bad = np.array([0, 5, 3], dtype=np.int32)
    assert L.dhsa_segment_capacity(bad.ctypes.data_as(ctypes.c_void_p), 2, 1, ctypes.byref(cap)) == 1
    ws = ctypes.c_size_t(0)
    assert L.dhsa_segment_workspace_size(356, ctypes.byref(ws)) == 0 and ws.value == 256 + 2 * 256
    assert L.dhsa_segment_workspace_size(131072, ctypes.byref(ws)) == 0 and ws.value == 256 + 2 * 16384
    assert L.dhsa_segment_workspace_size(-1, ctypes.byref(ws)) == 1


@pytest.mark.parametrize("case", ["ok_empty", "min0", "max_lt_min", "max_too_long", "nan", "capacity",
                                  "workspace", "misaligned", "head_dim", "dtype", "cu_start", "cu_order"])
def test_segment_rejects_before_launch(case):
    """dhsa_segment validates everything on the host and returns its code
    before launching anything (there is no GPU here)."""
    L = api.lib()
    cu = np.array([0, 300, 1000], dtype=np.int32)
    rule = api._SegmentRule(0.5, 16, 64)
    kwargs = dict(k=16, dtype=0, hkv=2, d=128, cap=int(np.ceil(300 / 16) + np.ceil(700 / 16)), ws=256 + 2 * 256)
    want = 1
    if case == "ok_empty":
        cu = np.array([0, 0], dtype=np.int32)
        kwargs.update(cap=0)
        want = 0
    elif case == "min0":
        rule = api._SegmentRule(0.5, 0, 64)
    elif case == "max_lt_min":
        rule = api._SegmentRule(0.5, 16, 15)
    elif case == "max_too_long":
        rule = api._SegmentRule(0.5, 16, 65537)
    elif case == "nan":
        rule = api._SegmentRule(float("nan"), 16, 64)
    elif case == "capacity":
        kwargs["cap"] -= 1
    elif case == "workspace":
        kwargs["ws"] = 256 + 2 * 256 - 1
        want = 3
    elif case == "misaligned":
        kwargs["k"] = 24
    elif case == "head_dim":
        kwargs["d"] = 96
        want = 2
    elif case == "dtype":
        kwargs["dtype"] = 7
    elif case == "cu_start":
        cu = np.array([1, 300, 1000], dtype=np.int32)
    elif case == "cu_order":
        cu = np.array([0, 300, 200], dtype=np.int32)
    P = ctypes.c_void_p
    B = cu.shape[0] - 1
    got = L.dhsa_segment(P(kwargs["k"]), kwargs["dtype"], kwargs["hkv"], kwargs["d"], B, P(16),
                         cu.ctypes.data_as(P), rule, P(16), kwargs["cap"], P(16), P(16), P(256),
                         kwargs["ws"], P(0))
    if case == "ok_empty":
        # a valid empty batch would launch the compaction kernel; only check
        # that validation passes by asking for too little workspace instead
        got = L.dhsa_segment(P(16), 0, 2, 128, B, P(16), cu.ctypes.data_as(P), rule, P(16), 0, P(16), P(16),
                             P(256), 255, P(0))
        want = 3
    assert got == want


def test_tensor_peak_follows_the_sampled_clock():
    """The roofline's bf16 denominator: the straight line through the two
    measured GEMM figures (sustained at its median clock, burst at the
    maximum), at the run's median SM clock, kept between the two."""
    import bench

    pk = {"bf16_tflops": 1630.0, "bf16_tflops_sustained": 1374.2, "sustained_sm_mhz": 1237.0,
          "sm_max_mhz": 1965.0, "source": "measured"}
    assert bench.tensor_peak(pk, {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0})[0] == 1630.0
    assert bench.tensor_peak(pk, {"sm_mhz": None})[0] == 1630.0
    assert bench.tensor_peak(pk, {"sm_mhz": 1237.0, "sm_max_mhz": 1965.0})[0] == 1374.2
    assert bench.tensor_peak(pk, {"sm_mhz": 1100.0, "sm_max_mhz": 1965.0})[0] == 1374.2
    mid = bench.tensor_peak(pk, {"sm_mhz": (1237.0 + 1965.0) / 2, "sm_max_mhz": 1965.0})[0]
    assert abs(mid - (1374.2 + 1630.0) / 2) < 1e-9
    # the loaded clock of a 128K bench run: 1702 MHz -> 1537.7 TFLOP/s, above the burst figure
    # scaled through the origin (1411.8), which the sustained point shows to be too low
    p1702 = bench.tensor_peak(pk, {"sm_mhz": 1702.0, "sm_max_mhz": 1965.0})[0]
    assert abs(p1702 - (1374.2 + 255.8 * 465.0 / 728.0)) < 1e-9 and p1702 > 1630.0 * 1702.0 / 1965.0
