"""Thin Python binding over libdhsa.so (ctypes).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  PyTorch supplies device memory and the current stream.  There is no
fallback: if the library is missing or a call fails, an exception is raised.
"""

from __future__ import annotations

import ctypes
import dataclasses
import os
import threading
from typing import Optional, Tuple

import numpy as np
import torch

from .workloads import Budget

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdhsa.so")
_lib = None
_lib_lock = threading.Lock()

DHSA_BF16 = 0
DHSA_F32 = 1

STATUS_NAMES = {0: "DHSA_OK", 1: "DHSA_ERR_INVALID_ARG", 2: "DHSA_ERR_UNSUPPORTED",
                3: "DHSA_ERR_WORKSPACE", 4: "DHSA_ERR_CUDA", 5: "DHSA_ERR_TIMEOUT",
                6: "DHSA_ERR_DEVICE_CHECK"}

EXPORTED = [
    "dhsa_status_string", "dhsa_validate", "dhsa_plan_nnz", "dhsa_chunk_reduce",
    "dhsa_chunk_similarity", "dhsa_topk_select", "dhsa_plan_workspace_size", "dhsa_plan",
    "dhsa_attention_workspace_size", "dhsa_attention", "dhsa_workspace_status",
    "dhsa_selftest_timeout", "dhsa_plan_noalloc", "dhsa_attention_kv_plan",
    "dhsa_segment_capacity", "dhsa_segment_workspace_size", "dhsa_segment", "dhsa_plan_check",
    "dhsa_plan_margins",
]

DHSA_BUDGET_PER_KV_HEAD = 0x100


class DhsaError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__("%s failed: %s" % (where, STATUS_NAMES.get(code, str(code))))
        self.code = code


class _Budget(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("k", ctypes.c_int32), ("num", ctypes.c_int32),
                ("den", ctypes.c_int32)]


class _Problem(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int32), ("num_seqs", ctypes.c_int32),
                ("total_tokens", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("num_chunks", ctypes.c_int32),
                ("cu_seqlens", ctypes.c_void_p), ("chunk_bounds", ctypes.c_void_p),
                ("seq_chunk_ptr", ctypes.c_void_p),
                ("h_cu_seqlens", ctypes.c_void_p), ("h_chunk_bounds", ctypes.c_void_p),
                ("h_seq_chunk_ptr", ctypes.c_void_p)]


class _SegmentRule(ctypes.Structure):
    _fields_ = [("threshold", ctypes.c_float), ("min_len", ctypes.c_int32), ("max_len", ctypes.c_int32)]


def library_path() -> str:
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    with _lib_lock:  # one thread loads the library and sets every signature
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError("libdhsa.so is missing (build it with "
                               "`python -m dynamic_hierarchical_sparse_b200.build`)")
        L = ctypes.CDLL(_LIB_PATH)
        P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        PP = ctypes.POINTER(_Problem)
        PB = ctypes.POINTER(_Budget)
        sig = {
            "dhsa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
            "dhsa_validate": (ctypes.c_int, [PP, PB]),
            "dhsa_plan_nnz": (ctypes.c_int, [PP, _Budget, ctypes.POINTER(I64)]),
            "dhsa_chunk_reduce": (ctypes.c_int, [P, I32, I32, I32, I32, P, I32, P, P]),
            "dhsa_chunk_similarity": (ctypes.c_int, [P, P, PP, P, P]),
            "dhsa_topk_select": (ctypes.c_int, [P, PP, _Budget, P, P, I64, P, SZ, P]),
            "dhsa_plan_workspace_size": (ctypes.c_int, [PP, _Budget, ctypes.POINTER(SZ)]),
            "dhsa_plan": (ctypes.c_int, [P, P, PP, _Budget, P, P, I64, P, SZ, P]),
            "dhsa_attention_workspace_size": (ctypes.c_int, [PP, ctypes.POINTER(SZ)]),
            "dhsa_attention": (ctypes.c_int, [P, P, P, PP, P, P, I64, ctypes.c_float, P, P, SZ, P]),
            "dhsa_workspace_status": (ctypes.c_int, [P, P]),
            "dhsa_selftest_timeout": (ctypes.c_int, [P, I32, P]),
            "dhsa_plan_noalloc": (ctypes.c_int, [P, P, PP, _Budget, P, P, I64, P]),
            "dhsa_attention_kv_plan": (ctypes.c_int, [P, P, P, PP, P, P, I64, ctypes.c_float, P, P, SZ, P]),
            "dhsa_segment_capacity": (ctypes.c_int, [P, I32, I32, ctypes.POINTER(I64)]),
            "dhsa_segment_workspace_size": (ctypes.c_int, [I32, ctypes.POINTER(SZ)]),
            "dhsa_segment": (ctypes.c_int, [P, I32, I32, I32, I32, P, P, _SegmentRule, P, I64, P, P, P, SZ, P]),
            "dhsa_plan_check": (ctypes.c_int, [PP, P, P, I64, I32, P, SZ, P]),
            "dhsa_plan_margins": (ctypes.c_int, [PP, _Budget, P, P, I64, P, SZ, P, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(code: int, where: str) -> None:
    if code != 0:
        raise DhsaError(code, where)


def _stream_ptr(stream: Optional[torch.cuda.Stream]) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _enter(stream) -> None:
    """A one-shot call on an explicit stream first waits for the work queued on
    the current stream (its inputs, and outputs this module just zeroed there)."""
    if stream is not None:
        stream.wait_stream(torch.cuda.current_stream(stream.device))


def _leave(stream) -> None:
    """... and the current stream waits for the call before its result is used
    (or freed) there."""
    if stream is not None:
        torch.cuda.current_stream(stream.device).wait_stream(stream)


def _ptr(t: Optional[torch.Tensor]) -> ctypes.c_void_p:
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _budget(b: Budget) -> _Budget:
    kind = int(b.kind) | (DHSA_BUDGET_PER_KV_HEAD if getattr(b, "per_kv_head", False) else 0)
    return _Budget(kind, int(b.k), int(b.num), int(b.den))


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return DHSA_BF16
    if t.dtype == torch.float32:
        return DHSA_F32
    raise TypeError("q/k/v must be bfloat16 or float32, got %s" % t.dtype)


class Problem:
    """Shapes + chunk structure of one packed batch, with host and device mirrors."""

    def __init__(self, cu_seqlens, chunk_bounds, seq_chunk_ptr, num_q_heads: int,
                 num_kv_heads: int, head_dim: int, dtype: torch.dtype,
                 device: Optional[torch.device] = None):
        self.h_cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
        self.h_bounds = np.ascontiguousarray(np.asarray(chunk_bounds, dtype=np.int32))
        self.h_sptr = np.ascontiguousarray(np.asarray(seq_chunk_ptr, dtype=np.int32))
        dev = torch.device("cuda") if device is None else device
        self.d_cu = torch.from_numpy(self.h_cu).to(dev)
        self.d_bounds = torch.from_numpy(self.h_bounds).to(dev)
        self.d_sptr = torch.from_numpy(self.h_sptr).to(dev)
        self.num_q_heads, self.num_kv_heads, self.head_dim = num_q_heads, num_kv_heads, head_dim
        self.dtype = dtype
        self.num_chunks = int(self.h_bounds.shape[0] - 1)
        self.num_seqs = int(self.h_cu.shape[0] - 1)
        self.total_tokens = int(self.h_cu[-1])
        self.c = _Problem(
            DHSA_BF16 if dtype == torch.bfloat16 else DHSA_F32, self.num_seqs, self.total_tokens,
            num_q_heads, num_kv_heads, head_dim, self.num_chunks,
            self.d_cu.data_ptr(), self.d_bounds.data_ptr(), self.d_sptr.data_ptr(),
            self.h_cu.ctypes.data, self.h_bounds.ctypes.data, self.h_sptr.ctypes.data)

    @staticmethod
    def from_inputs(inp, device: Optional[torch.device] = None) -> "Problem":
        s = inp.spec
        return Problem(inp.cu_seqlens, inp.chunk_bounds, inp.seq_chunk_ptr, s.num_q_heads,
                       s.num_kv_heads, s.head_dim, inp.q.dtype, device)

    def ref(self):
        return ctypes.byref(self.c)

    def validate(self, budget: Optional[Budget] = None) -> int:
        if budget is None:
            return lib().dhsa_validate(self.ref(), None)
        b = _budget(budget)
        return lib().dhsa_validate(self.ref(), ctypes.byref(b))

    def nnz(self, budget: Budget) -> int:
        out = ctypes.c_int64(0)
        _check(lib().dhsa_plan_nnz(self.ref(), _budget(budget), ctypes.byref(out)), "dhsa_plan_nnz")
        return int(out.value)

    def plan_workspace_bytes(self, budget: Budget) -> int:
        out = ctypes.c_size_t(0)
        _check(lib().dhsa_plan_workspace_size(self.ref(), _budget(budget), ctypes.byref(out)),
               "dhsa_plan_workspace_size")
        return int(out.value)

    def attention_workspace_bytes(self) -> int:
        out = ctypes.c_size_t(0)
        _check(lib().dhsa_attention_workspace_size(self.ref(), ctypes.byref(out)),
               "dhsa_attention_workspace_size")
        return int(out.value)


@dataclasses.dataclass
class Plan:
    row_ptr: torch.Tensor  # int32 [Hq*n+1] device ([Hkv*n+1] for a per-KV-head plan)
    col: torch.Tensor      # int32 [nnz] device
    nnz: int
    per_kv_head: bool = False


def _workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def _require(t: torch.Tensor, name: str) -> None:
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


def chunk_reduce(x: torch.Tensor, problem: Problem, stream=None) -> torch.Tensor:
    """Step 1 for one tensor: [T, H, d] -> fp32 [H, n, d]."""
    _require(x, "x")
    T, H, d = x.shape
    out = torch.empty(H, problem.num_chunks, d, dtype=torch.float32, device=x.device)
    _enter(stream)
    _check(lib().dhsa_chunk_reduce(_ptr(x), _dtype_code(x), T, H, d, _ptr(problem.d_bounds),
                                   problem.num_chunks, _ptr(out), _stream_ptr(stream)),
           "dhsa_chunk_reduce")
    _leave(stream)
    return out


def chunk_similarity(qc: torch.Tensor, kc: torch.Tensor, problem: Problem, stream=None) -> torch.Tensor:
    """Step 2: fp32 [Hq, n, n]; entries outside the causal same-sequence triangle are 0."""
    n = problem.num_chunks
    scores = torch.zeros(problem.num_q_heads, n, n, dtype=torch.float32, device=qc.device)
    _enter(stream)
    _check(lib().dhsa_chunk_similarity(_ptr(qc), _ptr(kc), problem.ref(), _ptr(scores),
                                       _stream_ptr(stream)), "dhsa_chunk_similarity")
    _leave(stream)
    return scores


def topk_select(scores: torch.Tensor, problem: Problem, budget: Budget, stream=None,
                check: bool = False) -> Plan:
    """Step 3 on a given score matrix."""
    nnz = problem.nnz(budget)
    dev = scores.device
    heads = problem.num_kv_heads if budget.per_kv_head else problem.num_q_heads
    row_ptr = torch.empty(heads * problem.num_chunks + 1, dtype=torch.int32, device=dev)
    col = torch.empty(max(nnz, 1), dtype=torch.int32, device=dev)
    ws = _workspace(256, dev)
    st = _stream_ptr(stream)
    _enter(stream)
    _check(lib().dhsa_topk_select(_ptr(scores), problem.ref(), _budget(budget), _ptr(row_ptr), _ptr(col),
                                  nnz, _ptr(ws), ws.numel(), st), "dhsa_topk_select")
    if check:
        _check(lib().dhsa_workspace_status(_ptr(ws), st), "dhsa_topk_select (device)")
    _leave(stream)
    return Plan(row_ptr, col[:nnz], nnz, bool(budget.per_kv_head))


class Planner:
    """Owns the plan workspace and output buffers for repeated dhsa_plan calls.
    With an explicit stream, ordering against other streams is the caller's
    (the one-shot functions below do it themselves)."""

    def __init__(self, problem: Problem, budget: Budget, device=None):
        self.problem, self.budget = problem, budget
        dev = problem.d_bounds.device if device is None else device
        self.nnz = problem.nnz(budget)
        self.ws = _workspace(problem.plan_workspace_bytes(budget), dev)
        heads = problem.num_kv_heads if budget.per_kv_head else problem.num_q_heads
        self.row_ptr = torch.empty(heads * problem.num_chunks + 1, dtype=torch.int32, device=dev)
        self.col = torch.empty(max(self.nnz, 1), dtype=torch.int32, device=dev)
        self._b = _budget(budget)

    def __call__(self, q: torch.Tensor, k: torch.Tensor, stream=None) -> Plan:
        _check(lib().dhsa_plan(_ptr(q), _ptr(k), self.problem.ref(), self._b, _ptr(self.row_ptr),
                               _ptr(self.col), self.nnz, _ptr(self.ws), self.ws.numel(),
                               _stream_ptr(stream)), "dhsa_plan")
        return Plan(self.row_ptr, self.col[:self.nnz], self.nnz, bool(self.budget.per_kv_head))

    def status(self, stream=None) -> int:
        return lib().dhsa_workspace_status(_ptr(self.ws), _stream_ptr(stream))

    def margins(self, stream=None) -> torch.Tensor:
        """Selection margins of the plan the last call wrote (dhsa_plan_margins):
        fp32 [rows, 2], the k-th and (k+1)-th largest admissible scores per row
        (NaN where there is none)."""
        rows = self.row_ptr.numel() - 1
        out = torch.empty(rows, 2, dtype=torch.float32, device=self.row_ptr.device)
        _check(lib().dhsa_plan_margins(self.problem.ref(), self._b, _ptr(self.row_ptr), _ptr(self.col), self.nnz,
                                       _ptr(self.ws), self.ws.numel(), _ptr(out), _stream_ptr(stream)),
               "dhsa_plan_margins")
        return out


def plan(q: torch.Tensor, k: torch.Tensor, problem: Problem, budget: Budget, stream=None,
         check: bool = False) -> Plan:
    """Steps 1-3: returns the per-(head, query chunk) list of kept key chunks."""
    _require(q, "q")
    _require(k, "k")
    p = Planner(problem, budget, q.device)
    _enter(stream)
    out = p(q, k, stream)
    if check:
        _check(p.status(stream), "dhsa_plan (device)")
    _leave(stream)
    return Plan(out.row_ptr.clone(), out.col.clone(), out.nnz, out.per_kv_head)


def check_plan(problem: Problem, row_ptr: torch.Tensor, col: torch.Tensor, per_kv_head: bool = False,
               stream=None) -> int:
    """Device-side structural check of a plan (dhsa_plan_check).  Waits for it
    and returns the status (0 = a valid plan, 6 = DHSA_ERR_DEVICE_CHECK).
    row_ptr / col: int32 device tensors; nnz = col.numel()."""
    _require(row_ptr, "row_ptr")
    _require(col, "col")
    if row_ptr.dtype != torch.int32 or col.dtype != torch.int32:
        raise TypeError("row_ptr and col must be int32")
    ws = _workspace(256, row_ptr.device)
    st = _stream_ptr(stream)
    _enter(stream)
    _check(lib().dhsa_plan_check(problem.ref(), _ptr(row_ptr), _ptr(col), int(col.numel()), int(bool(per_kv_head)),
                                 _ptr(ws), ws.numel(), st), "dhsa_plan_check")
    code = int(lib().dhsa_workspace_status(_ptr(ws), st))
    _leave(stream)
    return code


class Attention:
    """Owns the attention workspace for repeated dhsa_attention calls (stream
    ordering as for Planner)."""

    def __init__(self, problem: Problem, device=None):
        self.problem = problem
        dev = problem.d_bounds.device if device is None else device
        self.ws = _workspace(problem.attention_workspace_bytes(), dev)

    def __call__(self, q, k, v, plan: Plan, out: torch.Tensor, scale: Optional[float] = None,
                 stream=None) -> torch.Tensor:
        fn = lib().dhsa_attention_kv_plan if plan.per_kv_head else lib().dhsa_attention
        _check(fn(_ptr(q), _ptr(k), _ptr(v), self.problem.ref(), _ptr(plan.row_ptr), _ptr(plan.col), plan.nnz,
                  ctypes.c_float(0.0 if scale is None else scale), _ptr(out), _ptr(self.ws), self.ws.numel(),
                  _stream_ptr(stream)), "dhsa_attention")
        return out

    def status(self, stream=None) -> int:
        return lib().dhsa_workspace_status(_ptr(self.ws), _stream_ptr(stream))


def attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, problem: Problem, plan: Plan,
              scale: Optional[float] = None, stream=None, check: bool = False) -> torch.Tensor:
    """Step 4: sparse causal attention over the plan's kept token pairs."""
    for t, name in ((q, "q"), (k, "k"), (v, "v")):
        _require(t, name)
    out = torch.empty_like(q)
    a = Attention(problem, q.device)
    _enter(stream)
    a(q, k, v, plan, out, scale, stream)
    if check:
        _check(a.status(stream), "dhsa_attention (device)")
    _leave(stream)
    return out


class Segmenter:
    """Owns the buffers of repeated online chunking calls (dhsa_segment) for
    one batch layout: sequence offsets, KV heads, head dim and rule."""

    def __init__(self, cu_seqlens, num_kv_heads: int, head_dim: int, rule, device=None):
        self.h_cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
        self.num_seqs = int(self.h_cu.shape[0] - 1)
        self.num_kv_heads, self.head_dim = int(num_kv_heads), int(head_dim)
        self.rule = rule
        self._rule = _SegmentRule(float(rule.threshold), int(rule.min_len), int(rule.max_len))
        dev = torch.device("cuda") if device is None else torch.device(device)
        L = lib()
        cap = ctypes.c_int64(0)
        _check(L.dhsa_segment_capacity(self.h_cu.ctypes.data_as(ctypes.c_void_p), self.num_seqs,
                                       int(rule.min_len), ctypes.byref(cap)), "dhsa_segment_capacity")
        self.capacity = int(cap.value)
        ws = ctypes.c_size_t(0)
        _check(L.dhsa_segment_workspace_size(int(self.h_cu[-1]), ctypes.byref(ws)), "dhsa_segment_workspace_size")
        self.ws = _workspace(ws.value, dev)
        self.d_cu = torch.from_numpy(self.h_cu).to(dev)
        self.chunk_bounds = torch.empty(self.capacity + 1, dtype=torch.int32, device=dev)
        self.seq_chunk_ptr = torch.empty(self.num_seqs + 1, dtype=torch.int32, device=dev)
        self.num_chunks = torch.empty(1, dtype=torch.int32, device=dev)

    def __call__(self, k: torch.Tensor, stream=None):
        """Asynchronous: returns the device arrays (chunk_bounds holds
        num_chunks + 1 valid entries)."""
        _require(k, "k")
        _check(lib().dhsa_segment(_ptr(k), _dtype_code(k), self.num_kv_heads, self.head_dim, self.num_seqs,
                                  _ptr(self.d_cu), self.h_cu.ctypes.data_as(ctypes.c_void_p), self._rule,
                                  _ptr(self.chunk_bounds), self.capacity, _ptr(self.seq_chunk_ptr),
                                  _ptr(self.num_chunks), _ptr(self.ws), self.ws.numel(), _stream_ptr(stream)),
               "dhsa_segment")
        return self.chunk_bounds, self.seq_chunk_ptr, self.num_chunks

    def status(self, stream=None) -> int:
        return lib().dhsa_workspace_status(_ptr(self.ws), _stream_ptr(stream))


def segment(k: torch.Tensor, cu_seqlens, rule, stream=None, check: bool = False):
    """Online variable-length chunking of the packed batch ``k`` [T, Hkv, d].

    Waits for the result and returns host int32 arrays (chunk_bounds [n+1],
    seq_chunk_ptr [B+1]), ready for ``Problem``."""
    seg = Segmenter(cu_seqlens, k.shape[1], k.shape[2], rule, k.device)
    _enter(stream)
    bounds, ptr, n = seg(k, stream)
    if check:
        _check(seg.status(stream), "dhsa_segment (device)")
    _leave(stream)
    n = int(n.item())
    return bounds[:n + 1].cpu().numpy(), ptr.cpu().numpy()


def selftest_timeout(limit_us: int = 20000, device=None) -> int:
    """Runs the bounded-wait self test; returns the status it reports (expect 5)."""
    ws = _workspace(256, torch.device("cuda") if device is None else device)
    st = _stream_ptr(None)
    _check(lib().dhsa_selftest_timeout(_ptr(ws), int(limit_us), st), "dhsa_selftest_timeout")
    return int(lib().dhsa_workspace_status(_ptr(ws), st))
