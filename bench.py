"""DHSA prefill benchmark: one step = dhsa_plan + dhsa_attention over the whole
packed batch of one attention layer (all heads).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Default workload: LLaMA-3.1-8B-shaped 128K prefill (T=131072, 32 query / 8 KV
heads, d=128, bf16, chunk lengths U[256,1024], keep 5 % of admissible key
chunks + diagonal).  Inputs are seeded synthetic tensors; the Q/K/V of one
step (1.6 GB) exceed the 126 MB L2, so consecutive steps do not hit in L2.

Prints one JSON line (rank 0).  With N > 1 (torchrun) every rank runs an
independent replica of the workload (the path has no cross-GPU exchange), so
scaling is weak and `value` = N * T * K / (max over ranks of the timed span).
`--impl reference` times the fp64 CPU oracle on a bounded sample instead.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from dynamic_hierarchical_sparse_b200 import workloads as W  # noqa: E402

METRIC = "DHSA prefill tokens/s at 128K (1 B200); attn tensor-pipe % of peak on kept FLOPs"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = W.LLAMA_128K.name

# dram__bytes_read.sum + dram__bytes_write.sum of one attention_pair_kernel<128>
# launch at the default 128K workload, from a one-pass ncu capture (the
# command is in the record).  It is a stored figure, not measured by this run,
# and it holds only for the kernel source it was captured on: the record
# keeps the SHA-256 of that source (attention_bf16_pair.cu + common.cuh), and
# any other source reports traffic as null.
ATTN_TRAFFIC_CAPTURE = {
    "bytes": 10.466e9,  # 9.427 GB read + 1.040 GB written
    "source_sha256": "14d72c73ae0e794dede9b6cad0ccff10c01b6bb6c5dd53e49fd3ff01f4e94cbd",
    "command": ("ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum --clock-control none "
                "-k regex:attention_pair -s 1 -c 1 python bench.py --steps 2 --warmup 3 --no-cpu-baseline --no-micro"),
}
ATTN_KERNEL_SOURCES = ("dynamic_hierarchical_sparse_b200/csrc/attention_bf16_pair.cu",
                       "dynamic_hierarchical_sparse_b200/csrc/common.cuh")

# FP32 FFMA ceiling of one B200: 148 SMs x 128 FP32 lanes x 2 FLOP per FMA x 1965 MHz
FP32_FFMA_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                "sustained_sm_mhz": (p.get("clocks_under_load") or {}).get("sm_mhz_median"),
                "sm_max_mhz": p.get("sm_max_mhz"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "sustained_sm_mhz": 1300.0, "sm_max_mhz": 1965.0, "source": "fallback"}


def tensor_peak(peaks, clk):
    """The bf16 peak a kernel timed in this run is held against, from the SM
    clock sampled during the timed region.  Two GEMM figures were measured:
    the burst one (timed alone, taken at the maximum clock) and the sustained
    one (a seconds-long loop under the power cap, at its recorded median
    clock).  The peak is the straight line through those two (clock, TFLOP/s)
    points at this run's median clock, kept between the two figures: the burst
    figure at the maximum clock, the sustained one at or below its clock.  A
    run whose clock was not sampled gets the burst figure.  Returns (peak, kind)."""
    sm, smax = clk.get("sm_mhz"), clk.get("sm_max_mhz") or peaks.get("sm_max_mhz")
    burst, sust, s_mhz = peaks["bf16_tflops"], peaks["bf16_tflops_sustained"], peaks.get("sustained_sm_mhz")
    if sm is None or not smax or sm >= smax or not s_mhz or s_mhz >= smax:
        return burst, ("%s bf16 dense, burst (this run's median SM clock %s MHz, the maximum %s MHz)"
                       % (peaks["source"], "%.0f" % sm if sm is not None else "unsampled", smax))
    if sm <= s_mhz:
        return sust, ("%s bf16 dense, sustained (this run's median SM clock %.0f MHz is at or below the %.0f MHz "
                      "of the sustained figure)" % (peaks["source"], sm, s_mhz))
    peak = sust + (burst - sust) * (sm - s_mhz) / (smax - s_mhz)
    return peak, ("%s bf16 dense at this run's median SM clock %.0f MHz: the line through the sustained figure "
                  "(%.0f TFLOP/s at %.0f MHz) and the burst figure (%.0f at the maximum %.0f MHz)"
                  % (peaks["source"], sm, sust, s_mhz, burst, smax))


def attention_traffic():
    """The stored per-launch DRAM traffic of the attention kernel, or None when
    the kernel source differs from the one it was captured on."""
    import hashlib

    if ATTN_TRAFFIC_CAPTURE is None:
        return None, "no capture of the current kernel source"
    h = hashlib.sha256()
    for rel in ATTN_KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    if h.hexdigest() != ATTN_TRAFFIC_CAPTURE["source_sha256"]:
        return None, "kernel source changed since the capture"
    return ATTN_TRAFFIC_CAPTURE["bytes"], ("stored ncu capture (one pass, not this run) of this kernel source: %s"
                                           % ATTN_TRAFFIC_CAPTURE["command"])


def kept_pairs(bounds, row_ptr, col, num_chunks):
    """Exact (query token, key token, head) pairs kept by a plan."""
    lens = np.diff(np.asarray(bounds, dtype=np.int64))
    rp = np.asarray(row_ptr, dtype=np.int64)
    cl = np.asarray(col, dtype=np.int64)
    rows = np.repeat(np.arange(rp.shape[0] - 1), np.diff(rp))
    ci = rows % num_chunks
    Li = lens[ci]
    Lj = lens[cl]
    per = np.where(cl == ci, Li * (Li + 1) // 2, Li * Lj)
    return int(per.sum())


class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons while the timed region runs.

    nvidia-smi starts sampling before the timed region (it needs a moment to
    start), so each line is stamped with the host time it arrived, and only the
    lines that arrived between mark_start() and mark_stop() count.  If none did
    (output held back by buffering, or a region shorter than one interval), all
    lines are used and the record says so."""

    INTERVAL_MS = 100

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []  # (host time of arrival, line)
        self.thread = None
        self.t0 = None
        self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", str(self.INTERVAL_MS)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark_start(self):
        """Host time at which the timed region starts (call just before it)."""
        self.t0 = time.time()

    def mark_stop(self):
        """Host time at which the timed region has ended (call after the synchronize)."""
        self.t1 = time.time()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)
        return self.summarise(self.lines, self.t0, self.t1)

    @staticmethod
    def summarise(lines, t0, t1):
        """Median SM clock, maximum clock and throttle reasons of the samples
        that arrived in [t0, t1], else of all samples."""
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        rows = []  # (arrival, sm MHz, max MHz, active reasons)
        for t, ln in lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm, smax = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            rows.append((t, sm, smax, {nm for nm, val in zip(names, parts[5:9]) if val.lower().startswith("active")}))
        inside = [r for r in rows if t0 is not None and t1 is not None and t0 <= r[0] <= t1]
        use = inside if inside else rows
        reasons = set().union(*(r[3] for r in use)) if use else set()
        return {"sm_mhz": statistics.median(r[1] for r in use) if use else None,
                "sm_max_mhz": use[-1][2] if use else None,
                "reasons": sorted(reasons), "samples": len(use), "samples_total": len(rows),
                "window": "samples that arrived during the timed region" if inside else
                          "all samples (none arrived during the timed region)"}


def _dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def _barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """Largest value over all ranks (the timed span of the slowest replica)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tokens_per_s(world: int, tokens_per_replica: int, steps: int, max_elapsed_s: float) -> float:
    """Weak scaling: every rank runs one replica of the workload; the job's rate is
    all ranks' tokens over the slowest rank's timed span."""
    return world * tokens_per_replica * steps / max_elapsed_s


def run_cpu_oracle(inp, budget_seconds: float = 20.0, per_kv_head: bool = False, gpu_plan=None, gpu_out=None):
    """Times the fp64 oracle, as it stands, on a bounded sample of the workload.

    Sample: the oracle's full planning step (steps 1-3) on the whole workload,
    then attention (chunk-gather form) for seeded random (head, query chunk)
    pairs until about `budget_seconds` of attention work is done; that
    attention time is scaled to the whole layer by kept pairs.

    With the GPU's plan (host row_ptr, col) and output (device [T, Hq, d]),
    the figures it computed anyway also give the run's parity record: plan rows
    that differ from the oracle's, and the error of the GPU output on the
    sampled (head, query chunk) blocks (outside every timed region).
    """
    from oracle import dhsa_oracle as O

    b = inp.budget
    spec = inp.spec
    group = spec.num_q_heads // spec.num_kv_heads if per_kv_head else 1
    t0 = time.perf_counter()
    ref = O.build_plan(inp.q, inp.k, inp.chunk_bounds, inp.seq_chunk_ptr, b.kind, b.k, b.num, b.den,
                       per_kv_head=per_kv_head)
    t_plan = time.perf_counter() - t0
    n = inp.num_chunks
    lens = np.diff(inp.chunk_bounds.astype(np.int64))
    rp = ref["row_ptr"]
    total_pairs = kept_pairs(inp.chunk_bounds, rp, ref["col"], n) * group
    rng = np.random.default_rng(0)
    order = rng.permutation(spec.num_q_heads * n)
    done_pairs, t_attn, chunks_done = 0, 0.0, 0
    same_rows = None
    if gpu_plan is not None:
        grp, gcl = (np.asarray(x, dtype=np.int64) for x in gpu_plan)
        nrows = rp.shape[0] - 1
        same_rows = np.array([np.array_equal(gcl[grp[r]:grp[r + 1]], ref["col"][rp[r]:rp[r + 1]])
                              for r in range(nrows)])
    err_max, err_sq, ref_sq, ref_max, compared = 0.0, 0.0, 0.0, 0.0, 0
    for hr in order:
        h, i = int(hr) // n, int(hr) % n
        r = (h // group) * n + i
        t1 = time.perf_counter()
        o_ref = O.attention_query_chunk(inp.q, inp.k, inp.v, inp.chunk_bounds, rp, ref["col"], h, i,
                                        per_kv_head=per_kv_head)
        t_attn += time.perf_counter() - t1
        if gpu_out is not None and same_rows[r]:
            b0, b1 = int(inp.chunk_bounds[i]), int(inp.chunk_bounds[i + 1])
            got = gpu_out[b0:b1, h].double().cpu().numpy()
            e = got - o_ref
            err_max = max(err_max, float(np.abs(e).max()))
            err_sq += float((e * e).sum())
            ref_sq += float((o_ref * o_ref).sum())
            ref_max = max(ref_max, float(np.abs(o_ref).max()))
            compared += 1
        for j in ref["col"][rp[r]:rp[r + 1]]:
            done_pairs += int(lens[i] * (lens[i] + 1) // 2 if j == i else lens[i] * lens[j])
        chunks_done += 1
        if t_attn > budget_seconds:
            break
    t_attn_total = t_attn * total_pairs / max(done_pairs, 1)
    T = int(inp.cu_seqlens[-1])
    value = T / (t_plan + t_attn_total)
    threads = None
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        threads = max((x.get("num_threads") or 1) for x in info) if info else 1
    except Exception:
        threads = None
    cores = len(os.sched_getaffinity(0))
    parity = None
    if same_rows is not None:
        parity = {"plan_rows": int(same_rows.shape[0]), "plan_rows_differing": int((~same_rows).sum()),
                  "attention_blocks_compared": compared, "max_abs_err": err_max,
                  "rel_fro": math.sqrt(err_sq / ref_sq) if ref_sq > 0 else None, "max_abs_ref": ref_max,
                  "what": "GPU plan against the oracle's (row by row), and the GPU output on the oracle's sampled "
                          "(head, query chunk) blocks whose plan rows agree"}
    return {
        "parity": parity, "t_step_s": t_plan + t_attn, "sampled_pairs": done_pairs, "total_pairs": total_pairs,
        "value": value, "unit": UNIT, "cores": threads if threads else cores, "kind": "oracle",
        "sample": ("fp64 oracle: full plan (steps 1-3) on all %d tokens in %.1f s; attention for %d random "
                   "(head, query chunk) pairs of %d (%.2f%% of kept pairs) in %.1f s, scaled by kept pairs to "
                   "%.0f s for the whole layer; host has %d cores, BLAS threads %s"
                   % (T, t_plan, chunks_done, spec.num_q_heads * n, 100.0 * done_pairs / total_pairs, t_attn,
                      t_attn_total, cores, threads)),
    }


L2_BYTES = 126 * 10**6
L2_FLUSH_BYTES = 256 * 2**20


def qkv_bytes(spec) -> int:
    elt = 2 if spec.dtype == "bf16" else 4
    return spec.total_tokens * (spec.num_q_heads + 2 * spec.num_kv_heads) * spec.head_dim * elt


def needs_l2_flush(spec) -> bool:
    """Inputs that fit in L2 would be timed warm without a flush between steps."""
    return qkv_bytes(spec) <= L2_BYTES


def _config(spec, inp, budget, pairs, world):
    """The workload description both arms print (identical keys and values)."""
    qkv = qkv_bytes(spec)
    l2 = ("no flush: each step streams Q/K/V (%.2f GB) > 126 MB L2" % (qkv / 1e9) if not needs_l2_flush(spec) else
          "L2 flushed before every timed step (a %d MB write); Q/K/V %.3f GB fit in the 126 MB L2, so the "
          "value is the sum of the per-step event times, without the flushes" % (L2_FLUSH_BYTES >> 20, qkv / 1e9))
    return {
        "workload": spec.name, "tokens": spec.total_tokens, "num_seqs": len(spec.seq_lens),
        "q_heads": spec.num_q_heads, "kv_heads": spec.num_kv_heads, "head_dim": spec.head_dim,
        "num_chunks": inp.num_chunks, "budget": _budget_str(budget),
        "kept_pairs": pairs, "kept_pairs_frac_of_causal": pairs / (spec.num_q_heads * sum(
            L * (L + 1) // 2 for L in spec.seq_lens)),
        "parallelism": "replica per GPU" if world > 1 else "single GPU",
        "l2": l2,
    }


def plan_kernel_rates(prob, q, k, budget, reps: int = 10):
    """Each planning kernel timed alone, through its own entry point (chunk
    reduce of Q, of K, chunk similarity, select), with CUDA events around every
    launch, outside the benchmark's timed region.  Returns per kernel the
    mean milliseconds, the algorithmic bytes and the achieved GB/s.  (The plan
    itself reduces Q and K in one launch; here they are two.)"""
    import ctypes

    from dynamic_hierarchical_sparse_b200 import api

    L = api.lib()
    dev = q.device
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    n = prob.num_chunks
    qc = torch.empty(Hq, n, d, dtype=torch.float32, device=dev)
    kc = torch.empty(Hkv, n, d, dtype=torch.float32, device=dev)
    scores = torch.zeros(Hq, n, n, dtype=torch.float32, device=dev)
    nnz = prob.nnz(budget)
    row_ptr = torch.empty(Hq * n + 1, dtype=torch.int32, device=dev)
    col = torch.empty(max(nnz, 1), dtype=torch.int32, device=dev)
    ws = torch.empty(256, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    st = ctypes.c_void_p(stream.cuda_stream)
    P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    dt = api._dtype_code(q)
    b = api._budget(budget)
    launches = {
        "chunk_reduce_q": lambda: L.dhsa_chunk_reduce(P(q), dt, T, Hq, d, P(prob.d_bounds), n, P(qc), st),
        "chunk_reduce_k": lambda: L.dhsa_chunk_reduce(P(k), dt, T, Hkv, d, P(prob.d_bounds), n, P(kc), st),
        "chunk_similarity": lambda: L.dhsa_chunk_similarity(P(qc), P(kc), prob.ref(), P(scores), st),
        "topk_select": lambda: L.dhsa_topk_select(P(scores), prob.ref(), b, P(row_ptr), P(col), nnz, P(ws),
                                                  ws.numel(), st),
    }
    times = {}
    for name, fn in launches.items():
        for _ in range(2):
            if fn() != 0:
                raise RuntimeError("%s failed" % name)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for e0, e1 in evs:
            e0.record(stream)
            fn()
            e1.record(stream)
        torch.cuda.synchronize()
        times[name] = statistics.mean(e0.elapsed_time(e1) for e0, e1 in evs) / 1e3
    m = np.diff(np.asarray(prob.h_sptr, dtype=np.int64))
    elt = q.element_size()
    tri_incl = int(Hq * (m * (m + 1) // 2).sum() * 4)   # scores written, diagonal included
    tri_strict = int(Hq * (m * (m - 1) // 2).sum() * 4)  # scores the selection reads
    bytes_ = {
        "chunk_reduce": (q.numel() + k.numel()) * elt + (Hq + Hkv) * n * d * 4,
        "chunk_similarity": (Hq + Hkv) * n * d * 4 + tri_incl,
        "topk_select": tri_strict + (nnz + Hq * n + 1) * 4,
    }
    t = {"chunk_reduce": times["chunk_reduce_q"] + times["chunk_reduce_k"],
         "chunk_similarity": times["chunk_similarity"], "topk_select": times["topk_select"]}
    peaks = _peaks()
    out = {}
    for name in ("chunk_reduce", "chunk_similarity", "topk_select"):
        gbs = bytes_[name] / t[name] / 1e9
        out[name] = {"ms": t[name] * 1e3, "bytes": int(bytes_[name]), "gbs": gbs, "frac": gbs / peaks["hbm_gbs"]}
    out["chunk_reduce"]["note"] = "Q and K reduced in two launches here (one in the plan)"
    out["topk_select"]["note"] = ("the score triangle here is %.1f MB, below what HBM streaming needs; "
                                  "select_micro is the size where its bytes matter" % (tri_strict / 1e6))
    out["peak_kind"] = "%s copy bandwidth %.0f GB/s" % (peaks["source"], peaks["hbm_gbs"])
    return out


def bench_gpu(args):
    from dynamic_hierarchical_sparse_b200 import api

    world, rank, local = _dist_setup(args.gpus)
    spec = W.BY_NAME[args.workload]
    inp = W.generate(spec, seed=rank)
    dev = torch.device("cuda", local)
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    prob = api.Problem.from_inputs(inp, dev)
    budget = inp.budget.kv() if args.kv_plan else inp.budget
    group = spec.num_q_heads // spec.num_kv_heads if args.kv_plan else 1
    planner = api.Planner(prob, budget, dev)
    attn = api.Attention(prob, dev)
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream(dev)
    T = int(inp.cu_seqlens[-1])

    def step():
        p = planner(q, k)
        attn(q, k, v, p, out)
        return p

    for _ in range(args.warmup):
        plan = step()
    torch.cuda.synchronize()
    if planner.status() != 0 or attn.status() != 0:
        raise RuntimeError("device-side status set during warm-up")
    plan = planner(q, k)
    torch.cuda.synchronize()
    pairs = kept_pairs(inp.chunk_bounds, plan.row_ptr.cpu().numpy(), plan.col[:plan.nnz].cpu().numpy(),
                       inp.num_chunks) * group
    flops_attn = 4.0 * spec.head_dim * pairs
    reduce_bytes = (q.numel() + k.numel()) * q.element_size()

    # ---------------- device-timed region: K full steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev) if needs_l2_flush(spec) else None
    clocks = ClockSampler(local)
    _barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    clocks.mark_start()
    start.record(stream)
    for i in range(args.steps):
        if flush is not None:
            flush.fill_(i & 255)
        ev[i][0].record(stream)
        p = planner(q, k)
        ev[i][1].record(stream)
        attn(q, k, v, p, out)
        ev[i][2].record(stream)
    stop.record(stream)
    torch.cuda.synchronize()
    clocks.mark_stop()
    clk = clocks.stop()
    _barrier(world)
    elapsed_s = start.elapsed_time(stop) / 1e3
    if flush is not None:  # the flushes are not part of the work
        elapsed_s = sum(a.elapsed_time(c) for a, _, c in ev) / 1e3
    t_plan = statistics.mean(a.elapsed_time(b) for a, b, _ in ev) / 1e3
    t_attn = statistics.mean(b.elapsed_time(c) for _, b, c in ev) / 1e3
    if planner.status() != 0 or attn.status() != 0:
        raise RuntimeError("device-side status set during the timed region")
    max_elapsed = _max_over_ranks(elapsed_s, world)
    value = whole_job_tokens_per_s(world, T, args.steps, max_elapsed)

    # ---------------- end to end through the public API with host buffers
    # Every step copies its Q/K/V in from pinned host memory and its output
    # back out.  Three device buffer sets and three streams let step i's
    # copy-out, step i+1's copy-in and step i's plan + attention overlap (the
    # copies run in opposite directions over the host link), as a prefill
    # server streaming requests would run them; with three sets a copy-in
    # never waits for the copy-out of the step before.
    nbuf = 3
    hq = inp.q.pin_memory()
    hk = inp.k.pin_memory()
    hv = inp.v.pin_memory()
    houts = [torch.empty(inp.q.shape, dtype=inp.q.dtype).pin_memory() for _ in range(nbuf)]
    dq = [q] + [torch.empty_like(q) for _ in range(nbuf - 1)]
    dk = [k] + [torch.empty_like(k) for _ in range(nbuf - 1)]
    dv = [v] + [torch.empty_like(v) for _ in range(nbuf - 1)]
    douts = [out] + [torch.empty_like(out) for _ in range(nbuf - 1)]
    s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev_in, ev_cmp, ev_out = ([torch.cuda.Event() for _ in range(nbuf)] for _ in range(3))
    e2e_steps = max(2, min(args.steps, 24))  # the stream's fill and drain amortised over up to 24 steps

    def e2e_run(nsteps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        for i in range(nsteps):
            b = i % nbuf
            if i >= nbuf:  # buffer set b is free once step i-nbuf's attention and copy-out are done
                s_in.wait_event(ev_cmp[b])
                s_in.wait_event(ev_out[b])
            with torch.cuda.stream(s_in):
                dq[b].copy_(hq, non_blocking=True)
                dk[b].copy_(hk, non_blocking=True)
                dv[b].copy_(hv, non_blocking=True)
            ev_in[b].record(s_in)
            s_cmp.wait_event(ev_in[b])
            p = planner(dq[b], dk[b], stream=s_cmp)
            attn(dq[b], dk[b], dv[b], p, douts[b], stream=s_cmp)
            ev_cmp[b].record(s_cmp)
            s_out.wait_event(ev_cmp[b])
            with torch.cuda.stream(s_out):
                houts[b].copy_(douts[b], non_blocking=True)
            ev_out[b].record(s_out)
        e1.record(s_out)
        return e0, e1

    e2e_run(2)
    torch.cuda.synchronize()
    _barrier(world)
    e0, e1 = e2e_run(e2e_steps)
    torch.cuda.synchronize()
    if planner.status() != 0 or attn.status() != 0:
        raise RuntimeError("device-side status set during the end-to-end run")
    e2e_s = _max_over_ranks(e0.elapsed_time(e1) / 1e3, world)
    e2e_value = whole_job_tokens_per_s(world, T, e2e_steps, e2e_s)
    h2d = (hq.numel() + hk.numel() + hv.numel()) * hq.element_size()
    d2h = houts[0].numel() * houts[0].element_size()

    peaks = _peaks()
    achieved_tflops = flops_attn / t_attn / 1e12
    traffic, traffic_kind = None, "no capture of this workload"
    if spec.dtype == "bf16":
        kernel = ("attention_pair_kernel<%d>" % spec.head_dim if spec.head_dim in (64, 128)
                  else "attention_d256_kernel")
        bound = "tensor"
        peak, peak_kind = tensor_peak(peaks, clk)
        if spec.name == DEFAULT_WORKLOAD and not args.kv_plan:
            traffic, traffic_kind = attention_traffic()
    else:
        # fp32 inputs run the FFMA kernel: its ceiling is the FP32 pipe, not the tensor cores
        kernel, bound, peak = "attention_f32_kernel<%d>" % spec.head_dim, "alu", FP32_FFMA_TFLOPS
        peak_kind = "nominal fp32 FFMA: 148 SMs x 128 lanes x 2 FLOP x 1965 MHz"
    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": max_elapsed / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if spec.dtype == "bf16" else "f32",
        "data": "synthetic (seeded; rank-4 shared component, scale 2)",
        "config": _config(spec, inp, budget, pairs, world),
        "t_plan_ms": t_plan * 1e3, "t_attn_ms": t_attn * 1e3,
        "plan_hbm_gbs": reduce_bytes / t_plan / 1e9,
        "roofline": {
            "kernel": kernel, "bound": bound, "achieved": achieved_tflops,
            "peak": peak, "unit": "TFLOP/s", "frac": achieved_tflops / peak, "peak_kind": peak_kind,
            "frac_of_burst": (achieved_tflops / peaks["bf16_tflops"]) if bound == "tensor" else None,
            "frac_of_sustained": (achieved_tflops / peaks["bf16_tflops_sustained"]) if bound == "tensor" else None,
            "traffic": traffic, "traffic_kind": traffic_kind,
            "algorithmic_flops_per_launch": flops_attn,
            "how": "achieved = 4 * head_dim * kept pairs (counted from this run's plan) / mean event-timed "
                   "attention launch over the timed steps",
        },
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps,
                "schedule": "each step copies Q/K/V in from pinned host memory and O out; copy-in, "
                            "plan + attention and copy-out of consecutive steps overlap on three streams "
                            "(three device buffer sets)"},
        # per step: chunk reduce (Q and K in one launch), [group sum,] similarity, select, attention
        # reduce, similarity, (group sum,) select; the f16 copy of V (bf16) and attention
        "gpu_launches": ((5 if args.kv_plan else 4) + (1 if spec.dtype == "bf16" else 0)) * args.steps,
        "clocks": clk,
    }
    if rank == 0 and world == 1:
        if not args.kv_plan:
            result["kernels"] = plan_kernel_rates(prob, q, k, budget)
        if not args.no_micro and spec.name == DEFAULT_WORKLOAD:
            result["select_micro"] = select_micro_result(args.warmup, 20)
        if not args.no_cpu_baseline:
            attn(q, k, v, plan, out)
            cb = run_cpu_oracle(inp, args.cpu_seconds, per_kv_head=args.kv_plan,
                                gpu_plan=(plan.row_ptr.cpu().numpy(), plan.col[:plan.nnz].cpu().numpy()),
                                gpu_out=out)
            result["parity"] = cb.pop("parity")
            for key in ("t_step_s", "sampled_pairs", "total_pairs"):
                cb.pop(key)
            result["cpu_baseline"] = cb
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


SELECT_MICRO = W.WorkloadSpec(
    "select_micro_128k_h32_chunks16to64_frac5", [131072], 32, 8, 128, "bf16", 16, 64,
    W.Budget.fraction(1, 20), "normal")


def select_micro_inputs(seed: int = 0):
    """Chunk structure of the select micro-benchmark (no token tensors needed)."""
    rng = np.random.default_rng(seed)
    lens = W.chunk_lengths_until(rng, SELECT_MICRO.seq_lens[0], SELECT_MICRO.chunk_lo, SELECT_MICRO.chunk_hi)
    return W.make_bounds(SELECT_MICRO.seq_lens, [lens])


def triangle_bytes(seq_chunk_ptr, num_q_heads):
    ptr = np.asarray(seq_chunk_ptr, dtype=np.int64)
    m = np.diff(ptr)
    return int(num_q_heads * (m * (m - 1) // 2).sum() * 4)


def bench_select_micro(args):
    torch.cuda.set_device(0)
    print(json.dumps(select_micro_result(args.warmup, args.steps)), flush=True)


def select_micro_result(warmup: int, steps: int):
    """Step 3 alone at a size where its bytes matter: T=131072, 32 heads,
    chunk lengths U[16,64] (n ~ 3300), keep 5 % + diagonal, fp32 scores
    drawn N(0,1) on the device.  Reports achieved GB/s on the algorithmic bytes
    (causal score triangle read + plan written) against measured HBM."""
    from dynamic_hierarchical_sparse_b200 import api

    dev = torch.device("cuda", torch.cuda.current_device())
    cu, bounds, sptr = select_micro_inputs(0)
    spec = SELECT_MICRO
    prob = api.Problem(cu, bounds, sptr, spec.num_q_heads, spec.num_kv_heads, spec.head_dim, torch.bfloat16, dev)
    n = prob.num_chunks
    gen = torch.Generator(device=dev).manual_seed(0)
    scores = torch.randn(spec.num_q_heads, n, n, generator=gen, device=dev, dtype=torch.float32)
    budget = spec.budget
    plan = api.topk_select(scores, prob, budget, check=True)
    for _ in range(warmup):
        api.topk_select(scores, prob, budget)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # the triangle (0.69 GB) is read once per call and exceeds L2, so calls do not hit in L2
    e0.record(stream)
    for _ in range(steps):
        api.topk_select(scores, prob, budget)
    e1.record(stream)
    torch.cuda.synchronize()
    t = e0.elapsed_time(e1) / 1e3 / steps
    tri = triangle_bytes(sptr, spec.num_q_heads)
    out_bytes = (plan.nnz + plan.row_ptr.numel()) * 4
    gbs = (tri + out_bytes) / t / 1e9
    peaks = _peaks()
    del scores
    torch.cuda.empty_cache()
    return {
        "metric": "select kernel HBM GB/s (micro-benchmark)", "value": gbs, "unit": "GB/s",
        "n_gpus": 1, "steps": steps, "warmup": warmup, "ms_per_call": t * 1e3,
        "higher_is_better": True, "dtype": "f32", "data": "synthetic N(0,1) scores (seeded, on device)",
        "config": {"workload": spec.name, "tokens": int(cu[-1]), "q_heads": spec.num_q_heads, "num_chunks": n,
                   "budget": _budget_str(budget), "nnz": plan.nnz, "triangle_bytes": tri,
                   "l2": "no flush: triangle %.2f GB > 126 MB L2" % (tri / 1e9)},
        "roofline": {"kernel": "topk_select_kernel", "bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                     "peak_kind": "%s copy bandwidth" % peaks["source"]},
        "gpu_launches": steps,  # one select kernel per call
    }


SEGMENT_MICRO = dict(name="segment_micro_128k_kv8_d128_bf16_planted256to1024", tokens=131072, hkv=8, d=128,
                     lo=256, hi=1024, rule=W.SegmentRule(0.5, 256, 1024))


def bench_segment_micro(args):
    """Online chunking alone on the 128K LLaMA key shape (K [131072, 8, 128]
    bf16, 268 MB), keys with planted segments U[256, 1024] (the 128K
    workload's chunk lengths), rule threshold 0.5, min 256, max 1024.  One call
    is two launches (adjacent-key similarity bits, then the walk, which writes the chunk
    bounds itself for a batch of one sequence).
    Algorithmic bytes: every key read once plus the two bitmaps written and
    read (T/8 bytes each way) and the bounds written."""
    from dynamic_hierarchical_sparse_b200 import api
    from oracle import dhsa_oracle as O

    cfg = SEGMENT_MICRO
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    k_host, cu, bounds, ptr = W.planted_segment_keys(0, [cfg["tokens"]], cfg["hkv"], cfg["d"], cfg["lo"], cfg["hi"])
    k = k_host.to(dev)
    seg = api.Segmenter(cu, cfg["hkv"], cfg["d"], cfg["rule"], dev)
    b, p, n = seg(k)
    assert seg.status() == 0
    n = int(n.item())
    if not (np.array_equal(b[:n + 1].cpu().numpy(), bounds) and np.array_equal(p.cpu().numpy(), ptr)):
        raise RuntimeError("segmentation does not recover the planted segments")
    for _ in range(args.warmup):
        seg(k)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(0)
    clocks.start()
    time.sleep(0.3)
    clocks.mark_start()
    e0.record(stream)
    for _ in range(args.steps):
        seg(k)
    e1.record(stream)
    torch.cuda.synchronize()
    clocks.mark_stop()
    clk = clocks.stop()
    t = e0.elapsed_time(e1) / 1e3 / args.steps
    T = cfg["tokens"]
    key_bytes = T * cfg["hkv"] * cfg["d"] * 2
    algo = key_bytes + 4 * (T // 8) + 4 * (n + 1) + 4 * 2
    gbs = algo / t / 1e9
    peaks = _peaks()
    res = {
        "metric": "online chunking HBM GB/s (micro-benchmark)", "value": gbs, "unit": "GB/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_call": t * 1e3, "tokens_per_s": T / t,
        "higher_is_better": True, "dtype": "bf16 keys, f32 similarity",
        "data": "synthetic keys with planted segments (seeded)",
        "config": {"workload": cfg["name"], "tokens": T, "kv_heads": cfg["hkv"], "head_dim": cfg["d"],
                   "rule": {"threshold": cfg["rule"].threshold, "min_len": cfg["rule"].min_len,
                            "max_len": cfg["rule"].max_len},
                   "num_chunks": n, "l2": "no flush: keys %.2f GB > 126 MB L2" % (key_bytes / 1e9)},
        "roofline": {"kernel": "dhsa_segment (2 launches; adjacent_sim_kernel dominant)", "bound": "hbm",
                     "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                     "peak_kind": "%s copy bandwidth" % peaks["source"],
                     "note": "whole call timed: the walk and compaction count against it"},
        "gpu_launches": 2 * args.steps,  # similarity, walk (with the compaction: one sequence) per call
        "clocks": clk,
    }
    if not args.no_cpu_baseline:
        sample = 16384
        t0 = time.perf_counter()
        O.segment(k_host[:sample], [0, sample], cfg["rule"].threshold, cfg["rule"].min_len, cfg["rule"].max_len)
        dt = time.perf_counter() - t0
        res["cpu_baseline"] = {"value": sample / dt, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                               "sample": "first %d tokens of the same keys" % sample,
                               "gpu_value_same_unit": T / t}
    print(json.dumps(res), flush=True)


def bench_online_chunking(args):
    """The whole layer with online chunking: each step segments the keys on the
    device (dhsa_segment), reads the chunk count and boundaries back to build
    the problem on the host (the later steps size their launches from them),
    then plans and attends.  128K LLaMA shape; the keys carry planted segments
    U[256, 1024] (the default workload's chunk lengths), Q and V are the default
    workload's.  Device-timed with CUDA events around whole steps, so the
    host round trip is inside the timed region."""
    from dynamic_hierarchical_sparse_b200 import api

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    spec = W.LLAMA_128K
    inp = W.generate(spec, seed=0)
    T = spec.total_tokens
    k_host, cu, planted, planted_ptr = W.planted_segment_keys(0, [T], spec.num_kv_heads, spec.head_dim, 256, 1024)
    rule = W.SegmentRule(0.5, 256, 1024)
    q, k, v = inp.q.to(dev), k_host.to(dev), inp.v.to(dev)
    out = torch.empty_like(q)
    seg = api.Segmenter(cu, spec.num_kv_heads, spec.head_dim, rule, dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        b, p, n = seg(k)
        nh = int(n.item())  # waits for the segmentation
        hb = b[:nh + 1].cpu().numpy()
        hp = p.cpu().numpy()
        if ev is not None:
            ev[1].record(stream)
        prob = api.Problem(cu, hb, hp, spec.num_q_heads, spec.num_kv_heads, spec.head_dim, q.dtype, dev)
        plan = api.Planner(prob, inp.budget, dev)(q, k)
        if ev is not None:
            ev[2].record(stream)
        api.Attention(prob, dev)(q, k, v, plan, out)
        if ev is not None:
            ev[3].record(stream)
        return hb, hp

    for _ in range(args.warmup):
        hb, hp = step()
    torch.cuda.synchronize()
    if seg.status() != 0:
        raise RuntimeError("device-side status set during warm-up")
    if not (np.array_equal(hb, planted) and np.array_equal(hp, planted_ptr)):
        raise RuntimeError("online chunking did not recover the planted segments")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    clocks = ClockSampler(0)
    clocks.start()
    time.sleep(0.3)
    torch.cuda.synchronize()
    clocks.mark_start()
    for i in range(args.steps):
        step(evs[i])
    torch.cuda.synchronize()
    clocks.mark_stop()
    clk = clocks.stop()
    total = sum(e[0].elapsed_time(e[3]) for e in evs) / 1e3
    part = [statistics.mean(e[j].elapsed_time(e[j + 1]) for e in evs) for j in range(3)]
    print(json.dumps({
        "metric": "DHSA prefill tokens/s at 128K with online chunking (1 B200)", "value": T * args.steps / total,
        "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total / args.steps * 1e3, "higher_is_better": True, "dtype": "bf16",
        "data": "synthetic (seeded; keys with planted segments U[256,1024])",
        "config": {"workload": "llama31_8b_128k_h32kv8_d128_bf16_frac5 with online chunking",
                   "rule": {"threshold": rule.threshold, "min_len": rule.min_len, "max_len": rule.max_len},
                   "num_chunks": int(hb.shape[0] - 1), "budget": _budget_str(inp.budget)},
        "ms_segment_and_readback": part[0], "ms_plan": part[1], "ms_attention": part[2],
        "gpu_launches": 7 * args.steps,  # segment 2 (one sequence), plan 3, f16 copy of V 1, attention 1 per step
        "clocks": clk,
    }), flush=True)


def memory_report(spec, seed: int = 0, device=None):
    """Device memory of one DHSA layer call beyond its inputs and output.

    Returns a dict with the library's size queries (plan workspace, plan
    arrays, attention workspace), the measured peak of allocations made while
    planning and attending (torch's allocator statistics, inputs and output
    allocated beforehand), and, for scale, the bytes of Q/K/V/O and of a dense
    score matrix [Hq, T, T] in bf16 that attention without tiling would hold.
    """
    from dynamic_hierarchical_sparse_b200 import api

    dev = device or torch.device("cuda", 0)
    inp = W.generate(spec, seed=seed)
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    out = torch.empty_like(q)
    prob = api.Problem.from_inputs(inp, dev)
    torch.cuda.synchronize(dev)
    torch.cuda.reset_peak_memory_stats(dev)
    base = torch.cuda.memory_allocated(dev)
    planner = api.Planner(prob, inp.budget, dev)
    attn = api.Attention(prob, dev)
    plan = planner(q, k)
    attn(q, k, v, plan, out)
    torch.cuda.synchronize(dev)
    peak_extra = torch.cuda.max_memory_allocated(dev) - base
    T = int(inp.cu_seqlens[-1])
    io = (q.numel() + k.numel() + v.numel() + out.numel()) * q.element_size()
    seq = np.diff(np.asarray(inp.cu_seqlens, dtype=np.int64))
    rep = {
        "workload": spec.name, "tokens": T, "num_chunks": inp.num_chunks,
        "plan_workspace_bytes": prob.plan_workspace_bytes(inp.budget),
        "plan_bytes": (prob.num_q_heads * prob.num_chunks + 1 + prob.nnz(inp.budget)) * 4,
        "attention_workspace_bytes": prob.attention_workspace_bytes(),
        "measured_peak_extra_bytes": int(peak_extra),
        "qkvo_bytes": int(io),
        "dense_scores_bf16_bytes": int(spec.num_q_heads * int((seq * seq).sum()) * 2),
    }
    rep["extra_over_qkvo"] = rep["measured_peak_extra_bytes"] / io
    del planner, attn, plan, q, k, v, out
    torch.cuda.empty_cache()
    return rep


def bench_memory(args):
    """Peak device memory of plan + attention at each shape (one JSON line each)."""
    torch.cuda.set_device(0)
    for spec in (W.GEMMA2_8K, W.LLAMA_32K, W.RAGGED_NEEDLE, W.LLAMA_128K, W.BLOCKSPARSE_128K):
        rep = memory_report(spec)
        print(json.dumps(dict(metric="DHSA extra device memory per layer call", unit="bytes",
                              value=rep["measured_peak_extra_bytes"], higher_is_better=False, **rep)), flush=True)


DENSE_SHAPES = (W.GEMMA2_8K, W.LLAMA_32K, W.LLAMA_128K)


def _timed_steps(fn, steps, warmup, stream):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / 1e3 / steps


def _extra_bytes(fn, dev):
    """Peak bytes allocated while fn runs, beyond what was allocated before."""
    torch.cuda.synchronize(dev)
    torch.cuda.reset_peak_memory_stats(dev)
    base = torch.cuda.memory_allocated(dev)
    keep = fn()
    torch.cuda.synchronize(dev)
    peak = torch.cuda.max_memory_allocated(dev) - base
    del keep
    return int(peak)


def bench_dense(args):
    """Sparse DHSA against dense causal attention on the same inputs, one JSON
    line per shape (Gemma2 8K, LLaMA 32K, LLaMA 128K): time of plan +
    attention and the device memory a layer call allocates beyond Q/K/V/O.

    Dense arms: (1) the same library with a budget that keeps every admissible
    chunk (every row dense causal: the same kernels doing dense work), and (2)
    torch's scaled_dot_product_attention (a FlashAttention-style library
    kernel, causal, grouped-query), for context.  Inputs are resident; no L2
    flush (each step streams more than the L2 holds)."""
    from dynamic_hierarchical_sparse_b200 import api

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    steps = max(3, min(args.steps, 20))
    for spec in DENSE_SHAPES:
        inp = W.generate(spec, seed=0)
        q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
        out = torch.empty_like(q)
        prob = api.Problem.from_inputs(inp, dev)
        T = spec.total_tokens
        arms = {}
        for name, budget in (("sparse", inp.budget), ("dense_same_kernels", W.Budget.topk(10 ** 6))):
            def layer(budget=budget):
                pl = api.Planner(prob, budget, dev)
                at = api.Attention(prob, dev)
                at(q, k, v, pl(q, k), out)
                return pl, at
            extra = _extra_bytes(layer, dev)
            planner, attn = api.Planner(prob, budget, dev), api.Attention(prob, dev)
            t = _timed_steps(lambda: attn(q, k, v, planner(q, k), out), steps, args.warmup, stream)
            if planner.status() != 0 or attn.status() != 0:
                raise RuntimeError("device-side status set (%s, %s)" % (spec.name, name))
            plan = planner(q, k)
            torch.cuda.synchronize()
            pairs = kept_pairs(inp.chunk_bounds, plan.row_ptr.cpu().numpy(), plan.col[:plan.nnz].cpu().numpy(),
                               inp.num_chunks)
            arms[name] = {"ms": t * 1e3, "tokens_per_s": T / t, "extra_bytes": extra, "kept_pairs": pairs,
                          "attention_tflops_kept": 4.0 * spec.head_dim * pairs / t / 1e12,
                          "budget": _budget_str(budget)}
            del planner, attn, plan
        # dense library attention (context): [1, H, T, d] strided views of the THD tensors
        qh = q.view(T, spec.num_q_heads, spec.head_dim).transpose(0, 1)[None]
        kh = k.view(T, spec.num_kv_heads, spec.head_dim).transpose(0, 1)[None]
        vh = v.view(T, spec.num_kv_heads, spec.head_dim).transpose(0, 1)[None]
        sdpa = torch.nn.functional.scaled_dot_product_attention
        try:
            def dense_lib():
                return sdpa(qh, kh, vh, is_causal=True, enable_gqa=True)
            extra = _extra_bytes(dense_lib, dev) - out.numel() * out.element_size()
            t = _timed_steps(dense_lib, steps, args.warmup, stream)
            causal = spec.num_q_heads * T * (T + 1) // 2
            arms["dense_sdpa"] = {"ms": t * 1e3, "tokens_per_s": T / t, "extra_bytes_beyond_output": extra,
                                  "attention_tflops_causal": 4.0 * spec.head_dim * causal / t / 1e12,
                                  "what": "torch scaled_dot_product_attention, is_causal, enable_gqa (library)"}
        except RuntimeError as e:  # no dense kernel for this shape in this torch build
            arms["dense_sdpa"] = {"unavailable": str(e).splitlines()[0][:200]}
        sp, dn = arms["sparse"], arms["dense_same_kernels"]
        res = {
            "metric": "DHSA sparse vs dense causal attention, one layer (1 B200)", "workload": spec.name,
            "tokens": T, "steps": steps, "warmup": args.warmup, "unit": "ms", "higher_is_better": False,
            "sparse": sp, "dense_same_kernels": dn, "dense_sdpa": arms["dense_sdpa"],
            "latency_reduction_vs_dense_same_kernels": 1.0 - sp["ms"] / dn["ms"],
            "speedup_vs_dense_same_kernels": dn["ms"] / sp["ms"],
            "peak_extra_memory_ratio_vs_dense_same_kernels": sp["extra_bytes"] / max(1, dn["extra_bytes"]),
            "qkvo_bytes": int((q.numel() + k.numel() + v.numel() + out.numel()) * q.element_size()),
            "pages_context": ("On-Device page: 20-60 % lower prefill latency and ~35 % lower peak memory than dense "
                              "attention on Gemma2 (whole model, edge hardware); Memory-Constrained page: up to "
                              "10x prefill speed-up at 128K"),
        }
        if "ms" in arms["dense_sdpa"]:
            res["speedup_vs_dense_sdpa"] = arms["dense_sdpa"]["ms"] / sp["ms"]
        print(json.dumps(res), flush=True)
        del q, k, v, out, prob, inp
        torch.cuda.empty_cache()


def _budget_str(b):
    rows = ", one plan row per KV head (group-summed scores)" if getattr(b, "per_kv_head", False) else ""
    if b.kind == W.BUDGET_TOPK:
        return "top-%d + diagonal%s" % (b.k, rows)
    return "%d/%d of admissible (ceil) + diagonal%s" % (b.num, b.den, rows)


def bench_reference(args):
    """The fp64 CPU oracle as the reference arm (rank 0 only).

    Each step (warm-up and timed) is the oracle's full plan on the whole
    workload plus attention on a seeded sample of (head, query chunk) pairs,
    about `per_step` seconds of it; `ms_per_step` is that step's measured wall
    time.  `value` is the whole layer's tokens/s with the sampled attention
    time scaled to all kept pairs (median over the timed steps)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from oracle import dhsa_oracle as O

    spec = W.BY_NAME[args.workload]
    inp = W.generate(spec, seed=0)
    budget = inp.budget.kv() if args.kv_plan else inp.budget
    group = spec.num_q_heads // spec.num_kv_heads if args.kv_plan else 1
    per_step = max(3.0, min(40.0, 150.0 / max(1, args.steps + args.warmup)))
    vals, step_s = [], []
    base = None
    for i in range(args.warmup + args.steps):
        r = run_cpu_oracle(inp, per_step, per_kv_head=args.kv_plan)
        if i >= args.warmup:
            vals.append(r["value"])
            step_s.append(r["t_step_s"])
            base = r
    value = statistics.median(vals)
    ref = O.build_plan(inp.q, inp.k, inp.chunk_bounds, inp.seq_chunk_ptr, budget.kind, budget.k, budget.num,
                       budget.den, per_kv_head=args.kv_plan)
    pairs = kept_pairs(inp.chunk_bounds, ref["row_ptr"], ref["col"], inp.num_chunks) * group
    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.mean(step_s) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; rank-4 shared component, scale 2)", "impl": "reference",
        "config": _config(spec, inp, budget, pairs, int(os.environ.get("WORLD_SIZE", "1"))),
        "step": ("each step is the oracle's full plan plus attention on a seeded sample of (head, query chunk) "
                 "pairs (%.2f%% of kept pairs in the last step); ms_per_step is that sampled step's wall time, "
                 "and value scales its attention time to every kept pair"
                 % (100.0 * base["sampled_pairs"] / max(1, base["total_pairs"]))),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": base["cores"], "kind": "oracle",
                         "sample": base["sample"]},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(result), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(W.BY_NAME))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-micro", action="store_true", help="skip the select micro-benchmark in the main line")
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--memory", action="store_true", help="report device memory per layer call instead")
    ap.add_argument("--dense", action="store_true",
                    help="sparse against dense causal attention (time and memory) at the 8K, 32K and 128K shapes")
    ap.add_argument("--kv-plan", action="store_true",
                    help="grouped-query mode: one plan row per KV head (scored by the group's summed queries)")
    ap.add_argument("--online-chunking", action="store_true",
                    help="each step segments the keys online (dhsa_segment) before planning")
    ap.add_argument("--micro", default=None, choices=["select", "segment"],
                    help="time one kernel alone instead of the full step")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        print("note: warm-up raised to 3", file=sys.stderr)
        args.warmup = 3
    if args.memory:
        bench_memory(args)
    elif args.dense:
        bench_dense(args)
    elif args.micro == "select":
        bench_select_micro(args)
    elif args.micro == "segment":
        bench_segment_micro(args)
    elif args.online_chunking:
        bench_online_chunking(args)
    elif args.impl == "reference":
        bench_reference(args)
    else:
        bench_gpu(args)


if __name__ == "__main__":
    main()
