/*
 * dhsa.h - C ABI of libdhsa.so, the B200 (sm_100a) prefill hot path of
 * Dynamic Hierarchical Sparse Attention (DHSA).
 *
 * The method is described on two pages: "Long-Context Modeling with Dynamic
 * Hierarchical Sparse Attention for On-Device LLMs" (Abstract, AI Summary) and
 * "Long-Context Modeling with Dynamic Hierarchical Sparse Attention for
 * Memory-Constrained LLM Inference" (abstract).  The path has four steps:
 *
 *   1. chunk aggregation  dhsa_chunk_reduce      (On-Device page, Abstract:
 *      length-normalised aggregation, mean scaled by sqrt(chunk length))
 *   2. chunk similarity   dhsa_chunk_similarity  (On-Device page, Abstract:
 *      chunk-level similarity scores; dot product of representations)
 *   3. upsample + select  dhsa_topk_select       (On-Device page, Abstract:
 *      chunk scores upsampled to token level decide which token interactions
 *      are kept; Memory-Constrained page: importance estimated per chunk and
 *      propagated to token interactions, keeping causal dependencies)
 *   4. sparse attention   dhsa_attention         (causal softmax attention over
 *      the kept token pairs only)
 *
 * dhsa_plan runs steps 1-3 back to back.  dhsa_segment (optional) proposes the
 * chunk boundaries online from the keys, under a rule stated with it.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Token tensors are packed "THD": q [T, Hq, d], k and v [T, Hkv, d],
 *   contiguous, row-major, in the problem's dtype (bf16 or fp32), 16-byte
 *   aligned.  Query head h reads KV head h / (Hq / Hkv).
 * - Chunks are given by global token offsets chunk_bounds[0..n], strictly
 *   increasing, chunk_bounds[0] = 0, chunk_bounds[n] = T.  Chunks never cross a
 *   sequence: chunk_bounds[seq_chunk_ptr[b]] == cu_seqlens[b] for every b.
 * - Every pointer marked "device" is device memory owned by the caller; every
 *   pointer marked "host" is host memory owned by the caller, read during the
 *   call only.  The library allocates nothing: the caller passes workspace.
 * - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL
 *   means the legacy default stream).  Argument errors are detected on the host
 *   and returned before anything is launched.  Launch failures return
 *   DHSA_ERR_CUDA.  Errors found by the kernels themselves (a bounded wait that
 *   ran out, an index check) are written to a status word at the start of the
 *   workspace and read with dhsa_workspace_status.
 * - No C++ exception crosses this interface.  All entry points are reentrant,
 *   except that calls of dhsa_plan_noalloc share one device array (see there).
 */
#ifndef DHSA_H_
#define DHSA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DHSA_API __attribute__((visibility("default")))
#else
#define DHSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DHSA_OK = 0,
  DHSA_ERR_INVALID_ARG = 1,  /* bad shape, pointer, bounds or budget */
  DHSA_ERR_UNSUPPORTED = 2,  /* valid but not built (e.g. head_dim 96) */
  DHSA_ERR_WORKSPACE = 3,    /* workspace missing or too small */
  DHSA_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
  DHSA_ERR_TIMEOUT = 5,      /* a bounded device-side wait ran out */
  DHSA_ERR_DEVICE_CHECK = 6  /* a device-side index/consistency check failed */
} dhsa_status;

typedef enum { DHSA_BF16 = 0, DHSA_F32 = 1 } dhsa_dtype;

typedef enum { DHSA_BUDGET_TOPK = 0, DHSA_BUDGET_FRACTION = 1 } dhsa_budget_kind;

/* Flag OR-ed into dhsa_budget.kind: a per-KV-head plan.  The pages never
 * mention grouped-query attention; this is an added mode for GQA models.
 * Instead of one plan row per (query head h, query chunk i) there is one per
 * (KV head g, query chunk i), rows r = g * n + i, and its score for key chunk j
 * is the sum over the query heads h of group g of qc[h, i] . kc[g, j]
 * (equivalently (sum_h qc[h, i]) . kc[g, j]).  Every query head of the group
 * then attends over that row: pass the plan to dhsa_attention_kv_plan.  With
 * Hq == Hkv the two kinds of plan are identical. */
#define DHSA_BUDGET_PER_KV_HEAD 0x100

/* Key-chunk budget of one query chunk with i_local earlier chunks in its
 * sequence (the diagonal chunk is always kept on top of it):
 *   TOPK:     keep min(k, i_local)
 *   FRACTION: keep min(i_local, ceil(i_local * num / den)), integer arithmetic
 * Requires k >= 0, num >= 0, den >= 1. */
typedef struct {
  int32_t kind;
  int32_t k;
  int32_t num;
  int32_t den;
} dhsa_budget;

/* Shapes and chunk structure of one packed batch. */
typedef struct {
  int32_t dtype;         /* dhsa_dtype of q, k, v and out */
  int32_t num_seqs;      /* B >= 0 */
  int32_t total_tokens;  /* T >= 0 */
  int32_t num_q_heads;   /* Hq >= 1 */
  int32_t num_kv_heads;  /* Hkv >= 1, Hq % Hkv == 0 */
  int32_t head_dim;      /* d in {64, 128, 256} */
  int32_t num_chunks;    /* n >= 0 */
  const int32_t* cu_seqlens;       /* device [B+1] */
  const int32_t* chunk_bounds;     /* device [n+1] */
  const int32_t* seq_chunk_ptr;    /* device [B+1] */
  const int32_t* h_cu_seqlens;     /* host mirror [B+1] */
  const int32_t* h_chunk_bounds;   /* host mirror [n+1] */
  const int32_t* h_seq_chunk_ptr;  /* host mirror [B+1] */
} dhsa_problem;

/* Human-readable name of a status code (static storage). */
DHSA_API const char* dhsa_status_string(dhsa_status s);

/* Host-only checks of the problem (and budget when `budget` is non-NULL).
 * Returns DHSA_OK or the first error found. */
DHSA_API dhsa_status dhsa_validate(const dhsa_problem* p, const dhsa_budget* budget);

/* Number of plan entries: sum over plan heads and chunks of (budget + 1).
 * Host-only, from the host mirrors.  The plan's row count is Hq * n, or
 * Hkv * n when budget.kind carries DHSA_BUDGET_PER_KV_HEAD. */
DHSA_API dhsa_status dhsa_plan_nnz(const dhsa_problem* p, dhsa_budget budget, int64_t* nnz);

/* ---- step 1: length-normalised chunk aggregation --------------------------
 * out[h, c, :] = (sum over tokens t of chunk c of x[t, h, :]) / sqrt(L_c),
 * i.e. the chunk mean scaled by sqrt(L_c) (On-Device page, Abstract), with
 * fp32 accumulation.
 *   x     device [T, H, d] in `dtype`
 *   out   device fp32 [H, n, d]
 * Deterministic (fixed summation order). */
DHSA_API dhsa_status dhsa_chunk_reduce(const void* x, int32_t dtype, int32_t total_tokens,
                              int32_t num_heads, int32_t head_dim,
                              const int32_t* chunk_bounds, int32_t num_chunks,
                              float* out, void* stream);

/* ---- step 2: chunk similarity -------------------------------------------
 * scores[h, i, j] = qc[h, i, :] . kc[h / (Hq/Hkv), j, :] for every j <= i in
 * the same sequence (On-Device page, Abstract: chunk-level similarity scores).
 * Entries outside that causal, same-sequence triangle are not written.
 *   qc      device fp32 [Hq, n, d]
 *   kc      device fp32 [Hkv, n, d]
 *   scores  device fp32 [Hq, n, n] */
DHSA_API dhsa_status dhsa_chunk_similarity(const float* qc, const float* kc,
                                  const dhsa_problem* p, float* scores,
                                  void* stream);

/* ---- step 3: upsample + select ------------------------------------------
 * For each row r = h * n + i (h < Hq, or h < Hkv with
 * DHSA_BUDGET_PER_KV_HEAD, where scores are then [Hkv, n, n]): keep the
 * budget's number of admissible key
 * chunks j < i of i's sequence with the largest scores[h, i, j] (ties to the
 * lower j), plus the diagonal i.  Because every token pair of chunks (i, j)
 * inherits score(i, j), this is the token-level keep set of the pages'
 * upsampling step, stored per chunk.
 *   row_ptr  device int32 [rows + 1]  (CSR offsets, written; rows = Hq*n, or
 *                                      Hkv*n for a per-KV-head plan)
 *   col      device int32 [nnz]       (ascending chunk ids; the diagonal is
 *                                      the last entry of its row)
 *   nnz      must equal dhsa_plan_nnz() for the same problem and budget. */
DHSA_API dhsa_status dhsa_topk_select(const float* scores, const dhsa_problem* p,
                             dhsa_budget budget, int32_t* row_ptr, int32_t* col,
                             int64_t nnz, void* workspace, size_t workspace_bytes,
                             void* stream);

/* ---- steps 1-3 ------------------------------------------------------------
 * dhsa_chunk_reduce, dhsa_chunk_similarity and dhsa_topk_select in one call,
 * from q and k to the plan (On-Device page, Abstract: chunk representations,
 * chunk-level similarity, upsampled scores deciding the kept interactions;
 * Memory-Constrained page, abstract: importance estimated per chunk and
 * carried to the token pairs, causal dependencies kept).
 * Workspace: dhsa_plan_workspace_size bytes, 256-byte aligned, device.  It
 * holds the status word, qc, kc and the score matrix (and, for a per-KV-head
 * plan, the summed query chunks [Hkv, n, d] fp32; the score matrix is then
 * [Hkv, n, n]). */
DHSA_API dhsa_status dhsa_plan_workspace_size(const dhsa_problem* p, dhsa_budget budget,
                                     size_t* bytes);
DHSA_API dhsa_status dhsa_plan(const void* q, const void* k, const dhsa_problem* p,
                      dhsa_budget budget, int32_t* row_ptr, int32_t* col,
                      int64_t nnz, void* workspace, size_t workspace_bytes,
                      void* stream);

/* ---- step 4: sparse causal attention --------------------------------------
 * out[t, h, :] = sum over kept s of softmax_s(q[t,h].k[s,g] * scale) v[s,g],
 * kept s = {s <= t : chunk(s) in row (h, chunk(t)) of the plan}, g = h/(Hq/Hkv).
 * scale <= 0 selects 1/sqrt(d).  bf16 runs on tcgen05 tensor cores with fp32
 * accumulation and an fp32 online softmax; fp32 runs an fp32 kernel.
 *   q, k, v  device, THD, `dtype`; out device [T, Hq, d] in `dtype`
 *   row_ptr, col: a plan as written by dhsa_plan / dhsa_topk_select
 * Workspace: dhsa_attention_workspace_size bytes, 256-byte aligned: the status
 * word and the work-item counter of the persistent bf16 kernel, both reset by
 * each call, then (bf16 problems) an f16 copy of v, T*Hkv*d*2 bytes, written by
 * each call: the tensor cores take the softmax weights P and V in f16 (11
 * significant bits against bf16's 8: each weight rounds by at most 2^-11 of
 * itself, or by up to 2^-25 below 2^-14 where f16 is subnormal, so out moves
 * by at most 2^-11 max|v| plus 2^-25 max|v| / l per weight below 2^-14, l the
 * row's sum of weights).  A |v| above 65504 or a NaN is reported as
 * DHSA_ERR_DEVICE_CHECK through dhsa_workspace_status (the copy holds +-65504
 * for the former, NaN for the latter).
 * A workspace serves one call at a time: calls that may overlap on the GPU
 * (other streams) need workspaces of their own. */
DHSA_API dhsa_status dhsa_attention_workspace_size(const dhsa_problem* p, size_t* bytes);
DHSA_API dhsa_status dhsa_attention(const void* q, const void* k, const void* v,
                           const dhsa_problem* p, const int32_t* row_ptr,
                           const int32_t* col, int64_t nnz, float scale, void* out,
                           void* workspace, size_t workspace_bytes, void* stream);

/* Step 4 over a per-KV-head plan (built with DHSA_BUDGET_PER_KV_HEAD): query
 * head h reads plan row (h / (Hq/Hkv)) * n + chunk(t).  Arguments, layouts,
 * workspace and errors as dhsa_attention; nnz is the per-KV-head plan's. */
DHSA_API dhsa_status dhsa_attention_kv_plan(const void* q, const void* k, const void* v,
                                           const dhsa_problem* p, const int32_t* row_ptr,
                                           const int32_t* col, int64_t nnz, float scale, void* out,
                                           void* workspace, size_t workspace_bytes, void* stream);

/* Selection margins of a plan just written by dhsa_plan (step 3's top-k over
 * chunk scores: On-Device page, Abstract).  For every plan row r (r = h * n + i,
 * or g * n + i for a per-KV-head plan):
 *   margins[2r]     the smallest score among the kept earlier chunks, i.e. the
 *                   k-th largest admissible score (NaN when the row keeps none);
 *   margins[2r + 1] the largest admissible score that was left out, i.e. the
 *                   (k+1)-th (NaN when every admissible chunk is kept).
 * Rows whose two margins are close (relative to the row's scores) are the
 * near-tie rows, where rounding in the scores can change the selection.
 *   p, budget   the problem and budget of the dhsa_plan call
 *   row_ptr, col, nnz   that call's plan (device)
 *   workspace   that call's workspace, unchanged since (its score matrix is read)
 *   margins     device fp32 [rows, 2], written
 * A plan entry outside its row's candidate range is skipped and reported in the
 * workspace's status word (DHSA_ERR_DEVICE_CHECK via dhsa_workspace_status).
 * Argument errors (another nnz, a workspace too small) return before any launch. */
DHSA_API dhsa_status dhsa_plan_margins(const dhsa_problem* p, dhsa_budget budget, const int32_t* row_ptr,
                                       const int32_t* col, int64_t nnz, const void* workspace,
                                       size_t workspace_bytes, float* margins, void* stream);

/* Device-side check of a plan before it is handed to step 4 (for plans that
 * did not come from dhsa_plan / dhsa_topk_select, or that were stored and
 * reloaded).  A plan row (plan head, query chunk i) must hold the kept key
 * chunks of i plus its diagonal: a non-empty, strictly ascending list of
 * chunks of i's own sequence, none later than i, whose last entry is i (the
 * causal keep set of step 3: On-Device page, Abstract; Memory-Constrained
 * page: causally important dependencies are kept).  row_ptr must start at 0,
 * never decrease and end at nnz.
 *   row_ptr     device int32 [rows + 1], rows = Hq * n, or Hkv * n when
 *               per_kv_head is non-zero
 *   col         device int32 [nnz]
 *   workspace   device, >= 256 bytes: its status word is cleared, then set to
 *               DHSA_ERR_DEVICE_CHECK's bit by any violation; read it with
 *               dhsa_workspace_status.
 * The kernel reads only row_ptr[0..rows] and col[0..nnz), so a malformed
 * plan cannot make it read out of range.  Argument errors (nnz < rows, a
 * NULL pointer) return before the launch.  The attention kernels themselves
 * clamp plan entries into range and report out-of-range ones, but accept
 * other malformed rows (unsorted, later chunks) with unspecified output. */
DHSA_API dhsa_status dhsa_plan_check(const dhsa_problem* p, const int32_t* row_ptr, const int32_t* col,
                                     int64_t nnz, int32_t per_kv_head, void* workspace, size_t workspace_bytes,
                                     void* stream);

/* Waits for `stream`, then reads the status word that the kernels of the last
 * call given `workspace` may have set.  Returns DHSA_OK, DHSA_ERR_TIMEOUT or
 * DHSA_ERR_DEVICE_CHECK (or DHSA_ERR_CUDA if the wait itself failed). */
DHSA_API dhsa_status dhsa_workspace_status(const void* workspace, void* stream);

/* Diagnostic: launches one tiny kernel whose only wait is on a barrier that
 * nothing releases, with a limit of `limit_us` microseconds (1..2000000); the
 * kernel gives up, records DHSA_ERR_TIMEOUT in the status word at the start
 * of `workspace` (>= 256 bytes) and returns.  Exercises the timeout path of
 * the bounded waits without hanging the device. */
DHSA_API dhsa_status dhsa_selftest_timeout(void* workspace, int32_t limit_us, void* stream);

/* ---- step 0 (optional): online variable-length chunking -------------------
 * The On-Device page (Abstract, AI Summary) says that DHSA segments each
 * sequence adaptively and online into variable-length chunks, and gives no
 * rule.  This library's rule is a plain one, decided left to right as tokens
 * arrive: with the current chunk of a sequence starting at token b, token t
 * starts a new chunk when
 *     t - b >= max_len, or
 *     t - b >= min_len and sim(t) < threshold,
 * sim(t) = (1/Hkv) * sum_g cos(k[t-1, g], k[t, g]), cos(x, y) = x.y/(|x||y|),
 * and 1 when either key is zero (a zero key never breaks a chunk).  The first
 * chunk starts at the sequence's first token; the last may be shorter than
 * min_len.  threshold <= -1 gives fixed max_len chunks, threshold > 1 fixed
 * min_len chunks (while no key is zero).  sim is computed in fp32; a
 * decision on a sim within about d * 2^-23 of the threshold may differ from
 * one taken in exact arithmetic.
 * The outputs are the chunk_bounds / seq_chunk_ptr arrays of dhsa_problem. */
#define DHSA_SEGMENT_MAX_LEN 65536
typedef struct {
  float threshold;  /* finite, or +-infinity */
  int32_t min_len;  /* 1 <= min_len <= max_len */
  int32_t max_len;  /* max_len <= DHSA_SEGMENT_MAX_LEN */
} dhsa_segment_rule;

/* Host only: the most chunks any key values can give, sum over sequences of
 * ceil(L_b / min_len) (every chunk but a sequence's last has >= min_len
 * tokens).  h_cu_seqlens: host [B+1]. */
DHSA_API dhsa_status dhsa_segment_capacity(const int32_t* h_cu_seqlens, int32_t num_seqs, int32_t min_len,
                                           int64_t* max_chunks);
/* Workspace of dhsa_segment for T tokens: the status word plus two bitmaps of
 * ceil(T/32) words. */
DHSA_API dhsa_status dhsa_segment_workspace_size(int32_t total_tokens, size_t* bytes);
/*   k              device [T, Hkv, d] in `dtype` (bf16 or fp32), 16-byte aligned,
 *                  d in {64, 128, 256}
 *   cu_seqlens     device [B+1]; h_cu_seqlens its host mirror (T = h_cu_seqlens[B])
 *   chunk_bounds   device int32 [max_chunks + 1], written: entries 0..n
 *   max_chunks     >= dhsa_segment_capacity(...)
 *   seq_chunk_ptr  device int32 [B + 1], written
 *   num_chunks     device int32 [1], written: n
 * The caller reads n (and mirrors the arrays to the host) before building the
 * dhsa_problem of the later steps. */
DHSA_API dhsa_status dhsa_segment(const void* k, int32_t dtype, int32_t num_kv_heads, int32_t head_dim,
                                  int32_t num_seqs, const int32_t* cu_seqlens, const int32_t* h_cu_seqlens,
                                  dhsa_segment_rule rule, int32_t* chunk_bounds, int64_t max_chunks,
                                  int32_t* seq_chunk_ptr, int32_t* num_chunks, void* workspace,
                                  size_t workspace_bytes, void* stream);

/* ---- steps 1-3 without a caller workspace ----------------------------------
 * The computation is dhsa_plan's (On-Device page, Abstract; steps 1-3 above).
 * The pages have no counterpart of this entry point: an interface addition
 * for callers that cannot allocate device memory at the point where they plan,
 * such as code that runs inside another framework's allocator-free region, a
 * plugin that is handed only its input and output buffers, or a process whose
 * allocations go through a pool it does not own.  Same inputs, outputs and results as dhsa_plan; the
 * scratch (status word, qc, kc, score matrix) lives in one fixed device array
 * inside the library, DHSA_PLAN_NOALLOC_MAX_SCRATCH bytes per device, which
 * every GPU that loads the library holds until the process exits.
 * - Problems whose plan scratch (dhsa_plan_workspace_size) exceeds that size
 *   are rejected with DHSA_ERR_WORKSPACE before anything is launched.
 * - Allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
 * - The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current) and caches it; make that
 *   first call before any stream capture on the device.
 * - All calls share the one array and leave their intermediates in it.  Calls
 *   whose kernels overlap on the GPU (other streams, other threads) race on it
 *   and give wrong plans: serialise them.
 * - The array's status word is cleared by each call but cannot be read back;
 *   device-side consistency checks of this variant are not reported. */
#define DHSA_PLAN_NOALLOC_MAX_SCRATCH (16u << 20)
DHSA_API dhsa_status dhsa_plan_noalloc(const void* q, const void* k, const dhsa_problem* p,
                                       dhsa_budget budget, int32_t* row_ptr, int32_t* col,
                                       int64_t nnz, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DHSA_H_ */
