// C ABI of libdhsa.so: argument validation, workspace carving and launches.
// Every entry point returns a dhsa_status; nothing throws across the ABI.
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "dhsa.h"
#include "common.cuh"
#include "launchers.h"

namespace dhsa {
namespace {

constexpr size_t kAlign = 256;
constexpr size_t kStatusBytes = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int base_kind(const dhsa_budget& b) { return b.kind & 0xFF; }
bool per_kv_head(const dhsa_budget& b) { return (b.kind & DHSA_BUDGET_PER_KV_HEAD) != 0; }

int64_t budget_of(int i_local, const dhsa_budget& b) {
  if (base_kind(b) == DHSA_BUDGET_TOPK) return i_local < b.k ? i_local : b.k;
  const int64_t want = (static_cast<int64_t>(i_local) * b.num + b.den - 1) / b.den;
  return want < i_local ? want : i_local;
}

dhsa_status check_budget(const dhsa_budget& b) {
  if ((b.kind & ~(0xFF | DHSA_BUDGET_PER_KV_HEAD)) != 0) return DHSA_ERR_INVALID_ARG;
  if (base_kind(b) == DHSA_BUDGET_TOPK) return b.k >= 0 ? DHSA_OK : DHSA_ERR_INVALID_ARG;
  if (base_kind(b) == DHSA_BUDGET_FRACTION) return (b.num >= 0 && b.den >= 1) ? DHSA_OK : DHSA_ERR_INVALID_ARG;
  return DHSA_ERR_INVALID_ARG;
}

// Plan rows come in blocks of num_chunks, one block per query head, or per KV
// head for a per-KV-head plan.
int plan_heads(const dhsa_problem* p, const dhsa_budget& b) {
  return per_kv_head(b) ? p->num_kv_heads : p->num_q_heads;
}

dhsa_status check_problem(const dhsa_problem* p) {
  if (p == nullptr) return DHSA_ERR_INVALID_ARG;
  if (p->dtype != DHSA_BF16 && p->dtype != DHSA_F32) return DHSA_ERR_INVALID_ARG;
  if (p->num_seqs < 0 || p->total_tokens < 0 || p->num_chunks < 0) return DHSA_ERR_INVALID_ARG;
  if (p->num_q_heads < 1 || p->num_kv_heads < 1 || p->num_q_heads % p->num_kv_heads != 0)
    return DHSA_ERR_INVALID_ARG;
  if (p->head_dim != 64 && p->head_dim != 128 && p->head_dim != 256) {
    return p->head_dim > 0 ? DHSA_ERR_UNSUPPORTED : DHSA_ERR_INVALID_ARG;
  }
  if (p->num_chunks > 65535 || p->num_q_heads > 65535) return DHSA_ERR_UNSUPPORTED;
  if (p->h_cu_seqlens == nullptr || p->h_chunk_bounds == nullptr || p->h_seq_chunk_ptr == nullptr)
    return DHSA_ERR_INVALID_ARG;
  if (p->cu_seqlens == nullptr || p->chunk_bounds == nullptr || p->seq_chunk_ptr == nullptr)
    return DHSA_ERR_INVALID_ARG;
  const int B = p->num_seqs, n = p->num_chunks;
  const int32_t* cu = p->h_cu_seqlens;
  const int32_t* bd = p->h_chunk_bounds;
  const int32_t* sp = p->h_seq_chunk_ptr;
  if (cu[0] != 0 || cu[B] != p->total_tokens) return DHSA_ERR_INVALID_ARG;
  for (int b = 0; b < B; ++b)
    if (cu[b + 1] < cu[b]) return DHSA_ERR_INVALID_ARG;
  if (bd[0] != 0 || bd[n] != p->total_tokens) return DHSA_ERR_INVALID_ARG;
  for (int c = 0; c < n; ++c)
    if (bd[c + 1] <= bd[c]) return DHSA_ERR_INVALID_ARG;  // chunks are non-empty
  if (sp[0] != 0 || sp[B] != n) return DHSA_ERR_INVALID_ARG;
  for (int b = 0; b < B; ++b) {
    if (sp[b + 1] < sp[b]) return DHSA_ERR_INVALID_ARG;
    if (bd[sp[b]] != cu[b] || bd[sp[b + 1]] != cu[b + 1]) return DHSA_ERR_INVALID_ARG;  // no chunk crosses a sequence
  }
  return DHSA_OK;
}

int max_chunk_len(const dhsa_problem* p) {
  int m = 0;
  for (int c = 0; c < p->num_chunks; ++c) {
    const int L = p->h_chunk_bounds[c + 1] - p->h_chunk_bounds[c];
    if (L > m) m = L;
  }
  return m;
}

int64_t nnz_per_head(const dhsa_problem* p, const dhsa_budget& b) {
  int64_t total = 0;
  for (int s = 0; s < p->num_seqs; ++s) {
    const int cnt = p->h_seq_chunk_ptr[s + 1] - p->h_seq_chunk_ptr[s];
    for (int l = 0; l < cnt; ++l) total += budget_of(l, b) + 1;
  }
  return total;
}

struct PlanLayout {
  size_t qc, kc, qg, scores, total;  // qg: summed query chunks of a per-KV-head plan (else unused)
};

PlanLayout plan_layout(const dhsa_problem* p, const dhsa_budget& b) {
  PlanLayout L;
  const size_t n = static_cast<size_t>(p->num_chunks), d = static_cast<size_t>(p->head_dim);
  L.qc = kStatusBytes;
  L.kc = L.qc + align_up(static_cast<size_t>(p->num_q_heads) * n * d * 4);
  L.qg = L.kc + align_up(static_cast<size_t>(p->num_kv_heads) * n * d * 4);
  L.scores = L.qg + (per_kv_head(b) ? align_up(static_cast<size_t>(p->num_kv_heads) * n * d * 4) : 0);
  L.total = L.scores + align_up(static_cast<size_t>(plan_heads(p, b)) * n * n * 4);
  return L;
}

dhsa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? DHSA_OK : DHSA_ERR_CUDA; }

BudgetArgs to_args(const dhsa_budget& b) { return BudgetArgs{base_kind(b), b.k, b.num, b.den}; }

// Selection core shared by dhsa_topk_select and the planning steps (after
// validation): scores [plan_heads, n, n] -> plan rows (plan head, chunk).
dhsa_status run_select(const float* scores, const dhsa_problem* p, const dhsa_budget& budget, int32_t* row_ptr,
                       int32_t* col, uint32_t* status, cudaStream_t stream) {
  const int64_t per_head = nnz_per_head(p, budget);
  return cuda_status(launch_topk_select(scores, p->num_chunks, plan_heads(p, budget), p->seq_chunk_ptr,
                                        p->num_seqs, to_args(budget), row_ptr, col, static_cast<int>(per_head),
                                        status, stream));
}

// Steps 1-3 into a validated workspace laid out by plan_layout (status word
// cleared by the caller).
dhsa_status run_plan(const void* q, const void* k, const dhsa_problem* p, const dhsa_budget& budget,
                     int32_t* row_ptr, int32_t* col, unsigned char* ws, const PlanLayout& L, cudaStream_t st) {
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  float* qc = reinterpret_cast<float*>(ws + L.qc);
  float* kc = reinterpret_cast<float*>(ws + L.kc);
  float* scores = reinterpret_cast<float*>(ws + L.scores);
  cudaError_t e = launch_chunk_reduce(p->dtype, q, p->num_q_heads, qc, k, p->num_kv_heads, kc, p->head_dim,
                                      p->chunk_bounds, p->num_chunks, st);
  if (e != cudaSuccess) return DHSA_ERR_CUDA;
  if (per_kv_head(budget)) {
    float* qg = reinterpret_cast<float*>(ws + L.qg);
    e = launch_group_sum(qc, p->num_q_heads, p->num_kv_heads, p->num_chunks, p->head_dim, qg, st);
    if (e != cudaSuccess) return DHSA_ERR_CUDA;
    e = launch_chunk_similarity(qg, kc, p->num_kv_heads, p->num_kv_heads, p->num_chunks, p->head_dim,
                                p->seq_chunk_ptr, p->num_seqs, scores, st);
  } else {
    e = launch_chunk_similarity(qc, kc, p->num_q_heads, p->num_kv_heads, p->num_chunks, p->head_dim,
                                p->seq_chunk_ptr, p->num_seqs, scores, st);
  }
  if (e != cudaSuccess) return DHSA_ERR_CUDA;
  return run_select(scores, p, budget, row_ptr, col, status, st);
}

// Bytes of the attention workspace: the status word and the work-item
// counter, then (bf16) the f16 copy of V that the P V products read.
size_t attention_ws_bytes(const dhsa_problem* p) {
  size_t b = kStatusBytes;
  if (p->dtype == DHSA_BF16)
    b += align_up(static_cast<size_t>(p->total_tokens) * p->num_kv_heads * p->head_dim * 2);
  return b;
}

// Step 4 after validation; plan_group = query heads per plan row.
dhsa_status run_attention(const void* q, const void* k, const void* v, const dhsa_problem* p,
                          const int32_t* row_ptr, const int32_t* col, int64_t nnz, int plan_group, float scale,
                          void* out, void* workspace, size_t workspace_bytes, cudaStream_t st) {
  if (nnz < static_cast<int64_t>(p->num_q_heads / plan_group) * p->num_chunks || nnz > INT32_MAX)
    return DHSA_ERR_INVALID_ARG;  // >= diagonal per row
  if (workspace == nullptr || workspace_bytes < attention_ws_bytes(p) ||
      (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0)
    return DHSA_ERR_WORKSPACE;
  if (p->total_tokens == 0 || p->num_chunks == 0) return DHSA_OK;
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr || row_ptr == nullptr || col == nullptr)
    return DHSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return DHSA_ERR_INVALID_ARG;
  if (!(scale > 0.f)) scale = 1.0f / sqrtf(static_cast<float>(p->head_dim));
  uint32_t* status = static_cast<uint32_t*>(workspace);
  // status word, then the persistent attention kernel's work-item counter
  if (cudaMemsetAsync(status, 0, 2 * sizeof(uint32_t), st) != cudaSuccess) return DHSA_ERR_CUDA;
  if (p->dtype == DHSA_F32) {
    return cuda_status(launch_attention_f32(static_cast<const float*>(q), static_cast<const float*>(k),
                                            static_cast<const float*>(v), p->chunk_bounds, p->num_chunks, row_ptr,
                                            col, static_cast<int>(nnz), p->total_tokens, p->num_q_heads,
                                            p->num_kv_heads, p->head_dim, plan_group, scale,
                                            static_cast<float*>(out), status, st));
  }
  // V in f16 for the P V products (P is f16 too: see the kernels)
  void* v16 = static_cast<unsigned char*>(workspace) + kStatusBytes;
  const long long v_elems = static_cast<long long>(p->total_tokens) * p->num_kv_heads * p->head_dim;
  if (cudaError_t e = launch_v_to_f16(v, v16, v_elems, status, st); e != cudaSuccess) return cuda_status(e);
  AttnBf16Args a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.v16 = v16;
  a.out = out;
  a.bounds = p->chunk_bounds;
  a.row_ptr = row_ptr;
  a.col = col;
  a.nnz = static_cast<int>(nnz);
  a.num_chunks = p->num_chunks;
  a.total_tokens = p->total_tokens;
  a.num_q_heads = p->num_q_heads;
  a.num_kv_heads = p->num_kv_heads;
  a.head_dim = p->head_dim;
  a.max_chunk_len = max_chunk_len(p);
  a.plan_group = plan_group;
  a.scale = scale;
  a.status = status;
  return cuda_status(launch_attention_bf16(a, st));
}

__global__ void timeout_selftest_kernel(uint32_t* status, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar_storage;
  __shared__ int abort_flag;
  const uint32_t bar = smem_u32(&bar_storage);
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // nothing ever arrives on this barrier: the wait must give up by itself
  mbar_wait(bar, 0, reinterpret_cast<volatile int*>(&abort_flag), status, limit_ns);
}

}  // namespace

cudaError_t launch_timeout_selftest(uint32_t* status, unsigned long long limit_ns, cudaStream_t stream) {
  timeout_selftest_kernel<<<1, 32, 0, stream>>>(status, limit_ns);
  return cudaGetLastError();
}

// Fixed scratch of dhsa_plan_noalloc (status word, qc, kc, scores).  Host code
// must not use this name as a device address: it is a host-side stand-in, so
// the address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_plan_noalloc_scratch[DHSA_PLAN_NOALLOC_MAX_SCRATCH];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_addr[kMaxDevices] = {};

// Device address of the fixed scratch on the current device (looked up once).
dhsa_status noalloc_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DHSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (g_noalloc_addr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_plan_noalloc_scratch) != cudaSuccess || ptr == nullptr)
      return DHSA_ERR_CUDA;
    g_noalloc_addr[dev] = ptr;
  }
  *out = g_noalloc_addr[dev];
  return DHSA_OK;
}

}  // namespace

}  // namespace dhsa

using namespace dhsa;

extern "C" {

const char* dhsa_status_string(dhsa_status s) {
  switch (s) {
    case DHSA_OK: return "DHSA_OK";
    case DHSA_ERR_INVALID_ARG: return "DHSA_ERR_INVALID_ARG";
    case DHSA_ERR_UNSUPPORTED: return "DHSA_ERR_UNSUPPORTED";
    case DHSA_ERR_WORKSPACE: return "DHSA_ERR_WORKSPACE";
    case DHSA_ERR_CUDA: return "DHSA_ERR_CUDA";
    case DHSA_ERR_TIMEOUT: return "DHSA_ERR_TIMEOUT";
    case DHSA_ERR_DEVICE_CHECK: return "DHSA_ERR_DEVICE_CHECK";
  }
  return "DHSA_ERR_UNKNOWN";
}

dhsa_status dhsa_validate(const dhsa_problem* p, const dhsa_budget* budget) {
  dhsa_status s = check_problem(p);
  if (s != DHSA_OK) return s;
  if (budget != nullptr) return check_budget(*budget);
  return DHSA_OK;
}

dhsa_status dhsa_plan_nnz(const dhsa_problem* p, dhsa_budget budget, int64_t* nnz) {
  dhsa_status s = dhsa_validate(p, &budget);
  if (s != DHSA_OK) return s;
  if (nnz == nullptr) return DHSA_ERR_INVALID_ARG;
  *nnz = nnz_per_head(p, budget) * plan_heads(p, budget);
  return DHSA_OK;
}

dhsa_status dhsa_chunk_reduce(const void* x, int32_t dtype, int32_t total_tokens, int32_t num_heads,
                              int32_t head_dim, const int32_t* chunk_bounds, int32_t num_chunks, float* out,
                              void* stream) {
  if (dtype != DHSA_BF16 && dtype != DHSA_F32) return DHSA_ERR_INVALID_ARG;
  if (total_tokens < 0 || num_heads < 1 || num_chunks < 0) return DHSA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128 && head_dim != 256) return DHSA_ERR_UNSUPPORTED;
  if (num_chunks > 65535) return DHSA_ERR_UNSUPPORTED;
  if (num_chunks == 0) return DHSA_OK;
  if (x == nullptr || out == nullptr || chunk_bounds == nullptr || !aligned16(x)) return DHSA_ERR_INVALID_ARG;
  return cuda_status(launch_chunk_reduce(dtype, x, num_heads, out, nullptr, 0, nullptr, head_dim, chunk_bounds,
                                         num_chunks, static_cast<cudaStream_t>(stream)));
}

dhsa_status dhsa_chunk_similarity(const float* qc, const float* kc, const dhsa_problem* p, float* scores,
                                  void* stream) {
  dhsa_status s = check_problem(p);
  if (s != DHSA_OK) return s;
  if (p->num_chunks == 0) return DHSA_OK;
  if (qc == nullptr || kc == nullptr || scores == nullptr) return DHSA_ERR_INVALID_ARG;
  return cuda_status(launch_chunk_similarity(qc, kc, p->num_q_heads, p->num_kv_heads, p->num_chunks, p->head_dim,
                                             p->seq_chunk_ptr, p->num_seqs, scores,
                                             static_cast<cudaStream_t>(stream)));
}

dhsa_status dhsa_topk_select(const float* scores, const dhsa_problem* p, dhsa_budget budget, int32_t* row_ptr,
                             int32_t* col, int64_t nnz, void* workspace, size_t workspace_bytes, void* stream) {
  dhsa_status s = dhsa_validate(p, &budget);
  if (s != DHSA_OK) return s;
  const int64_t want = nnz_per_head(p, budget) * plan_heads(p, budget);
  if (nnz != want || want > INT32_MAX) return DHSA_ERR_INVALID_ARG;
  if (workspace == nullptr || workspace_bytes < kStatusBytes) return DHSA_ERR_WORKSPACE;
  if (p->num_chunks == 0) return DHSA_OK;
  if (scores == nullptr || row_ptr == nullptr || col == nullptr) return DHSA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t* status = static_cast<uint32_t*>(workspace);
  if (cudaMemsetAsync(status, 0, sizeof(uint32_t), st) != cudaSuccess) return DHSA_ERR_CUDA;
  return run_select(scores, p, budget, row_ptr, col, status, st);
}

dhsa_status dhsa_plan_workspace_size(const dhsa_problem* p, dhsa_budget budget, size_t* bytes) {
  dhsa_status s = dhsa_validate(p, &budget);
  if (s != DHSA_OK) return s;
  if (bytes == nullptr) return DHSA_ERR_INVALID_ARG;
  *bytes = plan_layout(p, budget).total;
  return DHSA_OK;
}

dhsa_status dhsa_plan(const void* q, const void* k, const dhsa_problem* p, dhsa_budget budget, int32_t* row_ptr,
                      int32_t* col, int64_t nnz, void* workspace, size_t workspace_bytes, void* stream) {
  dhsa_status s = dhsa_validate(p, &budget);
  if (s != DHSA_OK) return s;
  const int64_t want = nnz_per_head(p, budget) * plan_heads(p, budget);
  if (nnz != want || want > INT32_MAX) return DHSA_ERR_INVALID_ARG;
  const PlanLayout L = plan_layout(p, budget);
  if (workspace == nullptr || workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0)
    return DHSA_ERR_WORKSPACE;
  if (p->num_chunks == 0) return DHSA_OK;
  if (q == nullptr || k == nullptr || row_ptr == nullptr || col == nullptr || !aligned16(q) || !aligned16(k))
    return DHSA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  if (cudaMemsetAsync(ws, 0, sizeof(uint32_t), st) != cudaSuccess) return DHSA_ERR_CUDA;
  return run_plan(q, k, p, budget, row_ptr, col, ws, L, st);
}

dhsa_status dhsa_attention_workspace_size(const dhsa_problem* p, size_t* bytes) {
  dhsa_status s = check_problem(p);
  if (s != DHSA_OK) return s;
  if (bytes == nullptr) return DHSA_ERR_INVALID_ARG;
  *bytes = attention_ws_bytes(p);
  return DHSA_OK;
}

dhsa_status dhsa_attention(const void* q, const void* k, const void* v, const dhsa_problem* p,
                           const int32_t* row_ptr, const int32_t* col, int64_t nnz, float scale, void* out,
                           void* workspace, size_t workspace_bytes, void* stream) {
  dhsa_status s = check_problem(p);
  if (s != DHSA_OK) return s;
  return run_attention(q, k, v, p, row_ptr, col, nnz, 1, scale, out, workspace, workspace_bytes,
                       static_cast<cudaStream_t>(stream));
}

dhsa_status dhsa_attention_kv_plan(const void* q, const void* k, const void* v, const dhsa_problem* p,
                                   const int32_t* row_ptr, const int32_t* col, int64_t nnz, float scale, void* out,
                                   void* workspace, size_t workspace_bytes, void* stream) {
  dhsa_status s = check_problem(p);
  if (s != DHSA_OK) return s;
  return run_attention(q, k, v, p, row_ptr, col, nnz, p->num_q_heads / p->num_kv_heads, scale, out, workspace,
                       workspace_bytes, static_cast<cudaStream_t>(stream));
}

dhsa_status dhsa_plan_margins(const dhsa_problem* p, dhsa_budget budget, const int32_t* row_ptr, const int32_t* col,
                              int64_t nnz, const void* workspace, size_t workspace_bytes, float* margins,
                              void* stream) {
  dhsa_status s = dhsa_validate(p, &budget);
  if (s != DHSA_OK) return s;
  const int64_t want = nnz_per_head(p, budget) * plan_heads(p, budget);
  if (nnz != want || want > INT32_MAX) return DHSA_ERR_INVALID_ARG;
  const PlanLayout L = plan_layout(p, budget);
  if (workspace == nullptr || workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0)
    return DHSA_ERR_WORKSPACE;
  if (p->num_chunks == 0) return DHSA_OK;
  if (row_ptr == nullptr || col == nullptr || margins == nullptr) return DHSA_ERR_INVALID_ARG;
  const unsigned char* ws = static_cast<const unsigned char*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(const_cast<unsigned char*>(ws));
  const float* scores = reinterpret_cast<const float*>(ws + L.scores);
  const int rows = plan_heads(p, budget) * p->num_chunks;
  return cuda_status(launch_plan_margins(scores, row_ptr, col, nnz, rows, p->num_chunks, p->seq_chunk_ptr,
                                         p->num_seqs, margins, status, static_cast<cudaStream_t>(stream)));
}

dhsa_status dhsa_plan_check(const dhsa_problem* p, const int32_t* row_ptr, const int32_t* col, int64_t nnz,
                            int32_t per_kv_head, void* workspace, size_t workspace_bytes, void* stream) {
  dhsa_status s = check_problem(p);
  if (s != DHSA_OK) return s;
  const int64_t rows = static_cast<int64_t>(per_kv_head ? p->num_kv_heads : p->num_q_heads) * p->num_chunks;
  if (nnz < rows || nnz > INT32_MAX) return DHSA_ERR_INVALID_ARG;  // every row holds at least its diagonal
  if (workspace == nullptr || workspace_bytes < kStatusBytes) return DHSA_ERR_WORKSPACE;
  if (rows == 0) return DHSA_OK;
  if (row_ptr == nullptr || col == nullptr) return DHSA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t* status = static_cast<uint32_t*>(workspace);
  if (cudaMemsetAsync(status, 0, sizeof(uint32_t), st) != cudaSuccess) return DHSA_ERR_CUDA;
  return cuda_status(launch_plan_check(row_ptr, col, nnz, static_cast<int>(rows), p->num_chunks, p->seq_chunk_ptr,
                                       p->num_seqs, status, st));
}

dhsa_status dhsa_workspace_status(const void* workspace, void* stream) {
  if (workspace == nullptr) return DHSA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return DHSA_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return DHSA_ERR_CUDA;
  if (word & kDevTimeout) return DHSA_ERR_TIMEOUT;
  if (word & kDevCheck) return DHSA_ERR_DEVICE_CHECK;
  return DHSA_OK;
}

dhsa_status dhsa_plan_noalloc(const void* q, const void* k, const dhsa_problem* p, dhsa_budget budget,
                              int32_t* row_ptr, int32_t* col, int64_t nnz, void* stream) {
  dhsa_status s = dhsa_validate(p, &budget);
  if (s != DHSA_OK) return s;
  const int64_t want = nnz_per_head(p, budget) * plan_heads(p, budget);
  if (nnz != want || want > INT32_MAX) return DHSA_ERR_INVALID_ARG;
  const PlanLayout L = plan_layout(p, budget);
  if (L.total > DHSA_PLAN_NOALLOC_MAX_SCRATCH) return DHSA_ERR_WORKSPACE;  // problem too large for the fixed scratch
  if (p->num_chunks == 0) return DHSA_OK;
  if (q == nullptr || k == nullptr || row_ptr == nullptr || col == nullptr || !aligned16(q) || !aligned16(k))
    return DHSA_ERR_INVALID_ARG;
  void* base = nullptr;
  s = noalloc_scratch(&base);
  if (s != DHSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned char* ws = static_cast<unsigned char*>(base);
  // qc, kc, the summed query chunks and the score triangle are fully
  // rewritten before they are read; only the status word has to start at zero
  if (cudaMemsetAsync(ws, 0, sizeof(uint32_t), st) != cudaSuccess) return DHSA_ERR_CUDA;
  return run_plan(q, k, p, budget, row_ptr, col, ws, L, st);
}

dhsa_status dhsa_selftest_timeout(void* workspace, int32_t limit_us, void* stream) {
  if (workspace == nullptr) return DHSA_ERR_WORKSPACE;
  if (limit_us < 1 || limit_us > 2000000) return DHSA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t* status = static_cast<uint32_t*>(workspace);
  if (cudaMemsetAsync(status, 0, sizeof(uint32_t), st) != cudaSuccess) return DHSA_ERR_CUDA;
  return cuda_status(launch_timeout_selftest(status, static_cast<unsigned long long>(limit_us) * 1000ull, st));
}

dhsa_status dhsa_segment_capacity(const int32_t* h_cu_seqlens, int32_t num_seqs, int32_t min_len,
                                  int64_t* max_chunks) {
  if (h_cu_seqlens == nullptr || max_chunks == nullptr || num_seqs < 0 || min_len < 1) return DHSA_ERR_INVALID_ARG;
  if (h_cu_seqlens[0] != 0) return DHSA_ERR_INVALID_ARG;
  int64_t total = 0;
  for (int b = 0; b < num_seqs; ++b) {
    const int64_t L = static_cast<int64_t>(h_cu_seqlens[b + 1]) - h_cu_seqlens[b];
    if (L < 0) return DHSA_ERR_INVALID_ARG;
    total += (L + min_len - 1) / min_len;
  }
  *max_chunks = total;
  return DHSA_OK;
}

dhsa_status dhsa_segment_workspace_size(int32_t total_tokens, size_t* bytes) {
  if (total_tokens < 0 || bytes == nullptr) return DHSA_ERR_INVALID_ARG;
  const size_t words = (static_cast<size_t>(total_tokens) + 31) / 32;
  *bytes = kStatusBytes + 2 * align_up(words * sizeof(uint32_t));
  return DHSA_OK;
}

dhsa_status dhsa_segment(const void* k, int32_t dtype, int32_t num_kv_heads, int32_t head_dim, int32_t num_seqs,
                         const int32_t* cu_seqlens, const int32_t* h_cu_seqlens, dhsa_segment_rule rule,
                         int32_t* chunk_bounds, int64_t max_chunks, int32_t* seq_chunk_ptr, int32_t* num_chunks,
                         void* workspace, size_t workspace_bytes, void* stream) {
  if (dtype != DHSA_BF16 && dtype != DHSA_F32) return DHSA_ERR_INVALID_ARG;
  if (num_kv_heads < 1 || num_seqs < 0) return DHSA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128 && head_dim != 256) {
    return head_dim > 0 ? DHSA_ERR_UNSUPPORTED : DHSA_ERR_INVALID_ARG;
  }
  if (isnan(rule.threshold) || rule.min_len < 1 || rule.max_len < rule.min_len ||
      rule.max_len > DHSA_SEGMENT_MAX_LEN)
    return DHSA_ERR_INVALID_ARG;
  int64_t cap = 0;
  dhsa_status s = dhsa_segment_capacity(h_cu_seqlens, num_seqs, rule.min_len, &cap);
  if (s != DHSA_OK) return s;
  const int32_t T = h_cu_seqlens[num_seqs];
  if (max_chunks < cap || max_chunks > INT32_MAX - 1) return DHSA_ERR_INVALID_ARG;
  if (cu_seqlens == nullptr || chunk_bounds == nullptr || seq_chunk_ptr == nullptr || num_chunks == nullptr)
    return DHSA_ERR_INVALID_ARG;
  if (T > 0 && (k == nullptr || !aligned16(k))) return DHSA_ERR_INVALID_ARG;
  size_t need = 0;
  dhsa_segment_workspace_size(T, &need);
  if (workspace == nullptr || workspace_bytes < need) return DHSA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  const size_t words = (static_cast<size_t>(T) + 31) / 32;
  uint32_t* drop = reinterpret_cast<uint32_t*>(ws + kStatusBytes);
  uint32_t* start_bits = reinterpret_cast<uint32_t*>(ws + kStatusBytes + align_up(words * sizeof(uint32_t)));
  if (cudaMemsetAsync(status, 0, sizeof(uint32_t), st) != cudaSuccess) return DHSA_ERR_CUDA;
  return cuda_status(launch_segment(k, dtype, T, num_kv_heads, head_dim, cu_seqlens, num_seqs, rule.threshold,
                                    rule.min_len, rule.max_len, chunk_bounds, max_chunks, seq_chunk_ptr,
                                    num_chunks, drop, start_bits, status, st));
}

}  // extern "C"
