// Internal launchers of the DHSA kernels (C++ linkage, not exported).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace dhsa {

struct BudgetArgs {
  int kind;  // 0 = top-k, 1 = fraction
  int k;
  int num;
  int den;
};

// Step 1. Reduces xa ([T, heads_a, d]) into out_a and, when xb is non-null,
// xb ([T, heads_b, d]) into out_b, in one launch.  dtype 0 = bf16, 1 = fp32.
cudaError_t launch_chunk_reduce(int dtype, const void* xa, int heads_a, float* out_a, const void* xb,
                                int heads_b, float* out_b, int head_dim, const int* bounds,
                                int num_chunks, cudaStream_t stream);

// Per-KV-head planning: qg[g, c, :] = sum over r < group of qc[g * group + r, c, :]
// (fp32, fixed order r = 0, 1, ...).
cudaError_t launch_group_sum(const float* qc, int num_q_heads, int num_kv_heads, int num_chunks, int head_dim,
                             float* qg, cudaStream_t stream);

// Step 2.
cudaError_t launch_chunk_similarity(const float* qc, const float* kc, int num_q_heads, int num_kv_heads,
                                    int num_chunks, int head_dim, const int* seq_chunk_ptr,
                                    int num_seqs, float* scores, cudaStream_t stream);

// Step 3 (any number of candidates per row).
cudaError_t launch_topk_select(const float* scores, int num_chunks, int num_q_heads,
                               const int* seq_chunk_ptr, int num_seqs, BudgetArgs budget,
                               int* row_ptr, int* col, int nnz_per_head, uint32_t* status,
                               cudaStream_t stream);

// Step 4, fp32.  plan_group: query heads per plan row (1: a plan row per query
// head; Hq/Hkv: a plan row per KV head, read by every head of the group).
// Plan rows outside [0, nnz] and entries outside [0, num_chunks) are reported
// in *status (kDevCheck) and skipped.
cudaError_t launch_attention_f32(const float* q, const float* k, const float* v, const int* bounds,
                                 int num_chunks, const int* row_ptr, const int* col, int nnz, int total_tokens,
                                 int num_q_heads, int num_kv_heads, int head_dim, int plan_group, float scale,
                                 float* out, uint32_t* status, cudaStream_t stream);

// Step 4, bf16 on tcgen05.  h_bounds is the host mirror of bounds (used to
// size the grid).
struct AttnBf16Args {
  const void* q;
  const void* k;
  const void* v;
  const void* v16;  // f16 copy of v (launch_v_to_f16), the B operand of the P V product
  void* out;
  const int* bounds;
  const int* row_ptr;
  const int* col;
  int nnz;  // entries of col; plan rows reaching past it are reported (kDevCheck)
  int num_chunks;
  int total_tokens;
  int num_q_heads;
  int num_kv_heads;
  int head_dim;
  int max_chunk_len;
  int plan_group;  // query heads per plan row: 1 (per query head) or Hq / Hkv (per KV head)
  float scale;
  uint32_t* status;
};
cudaError_t launch_attention_bf16(const AttnBf16Args& a, cudaStream_t stream);
// head_dim 64 / 128: two query tiles per CTA, P kept in TMEM.
cudaError_t launch_attention_pair(const AttnBf16Args& a, cudaStream_t stream);
// head_dim 256: one query tile per CTA, 128-key tiles, S double-buffered and P in TMEM.
cudaError_t launch_attention_d256(const AttnBf16Args& a, cudaStream_t stream);
// TMA view of a packed THD bf16 tensor (see attention_bf16.cu).
CUresult encode_qkv_map(CUtensorMap* map, const void* base, int heads, int head_dim, int tokens, int box_rows,
                        bool f16 = false);
// v (bf16, n elements, n a multiple of 8) -> v16 (f16), exact for |v| <= 65504;
// larger magnitudes are reported (kDevCheck).
cudaError_t launch_v_to_f16(const void* v, void* v16, long long n, uint32_t* status, cudaStream_t stream);

// Online chunking (three launches: adjacent-key similarity bits, a walk per
// sequence, compaction).  drop and start_bits: ceil(T / 32) words each.
cudaError_t launch_segment(const void* k, int dtype, int total_tokens, int num_kv_heads, int head_dim,
                           const int* cu_seqlens, int num_seqs, float threshold, int min_len, int max_len,
                           int* chunk_bounds, long long capacity, int* seq_chunk_ptr, int* num_chunks,
                           uint32_t* drop, uint32_t* start_bits, uint32_t* status, cudaStream_t stream);

// Structural check of a plan (rows = plan heads x num_chunks): sets kDevCheck
// in *status on any violation; reads only row_ptr[0..rows] and col[0..nnz).
cudaError_t launch_plan_check(const int* row_ptr, const int* col, long long nnz, int rows, int num_chunks,
                              const int* seq_chunk_ptr, int num_seqs, uint32_t* status, cudaStream_t stream);

// Per plan row r: margins[2r] = smallest kept score (k-th largest admissible),
// margins[2r + 1] = largest admissible score left out; NaN where there is none.
// scores: [rows, num_chunks] fp32 (a plan workspace's score matrix).
cudaError_t launch_plan_margins(const float* scores, const int* row_ptr, const int* col, long long nnz, int rows,
                                int num_chunks, const int* seq_chunk_ptr, int num_seqs, float* margins,
                                uint32_t* status, cudaStream_t stream);

// Diagnostic: a kernel whose only wait can never be satisfied, bounded by limit_ns.
cudaError_t launch_timeout_selftest(uint32_t* status, unsigned long long limit_ns, cudaStream_t stream);

}  // namespace dhsa
