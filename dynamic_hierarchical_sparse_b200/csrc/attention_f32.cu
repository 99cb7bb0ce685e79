// Step 4 of the DHSA path for fp32 inputs: sparse causal attention in true
// fp32 (FFMA), for problems whose accuracy target rules out reduced-precision
// tensor-core arithmetic.
//
// out[t, h] = sum_s softmax_s(q[t,h] . k[s,g] * scale) v[s,g] over the kept
// key tokens s <= t: tokens of the chunks listed in plan row (h, chunk(t))
// ("Long-Context Modeling with Dynamic Hierarchical Sparse Attention for
// On-Device LLMs", Abstract: only the token interactions selected through the
// upsampled chunk scores are preserved; causal order kept).
//
// One warp per (query token, head).  Keys are processed 32 at a time: each
// logit is a warp-wide dot product (lane-strided over d, shuffle reduction),
// the batch updates an online softmax (running max and sum), and each lane
// accumulates d/32 output columns.
#include "common.cuh"
#include "launchers.h"

namespace dhsa {
namespace {

constexpr int kRowsPerCta = 4;

template <int D>
__global__ void __launch_bounds__(kRowsPerCta * 32)
    attention_f32_kernel(const float* __restrict__ q, const float* __restrict__ k,
                         const float* __restrict__ v, const int* __restrict__ bounds, int num_chunks,
                         const int* __restrict__ row_ptr, const int* __restrict__ col, int nnz, int total_tokens,
                         int num_q_heads, int num_kv_heads, int plan_group, float scale,
                         float* __restrict__ out, uint32_t* status) {
  constexpr int PER = D / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kRowsPerCta + warp;
  const int h = blockIdx.y;
  if (t >= total_tokens) return;
  const int g = h / (num_q_heads / num_kv_heads);

  // chunk of t: last c with bounds[c] <= t
  int lo = 0, hi = num_chunks - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (bounds[mid] <= t) lo = mid; else hi = mid - 1;
  }
  const int ci = lo;

  float qv[PER];
  const float* qrow = q + (static_cast<size_t>(t) * num_q_heads + h) * D;
#pragma unroll
  for (int e = 0; e < PER; ++e) qv[e] = qrow[lane + 32 * e];

  float m_run = -INFINITY, l_run = 0.f;
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;

  const size_t kv_stride = static_cast<size_t>(num_kv_heads) * D;
  const int r = (h / plan_group) * num_chunks + ci;
  int p0 = row_ptr[r], p1 = row_ptr[r + 1];
  if (p0 < 0 || p1 < p0 || p1 > nnz) {
    // a malformed plan row: reported, and walked as an empty row
    if (lane == 0) report(status, kDevCheck);
    p0 = p1 = 0;
  }
  for (int p = p0; p < p1; ++p) {
    int cj = col[p];
    if (static_cast<unsigned>(cj) >= static_cast<unsigned>(num_chunks)) {
      // an entry outside the chunk range: reported and skipped
      if (lane == 0) report(status, kDevCheck);
      continue;
    }
    const int s0 = bounds[cj];
    const int s1 = min(bounds[cj + 1], t + 1);  // causal
    for (int sb = s0; sb < s1; sb += 32) {
      const int nb = min(32, s1 - sb);
      float my_logit = -INFINITY;
      for (int u = 0; u < nb; ++u) {
        const float* krow = k + (sb + u) * kv_stride + static_cast<size_t>(g) * D;
        float part = 0.f;
#pragma unroll
        for (int e = 0; e < PER; ++e) part = fmaf(qv[e], krow[lane + 32 * e], part);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if (lane == u) my_logit = part * scale;
      }
      float bmax = my_logit;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, o));
      const float m_new = fmaxf(m_run, bmax);
      const float alpha = expf(m_run - m_new);  // m_run = -inf on the first batch -> 0
      const float pw = lane < nb ? expf(my_logit - m_new) : 0.f;
      float psum = pw;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, o);
      l_run = l_run * alpha + psum;
#pragma unroll
      for (int e = 0; e < PER; ++e) acc[e] *= alpha;
      for (int u = 0; u < nb; ++u) {
        const float pu = __shfl_sync(0xffffffffu, pw, u);
        const float* vrow = v + (sb + u) * kv_stride + static_cast<size_t>(g) * D;
#pragma unroll
        for (int e = 0; e < PER; ++e) acc[e] = fmaf(pu, vrow[lane + 32 * e], acc[e]);
      }
      m_run = m_new;
    }
  }
  const float inv = 1.f / l_run;
  float* orow = out + (static_cast<size_t>(t) * num_q_heads + h) * D;
#pragma unroll
  for (int e = 0; e < PER; ++e) orow[lane + 32 * e] = acc[e] * inv;
}

}  // namespace

cudaError_t launch_attention_f32(const float* q, const float* k, const float* v, const int* bounds,
                                 int num_chunks, const int* row_ptr, const int* col, int nnz, int total_tokens,
                                 int num_q_heads, int num_kv_heads, int head_dim, int plan_group, float scale,
                                 float* out, uint32_t* status, cudaStream_t stream) {
  if (total_tokens <= 0) return cudaSuccess;
  dim3 grid((total_tokens + kRowsPerCta - 1) / kRowsPerCta, num_q_heads);
  switch (head_dim) {
    case 64:
      attention_f32_kernel<64><<<grid, kRowsPerCta * 32, 0, stream>>>(
          q, k, v, bounds, num_chunks, row_ptr, col, nnz, total_tokens, num_q_heads, num_kv_heads, plan_group,
          scale, out, status);
      break;
    case 128:
      attention_f32_kernel<128><<<grid, kRowsPerCta * 32, 0, stream>>>(
          q, k, v, bounds, num_chunks, row_ptr, col, nnz, total_tokens, num_q_heads, num_kv_heads, plan_group,
          scale, out, status);
      break;
    case 256:
      attention_f32_kernel<256><<<grid, kRowsPerCta * 32, 0, stream>>>(
          q, k, v, bounds, num_chunks, row_ptr, col, nnz, total_tokens, num_q_heads, num_kv_heads, plan_group,
          scale, out, status);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace dhsa
