// Step 3 of the DHSA path: upsampling + selection.
//
// Every token pair of chunks (i, j) inherits score(i, j), so the token-level
// keep decision of the pages ("Long-Context Modeling with Dynamic Hierarchical
// Sparse Attention for On-Device LLMs", Abstract: chunk similarity upsampled to
// token level decides which token interactions are kept; "... for
// Memory-Constrained LLM Inference": chunk-level importance propagated to
// token-level interactions, keeping causal dependencies) reduces to keeping
// whole key chunks.  Row (h, i) keeps the budget's number of admissible key
// chunks j < i of the same sequence with the largest S[h, i, j] (ties to the
// lower j), plus the diagonal chunk i, written in ascending order.
//
// One warp per row.  The row's scores are read once (coalesced) into shared
// memory as order-preserving 32-bit keys; an MSB-first radix select (four
// 8-bit digit passes over a warp-private 256-bin histogram) finds the k-th
// largest key exactly; a ballot/popcount sweep in index order then emits every
// key above the threshold and the lowest-indexed keys equal to it.
#include "common.cuh"
#include "launchers.h"

namespace dhsa {
namespace {

constexpr int kSelWarps = 4;

__device__ __forceinline__ int row_budget(int i_local, const BudgetArgs& b) {
  if (b.kind == 0) return min(b.k, i_local);
  // ceil(i_local * num / den), capped at i_local (64-bit to avoid overflow)
  const long long want = (static_cast<long long>(i_local) * b.num + b.den - 1) / b.den;
  return static_cast<int>(min(static_cast<long long>(i_local), want));
}

__device__ __forceinline__ uint32_t order_key(float s) {
  uint32_t u = __float_as_uint(s);
  if (u == 0x80000000u) u = 0u;  // -0 ranks equal to +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ int seq_of_chunk(const int* __restrict__ ptr, int num_seqs, int c) {
  int lo = 0, hi = num_seqs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (ptr[mid] <= c) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// grid: x = chunk i, y = group of kSelWarps query heads.
__global__ void __launch_bounds__(kSelWarps * 32)
    topk_select_kernel(const float* __restrict__ scores, int num_chunks, int num_q_heads,
                       const int* __restrict__ seq_chunk_ptr, int num_seqs, BudgetArgs budget,
                       int* __restrict__ row_ptr, int* __restrict__ col, int nnz_per_head,
                       int key_capacity, uint32_t* status) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ int s_red[kSelWarps];
  const int i = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // plan offset of chunk i within one head: sum over earlier chunks of (budget + 1)
  int local = 0;
  for (int b = 0; b < num_seqs; ++b) {
    const int c0 = seq_chunk_ptr[b];
    if (c0 >= i) break;
    const int cnt = min(seq_chunk_ptr[b + 1], i) - c0;
    for (int l = threadIdx.x; l < cnt; l += blockDim.x) local += row_budget(l, budget) + 1;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) local += __shfl_xor_sync(0xffffffffu, local, o);
  if (lane == 0) s_red[warp] = local;
  __syncthreads();
  int prefix = 0;
#pragma unroll
  for (int w = 0; w < kSelWarps; ++w) prefix += s_red[w];

  const int h = blockIdx.y * kSelWarps + warp;
  if (h >= num_q_heads) return;
  const int b = seq_of_chunk(seq_chunk_ptr, num_seqs, i);
  const int c0 = seq_chunk_ptr[b];
  const int m = i - c0;  // admissible candidates c0 .. i-1
  const int keep = row_budget(m, budget);
  const int row = h * num_chunks + i;
  const int off = h * nnz_per_head + prefix;
  if (lane == 0) {
    row_ptr[row] = off;
    if (row == num_q_heads * num_chunks - 1) row_ptr[row + 1] = off + keep + 1;
  }
  int* out = col + off;
  if (keep >= m) {  // every admissible chunk is kept
    for (int j = lane; j < m; j += 32) out[j] = c0 + j;
    if (lane == 0) out[m] = i;
    return;
  }
  if (keep == 0) {
    if (lane == 0) out[0] = i;
    return;
  }
  if (m > key_capacity) {  // host sizing guarantees this cannot happen
    if (lane == 0) report(status, kDevCheck);
    return;
  }

  uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw) + static_cast<size_t>(warp) * (key_capacity + 256);
  int* hist = reinterpret_cast<int*>(keys + key_capacity);
  const float* srow = scores + (static_cast<size_t>(h) * num_chunks + i) * num_chunks + c0;
  for (int j = lane; j < m; j += 32) keys[j] = order_key(srow[j]);

  uint32_t prefix_bits = 0, prefix_mask = 0;
  int remaining = keep;  // how many still to take among keys matching prefix_bits
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
#pragma unroll
    for (int q = 0; q < 8; ++q) hist[lane * 8 + q] = 0;
    __syncwarp();
    for (int j = lane; j < m; j += 32) {
      const uint32_t kj = keys[j];
      if ((kj & prefix_mask) == prefix_bits) atomicAdd(&hist[(kj >> shift) & 255u], 1);
    }
    __syncwarp();
    // lane L owns digits 255-8L down to 248-8L (descending order across lanes)
    int cnt[8];
    int mine = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      cnt[q] = hist[255 - 8 * lane - q];
      mine += cnt[q];
    }
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const int excl = incl - mine;
    const bool here = excl < remaining && remaining <= incl;
    const unsigned hit = __ballot_sync(0xffffffffu, here);
    const int src = __ffs(hit) - 1;
    int digit = 0, above = 0;
    if (here) {
      int run = excl;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (run + cnt[q] >= remaining) {
          digit = 255 - 8 * lane - q;
          above = run;
          break;
        }
        run += cnt[q];
      }
    }
    digit = __shfl_sync(0xffffffffu, digit, src);
    above = __shfl_sync(0xffffffffu, above, src);
    remaining -= above;
    prefix_bits |= static_cast<uint32_t>(digit) << shift;
    prefix_mask |= 0xFFu << shift;
    __syncwarp();
  }
  const uint32_t thr = prefix_bits;
  const int need_eq = remaining;  // keys equal to thr to take, lowest index first

  int written = 0, eq_seen = 0;
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int base = 0; base < m; base += 32) {
    const int j = base + lane;
    const uint32_t kj = j < m ? keys[j] : 0u;
    const bool gt = j < m && kj > thr;
    const bool eq = j < m && kj == thr;
    const unsigned eqm = __ballot_sync(0xffffffffu, eq);
    const bool sel = gt || (eq && (eq_seen + __popc(eqm & lt_mask)) < need_eq);
    const unsigned selm = __ballot_sync(0xffffffffu, sel);
    if (sel) out[written + __popc(selm & lt_mask)] = c0 + j;
    written += __popc(selm);
    eq_seen += __popc(eqm);
  }
  if (lane == 0) {
    out[keep] = i;
    if (written != keep) report(status, kDevCheck);
  }
}

}  // namespace

size_t topk_select_smem_bytes(int key_capacity) {
  return static_cast<size_t>(kSelWarps) * (static_cast<size_t>(key_capacity) + 256) * 4;
}

cudaError_t launch_topk_select(const float* scores, int num_chunks, int num_q_heads,
                               const int* seq_chunk_ptr, int num_seqs, BudgetArgs budget,
                               int* row_ptr, int* col, int nnz_per_head, int key_capacity,
                               uint32_t* status, cudaStream_t stream) {
  if (num_chunks <= 0) return cudaSuccess;
  const size_t smem = topk_select_smem_bytes(key_capacity);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(topk_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  dim3 grid(num_chunks, (num_q_heads + kSelWarps - 1) / kSelWarps);
  topk_select_kernel<<<grid, kSelWarps * 32, smem, stream>>>(scores, num_chunks, num_q_heads, seq_chunk_ptr,
                                                             num_seqs, budget, row_ptr, col, nnz_per_head,
                                                             key_capacity, status);
  return cudaGetLastError();
}

}  // namespace dhsa
