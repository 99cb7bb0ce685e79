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
// One 256-thread CTA per row.  The row's scores are read once (coalesced) into
// shared memory as order-preserving 32-bit keys, the first digit histogram
// being built during that load; an MSB-first radix select (8-bit digits over a
// block-shared 256-bin histogram) finds the k-th largest key exactly, stopping
// early once the threshold bucket is taken whole.  Compaction is in index
// order: each warp owns a contiguous segment, per-warp counts of keys above and
// equal to the threshold give every warp its output offset and its share of
// the equal keys (lowest index first), and ballots place the keys.  The row's
// plan offset comes in closed form (plan_entries), not from a loop over the
// earlier chunks.
#include "common.cuh"
#include "launchers.h"

namespace dhsa {
namespace {

constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;

__device__ __forceinline__ int row_budget(int i_local, const BudgetArgs& b) {
  if (b.kind == 0) return min(b.k, i_local);
  // ceil(i_local * num / den), capped at i_local (64-bit to avoid overflow)
  const long long want = (static_cast<long long>(i_local) * b.num + b.den - 1) / b.den;
  return static_cast<int>(min(static_cast<long long>(i_local), want));
}

// sum_{l=0}^{n-1} floor((a*l + c) / m) for n, a, c >= 0 and m >= 1: lattice
// points under a line, counted by the Euclid-like reduction (swap the roles of
// a and m after taking out the integer parts), O(log) steps.
__device__ long long floor_sum(long long n, long long m, long long a, long long c) {
  long long total = 0;
  while (n > 0) {
    if (a >= m) {
      total += (n * (n - 1) / 2) * (a / m);
      a %= m;
    }
    if (c >= m) {
      total += n * (c / m);
      c %= m;
    }
    const long long y_max = a * n + c;
    if (y_max < m) break;
    n = y_max / m;
    c = y_max % m;
    const long long t = m;
    m = a;
    a = t;
  }
  return total;
}

// sum over l in [0, L) of (budget(l) + 1): plan entries of the first L chunks
// of a sequence, in closed form.
__device__ long long plan_entries(long long L, const BudgetArgs& b) {
  if (L <= 0) return 0;
  long long s;
  if (b.kind == 0) {
    const long long k = b.k;
    s = L <= k ? L * (L - 1) / 2 : k * (k - 1) / 2 + k * (L - k);
  } else if (b.num >= b.den) {
    s = L * (L - 1) / 2;  // ceil(l * num / den) >= l: every earlier chunk
  } else {
    s = floor_sum(L, b.den, b.num, b.den - 1);  // sum of ceil(l * num / den)
  }
  return s + L;
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

// grid: x = chunk i, y = query head; one 256-thread CTA per row (h, i).
__global__ void __launch_bounds__(kSelThreads)
    topk_select_kernel(const float* __restrict__ scores, int num_chunks, int num_q_heads,
                       const int* __restrict__ seq_chunk_ptr, int num_seqs, BudgetArgs budget,
                       int* __restrict__ row_ptr, int* __restrict__ col, int nnz_per_head,
                       int key_capacity, uint32_t* status) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ int hist[256];
  __shared__ int s_gt[kSelWarps], s_eq[kSelWarps];
  __shared__ int s_prefix, s_digit, s_above, s_count;
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw);
  const int i = blockIdx.x, h = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // plan offset of chunk i within one head: entries of every earlier chunk
  if (tid == 0) {
    long long acc = 0;
    for (int b = 0; b < num_seqs; ++b) {
      const int c0 = seq_chunk_ptr[b];
      if (c0 >= i) break;
      acc += plan_entries(min(seq_chunk_ptr[b + 1], i) - c0, budget);
    }
    s_prefix = static_cast<int>(acc);
  }
  for (int q = tid; q < 256; q += kSelThreads) hist[q] = 0;
  __syncthreads();
  const int prefix = s_prefix;

  const int b = seq_of_chunk(seq_chunk_ptr, num_seqs, i);
  const int c0 = seq_chunk_ptr[b];
  const int m = i - c0;  // admissible candidates c0 .. i-1
  const int keep = row_budget(m, budget);
  const int row = h * num_chunks + i;
  const int off = h * nnz_per_head + prefix;
  if (tid == 0) {
    row_ptr[row] = off;
    if (row == num_q_heads * num_chunks - 1) row_ptr[row + 1] = off + keep + 1;
  }
  int* out = col + off;
  if (keep >= m) {  // every admissible chunk is kept
    for (int j = tid; j < m; j += kSelThreads) out[j] = c0 + j;
    if (tid == 0) out[m] = i;
    return;
  }
  if (keep == 0) {
    if (tid == 0) out[0] = i;
    return;
  }
  if (m > key_capacity) {  // host sizing guarantees this cannot happen
    if (tid == 0) report(status, kDevCheck);
    return;
  }

  // load the row once (coalesced) as order-preserving keys; first digit pass fused in
  const float* srow = scores + (static_cast<size_t>(h) * num_chunks + i) * num_chunks + c0;
#pragma unroll 4
  for (int j = tid; j < m; j += kSelThreads) {
    const uint32_t kj = order_key(__ldcs(srow + j));
    keys[j] = kj;
    atomicAdd(&hist[kj >> 24], 1);
  }
  __syncthreads();

  uint32_t prefix_bits = 0, prefix_mask = 0;
  int remaining = keep;  // still to take among keys matching prefix_bits under prefix_mask
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    if (pass > 0) {
      for (int j = tid; j < m; j += kSelThreads) {
        const uint32_t kj = keys[j];
        if ((kj & prefix_mask) == prefix_bits) atomicAdd(&hist[(kj >> shift) & 255u], 1);
      }
      __syncthreads();
    }
    if (warp == 0) {
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
      if (excl < remaining && remaining <= incl) {
        int run = excl;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (run + cnt[q] >= remaining) {
            s_digit = 255 - 8 * lane - q;
            s_above = run;
            s_count = cnt[q];
            break;
          }
          run += cnt[q];
        }
      }
    }
    __syncthreads();
    const int digit = s_digit, above = s_above, count = s_count;
    remaining -= above;
    prefix_bits |= static_cast<uint32_t>(digit) << shift;
    prefix_mask |= 0xFFu << shift;
    if (remaining == count) break;  // the whole bucket is taken: no finer digits needed
    for (int q = tid; q < 256; q += kSelThreads) hist[q] = 0;
    __syncthreads();
  }
  // selected: (key & mask) > prefix, plus the lowest-indexed `need_eq` keys with
  // (key & mask) == prefix (all of them when the bucket was taken whole)
  const uint32_t thr = prefix_bits, msk = prefix_mask;
  const int need_eq = remaining;

  // compaction in index order: warp w owns the contiguous segment [lo, hi)
  const int seg = (m + kSelWarps - 1) / kSelWarps;
  const int lo = min(m, warp * seg), hi = min(m, lo + seg);
  int n_gt = 0, n_eq = 0;
  for (int base = lo; base < hi; base += 32) {
    const int j = base + lane;
    const uint32_t kj = j < hi ? (keys[j] & msk) : 0u;
    n_gt += __popc(__ballot_sync(0xffffffffu, j < hi && kj > thr));
    n_eq += __popc(__ballot_sync(0xffffffffu, j < hi && kj == thr));
  }
  if (lane == 0) {
    s_gt[warp] = n_gt;
    s_eq[warp] = n_eq;
  }
  __syncthreads();
  int eq_before = 0, sel_before = 0;
  for (int w = 0; w < warp; ++w) {
    const int eqb = eq_before;
    eq_before += s_eq[w];
    sel_before += s_gt[w] + min(max(need_eq - eqb, 0), s_eq[w]);
  }
  int written = sel_before, eq_seen = eq_before;
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int base = lo; base < hi; base += 32) {
    const int j = base + lane;
    const uint32_t kj = j < hi ? (keys[j] & msk) : 0u;
    const bool gt = j < hi && kj > thr;
    const bool eq = j < hi && kj == thr;
    const unsigned eqm = __ballot_sync(0xffffffffu, eq);
    const bool sel = gt || (eq && (eq_seen + __popc(eqm & lt_mask)) < need_eq);
    const unsigned selm = __ballot_sync(0xffffffffu, sel);
    if (sel) out[written + __popc(selm & lt_mask)] = c0 + j;
    written += __popc(selm);
    eq_seen += __popc(eqm);
  }
  if (warp == kSelWarps - 1 && lane == 0) {
    out[keep] = i;
    if (written != keep) report(status, kDevCheck);
  }
}

}  // namespace

size_t topk_select_smem_bytes(int key_capacity) { return static_cast<size_t>(key_capacity) * 4; }

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
  dim3 grid(num_chunks, num_q_heads);
  topk_select_kernel<<<grid, kSelThreads, smem, stream>>>(scores, num_chunks, num_q_heads, seq_chunk_ptr,
                                                             num_seqs, budget, row_ptr, col, nnz_per_head,
                                                             key_capacity, status);
  return cudaGetLastError();
}

}  // namespace dhsa
