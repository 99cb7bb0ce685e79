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
// One warp per row, eight consecutive rows (chunks i) of one query head per
// CTA.  Row offsets in the CSR follow from one closed-form offset per CTA
// (plan_entries) plus the budgets of the CTA's earlier rows.
//
// Rows longer than kFilterMin with a budget of at most 1/8 of the row first
// try a filter: the warp sorts 64 evenly spaced samples and takes as threshold
// tau the sample a few ranks below the budget's quantile; one coalesced sweep
// keeps the scores >= tau ("survivors", in index order, with their indices).
// When at least `keep` scores survive and they fit, the k-th largest score is
// among them and the exact selection runs on them only.  Otherwise (an unlucky
// sample, heavy ties, large budgets, short rows) the row is staged whole in the
// warp's shared memory, or, when it does not fit, selected from global memory
// directly; so the result never depends on the sample and no row is too long.
// Every route ends in the same exact selection: an MSB-first radix select over
// a warp-private 256-bin histogram on order-preserving 32-bit keys.  All keys
// lie between a known lower bound (tau, or the row minimum) and the row
// maximum, so they share every bit above the highest bit where the two differ;
// the radix starts there, takes up to 8 bits per pass and stops once the
// threshold bucket is taken whole.  One pass in index order then writes the
// keys above the threshold plus the lowest-indexed keys equal to it.
#include "common.cuh"
#include "launchers.h"

namespace dhsa {
namespace {

constexpr int kSelWarps = 8;  // rows per CTA
constexpr int kSelThreads = 32 * kSelWarps;
constexpr int kSurvCap = 896;           // staged keys per warp
constexpr int kFilterMin = 384;         // rows at most this long are staged whole
constexpr int kFilterMaxCandidates = 65535;  // survivor indices are 16-bit
constexpr int kSamples = 64;
constexpr int kSampleMargin = 5;  // ranks below the budget's sample quantile
constexpr int kBatch = 16;        // loads in flight per lane in the sweeps

struct WarpScratch {
  int hist[256];
  uint32_t key[kSurvCap];
  uint16_t idx[kSurvCap];
};

// a / b and a % b on non-negative 64-bit values, in 32-bit arithmetic when both fit
__device__ __forceinline__ unsigned long long udiv(unsigned long long a, unsigned long long b) {
  if (((a | b) >> 32) == 0) return static_cast<uint32_t>(a) / static_cast<uint32_t>(b);
  return a / b;
}

__device__ __forceinline__ int row_budget(int i_local, const BudgetArgs& b) {
  if (b.kind == 0) return min(b.k, i_local);
  // ceil(i_local * num / den), capped at i_local
  const unsigned long long want =
      udiv(static_cast<unsigned long long>(i_local) * b.num + b.den - 1, static_cast<unsigned long long>(b.den));
  return static_cast<int>(min(static_cast<unsigned long long>(i_local), want));
}

// sum_{l=0}^{n-1} floor((a*l + c) / m) for n, a, c >= 0 and m >= 1: lattice
// points under a line, counted by the Euclid-like reduction (swap the roles of
// a and m after taking out the integer parts), O(log) steps.
__device__ unsigned long long floor_sum(unsigned long long n, unsigned long long m, unsigned long long a,
                                        unsigned long long c) {
  unsigned long long total = 0;
  while (n > 0) {
    if (a >= m) {
      const unsigned long long q = udiv(a, m);
      total += (n * (n - 1) / 2) * q;
      a -= q * m;
    }
    if (c >= m) {
      const unsigned long long q = udiv(c, m);
      total += n * q;
      c -= q * m;
    }
    const unsigned long long y_max = a * n + c;
    if (y_max < m) break;
    n = udiv(y_max, m);
    c = y_max - n * m;
    const unsigned long long t = m;
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
    s = static_cast<long long>(floor_sum(L, b.den, b.num, b.den - 1));  // sum of ceil(l * num / den)
  }
  return s + L;
}

__device__ __forceinline__ uint32_t order_key(float s) {
  uint32_t u = __float_as_uint(s);
  if (u == 0x80000000u) u = 0u;  // -0 ranks equal to +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// the float whose order key is k (+0 for the key of both zeros)
__device__ __forceinline__ float key_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

__device__ __forceinline__ int seq_of_chunk(const int* __restrict__ ptr, int num_seqs, int c) {
  int lo = 0, hi = num_seqs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (ptr[mid] <= c) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Sorts 64 keys held two per lane (element e = slot * 32 + lane) into
// descending order with a bitonic network.
__device__ __forceinline__ void bitonic64_desc(uint32_t& v0, uint32_t& v1, int lane) {
#pragma unroll
  for (int k = 2; k <= 64; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j == 32) {
        const uint32_t hi = max(v0, v1), lo = min(v0, v1);
        v0 = hi;
        v1 = lo;
      } else {
        const uint32_t p0 = __shfl_xor_sync(0xffffffffu, v0, j);
        const uint32_t p1 = __shfl_xor_sync(0xffffffffu, v1, j);
        const bool low = (lane & j) == 0;
        // a block of size k sorts descending when (e & k) == 0
        const bool d0 = (lane & k) == 0;
        const bool d1 = k == 32 ? false : (lane & k) == 0;
        v0 = (d0 == low) ? max(v0, p0) : min(v0, p0);
        v1 = (d1 == low) ? max(v1, p1) : min(v1, p1);
      }
    }
  }
}

// Exact selection of the `keep` largest of n keys (ties to the lower index),
// written ascending by index to out[0..keep).  Keys come from get_key(t),
// their chunk ids from get_col(t), t ascending = index ascending; every key
// lies in [lo, hi].  The keys then share every bit above the highest bit where
// lo and hi differ, so the MSB-first radix starts there: each pass takes the
// (up to) 8 bits below the bits already fixed.  hist[] is zero on entry and is
// left zero.  Should fewer than `keep` keys be written (a defect, which the
// caller reports), the remaining slots get `fill` (the row's diagonal chunk), so
// the row never holds an index outside the chunk range.
template <typename GetKey, typename GetCol>
__device__ __forceinline__ bool warp_select(int n, int keep, uint32_t lo, uint32_t hi, int* hist, GetKey get_key,
                                            GetCol get_col, int* __restrict__ out, int fill, int lane) {
  const uint32_t diff = lo ^ hi;
  int top = diff == 0u ? -1 : 31 - __clz(static_cast<int>(diff));  // highest undecided bit
  uint32_t mask = top < 0 ? 0xFFFFFFFFu : ~((2u << top) - 1u);      // bits already decided
  uint32_t bits = lo & mask;
  int remaining = keep;  // still to take among keys matching bits under mask
  int count = n;         // keys matching bits under mask
#pragma unroll 1
  while (top >= 0) {
    const int shift = max(0, top - 7);
    const uint32_t dmask = (2u << (top - shift)) - 1u;
    for (int t = lane; t < n; t += 32) {
      const uint32_t k = get_key(t);
      if ((k & mask) == bits) atomicAdd(&hist[(k >> shift) & dmask], 1);
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
#pragma unroll
    for (int q = 0; q < 8; ++q) hist[255 - 8 * lane - q] = 0;
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const int excl = incl - mine;
    const bool here = excl < remaining && remaining <= incl;
    int digit = 0, above = 0, cdig = 0;
    if (here) {
      int run = excl;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (run + cnt[q] >= remaining) {
          digit = 255 - 8 * lane - q;
          above = run;
          cdig = cnt[q];
          break;
        }
        run += cnt[q];
      }
    }
    const int src = __ffs(__ballot_sync(0xffffffffu, here)) - 1;
    digit = __shfl_sync(0xffffffffu, digit, src);
    above = __shfl_sync(0xffffffffu, above, src);
    count = __shfl_sync(0xffffffffu, cdig, src);
    __syncwarp();
    remaining -= above;
    bits |= static_cast<uint32_t>(digit) << shift;
    mask |= dmask << shift;
    if (remaining == count) break;  // the whole bucket is taken: no finer digits needed
    top = shift - 1;
  }
  // selected: (key & mask) > bits, plus the lowest-indexed `remaining` keys with
  // (key & mask) == bits (all of them when the bucket is taken whole)
  const unsigned lt = (1u << lane) - 1u;
  int written = 0;
  if (remaining == count) {
    for (int base = 0; base < n && written < keep; base += 32) {
      const int t = base + lane;
      const bool sel = t < n && (get_key(t) & mask) >= bits;
      const unsigned selm = __ballot_sync(0xffffffffu, sel);
      const int pos = written + __popc(selm & lt);
      if (sel && pos < keep) out[pos] = get_col(t);
      written += __popc(selm);
    }
  } else {
    int eq_seen = 0;
    for (int base = 0; base < n && written < keep; base += 32) {
      const int t = base + lane;
      const uint32_t k = t < n ? (get_key(t) & mask) : 0u;
      const bool gt = t < n && k > bits;
      const bool eq = t < n && k == bits;
      const unsigned eqm = __ballot_sync(0xffffffffu, eq);
      const bool sel = gt || (eq && (eq_seen + __popc(eqm & lt)) < remaining);
      const unsigned selm = __ballot_sync(0xffffffffu, sel);
      const int pos = written + __popc(selm & lt);
      if (sel && pos < keep) out[pos] = get_col(t);
      written += __popc(selm);
      eq_seen += __popc(eqm);
    }
  }
  if (written < keep) {
    for (int t = written + lane; t < keep; t += 32) out[t] = fill;
  }
  return written == keep;  // more or fewer would be a defect: reported, never written past the row
}

// grid: x = group of kSelWarps consecutive chunks, y = query head.
__global__ void __launch_bounds__(kSelThreads)
    topk_select_kernel(const float* __restrict__ scores, int num_chunks, int num_q_heads,
                       const int* __restrict__ seq_chunk_ptr, int num_seqs, BudgetArgs budget,
                       int* __restrict__ row_ptr, int* __restrict__ col, int nnz_per_head, uint32_t* status) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ int s_entries[kSelWarps];
  __shared__ long long s_base;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int i0 = blockIdx.x * kSelWarps;
  const int i = i0 + warp;
  const bool valid = i < num_chunks;
  WarpScratch& ws = reinterpret_cast<WarpScratch*>(smem_raw)[warp];

  int c0 = 0, m = 0, keep = 0;
  if (valid) {
    c0 = seq_chunk_ptr[seq_of_chunk(seq_chunk_ptr, num_seqs, i)];
    m = i - c0;  // admissible candidates c0 .. i-1
    keep = row_budget(m, budget);
  }
  if (lane == 0) s_entries[warp] = valid ? keep + 1 : 0;
  if (threadIdx.x == 0) {
    // plan entries of every chunk before i0, within one head
    long long acc = 0;
    for (int bb = 0; bb < num_seqs; ++bb) {
      const int cb = seq_chunk_ptr[bb];
      if (cb >= i0) break;
      acc += plan_entries(min(seq_chunk_ptr[bb + 1], i0) - cb, budget);
    }
    s_base = acc;
  }
#pragma unroll
  for (int q = 0; q < 8; ++q) ws.hist[32 * q + lane] = 0;
  __syncthreads();
  if (!valid) return;
  long long off = s_base + static_cast<long long>(h) * nnz_per_head;
  for (int w = 0; w < warp; ++w) off += s_entries[w];
  const int row = h * num_chunks + i;
  if (lane == 0) {
    row_ptr[row] = static_cast<int>(off);
    if (row == num_q_heads * num_chunks - 1) row_ptr[row + 1] = static_cast<int>(off) + keep + 1;
  }
  int* out = col + off;
  if (lane == 0) out[keep] = i;  // the diagonal chunk, last
  if (keep >= m) {  // every admissible chunk is kept
    for (int j = lane; j < m; j += 32) out[j] = c0 + j;
    return;
  }
  if (keep == 0) return;

  const float* srow = scores + (static_cast<size_t>(h) * num_chunks + i) * num_chunks + c0;
  const unsigned lt = (1u << lane) - 1u;
  bool ok;
  if (m > kFilterMin && m <= kFilterMaxCandidates && keep * 8 <= m) {
    float xv[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int j = 32 * u + lane;
      xv[u] = j < m ? __ldcs(srow + j) : 0.f;
    }
    // threshold from 64 samples at the midpoints of equal strides
    uint32_t v0 = order_key(__ldg(srow + static_cast<int>(((2LL * lane + 1) * m) / (2 * kSamples))));
    uint32_t v1 = order_key(__ldg(srow + static_cast<int>(((2LL * (32 + lane) + 1) * m) / (2 * kSamples))));
    bitonic64_desc(v0, v1, lane);
    const int r = min(kSamples - 1, static_cast<int>((static_cast<long long>(kSamples) * keep) / m) + kSampleMargin);
    const uint32_t tau_key = __shfl_sync(0xffffffffu, r < 32 ? v0 : v1, r & 31);
    const float tau = key_float(tau_key);
    // sweep: keep the scores >= tau, in index order, as raw bits with their
    // indices (positions past the space are clamped; such a row falls back)
    int n = 0;
    for (int base = 0; base < m; base += 32 * kBatch) {
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int j = base + 32 * u + lane;
        const bool sv = j < m && xv[u] >= tau;
        const unsigned msk = __ballot_sync(0xffffffffu, sv);
        const int pos = min(n + __popc(msk & lt), kSurvCap - 1);
        if (sv) {
          ws.key[pos] = __float_as_uint(xv[u]);
          ws.idx[pos] = static_cast<uint16_t>(j);
        }
        n += __popc(msk);
      }
      if (base + 32 * kBatch < m) {
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
          const int j = base + 32 * kBatch + 32 * u + lane;
          xv[u] = j < m ? __ldcs(srow + j) : 0.f;
        }
      }
    }
    __syncwarp();
    if (n >= keep && n <= kSurvCap) {
      // every survivor's key is >= tau_key; the row maximum bounds them above
      uint32_t hi = 0u;
      for (int t = lane; t < n; t += 32) {
        const uint32_t k = order_key(__uint_as_float(ws.key[t]));
        ws.key[t] = k;
        hi = max(hi, k);
      }
      hi = __reduce_max_sync(0xffffffffu, hi);
      __syncwarp();
      ok = warp_select(
          n, keep, tau_key, hi, ws.hist, [&](int t) { return ws.key[t]; },
          [&](int t) { return c0 + static_cast<int>(ws.idx[t]); }, out, i, lane);
      if (!ok && lane == 0) report(status, kDevCheck);
      return;
    }
  }
  uint32_t lo = 0xFFFFFFFFu, hi = 0u;
  if (m <= kSurvCap) {
    // stage the row whole as order keys, with its key range
    for (int base = 0; base < m; base += 32 * 8) {
      float x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int j = base + 32 * u + lane;
        x[u] = j < m ? __ldcs(srow + j) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int j = base + 32 * u + lane;
        if (j < m) {
          const uint32_t k = order_key(x[u]);
          ws.key[j] = k;
          lo = min(lo, k);
          hi = max(hi, k);
        }
      }
    }
    lo = __reduce_min_sync(0xffffffffu, lo);
    hi = __reduce_max_sync(0xffffffffu, hi);
    __syncwarp();
    ok = warp_select(
        m, keep, lo, hi, ws.hist, [&](int t) { return ws.key[t]; }, [&](int t) { return c0 + t; }, out, i, lane);
  } else {
    // select from the row in global memory (read through L2 once per pass)
    for (int j = lane; j < m; j += 32) {
      const uint32_t k = order_key(__ldg(srow + j));
      lo = min(lo, k);
      hi = max(hi, k);
    }
    lo = __reduce_min_sync(0xffffffffu, lo);
    hi = __reduce_max_sync(0xffffffffu, hi);
    ok = warp_select(
        m, keep, lo, hi, ws.hist, [&](int t) { return order_key(__ldg(srow + t)); }, [&](int t) { return c0 + t; },
        out, i, lane);
  }
  if (!ok && lane == 0) report(status, kDevCheck);
}

}  // namespace

cudaError_t launch_topk_select(const float* scores, int num_chunks, int num_q_heads,
                               const int* seq_chunk_ptr, int num_seqs, BudgetArgs budget,
                               int* row_ptr, int* col, int nnz_per_head, uint32_t* status,
                               cudaStream_t stream) {
  if (num_chunks <= 0) return cudaSuccess;
  constexpr int smem = kSelWarps * static_cast<int>(sizeof(WarpScratch));
  cudaError_t e = cudaFuncSetAttribute(topk_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((num_chunks + kSelWarps - 1) / kSelWarps, num_q_heads);
  topk_select_kernel<<<grid, kSelThreads, smem, stream>>>(scores, num_chunks, num_q_heads, seq_chunk_ptr,
                                                             num_seqs, budget, row_ptr, col, nnz_per_head,
                                                             status);
  return cudaGetLastError();
}

}  // namespace dhsa
