// Selection margins of a plan: for every plan row, the smallest score among
// the kept earlier chunks (the k-th largest admissible score) and the largest
// score among the admissible chunks left out (the (k+1)-th).  The selection
// keeps the top-k admissible chunks by score, ties to the lower index ("Long-
// Context Modeling with Dynamic Hierarchical Sparse Attention for On-Device
// LLMs", Abstract: chunk scores decide which interactions are kept), so the
// gap between the two says how close the row is to a different selection:
// rows whose two margins are nearly equal are the ones where rounding in the
// scores can change the plan.
//
// One warp per plan row (grid-stride).  The kept set is the plan row without
// its last entry (the diagonal); membership of a candidate is a binary search
// in the ascending row.  Entries outside the row's candidate range are
// reported (kDevCheck) and skipped.
#include <math.h>

#include "common.cuh"
#include "launchers.h"

namespace dhsa {
namespace {

constexpr int kWarpsPerCta = 8;

__device__ __forceinline__ int sequence_start(const int* __restrict__ seq_chunk_ptr, int num_seqs, int c) {
  int lo = 0, hi = num_seqs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (seq_chunk_ptr[mid] <= c) lo = mid; else hi = mid - 1;
  }
  return seq_chunk_ptr[lo];
}

__global__ void __launch_bounds__(kWarpsPerCta * 32)
    plan_margins_kernel(const float* __restrict__ scores, const int* __restrict__ row_ptr,
                        const int* __restrict__ col, long long nnz, int rows, int num_chunks,
                        const int* __restrict__ seq_chunk_ptr, int num_seqs, float* __restrict__ margins,
                        uint32_t* status) {
  const int lane = threadIdx.x & 31;
  const int warps = gridDim.x * kWarpsPerCta;
  for (int r = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5); r < rows; r += warps) {
    const int i = r % num_chunks;
    const long long p0 = row_ptr[r], p1 = row_ptr[r + 1];
    float kept_min = INFINITY, left_max = -INFINITY;
    bool any_kept = false, any_left = false, bad = false;
    if (p0 < 0 || p1 <= p0 || p1 > nnz) {
      bad = true;
    } else {
      const int c0 = sequence_start(seq_chunk_ptr, num_seqs, i);
      const float* srow = scores + static_cast<size_t>(r) * num_chunks;  // S[plan head, i, :]
      const long long kend = p1 - 1;  // kept earlier chunks: [p0, p1 - 1), the diagonal last
      for (long long p = p0 + lane; p < kend; p += 32) {
        const int j = col[p];
        if (j < c0 || j >= i) {
          bad = true;
          continue;
        }
        kept_min = fminf(kept_min, srow[j]);
        any_kept = true;
      }
      for (int j = c0 + lane; j < i; j += 32) {
        long long lo = p0, hi = kend;  // is j in col[p0 .. kend)?
        while (lo < hi) {
          const long long mid = (lo + hi) >> 1;
          if (col[mid] < j) lo = mid + 1; else hi = mid;
        }
        if (lo < kend && col[lo] == j) continue;
        left_max = fmaxf(left_max, srow[j]);
        any_left = true;
      }
    }
    for (int o = 16; o > 0; o >>= 1) {
      kept_min = fminf(kept_min, __shfl_xor_sync(0xffffffffu, kept_min, o));
      left_max = fmaxf(left_max, __shfl_xor_sync(0xffffffffu, left_max, o));
    }
    any_kept = __any_sync(0xffffffffu, any_kept);
    any_left = __any_sync(0xffffffffu, any_left);
    bad = __any_sync(0xffffffffu, bad);
    if (lane == 0) {
      margins[2 * static_cast<size_t>(r)] = any_kept ? kept_min : NAN;
      margins[2 * static_cast<size_t>(r) + 1] = any_left ? left_max : NAN;
      if (bad) report(status, kDevCheck);
    }
  }
}

}  // namespace

cudaError_t launch_plan_margins(const float* scores, const int* row_ptr, const int* col, long long nnz, int rows,
                                int num_chunks, const int* seq_chunk_ptr, int num_seqs, float* margins,
                                uint32_t* status, cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int need = (rows + kWarpsPerCta - 1) / kWarpsPerCta;
  const int grid = need < 8 * sms ? need : 8 * sms;
  plan_margins_kernel<<<grid, kWarpsPerCta * 32, 0, stream>>>(scores, row_ptr, col, nnz, rows, num_chunks,
                                                               seq_chunk_ptr, num_seqs, margins, status);
  return cudaGetLastError();
}

}  // namespace dhsa
