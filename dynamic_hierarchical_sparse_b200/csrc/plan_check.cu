// Device-side validation of a plan handed to the attention step.
//
// A plan is valid for the attention kernels when every row (plan head, query
// chunk i) is a non-empty, strictly ascending list of chunks of i's own
// sequence that are not later than i, ending with i itself: the admissible
// key chunks kept for i plus its diagonal chunk ("Long-Context Modeling with
// Dynamic Hierarchical Sparse Attention for On-Device LLMs", Abstract: the
// kept token interactions follow causal order; "... for Memory-Constrained
// LLM Inference": causally important dependencies are kept), and the row
// offsets run from 0 to nnz without decreasing.  The kernel reads only
// row_ptr[0 .. rows] and col[0 .. nnz), the sizes the caller declares, so a
// malformed plan cannot make it read out of range; every violation sets the
// device-check bit of the status word.
#include "common.cuh"
#include "launchers.h"

namespace dhsa {
namespace {

constexpr int kWarpsPerCta = 8;

__device__ __forceinline__ int sequence_start_chunk(const int* __restrict__ seq_chunk_ptr, int num_seqs, int c) {
  int lo = 0, hi = num_seqs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (seq_chunk_ptr[mid] <= c) lo = mid; else hi = mid - 1;
  }
  return seq_chunk_ptr[lo];
}

// One warp per plan row (grid-stride over rows).
__global__ void __launch_bounds__(kWarpsPerCta * 32)
    plan_check_kernel(const int* __restrict__ row_ptr, const int* __restrict__ col, long long nnz, int rows,
                      int num_chunks, const int* __restrict__ seq_chunk_ptr, int num_seqs, uint32_t* status) {
  const int lane = threadIdx.x & 31;
  const int warps = gridDim.x * kWarpsPerCta;
  bool bad = false;
  for (int r = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5); r < rows; r += warps) {
    const long long p0 = row_ptr[r], p1 = row_ptr[r + 1];
    if (r == 0 && p0 != 0) bad = true;
    if (r == rows - 1 && p1 != nnz) bad = true;
    if (p0 < 0 || p1 <= p0 || p1 > nnz) {  // empty (no diagonal), decreasing, or past the end
      bad = true;
      continue;
    }
    const int i = r % num_chunks;
    const int c0 = sequence_start_chunk(seq_chunk_ptr, num_seqs, i);
    for (long long p = p0 + lane; p < p1; p += 32) {
      const int c = col[p];
      if (c < c0 || c > i) bad = true;                  // another sequence, or a later chunk
      if (p + 1 < p1 && col[p + 1] <= c) bad = true;    // not strictly ascending
      if (p + 1 == p1 && c != i) bad = true;            // the diagonal is the last entry
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) report(status, kDevCheck);
}

}  // namespace

cudaError_t launch_plan_check(const int* row_ptr, const int* col, long long nnz, int rows, int num_chunks,
                              const int* seq_chunk_ptr, int num_seqs, uint32_t* status, cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int need = (rows + kWarpsPerCta - 1) / kWarpsPerCta;
  const int grid = need < 8 * sms ? need : 8 * sms;
  plan_check_kernel<<<grid, kWarpsPerCta * 32, 0, stream>>>(row_ptr, col, nnz, rows, num_chunks, seq_chunk_ptr,
                                                             num_seqs, status);
  return cudaGetLastError();
}

}  // namespace dhsa
