// Step 2 of the DHSA path: chunk-level similarity scores.
//
// S[h, i, j] = qc[h, i, :] . kc[g(h), j, :] for j <= i in the same sequence
// ("Long-Context Modeling with Dynamic Hierarchical Sparse Attention for
// On-Device LLMs", Abstract: chunk-level similarity scores; the dot product of
// the chunk representations).  No 1/sqrt(d): it does not change any ranking.
//
// A small, ragged fp32 contraction (at most a few hundred MFLOP): plain FFMA
// with 32x32 output tiles staged through shared memory.  Tiles entirely above
// the diagonal or outside every sequence's triangle exit at once.
#include "common.cuh"
#include "launchers.h"

namespace dhsa {
namespace {

constexpr int kTile = 32;
constexpr int kDk = 32;  // depth slice staged per step

__device__ __forceinline__ int seq_of_chunk(const int* __restrict__ seq_chunk_ptr, int num_seqs, int c) {
  int lo = 0, hi = num_seqs - 1;  // last b with seq_chunk_ptr[b] <= c
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (seq_chunk_ptr[mid] <= c) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// grid: x = j tile, y = i tile, z = query head.  256 threads, 4 outputs each.
__global__ void __launch_bounds__(256)
    chunk_similarity_kernel(const float* __restrict__ qc, const float* __restrict__ kc, int num_chunks,
                            int head_dim, int group, const int* __restrict__ seq_chunk_ptr,
                            int num_seqs, float* __restrict__ scores) {
  const int jt = blockIdx.x, it = blockIdx.y, h = blockIdx.z;
  const int i0 = it * kTile, j0 = jt * kTile;
  if (j0 > i0 + kTile - 1) return;  // strictly above the diagonal
  // first chunk of the sequence of the earliest query chunk in this tile
  const int seq_first = seq_chunk_ptr[seq_of_chunk(seq_chunk_ptr, num_seqs, i0)];
  if (j0 + kTile - 1 < seq_first) return;  // every pair crosses a sequence edge

  __shared__ float sq[kTile][kDk + 1];
  __shared__ float sk[kTile][kDk + 1];
  const float* qh = qc + static_cast<size_t>(h) * num_chunks * head_dim;
  const float* kh = kc + static_cast<size_t>(h / group) * num_chunks * head_dim;

  const int tx = threadIdx.x & 31;   // j within tile
  const int ty = threadIdx.x >> 5;   // 8 rows of i, 4 apart
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int k0 = 0; k0 < head_dim; k0 += kDk) {
    for (int e = threadIdx.x; e < kTile * kDk; e += 256) {
      const int r = e / kDk, cc = e % kDk;
      const int ii = i0 + r, jj = j0 + r;
      sq[r][cc] = ii < num_chunks ? qh[static_cast<size_t>(ii) * head_dim + k0 + cc] : 0.f;
      sk[r][cc] = jj < num_chunks ? kh[static_cast<size_t>(jj) * head_dim + k0 + cc] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int cc = 0; cc < kDk; ++cc) {
      const float kv = sk[tx][cc];
#pragma unroll
      for (int r = 0; r < 4; ++r) acc[r] = fmaf(sq[ty + 8 * r][cc], kv, acc[r]);
    }
    __syncthreads();
  }
  const int j = j0 + tx;
  if (j >= num_chunks) return;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int i = i0 + ty + 8 * r;
    if (i >= num_chunks || j > i) continue;
    const int first = seq_chunk_ptr[seq_of_chunk(seq_chunk_ptr, num_seqs, i)];
    if (j < first) continue;
    scores[(static_cast<size_t>(h) * num_chunks + i) * num_chunks + j] = acc[r];
  }
}

}  // namespace

cudaError_t launch_chunk_similarity(const float* qc, const float* kc, int num_q_heads, int num_kv_heads,
                                    int num_chunks, int head_dim, const int* seq_chunk_ptr,
                                    int num_seqs, float* scores, cudaStream_t stream) {
  if (num_chunks <= 0) return cudaSuccess;
  const int tiles = (num_chunks + kTile - 1) / kTile;
  dim3 grid(tiles, tiles, num_q_heads);
  chunk_similarity_kernel<<<grid, 256, 0, stream>>>(qc, kc, num_chunks, head_dim,
                                                    num_q_heads / num_kv_heads, seq_chunk_ptr,
                                                    num_seqs, scores);
  return cudaGetLastError();
}

}  // namespace dhsa
