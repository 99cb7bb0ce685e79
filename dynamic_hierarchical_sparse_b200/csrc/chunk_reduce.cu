// Step 1 of the DHSA path: length-normalised chunk aggregation.
//
// rep[h, c, :] = (sum_{t in chunk c} x[t, h, :]) / sqrt(L_c)   ("Long-Context
// Modeling with Dynamic Hierarchical Sparse Attention for On-Device LLMs",
// Abstract: a chunk is represented by the mean of its tokens' vectors,
// multiplied by sqrt(L_c) to normalise for its length).
//
// HBM-bound streaming reduction.  One CTA owns one chunk and one 16-byte-per-
// lane column slice of the token row (H*d elements): every warp reads whole
// 512-byte row segments with 128-bit loads (fully coalesced), each lane keeps
// fp32 partial sums of its 8 (bf16) or 4 (fp32) columns over a strided subset
// of the chunk's tokens, and the warps' partials are combined through shared
// memory in a fixed order, so the result is deterministic.
#include "common.cuh"
#include "launchers.h"

namespace dhsa {
namespace {

constexpr int kReduceWarps = 8;
constexpr int kUnroll = 4;

template <typename T>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int kN = 8;
  __device__ static void add(const uint4& u, float* acc) {
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(p[i]);
      acc[2 * i] += f.x;
      acc[2 * i + 1] += f.y;
    }
  }
};
template <>
struct Vec<float> {
  static constexpr int kN = 4;
  __device__ static void add(const uint4& u, float* acc) {
    acc[0] += __uint_as_float(u.x);
    acc[1] += __uint_as_float(u.y);
    acc[2] += __uint_as_float(u.z);
    acc[3] += __uint_as_float(u.w);
  }
};

// grid: x = column slices of q then k (slices_a + slices_b), y = chunk.
template <typename T>
__global__ void __launch_bounds__(kReduceWarps * 32)
    chunk_reduce_kernel(const T* __restrict__ xa, int width_a, int slices_a, float* __restrict__ out_a,
                        const T* __restrict__ xb, int width_b, float* __restrict__ out_b,
                        int head_dim, const int* __restrict__ bounds, int num_chunks) {
  constexpr int VN = Vec<T>::kN;
  constexpr int kCols = 32 * VN;  // columns of one slice
  __shared__ float part[kReduceWarps][kCols];

  const int c = blockIdx.y;
  int slice = blockIdx.x;
  const T* x = xa;
  int width = width_a;
  float* out = out_a;
  if (slice >= slices_a) {
    slice -= slices_a;
    x = xb;
    width = width_b;
    out = out_b;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = bounds[c], t1 = bounds[c + 1];
  const int col = slice * kCols + lane * VN;
  const bool active = col < width;  // width is a multiple of VN (d >= 64)

  float acc[VN];
#pragma unroll
  for (int i = 0; i < VN; ++i) acc[i] = 0.f;

  if (active) {
    const T* base = x + col;
    int t = t0 + warp;
    // kUnroll independent 16-byte loads in flight per lane
    for (; t + (kUnroll - 1) * kReduceWarps < t1; t += kUnroll * kReduceWarps) {
      uint4 u[kUnroll];
#pragma unroll
      for (int j = 0; j < kUnroll; ++j)
        u[j] = __ldcs(reinterpret_cast<const uint4*>(base + static_cast<size_t>(t + j * kReduceWarps) * width));
#pragma unroll
      for (int j = 0; j < kUnroll; ++j) Vec<T>::add(u[j], acc);
    }
    for (; t < t1; t += kReduceWarps) {
      uint4 u = __ldcs(reinterpret_cast<const uint4*>(base + static_cast<size_t>(t) * width));
      Vec<T>::add(u, acc);
    }
  }
#pragma unroll
  for (int i = 0; i < VN; ++i) part[warp][lane * VN + i] = acc[i];
  __syncthreads();

  const float inv_sqrt_len = 1.0f / sqrtf(static_cast<float>(t1 - t0));
  for (int k = threadIdx.x; k < kCols; k += blockDim.x) {
    const int cc = slice * kCols + k;
    if (cc >= width) continue;
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kReduceWarps; ++w) s += part[w][k];
    const int h = cc / head_dim, dd = cc - h * head_dim;
    out[(static_cast<size_t>(h) * num_chunks + c) * head_dim + dd] = s * inv_sqrt_len;
  }
}

template <typename T>
cudaError_t launch_typed(const void* xa, int ha, float* out_a, const void* xb, int hb, float* out_b,
                         int head_dim, const int* bounds, int num_chunks, cudaStream_t stream) {
  constexpr int kCols = 32 * Vec<T>::kN;
  const int wa = ha * head_dim, wb = hb * head_dim;
  const int sa = (wa + kCols - 1) / kCols;
  const int sb = xb ? (wb + kCols - 1) / kCols : 0;
  dim3 grid(sa + sb, num_chunks);
  chunk_reduce_kernel<T><<<grid, kReduceWarps * 32, 0, stream>>>(
      static_cast<const T*>(xa), wa, sa, out_a, static_cast<const T*>(xb), wb, out_b, head_dim,
      bounds, num_chunks);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_reduce(int dtype, const void* xa, int heads_a, float* out_a, const void* xb,
                                int heads_b, float* out_b, int head_dim, const int* bounds,
                                int num_chunks, cudaStream_t stream) {
  if (num_chunks <= 0) return cudaSuccess;
  if (dtype == 0)
    return launch_typed<__nv_bfloat16>(xa, heads_a, out_a, xb, heads_b, out_b, head_dim, bounds,
                                       num_chunks, stream);
  return launch_typed<float>(xa, heads_a, out_a, xb, heads_b, out_b, head_dim, bounds, num_chunks,
                             stream);
}

namespace {

// Per-KV-head planning scores a KV group by the sum of its query heads' chunk
// scores, which by linearity is the dot product of the summed query-chunk
// representations with the KV head's key-chunk representation.
__global__ void group_sum_kernel(const float* __restrict__ qc, int group, int num_kv_heads, int per_head,
                                 float* __restrict__ qg) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<int64_t>(num_kv_heads) * per_head) return;
  const int g = static_cast<int>(idx / per_head);
  const int e = static_cast<int>(idx - static_cast<int64_t>(g) * per_head);
  const float* src = qc + static_cast<int64_t>(g) * group * per_head + e;
  float s = 0.f;
  for (int r = 0; r < group; ++r) s += src[static_cast<int64_t>(r) * per_head];
  qg[idx] = s;
}

}  // namespace

cudaError_t launch_group_sum(const float* qc, int num_q_heads, int num_kv_heads, int num_chunks, int head_dim,
                             float* qg, cudaStream_t stream) {
  const int per_head = num_chunks * head_dim;
  const int64_t total = static_cast<int64_t>(num_kv_heads) * per_head;
  if (total <= 0) return cudaSuccess;
  const int threads = 256;
  group_sum_kernel<<<static_cast<unsigned>((total + threads - 1) / threads), threads, 0, stream>>>(
      qc, num_q_heads / num_kv_heads, num_kv_heads, per_head, qg);
  return cudaGetLastError();
}

}  // namespace dhsa
