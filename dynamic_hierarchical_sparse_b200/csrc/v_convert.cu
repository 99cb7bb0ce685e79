// The f16 copy of V that the bf16 attention kernels read as the B operand of
// O += P V, with P in f16 (tcgen05.mma kind::f16 takes A and B of one type).
// bf16 -> f16 is exact for magnitudes up to 65504 (f16 has the more
// significant bits; below 2^-14 it goes subnormal, an absolute error of at
// most 2^-25).  Larger magnitudes and NaN are reported (kDevCheck): a larger
// magnitude is written saturated to +-65504, a NaN as a NaN.
//
// HBM-bound: 2 bytes read and 2 written per element, 16-byte vectors,
// grid-stride over a grid of whole waves.
#include "common.cuh"
#include "launchers.h"

namespace dhsa {
namespace {

constexpr int kConvThreads = 256;

__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w, bool& bad) {
  const float lo = __uint_as_float(w << 16), hi = __uint_as_float(w & 0xffff0000u);
  bad |= !(fabsf(lo) <= 65504.f) || !(fabsf(hi) <= 65504.f);
  uint32_t r;
  asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));  // first operand -> upper half
  return r;
}

__global__ void __launch_bounds__(kConvThreads)
    v_to_f16_kernel(const uint4* __restrict__ v, uint4* __restrict__ v16, long long nvec, uint32_t* status) {
  // kUnroll independent 16-byte loads in flight per thread before any store
  constexpr int kUnroll = 4;
  bool bad = false;
  const long long stride = static_cast<long long>(gridDim.x) * kConvThreads;
  for (long long i0 = blockIdx.x * static_cast<long long>(kConvThreads) + threadIdx.x; i0 < nvec;
       i0 += kUnroll * stride) {
    uint4 x[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const long long i = i0 + u * stride;
      x[u] = i < nvec ? __ldcs(v + i) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const long long i = i0 + u * stride;
      if (i >= nvec) break;
      uint4 y;
      y.x = bf16x2_to_f16x2(x[u].x, bad);
      y.y = bf16x2_to_f16x2(x[u].y, bad);
      y.z = bf16x2_to_f16x2(x[u].z, bad);
      y.w = bf16x2_to_f16x2(x[u].w, bad);
      v16[i] = y;
    }
  }
  if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) report(status, kDevCheck);
}

}  // namespace

cudaError_t launch_v_to_f16(const void* v, void* v16, long long n, uint32_t* status, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const long long nvec = n / 8;
  const long long need = (nvec + 4LL * kConvThreads - 1) / (4LL * kConvThreads);  // four vectors per thread
  const int grid = static_cast<int>(need < 8LL * sms ? need : 8LL * sms);
  v_to_f16_kernel<<<grid, kConvThreads, 0, stream>>>(static_cast<const uint4*>(v), static_cast<uint4*>(v16), nvec,
                                                     status);
  return cudaGetLastError();
}

}  // namespace dhsa
