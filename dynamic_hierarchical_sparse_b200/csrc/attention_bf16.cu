// Step 4 of the DHSA path for bf16 inputs: varlen block-sparse causal flash
// attention on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// out[t, h] = sum_s softmax_s(q[t,h] . k[s,g] * scale) v[s,g] over the kept
// key tokens s <= t, i.e. the tokens of the chunks in plan row (h, chunk(t))
// ("Long-Context Modeling with Dynamic Hierarchical Sparse Attention for
// On-Device LLMs", Abstract: only the token-level interactions selected by the
// upsampled chunk scores are preserved; "... for Memory-Constrained LLM
// Inference": causally important dependencies are kept).
//
// Work item = one CTA = (query chunk i, head h, 128-row tile of chunk i).  The
// kept key chunks of row (h, i) are merged into runs of consecutive chunks;
// each run is cut into BN-key tiles starting at the run's first token, and the
// run that ends at the diagonal chunk is clipped at the tile's last query row.
// Keys past a run's end and keys above the causal diagonal are masked.
//
// Warp roles (192 threads):
//   warps 0-3  softmax + epilogue; thread r owns query row r (= TMEM lane r)
//   warp 4     TMA producer: Q once, then K/V tiles into a 2-stage ring
//   warp 5     TMEM allocator and the single MMA-issuing thread
// TMEM (512 columns): S double buffer at [0, BN) and [BN, 2BN), O at [2BN, 2BN+D).
// S_j = Q K_j^T runs two tiles ahead of the softmax; P_j (bf16) goes to shared
// memory in the 128-byte-swizzled K-major layout and O += P_j V_j reads it
// there, with V as an N-major (d-contiguous) operand.  The online softmax is
// fp32 in the exp2 domain with lazy rescaling: O in TMEM is rescaled only when
// a warp's running maximum grows by more than 2^8.
#include "common.cuh"
#include "launchers.h"

namespace dhsa {
namespace {

constexpr int kBM = 128;
constexpr int kThreads = 192;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;

template <int D, int BN>
struct Cfg {
  static constexpr int kQSub = kBM * 128;     // bytes of one 64-column slice of Q
  static constexpr int kKVSub = BN * 128;     // bytes of one 64-column slice of a K/V tile
  static constexpr int kPSub = kBM * 128;     // bytes of one 64-key slice of P
  static constexpr int kQBytes = kBM * D * 2;
  static constexpr int kKVBytes = BN * D * 2;
  static constexpr int kPBytes = kBM * BN * 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + 2 * kKVBytes;
  static constexpr int kOffP = kOffV + 2 * kKVBytes;
  static constexpr int kOffBar = kOffP + kPBytes;
  static constexpr int kSmemBytes = kOffBar + 256 + 1024;  // + barriers + 1 KB alignment slack
  static constexpr uint32_t kColS0 = 0;
  static constexpr uint32_t kColO = 2 * BN;
  static_assert(2 * BN + D <= 512, "TMEM budget");
  static_assert(D % 64 == 0 && BN % 64 == 0, "tile shape");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

// barrier slots (8 bytes each) after kOffBar
enum {
  kBarQ = 0,
  kBarKFull = 1,   // +stage
  kBarKEmpty = 3,  // +stage
  kBarVFull = 5,
  kBarVEmpty = 7,
  kBarSFull = 9,   // +buffer
  kBarSFree = 11,  // +buffer
  kBarPFull = 13,
  kBarOReady = 14,
  kBarDrain = 15,
  kNumBars = 16
};

// Walks the key tiles of one work item: runs of consecutive kept chunks, cut
// into BN-token tiles; every run is clipped at `cap` (one past the tile's last
// valid query row), which only ever shortens the run holding the diagonal.
// Plan entries outside [0, num_chunks) are clamped into it (so the bounds are
// never read out of range) and counted in `bad`, which the caller reports.
template <int BN>
struct KeyTiles {
  const int* col;
  const int* bounds;
  int p, pend, re, k0, cap, nch, bad;
  __device__ void init(const int* col_, const int* bounds_, int p0, int p1, int cap_, int num_chunks) {
    col = col_;
    bounds = bounds_;
    p = p0;
    pend = p1;
    re = 0;
    k0 = 0;
    cap = cap_;
    nch = num_chunks;
    bad = 0;
  }
  __device__ int chunk(int q) {
    const int c = col[q];
    if (static_cast<unsigned>(c) >= static_cast<unsigned>(nch)) {
      ++bad;
      return min(max(c, 0), nch - 1);
    }
    return c;
  }
  __device__ bool next(int& tile_k0, int& tile_end) {
    if (k0 + BN < re) {
      k0 += BN;
    } else {
      if (p >= pend) return false;
      int c = chunk(p++);
      const int rs = bounds[c];
      int e = bounds[c + 1];
      while (p < pend && chunk(p) == c + 1) {
        c = chunk(p++);
        e = bounds[c + 1];
      }
      re = min(e, cap);
      k0 = rs;
    }
    tile_k0 = k0;
    tile_end = re;
    return true;
  }
};

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

template <int D, int BN>
__global__ void __launch_bounds__(kThreads, 1)
    attention_bf16_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, __nv_bfloat16* __restrict__ out,
                          const int* __restrict__ bounds, const int* __restrict__ row_ptr,
                          const int* __restrict__ col, int nnz, int num_chunks, int num_q_heads, int group,
                          int plan_group, float scale_log2, uint32_t* status) {
  using C = Cfg<D, BN>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle atoms
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::kOffBar;
  auto bar = [&](int idx) { return bar0 + 8u * static_cast<uint32_t>(idx); };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kOffBar + 8 * kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffBar + 8 * kNumBars + 4);

  const int mt = blockIdx.x;
  const int h = blockIdx.y;
  const int ci = num_chunks - 1 - static_cast<int>(blockIdx.z);  // longest rows first
  const int c_start = bounds[ci], c_end = bounds[ci + 1];
  const int q0 = c_start + mt * kBM;
  if (q0 >= c_end) return;  // uniform for the CTA: this chunk has fewer tiles
  const int q_end = min(q0 + kBM, c_end);
  const int g = h / group;
  const int r = (h / plan_group) * num_chunks + ci;
  int p0 = row_ptr[r], p1 = row_ptr[r + 1];
  const bool bad_row = p0 < 0 || p1 < p0 || p1 > nnz;
  if (bad_row) p0 = p1 = 0;  // a malformed plan row is reported below and walked as an empty row

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bar(kBarQ), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(kBarKFull + s), 1);
      mbar_init(bar(kBarKEmpty + s), 1);
      mbar_init(bar(kBarVFull + s), 1);
      mbar_init(bar(kBarVEmpty + s), 1);
      mbar_init(bar(kBarSFull + s), 1);
      mbar_init(bar(kBarSFree + s), kBM);
    }
    mbar_init(bar(kBarPFull), kBM);
    mbar_init(bar(kBarOReady), 1);
    mbar_init(bar(kBarDrain), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_holder), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  // number of key tiles (identical walk in every role)
  int ntiles = 0;
  {
    KeyTiles<BN> it;
    it.init(col, bounds, p0, p1, q_end, num_chunks);
    int a, b;
    while (it.next(a, b)) ++ntiles;
    if (threadIdx.x == 0 && (bad_row || it.bad)) report(status, kDevCheck);
  }

  if (warp == kProducerWarp) {
    if (lane == 0 && ntiles > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(bar(kBarQ), C::kQBytes);
#pragma unroll
      for (int a = 0; a < D / 64; ++a)
        tma_load_3d(sbase + C::kOffQ + a * C::kQSub, &tm_q, bar(kBarQ), a * 64, h, q0);
      KeyTiles<BN> it;
      it.init(col, bounds, p0, p1, q_end, num_chunks);
      int k0, ke;
      int issued = 0;
      for (int t = 0; it.next(k0, ke); ++t) {
        const int s = t & 1;
        const uint32_t par = ((t >> 1) & 1) ^ 1;
        if (!mbar_wait(bar(kBarKEmpty + s), par, abort_flag, status)) break;
        mbar_arrive_expect_tx(bar(kBarKFull + s), C::kKVBytes);
#pragma unroll
        for (int a = 0; a < D / 64; ++a)
          tma_load_3d(sbase + C::kOffK + s * C::kKVBytes + a * C::kKVSub, &tm_k, bar(kBarKFull + s), a * 64, g,
                      k0);
        ++issued;
        if (!mbar_wait(bar(kBarVEmpty + s), par, abort_flag, status)) break;
        mbar_arrive_expect_tx(bar(kBarVFull + s), C::kKVBytes);
#pragma unroll
        for (int a = 0; a < D / 64; ++a)
          tma_load_3d(sbase + C::kOffV + s * C::kKVBytes + a * C::kKVSub, &tm_v, bar(kBarVFull + s), a * 64, g,
                      k0);
      }
      if (*abort_flag) {
        // let copies already in flight land before the CTA exits (bounded)
        volatile int never = 0;
        mbar_wait(bar(kBarQ), 0, &never, nullptr, 10000000ull);
        for (int t = max(0, issued - 2); t < issued; ++t) {
          mbar_wait(bar(kBarKFull + (t & 1)), (t >> 1) & 1, &never, nullptr, 10000000ull);
          mbar_wait(bar(kBarVFull + (t & 1)), (t >> 1) & 1, &never, nullptr, 10000000ull);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0 && ntiles > 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(kBM, BN, 0);
      constexpr uint32_t idesc_o = idesc_bf16_f32(kBM, D, 1);
      bool ok = mbar_wait(bar(kBarQ), 0, abort_flag, status);
      tc_fence_after();
      auto issue_s = [&](int t) -> bool {
        const int s = t & 1;
        if (!mbar_wait(bar(kBarKFull + s), (t >> 1) & 1, abort_flag, status)) return false;
        tc_fence_after();
        const uint32_t kbase = sbase + C::kOffK + s * C::kKVBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t ad = smem_desc_sw128(sbase + C::kOffQ + (kk >> 2) * C::kQSub + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(kbase + (kk >> 2) * C::kKVSub + (kk & 3) * 32, 16, 1024);
          umma_f16_ss(tmem + C::kColS0 + (t & 1) * BN, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(bar(kBarSFull + (t & 1)));
        umma_commit(bar(kBarKEmpty + s));
        return true;
      };
      if (ok) ok = issue_s(0);
      if (ok && ntiles > 1) ok = issue_s(1);
      for (int j = 0; ok && j < ntiles; ++j) {
        if (!mbar_wait(bar(kBarPFull), j & 1, abort_flag, status)) break;
        const int s = j & 1;
        if (!mbar_wait(bar(kBarVFull + s), (j >> 1) & 1, abort_flag, status)) break;
        tc_fence_after();
        const uint32_t vbase = sbase + C::kOffV + s * C::kKVBytes;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint64_t ad = smem_desc_sw128(sbase + C::kOffP + (kk >> 2) * C::kPSub + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(vbase + kk * 16 * 128, C::kKVSub, 1024);
          umma_f16_ss(tmem + C::kColO, ad, bd, idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(bar(kBarOReady));
        umma_commit(bar(kBarVEmpty + s));
        if (j + 2 < ntiles) {
          if (!mbar_wait(bar(kBarSFree + (j & 1)), (j >> 1) & 1, abort_flag, status)) break;
          tc_fence_after();
          if (!issue_s(j + 2)) break;
        }
      }
      // every MMA issued above completes before TMEM is released
      umma_commit(bar(kBarDrain));
      volatile int never = 0;
      mbar_wait(bar(kBarDrain), 0, &never, nullptr);
    }
  } else {
    // ---------------------------------------------------- softmax warps 0-3
    const int row = threadIdx.x;  // 0..127
    const int t_row = q0 + row;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    float m_run = -INFINITY;  // running max of logits * scale * log2(e)
    float l_run = 0.f;
    KeyTiles<BN> it;
    it.init(col, bounds, p0, p1, q_end, num_chunks);
    int k0, ke;
    bool ok = true;
    for (int j = 0; it.next(k0, ke); ++j) {
      if (!mbar_wait(bar(kBarSFull + (j & 1)), (j >> 1) & 1, abort_flag, status)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[BN];
      {
        uint32_t raw[32];
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) {
          tmem_ld32(tmem + lane_base + C::kColS0 + (j & 1) * BN + 32 * c, raw);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) s[32 * c + e] = __uint_as_float(raw[e]);
        }
      }
      tc_fence_before();
      mbar_arrive(bar(kBarSFree + (j & 1)));

      const bool need_mask = (k0 + BN > ke) || (k0 + BN - 1 > q0);
      if (need_mask) {
        const int lim = min(ke - k0, t_row - k0 + 1);  // valid columns: c < lim
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (c >= lim) s[c] = -INFINITY;
      }
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < BN; ++c) mx = fmaxf(mx, s[c]);
      const float m_tile = mx * scale_log2;
      const bool need = m_tile > m_run + kRescaleLog2;
      const bool any = __any_sync(0xffffffffu, need);
      float alpha = 1.f;
      if (any) {
        const float m_new = fmaxf(m_run, m_tile);
        alpha = exp2f(m_run - m_new);
        m_run = m_new;
      }
      const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
      float psum = 0.f;
      uint32_t pk[BN / 2];
#pragma unroll
      for (int c = 0; c < BN; c += 2) {
        const float a0 = exp2f(fmaf(s[c], scale_log2, -m_use));
        const float a1 = exp2f(fmaf(s[c + 1], scale_log2, -m_use));
        psum += a0 + a1;
        pk[c / 2] = pack_bf16(a0, a1);
      }
      l_run = l_run * alpha + psum;

      if (j > 0) {
        // PV_{j-1} done: O is stable and the P buffer is free
        if (!mbar_wait(bar(kBarOReady), (j - 1) & 1, abort_flag, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (any) {
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            const uint32_t ta = tmem + lane_base + C::kColO + 32 * c;
            tmem_ld32(ta, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(ta, o);
          }
          tmem_wait_st();
        }
      }
      // P row -> shared memory, 128-byte-swizzled K-major layout
      unsigned char* prow = smem + C::kOffP + row * 128;
#pragma unroll
      for (int c8 = 0; c8 < BN / 8; ++c8) {
        const int sub = c8 >> 3, ch = c8 & 7;
        uint4 val = make_uint4(pk[4 * c8], pk[4 * c8 + 1], pk[4 * c8 + 2], pk[4 * c8 + 3]);
        *reinterpret_cast<uint4*>(prow + sub * C::kPSub + ((ch ^ (row & 7)) << 4)) = val;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(kBarPFull));
    }
    if (ok && ntiles > 0 && mbar_wait(bar(kBarOReady), (ntiles - 1) & 1, abort_flag, status)) {
      tc_fence_after();
      const float inv_l = 1.f / l_run;
      const bool valid = t_row < q_end;
      __nv_bfloat16* orow = out + (static_cast<size_t>(t_row) * num_q_heads + h) * D;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_base + C::kColO + 32 * c, o);
        tmem_wait_ld();
        if (valid) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 w;
            w.x = pack_bf16(__uint_as_float(o[e + 0]) * inv_l, __uint_as_float(o[e + 1]) * inv_l);
            w.y = pack_bf16(__uint_as_float(o[e + 2]) * inv_l, __uint_as_float(o[e + 3]) * inv_l);
            w.z = pack_bf16(__uint_as_float(o[e + 4]) * inv_l, __uint_as_float(o[e + 5]) * inv_l);
            w.w = pack_bf16(__uint_as_float(o[e + 6]) * inv_l, __uint_as_float(o[e + 7]) * inv_l);
            *reinterpret_cast<uint4*>(orow + 32 * c + e) = w;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

// 3-D (d, heads, tokens) view of a packed THD bf16 tensor with a (64, 1,
// box_rows) box and 128-byte swizzle: one box lands as box_rows x 128 bytes,
// the canonical K-major SW128 operand layout of tcgen05.mma.
CUresult encode_qkv_map(CUtensorMap* map, const void* base, int heads, int head_dim, int tokens, int box_rows) {
  using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
  static EncodeFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || p == nullptr)
      return CUDA_ERROR_NOT_FOUND;
    fn = reinterpret_cast<EncodeFn>(p);
  }
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(heads),
                              static_cast<cuuint64_t>(tokens)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(head_dim) * 2,
                                 static_cast<cuuint64_t>(heads) * head_dim * 2};
  const cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

namespace {

template <int D, int BN>
cudaError_t launch_dim(const AttnBf16Args& a, cudaStream_t stream) {
  using C = Cfg<D, BN>;
  CUtensorMap mq, mk, mv;
  if (encode_qkv_map(&mq, a.q, a.num_q_heads, D, a.total_tokens, kBM) != CUDA_SUCCESS ||
      encode_qkv_map(&mk, a.k, a.num_kv_heads, D, a.total_tokens, BN) != CUDA_SUCCESS ||
      encode_qkv_map(&mv, a.v, a.num_kv_heads, D, a.total_tokens, BN) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  auto kern = attention_bf16_kernel<D, BN>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  const int mtiles = (a.max_chunk_len + kBM - 1) / kBM;
  dim3 grid(mtiles, a.num_q_heads, a.num_chunks);
  const float scale_log2 = a.scale * 1.4426950408889634f;
  kern<<<grid, kThreads, C::kSmemBytes, stream>>>(mq, mk, mv, static_cast<__nv_bfloat16*>(a.out), a.bounds,
                                                  a.row_ptr, a.col, a.nnz, a.num_chunks, a.num_q_heads,
                                                  a.num_q_heads / a.num_kv_heads, a.plan_group, scale_log2,
                                                  a.status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention_bf16(const AttnBf16Args& a, cudaStream_t stream) {
  if (a.total_tokens <= 0 || a.num_chunks <= 0) return cudaSuccess;
  switch (a.head_dim) {
    case 64:
    case 128:
      return launch_attention_pair(a, stream);  // two query tiles per CTA (attention_bf16_pair.cu)
    case 256:
      return launch_dim<256, 64>(a, stream);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace dhsa
