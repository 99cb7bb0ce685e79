// Step 4 of the DHSA path for bf16 inputs with head_dim 256: varlen
// block-sparse causal flash attention on tcgen05 tensor cores.
//
// out[t, h] = sum_s softmax_s(q[t,h] . k[s,g] * scale) v[s,g] over the kept
// key tokens s <= t: the tokens of the chunks in plan row (h, chunk(t))
// ("Long-Context Modeling with Dynamic Hierarchical Sparse Attention for
// On-Device LLMs", Abstract: only the token interactions selected through the
// upsampled chunk scores are preserved; "... for Memory-Constrained LLM
// Inference": causally important dependencies are kept).
//
// Work item = one CTA = (query chunk i, head h, 128-row tile of chunk i).  The
// kept chunks of row (h, i) are merged into runs of consecutive chunks, each
// run is cut into 128-key tiles, and the run holding the diagonal is clipped
// at the tile's last valid query row.
//
// With d = 256 the output accumulator O takes half of the 512 TMEM columns, so
// the design is built around TMEM:
//   S_0, S_1  columns [0, 128) and [128, 256): S = Q K^T, double-buffered, so
//             QK^T of tile j+1 runs on the tensor core while the softmax
//             turns S(j) into P(j);
//   P(j)      f16, two per column, written by the softmax over the first 64
//             columns of S(j%2): the A operand of O += P V straight from TMEM
//             (B: an f16 copy of V, made before the launch),
//             so PV is one M=128, N=256 (= d) MMA per 16 keys, the tensor
//             core's full-rate shape, with no P traffic through shared memory;
//   O         columns [256, 512).
// Shared memory: Q (64 KB, four 64-column slices), K as 16 KB slices (128
// keys x 64 columns) in a 6-slot ring, slice s of key tile t in slot
// (4t + s) % 6, and V as one 64 KB tile.
//
// Warp roles (192 threads):
//   warps 0-3  softmax + epilogue; thread r owns query row r (= TMEM lane r)
//   warp 4     TMA producer (no multicast): Q, then K(j+1) ahead of V(j)
//   warp 5     TMEM allocator; lane 0 issues every MMA, in the order
//              QK(0), QK(1), PV(0), QK(2), PV(1), ..., PV(nt-1)
// The tensor core executes one thread's tcgen05 operations in issue order, so
// QK(j+2), issued after PV(j), overwrites S(j%2) (and P(j) in it) only after
// PV(j) has read P(j).  The online softmax is fp32 in the exp2 domain; O is
// rescaled whenever a warp's running max grows, after PV(j-1) is complete
// (O-ready barrier) and before P(j) is released.
//
// The issuing thread runs in step with the tensor pipe, and each barrier test
// or commit it makes between MMAs leaves the pipe waiting, so the protocol
// keeps them to three waits (P-full, V-full, K-full) and two commits (O-ready,
// S-full) per key tile: the four slices of a K tile land on one barrier (one
// per tile parity), the producer takes the S-full commit of QK(t-1) as the
// release of the slots that K(t) overwrites (tiles t-2 and t-1), and the
// O-ready commit of PV(j-1) as the release of V.
#include "common.cuh"
#include "launchers.h"

namespace dhsa {
namespace {

constexpr int kD = 256;
constexpr int kBM = 128;
constexpr int kBN = 128;
constexpr int kThreads = 192;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr uint32_t kTmemCols = 512;
// O is rescaled whenever a warp's running max grows, so the largest weight
// of a row is exp2(0) = 1, exact (a lagging max would leave it rounded,
// and that rounding would reach O directly).
constexpr float kRescaleLog2 = 0.0f;
constexpr int kSlices = kD / 64;        // 64-column slices of a Q / K / V row
constexpr int kKSlots = 6;              // K ring: 16 KB slices
constexpr int kSliceBytes = kBN * 128;  // one 64-column slice of a 128-row tile
constexpr int kQBytes = kBM * kD * 2;
constexpr int kVBytes = kBN * kD * 2;
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kQBytes;
constexpr int kOffV = kOffK + kKSlots * kSliceBytes;
constexpr int kOffBar = kOffV + kVBytes;
constexpr int kSmemBytes = kOffBar + 256 + 1024;  // + barriers + 1 KB alignment slack
constexpr uint32_t kColS = 0;    // + 128 * buffer
constexpr uint32_t kColO = 256;
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
static_assert(2 * kBN + kD <= 512, "TMEM budget");

enum {
  kBarQ = 0,
  kBarKFull = 1,              // + (key tile & 1): all four slices of the tile landed
  kBarVFull = kBarKFull + 2,
  kBarSFull = kBarVFull + 1,  // + buffer
  kBarPFull = kBarSFull + 2,
  kBarOReady = kBarPFull + 1,
  kBarDrain = kBarOReady + 1,
  kNumBars = kBarDrain + 1
};
static_assert(8 * kNumBars + 8 <= 256, "barrier area");

// Key tiles of one work item: runs of consecutive kept chunks cut into
// kBN-token tiles, every run clipped at `cap` (one past the tile's last valid
// query row).  Plan entries outside [0, num_chunks) are clamped into it (so
// the chunk bounds are never read out of range) and counted in `bad`.
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
    if (k0 + kBN < re) {
      k0 += kBN;
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

__global__ void __launch_bounds__(kThreads, 1)
    attention_d256_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, __nv_bfloat16* __restrict__ out,
                          const int* __restrict__ bounds, const int* __restrict__ row_ptr,
                          const int* __restrict__ col, int nnz, int num_chunks, int num_q_heads, int group,
                          int plan_group, float scale_log2, uint32_t* status) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle atoms
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + kOffBar;
  auto bar = [&](int idx) { return bar0 + 8u * static_cast<uint32_t>(idx); };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kOffBar + 8 * kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffBar + 8 * kNumBars + 4);

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
    mbar_init(bar(kBarKFull + 0), 1);
    mbar_init(bar(kBarKFull + 1), 1);
    mbar_init(bar(kBarVFull), 1);
    mbar_init(bar(kBarSFull + 0), 1);
    mbar_init(bar(kBarSFull + 1), 1);
    mbar_init(bar(kBarPFull), 4);  // one arrival per softmax warp
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
    KeyTiles it;
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
      mbar_arrive_expect_tx(bar(kBarQ), kQBytes);
#pragma unroll
      for (int a = 0; a < kSlices; ++a)
        tma_load_3d(sbase + kOffQ + a * kSliceBytes, &tm_q, bar(kBarQ), a * 64, h, q0);
      // K(j+1) is loaded ahead of V(j), the order in which the MMAs use them
      KeyTiles kt, vt;
      kt.init(col, bounds, p0, p1, q_end, num_chunks);
      vt.init(col, bounds, p0, p1, q_end, num_chunks);
      int ktiles = 0, vtiles = 0, qk_seen = -1;
      bool ok = true;
      // QK(t) done: the S-full commit of its buffer (the MMAs of one thread
      // complete in issue order, so it also covers every earlier QK)
      auto wait_qk = [&](int t) -> bool {
        if (t <= qk_seen) return true;
        if (!mbar_wait(bar(kBarSFull + (t & 1)), (t >> 1) & 1, abort_flag, status)) return false;
        qk_seen = t;
        return true;
      };
      // K(t) as four 16 KB slices, slice u = 4t + s into slot u % kKSlots, all
      // behind one barrier per tile parity.  The slots' previous slices belong
      // to tiles t-2 and t-1, free once QK(t-1) is done; waiting for that
      // before arming means no tile is ever left partly issued.
      auto load_k = [&]() -> bool {
        int k0, ke;
        if (!kt.next(k0, ke)) return true;
        const int t = ktiles;
        if (t >= 1 && !wait_qk(t - 1)) return false;
        mbar_arrive_expect_tx(bar(kBarKFull + (t & 1)), kSlices * kSliceBytes);
#pragma unroll
        for (int s = 0; s < kSlices; ++s)
          tma_load_3d(sbase + kOffK + ((kSlices * t + s) % kKSlots) * kSliceBytes, &tm_k, bar(kBarKFull + (t & 1)),
                      s * 64, g, k0);
        ktiles = t + 1;
        return true;
      };
      ok = load_k();
      for (int j = 0; ok && j < ntiles; ++j) {
        ok = load_k();  // K(j+1)
        if (!ok) break;
        int k0, ke;
        vt.next(k0, ke);
        // V(j) replaces V(j-1) once PV(j-1) is done (its O-ready commit)
        if (j >= 1 && !mbar_wait(bar(kBarOReady), (j - 1) & 1, abort_flag, status)) break;
        mbar_arrive_expect_tx(bar(kBarVFull), kVBytes);
#pragma unroll
        for (int a = 0; a < kSlices; ++a)
          tma_load_3d(sbase + kOffV + a * kSliceBytes, &tm_v, bar(kBarVFull), a * 64, g, k0);
        vtiles = j + 1;
      }
      if (*abort_flag) {
        // let copies already in flight land before the CTA exits (bounded)
        volatile int never = 0;
        mbar_wait(bar(kBarQ), 0, &never, nullptr, 10000000ull);
        for (int t = max(0, ktiles - 2); t < ktiles; ++t)
          mbar_wait(bar(kBarKFull + (t & 1)), (t >> 1) & 1, &never, nullptr, 10000000ull);
        if (vtiles > 0) mbar_wait(bar(kBarVFull), (vtiles - 1) & 1, &never, nullptr, 10000000ull);
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0 && ntiles > 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(kBM, kBN, 0);
      constexpr uint32_t idesc_o = idesc_f16_f32(kBM, kD, 1);  // P and V in f16
      bool ok = mbar_wait(bar(kBarQ), 0, abort_flag, status);
      tc_fence_after();
      // S(j) = Q K(j)^T into buffer j % 2: one wait for the whole tile
      auto issue_s = [&](int j) -> bool {
        const uint32_t d = tmem + kColS + (j & 1) * kBN;
        if (!mbar_wait_spin(bar(kBarKFull + (j & 1)), (j >> 1) & 1, abort_flag, status)) return false;
        tc_fence_after();
#pragma unroll
        for (int s = 0; s < kSlices; ++s) {
          const uint32_t kbase = sbase + kOffK + ((kSlices * j + s) % kKSlots) * kSliceBytes;
          const uint32_t qbase = sbase + kOffQ + s * kSliceBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = smem_desc_sw128(qbase + kk * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(kbase + kk * 32, 16, 1024);
            umma_f16_ss(d, ad, bd, idesc_s, (s > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit(bar(kBarSFull + (j & 1)));  // also frees the tile's K slots
        return true;
      };
      if (ok) ok = issue_s(0);
      if (ok && ntiles > 1) ok = issue_s(1);
      for (int j = 0; ok && j < ntiles; ++j) {
        if (!mbar_wait_spin(bar(kBarPFull), j & 1, abort_flag, status)) break;
        if (!mbar_wait_spin(bar(kBarVFull), j & 1, abort_flag, status)) break;
        tc_fence_after();
        const uint32_t pa = tmem + kColS + (j & 1) * kBN;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint64_t bd = smem_desc_sw128(sbase + kOffV + kk * 16 * 128, kSliceBytes, 1024);
          umma_f16_ts(tmem + kColO, pa + kk * 8, bd, idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(bar(kBarOReady));  // also frees V
        if (j + 2 < ntiles && !issue_s(j + 2)) break;
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
    KeyTiles it;
    it.init(col, bounds, p0, p1, q_end, num_chunks);
    int k0, ke;
    bool ok = true;
    for (int j = 0; it.next(k0, ke); ++j) {
      if (!mbar_wait(bar(kBarSFull + (j & 1)), (j >> 1) & 1, abort_flag, status)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tS = tmem + lane_base + kColS + (j & 1) * kBN;
      float s[kBN];
      float mp[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      const bool masked = (k0 + kBN > ke) || (k0 + kBN - 1 > q0);
      const int lim = min(ke - k0, t_row - k0 + 1);  // valid columns: c < lim
      auto take_half = [&](int base, uint32_t (&ra)[32], uint32_t (&rb)[32]) {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          s[base + e] = __uint_as_float(ra[e]);
          s[base + 32 + e] = __uint_as_float(rb[e]);
        }
        if (masked) {
#pragma unroll
          for (int blk = base; blk < base + kBN / 2; blk += 32) {
            if (lim < blk + 32) {
#pragma unroll
              for (int c = blk; c < blk + 32; ++c)
                if (c >= lim) s[c] = -INFINITY;
            }
          }
        }
#pragma unroll
        for (int c = base; c < base + kBN / 2; c += 8) {
#pragma unroll
          for (int q = 0; q < 4; ++q) mp[q] = fmax3(mp[q], s[c + q], s[c + 4 + q]);
        }
      };
      {
        uint32_t ra[32], rb[32], rc[32], rd[32];
        tmem_ld32(tS + 0, ra);
        tmem_ld32(tS + 32, rb);
        tmem_wait_ld();
        reg_dep32(ra);
        reg_dep32(rb);
        tmem_ld32(tS + 64, rc);
        tmem_ld32(tS + 96, rd);
        take_half(0, ra, rb);
        tmem_wait_ld();
        reg_dep32(rc);
        reg_dep32(rd);
        take_half(kBN / 2, rc, rd);
      }
      const float m_tile = fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])) * scale_log2;
      const bool any = __any_sync(0xffffffffu, m_tile > m_run + kRescaleLog2);
      float alpha = 1.f;
      if (any) {
        const float m_new = fmaxf(m_run, m_tile);
        alpha = (m_new == -INFINITY) ? 1.f : ex2_approx(m_run - m_new);
        m_run = m_new;
      }
      const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
      uint64_t ps2[2] = {0ull, 0ull};  // packed (lo, hi) partial sums
      const uint64_t scale2 = f2_pack(scale_log2, scale_log2);
      const uint64_t shift2 = f2_pack(-m_use, -m_use);
      uint32_t pk[kBN / 2];
#pragma unroll
      for (int c = 0; c < kBN; c += 2) {
        float x0, x1;
        f2_unpack(f2_fma(f2_pack(s[c], s[c + 1]), scale2, shift2), x0, x1);
        const float e0 = ex2_approx(x0);
        const float e1 = ex2_approx(x1);
        pk[c / 2] = pack_f16(e0, e1);
        ps2[(c / 2) & 1] = f2_add(ps2[(c / 2) & 1], f2_pack(e0, e1));
      }
      // P(j) over the first 64 columns of S(j % 2) (its S values are in registers)
      tmem_st32p(tS + 0, pk);
      tmem_st32p(tS + 32, pk + 32);
      {
        float a0, a1, b0, b1;
        f2_unpack(ps2[0], a0, a1);
        f2_unpack(ps2[1], b0, b1);
        l_run = l_run * alpha + ((a0 + a1) + (b0 + b1));
      }
      // P(j) is released only once PV(j-1) is done.  With S double-buffered
      // a warp can read S(j+1) before a slower warp has released P(j); waiting
      // here keeps every warp's release of P(j+1) behind the completion of
      // the P-full phase of tile j (PV(j-1) finishes long before P(j) is
      // ready in the steady state, so the wait costs nothing there).  O is
      // rescaled in the same window: after PV(j-1), before PV(j).
      if (j > 0) {
        if (!mbar_wait(bar(kBarOReady), (j - 1) & 1, abort_flag, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
      if (any && j > 0) {
        const uint64_t alpha2 = f2_pack(alpha, alpha);
        const uint32_t tO = tmem + lane_base + kColO;
#pragma unroll 1
        for (int c = 0; c < kD / 32; c += 2) {
          uint32_t o0[32], o1[32];
          tmem_ld32(tO + 32 * c, o0);
          tmem_ld32(tO + 32 * (c + 1), o1);
          tmem_wait_ld();
          reg_dep32(o0);
          reg_dep32(o1);
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            float x0, x1;
            f2_unpack(f2_mul(f2_pack(__uint_as_float(o0[e]), __uint_as_float(o0[e + 1])), alpha2), x0, x1);
            o0[e] = __float_as_uint(x0);
            o0[e + 1] = __float_as_uint(x1);
            f2_unpack(f2_mul(f2_pack(__uint_as_float(o1[e]), __uint_as_float(o1[e + 1])), alpha2), x0, x1);
            o1[e] = __float_as_uint(x0);
            o1[e + 1] = __float_as_uint(x1);
          }
          tmem_st32(tO + 32 * c, o0);
          tmem_st32(tO + 32 * (c + 1), o1);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kBarPFull));
    }
    if (ok && ntiles > 0 && mbar_wait(bar(kBarOReady), (ntiles - 1) & 1, abort_flag, status)) {
      tc_fence_after();
      const float inv_l = 1.f / l_run;
      const bool valid = t_row < q_end;
      __nv_bfloat16* orow = out + (static_cast<size_t>(t_row) * num_q_heads + h) * kD;
#pragma unroll 1
      for (int c = 0; c < kD / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_base + kColO + 32 * c, o);
        tmem_wait_ld();
        reg_dep32(o);
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

cudaError_t launch_attention_d256(const AttnBf16Args& a, cudaStream_t stream) {
  if (a.head_dim != kD) return cudaErrorInvalidValue;
  CUtensorMap mq, mk, mv;
  if (encode_qkv_map(&mq, a.q, a.num_q_heads, kD, a.total_tokens, kBM) != CUDA_SUCCESS ||
      encode_qkv_map(&mk, a.k, a.num_kv_heads, kD, a.total_tokens, kBN) != CUDA_SUCCESS ||
      encode_qkv_map(&mv, a.v16, a.num_kv_heads, kD, a.total_tokens, kBN, true) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  cudaError_t e =
      cudaFuncSetAttribute(attention_d256_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  const int mtiles = (a.max_chunk_len + kBM - 1) / kBM;
  dim3 grid(mtiles, a.num_q_heads, a.num_chunks);
  const float scale_log2 = a.scale * 1.4426950408889634f;
  attention_d256_kernel<<<grid, kThreads, kSmemBytes, stream>>>(
      mq, mk, mv, static_cast<__nv_bfloat16*>(a.out), a.bounds, a.row_ptr, a.col, a.nnz, a.num_chunks,
      a.num_q_heads, a.num_q_heads / a.num_kv_heads, a.plan_group, scale_log2, a.status);
  return cudaGetLastError();
}

}  // namespace dhsa
