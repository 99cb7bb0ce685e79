// Online variable-length chunking: proposes the chunk boundaries that the rest
// of the path takes as input.
//
// The pages ("Long-Context Modeling with Dynamic Hierarchical Sparse Attention
// for On-Device LLMs", Abstract and AI Summary) say that DHSA segments each
// sequence adaptively and online into variable-length chunks, and give no
// rule.  The rule built here is a plain left-to-right one, decided as tokens
// arrive: with the current chunk starting at token b, token t starts a new
// chunk when t - b >= max_len, or when t - b >= min_len and
//   sim(t) = (1 / Hkv) * sum_g cos(k[t-1, g], k[t, g])
// is below the threshold (strict; a zero key has cosine 1).
//
// Three launches:
//  1. adjacent_sim_kernel: sim(t) for every token, four consecutive tokens per
//     warp (each key row read once per warp, 16-byte vector loads, up to two
//     per lane and head, one squared norm per row), 32 tokens per CTA; one bit
//     per token ("drop": sim(t) < threshold) into a bitmap.  HBM-bound: every key row is read once from
//     DRAM (the row before a warp's first token, read by the neighbouring warp
//     too, hits in cache).
//  2. segment_walk_kernel: one CTA per sequence.  The rule: from chunk start
//     b, the next start is the first drop in [b + min_len, b + max_len), else
//     b + max_len.  The sequence's drop bits are brought into shared memory by
//     a bulk copy, a window of kWinWords words at a time.  Every drop of the
//     window is a possible chunk start, so the CTA lists them (ascending) and
//     takes, in parallel, the rule's step from each: the next drop that
//     becomes a start and the forced starts (x + max_len, x + 2 max_len, ...)
//     before it, found by binary search in the list.  The drops reached from
//     the window's first start are then found by pointer jumping (log2 of the
//     drop count rounds), and every thread sets the starts of the drops it
//     holds.  A window with more drops than the list holds is walked step by
//     step by one thread instead.  Chunk starts are set in a second bitmap.
//  3. segment_compact_kernel: one CTA turns the start bitmap into chunk_bounds
//     (a block-wide scan of per-thread bit counts), then seq_chunk_ptr by binary
//     search of each sequence's first token.  A batch of one sequence skips this
//     launch: its walk CTA, which holds every start, writes the bounds itself.
#include <cuda_bf16.h>

#include "common.cuh"
#include "launchers.h"

namespace dhsa {
namespace {

constexpr int kSimWarps = 8;             // warps per CTA; 32 tokens per CTA
constexpr int kWinWords = 4096;          // walk window: 131072 tokens (max_len <= 65536)
constexpr int kWalkThreads = 256;
constexpr int kStartBuf = 1024;          // chain entries the walking thread lists before the CTA writes them
constexpr int kNodeCap = 8192;           // drops per window the walk tabulates (more: step by step)
constexpr int kCompactThreads = 1024;

__device__ __forceinline__ void to_float(const uint4& v, float* f, const __nv_bfloat16*) {
  const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 x = __bfloat1622float2(p[i]);
    f[2 * i] = x.x;
    f[2 * i + 1] = x.y;
  }
}

__device__ __forceinline__ void to_float(const uint4& v, float* f, const float*) {
  f[0] = __uint_as_float(v.x);
  f[1] = __uint_as_float(v.y);
  f[2] = __uint_as_float(v.z);
  f[3] = __uint_as_float(v.w);
}

// One warp takes R consecutive tokens tb .. tb+R-1 and reads each of the rows
// tb-1 .. tb+R-1 once (all R+1 rows' loads are issued before any arithmetic):
// every row's squared norm is formed once and feeds the two cosines it takes
// part in.  A lane holds IT 16-byte vectors of one head (up to 2), so a head
// is covered by G = V / IT lanes (a reduction of log2(G) shuffle steps) and a
// pass over the heads takes P = 32 / G of them.
template <typename T, int D>
__global__ void __launch_bounds__(32 * kSimWarps)
    adjacent_sim_kernel(const T* __restrict__ k, int total_tokens, int hkv, float threshold,
                        uint32_t* __restrict__ drop, uint32_t* __restrict__ start_bits) {
  constexpr int E = 16 / static_cast<int>(sizeof(T));  // elements per 16-byte vector
  constexpr int V = D / E;                            // vectors per head
  constexpr int IT = V < 2 ? V : 2;                   // vectors per lane per head
  constexpr int G = V / IT;                           // lanes per head
  constexpr int P = 32 / G;                           // heads per pass
  constexpr int F = IT * E;                           // floats per lane per row
  constexpr int R = 32 / kSimWarps;                   // tokens per warp
  static_assert(G >= 1 && G <= 32 && (G & (G - 1)) == 0, "lanes per head");
  __shared__ uint32_t s_word;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * 32;
  const int tb = t0 + warp * R;
  if (threadIdx.x == 0) s_word = 0u;
  const uint4* kv = reinterpret_cast<const uint4*>(k);
  const size_t rowv = static_cast<size_t>(hkv) * V;  // vectors per token row
  const int sub = lane % G;
  float acc[R];
#pragma unroll
  for (int j = 0; j < R; ++j) acc[j] = 0.f;
  for (int g0 = 0; g0 < hkv; g0 += P) {
    const int g = g0 + lane / G;
    const bool on = g < hkv;
    uint4 raw[R + 1][IT];
#pragma unroll
    for (int r = 0; r <= R; ++r) {
      const int t = tb - 1 + r;
      const bool valid = on && t >= 0 && t < total_tokens;
#pragma unroll
      for (int it = 0; it < IT; ++it)
        raw[r][it] = valid ? __ldg(kv + static_cast<size_t>(t) * rowv + g * V + it * G + sub)
                           : make_uint4(0u, 0u, 0u, 0u);
    }
    float prev[F], cur[F];
#pragma unroll
    for (int it = 0; it < IT; ++it) to_float(raw[0][it], &prev[it * E], static_cast<const T*>(nullptr));
    float nprev = 0.f;
#pragma unroll
    for (int e = 0; e < F; ++e) nprev = fmaf(prev[e], prev[e], nprev);
#pragma unroll
    for (int o = G / 2; o >= 1; o >>= 1) nprev += __shfl_xor_sync(0xffffffffu, nprev, o);
#pragma unroll
    for (int j = 0; j < R; ++j) {
#pragma unroll
      for (int it = 0; it < IT; ++it) to_float(raw[j + 1][it], &cur[it * E], static_cast<const T*>(nullptr));
      float ncur = 0.f, dot = 0.f;
#pragma unroll
      for (int e = 0; e < F; ++e) {
        ncur = fmaf(cur[e], cur[e], ncur);
        dot = fmaf(prev[e], cur[e], dot);
      }
#pragma unroll
      for (int o = G / 2; o >= 1; o >>= 1) {
        ncur += __shfl_xor_sync(0xffffffffu, ncur, o);
        dot += __shfl_xor_sync(0xffffffffu, dot, o);
      }
      if (sub == 0 && on) acc[j] += (nprev > 0.f && ncur > 0.f) ? dot * rsqrtf(nprev) * rsqrtf(ncur) : 1.f;
#pragma unroll
      for (int e = 0; e < F; ++e) prev[e] = cur[e];
      nprev = ncur;
    }
  }
#pragma unroll
  for (int j = 0; j < R; ++j) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], o);
  }
  __syncthreads();  // s_word initialised
  if (lane == 0) {
    uint32_t bits = 0u;
#pragma unroll
    for (int j = 0; j < R; ++j) {
      const int t = tb + j;
      if (t >= 1 && t < total_tokens && acc[j] / static_cast<float>(hkv) < threshold) bits |= 1u << (warp * R + j);
    }
    if (bits) atomicOr(&s_word, bits);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    drop[blockIdx.x] = s_word;
    start_bits[blockIdx.x] = 0u;
  }
}

// Shared memory of the walk (dynamic: about 180 KB).
struct WalkSmem {
  uint32_t win[kWinWords];            // the window's drop bits
  int nd[kWinWords + 1];              // step-by-step walk only: first drop at or after word wb + i, else kNone
  int node_pos[kNodeCap];             // the window's drops, ascending
  int node_next[kNodeCap];            // walk from a chunk start at that drop: next drop start, or kEnd / kOut
  int node_k[kNodeCap];               // forced starts (x + max_len, x + 2 max_len, ...) before it
  int jump[kNodeCap];                 // pointer jumping: the node 2^r starts further on
  unsigned char on_chain[kNodeCap];   // reached from the window's first start
  int e_pos[kStartBuf];               // step-by-step walk: the starts it found this round
  int warp_cnt[kWalkThreads / 32];
  int carry[kWalkThreads / 32];
};

constexpr int kNone = 0x7fffffff;
constexpr int kEnd = -1;  // the walk reaches the end of the sequence
constexpr int kOut = -2;  // the walk needs bits past the window
constexpr int kNodesPerThread = kNodeCap / kWalkThreads;

// first drop at or after x among the window's drops (ascending node_pos[0, nodes)):
// its index, or nodes when there is none
__device__ __forceinline__ int first_node_at_or_after(const WalkSmem& S, int nodes, long long x) {
  int lo = 0, hi = nodes;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (S.node_pos[mid] < x) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// The walk's rule from a chunk start x, within the window: the next start is
// the first drop in [x + min_len, x + max_len), else x + max_len (a forced
// start) while that is inside the sequence.  Runs of forced starts are taken
// in closed form: with no drop before f, every start x + k max_len below f is
// forced.  Returns the index of the first drop that becomes a start (>= 0),
// kEnd or kOut; *forced counts the forced starts on the way and *last is the
// last start reached (x itself, or its last forced start).
__device__ int walk_from(const WalkSmem& S, int nodes, int x, int wb, int n, bool full, int s1, int min_len,
                         int max_len, int* forced, int* last) {
  int k_forced = 0;
  int result;
  while (true) {
    const long long clo = static_cast<long long>(x) + min_len;
    if (clo >= s1) { result = kEnd; break; }
    const long long xm = static_cast<long long>(x) + max_len;
    const int chi = static_cast<int>(xm < s1 ? xm : s1);
    if (((chi - 1) >> 5) >= wb + n) { result = kOut; break; }
    // first drop at or after clo (none needed when min_len == max_len: the
    // rule's interval is empty, and every start is forced)
    int idx = nodes, f = kNone;
    if (clo < chi) {
      idx = first_node_at_or_after(S, nodes, clo);
      if (idx < nodes) f = S.node_pos[idx];
    }
    if (f < chi) { result = idx; break; }
    if (xm >= s1) { result = kEnd; break; }
    if (f == kNone) {
      if (full) {  // no drop up to the end: forced starts while below s1
        const int k = static_cast<int>((static_cast<long long>(s1) - 1 - x) / max_len);
        k_forced += k;
        x += k * max_len;
        result = kEnd;
        break;
      }
      // no drop in the rest of the window: forced starts while their rule
      // window stays inside it (at least the one forced start x + max_len,
      // which is certain: no drop in [x + min_len, x + max_len) and
      // x + max_len < s1; so every call that leaves the window has moved the
      // walk on), then the walk needs the next window
      const long long room = (static_cast<long long>(wb + n) << 5) - x;
      const int k = max(1, static_cast<int>(room / max_len) - 1);
      x += k * max_len;
      k_forced += k;
      continue;
    }
    // f >= x + max_len: the starts x + max_len, ..., x + k max_len <= f are forced
    const int k = (f - x) / max_len;
    x += k * max_len;
    k_forced += k;
  }
  *forced = k_forced;
  *last = x;
  return result;
}

__device__ __forceinline__ void set_start(uint32_t* start_bits, int p) {
  atomicOr(start_bits + (p >> 5), 1u << (p & 31));
}

__global__ void __launch_bounds__(kWalkThreads)
    segment_walk_kernel(const uint32_t* __restrict__ drop, const int* __restrict__ cu_seqlens, int min_len,
                        int max_len, uint32_t* __restrict__ start_bits, uint32_t* status, int compact,
                        int* __restrict__ chunk_bounds, long long capacity, int* __restrict__ seq_chunk_ptr,
                        int* __restrict__ num_chunks) {
  extern __shared__ __align__(128) unsigned char walk_smem_raw[];
  WalkSmem& S = *reinterpret_cast<WalkSmem*>(walk_smem_raw);
  __shared__ __align__(8) uint64_t bar;
  __shared__ int s_abort, s_b, s_done, s_ne, s_nodes, s_first, s_forced;
  const int seq = blockIdx.x;
  const int s0 = cu_seqlens[seq], s1 = cu_seqlens[seq + 1];
  if (s1 <= s0) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int last_word = (s1 - 1) >> 5;
  const uint32_t mbar = smem_u32(&bar);
  if (tid == 0) {
    s_abort = 0;
    mbar_init(mbar, 1);
    fence_mbar_init();
    set_start(start_bits, s0);
  }
  __syncthreads();
  int b = s0;
  int wb = -1;  // first word held in the window (a multiple of 4: 16-byte copies)
  int n = 0;
  bool full = false;
  uint32_t phase = 0;
  constexpr int kWarpWords = kWinWords / (kWalkThreads / 32);  // words of the window per warp
  while (true) {
    const int lo = b + min_len;
    if (lo >= s1) break;
    const int hi = min(b + max_len, s1);
    if (wb < 0 || ((hi - 1) >> 5) >= wb + kWinWords) {
      // [lo, hi) spans at most (max_len + 29) / 32 + 1 words and wb is at most
      // 3 words below lo's word, so the new window holds it
      wb = (lo >> 5) & ~3;
      n = min(kWinWords, last_word + 1 - wb);
      full = wb + n > last_word;
      const uint32_t bytes = static_cast<uint32_t>((n + 3) & ~3) * 4u;  // inside the 256-byte-aligned bitmap
      __syncthreads();  // every thread is done with the old window
      if (tid == 0) {
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(mbar, bytes);
        bulk_load_1d(smem_u32(S.win), drop + wb, bytes, mbar);
      }
      const bool ok = mbar_wait(mbar, phase, &s_abort, status);
      phase ^= 1u;
      if (__syncthreads_or(!ok)) return;  // recorded in the status word
      // drops per warp: warp w holds words [w * kWarpWords, (w + 1) * kWarpWords),
      // its lanes consecutive words (no bank conflicts)
      const int w0 = warp * kWarpWords;
      int cnt = 0;
      for (int c = 0; c < kWarpWords; c += 32) {
        const int i = w0 + c + lane;
        if (i < n) cnt += __popc(S.win[i]);
      }
      cnt = __reduce_add_sync(0xffffffffu, cnt);
      if (lane == 0) S.warp_cnt[warp] = cnt;
      __syncthreads();
      int base = 0, nodes = 0;
      for (int w = 0; w < kWalkThreads / 32; ++w) {
        if (w < warp) base += S.warp_cnt[w];
        nodes += S.warp_cnt[w];
      }
      if (nodes <= kNodeCap) {
        // the window's drops in ascending order: a warp prefix per 32 words
        for (int c = 0; c < kWarpWords; c += 32) {
          const int i = w0 + c + lane;
          uint32_t m = i < n ? S.win[i] : 0u;
          if (!__any_sync(0xffffffffu, m != 0u)) continue;  // no drop in these 32 words
          const int pc = __popc(m);
          int incl = pc;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += u;
          }
          int r = base + incl - pc;
          while (m != 0u) {
            S.node_pos[r++] = ((wb + i) << 5) + __ffs(m) - 1;
            m &= m - 1u;
          }
          base += __shfl_sync(0xffffffffu, incl, 31);
        }
        __syncthreads();
        // the walk's step from a start at each drop
        for (int j = tid; j < nodes; j += kWalkThreads) {
          int forced, last;
          S.node_next[j] = walk_from(S, nodes, S.node_pos[j], wb, n, full, s1, min_len, max_len, &forced, &last);
          S.node_k[j] = forced;
        }
      } else {
        // too many drops to tabulate: nd = suffix minimum of each word's first
        // drop, for the step-by-step walk (within each thread's run of words,
        // then across threads)
        constexpr int kPer = kWinWords / kWalkThreads;
        const int i0 = tid * kPer, i1 = min(n, i0 + kPer);
        int run = kNone;
        for (int i = i1 - 1; i >= i0; --i) {
          const uint32_t m = S.win[i];
          if (m != 0u) run = ((wb + i) << 5) + __ffs(m) - 1;
          S.nd[i] = run;
        }
        int suf = run;  // suffix minimum over threads tid .. (inclusive) in this warp
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_down_sync(0xffffffffu, suf, o);
          if (lane + o < 32) suf = min(suf, v);
        }
        if (lane == 0) S.carry[warp] = suf;
        __syncthreads();
        int carry = __shfl_down_sync(0xffffffffu, suf, 1);
        if (lane == 31) carry = kNone;
        for (int w = warp + 1; w < kWalkThreads / 32; ++w) carry = min(carry, S.carry[w]);
        for (int i = i0; i < i1; ++i)
          if (S.nd[i] == kNone) S.nd[i] = carry;
        if (tid == 0) S.nd[n] = kNone;
      }
      if (tid == 0) s_nodes = nodes;
      __syncthreads();
    }
    const int nodes = s_nodes;
    if (nodes <= kNodeCap) {
      // the chain from b: its first drop start (thread 0), then every drop
      // start reached from it, found by pointer jumping (round r marks the
      // nodes 2^r .. 2^(r+1) - 1 steps on), all in parallel
      if (tid == 0) {
        int forced, last;
        const int f = walk_from(S, nodes, b, wb, n, full, s1, min_len, max_len, &forced, &last);
        s_first = f;
        s_forced = forced;
        s_b = last;
        s_done = f == kEnd;
      }
      __syncthreads();
      const int first = s_first;
      for (int k = 1 + tid; k <= s_forced; k += kWalkThreads) set_start(start_bits, b + k * max_len);
      if (first >= 0) {
        for (int j = tid; j < nodes; j += kWalkThreads) {
          S.on_chain[j] = j == first;
          S.jump[j] = S.node_next[j];
        }
        __syncthreads();
        for (int span = 1; span <= nodes; span <<= 1) {
          int nxt[kNodesPerThread];
#pragma unroll
          for (int q = 0; q < kNodesPerThread; ++q) {
            if (q * kWalkThreads >= nodes) break;  // the same for every thread
            const int j = tid + q * kWalkThreads;
            nxt[q] = kEnd;
            if (j < nodes) {
              const int t = S.jump[j];
              if (t >= 0) {
                if (S.on_chain[j]) S.on_chain[t] = 1;  // every node written here is on the chain
                nxt[q] = S.jump[t];
              } else {
                nxt[q] = t;
              }
            }
          }
          __syncthreads();
#pragma unroll
          for (int q = 0; q < kNodesPerThread; ++q) {
            if (q * kWalkThreads >= nodes) break;
            const int j = tid + q * kWalkThreads;
            if (j < nodes) S.jump[j] = nxt[q];
          }
          __syncthreads();
        }
        // the starts: every node on the chain and its forced starts; the one
        // whose step leaves the chain (end of sequence or of window) sets b
        for (int j = tid; j < nodes; j += kWalkThreads) {
          if (!S.on_chain[j]) continue;
          const int pos = S.node_pos[j], k = S.node_k[j];
          for (int q = 0; q <= k; ++q) set_start(start_bits, pos + q * max_len);
          const int nx = S.node_next[j];
          if (nx < 0) {
            s_b = pos + k * max_len;
            s_done = nx == kEnd;
          }
        }
      }
      __syncthreads();
      b = s_b;
      if (s_done) break;
      __syncthreads();  // s_b and s_done are rewritten by the next round
      continue;
    }
    // step by step, two shared-memory loads per chunk
    if (tid == 0) {
      int ne = 0, done = 0, cb = b;
      while (ne < kStartBuf) {
        const int clo = cb + min_len;
        if (clo >= s1) { done = 1; break; }
        const int chi = min(cb + max_len, s1);
        if (((chi - 1) >> 5) >= wb + n) break;  // the window must move first
        int f = kNone;  // first drop at or after clo (the interval is empty when min_len == max_len)
        if (clo < chi) {
          const int wl = clo >> 5;
          const uint32_t m = S.win[wl - wb] & (0xffffffffu << (clo & 31));
          f = m != 0u ? (wl << 5) + __ffs(m) - 1 : S.nd[wl - wb + 1];
        }
        int next;
        if (f < chi) {
          next = f;
        } else if (cb + max_len < s1) {
          next = cb + max_len;
        } else {
          done = 1;
          break;
        }
        S.e_pos[ne++] = next;
        cb = next;
      }
      s_b = cb;
      s_done = done;
      s_ne = ne;
    }
    __syncthreads();
    b = s_b;
    const int fin = s_done;
    for (int e = tid; e < s_ne; e += kWalkThreads) set_start(start_bits, S.e_pos[e]);
    __syncthreads();  // s_b, s_done and the start list are rewritten by the next round
    if (fin) break;
  }
  if (!compact) return;
  // A batch of one sequence: the start bitmap -> chunk_bounds here, without
  // the compaction launch (every start is set, and the block's atomics are
  // visible to it after the barrier).  An exclusive prefix of the threads'
  // start counts over runs of consecutive words.
  __syncthreads();
  const int nw = (s1 + 31) >> 5;
  const int per = (nw + kWalkThreads - 1) / kWalkThreads;
  const int w0 = min(nw, tid * per), w1 = min(nw, w0 + per);
  int cnt = 0;
  for (int w = w0; w < w1; ++w) cnt += __popc(start_bits[w]);
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) S.warp_cnt[warp] = incl;
  __syncthreads();
  long long pos = incl - cnt;
  int total = 0;
  for (int w = 0; w < kWalkThreads / 32; ++w) {
    if (w < warp) pos += S.warp_cnt[w];
    total += S.warp_cnt[w];
  }
  for (int w = w0; w < w1; ++w) {
    uint32_t bits = start_bits[w];
    while (bits) {
      const int bit = __ffs(bits) - 1;
      bits &= bits - 1u;
      if (pos < capacity) chunk_bounds[pos] = (w << 5) + bit;
      ++pos;
    }
  }
  if (tid == 0) {
    if (total > capacity) report(status, kDevCheck);
    const int n = static_cast<int>(min(static_cast<long long>(total), capacity));
    chunk_bounds[n] = s1;
    *num_chunks = total;
    seq_chunk_ptr[0] = 0;
    seq_chunk_ptr[1] = n;
  }
}

__global__ void __launch_bounds__(kCompactThreads)
    segment_compact_kernel(const uint32_t* __restrict__ start_bits, int total_tokens,
                           const int* __restrict__ cu_seqlens, int num_seqs, int* __restrict__ chunk_bounds,
                           long long capacity, int* __restrict__ seq_chunk_ptr, int* __restrict__ num_chunks,
                           uint32_t* status) {
  __shared__ int s_warp[kCompactThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nw = (total_tokens + 31) >> 5;
  const int per = (nw + kCompactThreads - 1) / kCompactThreads;
  const int w0 = min(nw, tid * per), w1 = min(nw, w0 + per);
  int cnt = 0;
  for (int w = w0; w < w1; ++w) cnt += __popc(start_bits[w]);
  // block-wide exclusive scan of cnt
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int x = s_warp[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += v;
    }
    s_warp[lane] = x;  // inclusive over warps
  }
  __syncthreads();
  const int total = s_warp[kCompactThreads / 32 - 1];
  long long pos = incl - cnt + (warp > 0 ? s_warp[warp - 1] : 0);
  for (int w = w0; w < w1; ++w) {
    uint32_t bits = start_bits[w];
    while (bits) {
      const int b = __ffs(bits) - 1;
      bits &= bits - 1u;
      if (pos < capacity) chunk_bounds[pos] = (w << 5) + b;
      ++pos;
    }
  }
  if (tid == 0) {
    if (total > capacity) report(status, kDevCheck);
    chunk_bounds[min(static_cast<long long>(total), capacity)] = total_tokens;
    *num_chunks = total;
  }
  __syncthreads();  // chunk_bounds visible to the whole block
  const int n = static_cast<int>(min(static_cast<long long>(total), capacity));
  for (int s = tid; s <= num_seqs; s += kCompactThreads) {
    if (s == num_seqs) {
      seq_chunk_ptr[s] = n;
      continue;
    }
    const int x = cu_seqlens[s];
    int lo = 0, hi = n;  // first chunk whose start is >= x
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (chunk_bounds[mid] < x) lo = mid + 1;
      else hi = mid;
    }
    seq_chunk_ptr[s] = lo;
  }
}

template <typename T, int D>
cudaError_t launch_sim(const void* k, int total_tokens, int hkv, float threshold, uint32_t* drop,
                       uint32_t* start_bits, cudaStream_t stream) {
  const int words = (total_tokens + 31) / 32;
  adjacent_sim_kernel<T, D><<<words, 32 * kSimWarps, 0, stream>>>(static_cast<const T*>(k), total_tokens, hkv,
                                                                  threshold, drop, start_bits);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_segment(const void* k, int dtype, int total_tokens, int num_kv_heads, int head_dim,
                           const int* cu_seqlens, int num_seqs, float threshold, int min_len, int max_len,
                           int* chunk_bounds, long long capacity, int* seq_chunk_ptr, int* num_chunks,
                           uint32_t* drop, uint32_t* start_bits, uint32_t* status, cudaStream_t stream) {
  cudaError_t e = cudaSuccess;
  if (total_tokens > 0) {
    if (dtype == 0) {
      if (head_dim == 64) e = launch_sim<__nv_bfloat16, 64>(k, total_tokens, num_kv_heads, threshold, drop, start_bits, stream);
      else if (head_dim == 128) e = launch_sim<__nv_bfloat16, 128>(k, total_tokens, num_kv_heads, threshold, drop, start_bits, stream);
      else e = launch_sim<__nv_bfloat16, 256>(k, total_tokens, num_kv_heads, threshold, drop, start_bits, stream);
    } else {
      if (head_dim == 64) e = launch_sim<float, 64>(k, total_tokens, num_kv_heads, threshold, drop, start_bits, stream);
      else if (head_dim == 128) e = launch_sim<float, 128>(k, total_tokens, num_kv_heads, threshold, drop, start_bits, stream);
      else e = launch_sim<float, 256>(k, total_tokens, num_kv_heads, threshold, drop, start_bits, stream);
    }
    if (e != cudaSuccess) return e;
    if (num_seqs > 0) {
      constexpr int walk_smem = static_cast<int>(sizeof(WalkSmem));
      e = cudaFuncSetAttribute(segment_walk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, walk_smem);
      if (e != cudaSuccess) return e;
      // one sequence: the walk writes the chunk bounds itself
      const int compact = num_seqs == 1 ? 1 : 0;
      segment_walk_kernel<<<num_seqs, kWalkThreads, walk_smem, stream>>>(drop, cu_seqlens, min_len, max_len,
                                                                         start_bits, status, compact,
                                                                         chunk_bounds, capacity, seq_chunk_ptr,
                                                                         num_chunks);
      e = cudaGetLastError();
      if (e != cudaSuccess || compact) return e;
    }
  }
  segment_compact_kernel<<<1, kCompactThreads, 0, stream>>>(start_bits, total_tokens, cu_seqlens, num_seqs,
                                                           chunk_bounds, capacity, seq_chunk_ptr, num_chunks,
                                                           status);
  return cudaGetLastError();
}

}  // namespace dhsa
