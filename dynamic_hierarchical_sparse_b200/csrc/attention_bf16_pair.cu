// Step 4 of the DHSA path for bf16 inputs, head_dim 64 and 128: varlen
// block-sparse causal flash attention on tcgen05 tensor cores, two query tiles
// per work item, one persistent CTA per SM.
//
// out[t, h] = sum_s softmax_s(q[t,h] . k[s,g] * scale) v[s,g] over the kept
// key tokens s <= t: the tokens of the chunks in plan row (h, chunk(t))
// ("Long-Context Modeling with Dynamic Hierarchical Sparse Attention for
// On-Device LLMs", Abstract: only the token interactions selected through the
// upsampled chunk scores are preserved; "... for Memory-Constrained LLM
// Inference": causally important dependencies are kept).
//
// Work item = (query chunk i, head h, pair of 128-row tiles of chunk i).  Both
// tiles walk the same key tiles, so every K/V tile brought into shared memory
// by TMA feeds two QK^T and two PV products.  The kept chunks of row (h, i) are
// merged into runs of consecutive chunks once per item (a list in shared
// memory; rows with more runs than it holds continue from the plan in global
// memory), each run is cut into 128-key tiles, and the run holding the
// diagonal is clipped at the last valid query row of the pair.  The first tile
// of the pair stops at its own last row, so its tiles are a prefix of the
// second's.
//
// The kernel is persistent: one CTA per SM takes items from a counter in the
// workspace until none are left, and every ring position and barrier phase
// runs on across items, so an item's Q and K/V loads and its first QK^T
// overlap the previous item's last softmax and epilogue.
//
// Warp roles (384 threads = three warpgroups):
//   warps 0-3   softmax + epilogue of query tile 0 (thread r = row r = TMEM lane r)
//   warps 4-7   softmax + epilogue of query tile 1
//   warp 8      TMA producer: both Q tiles of each item (once the previous
//               item's last QK^T is done), K tiles into a 2-stage ring, V
//               tiles into a 3-stage ring; tile t+2 loads once the MMAs
//               through S(t) are done (one release commit per key tile)
//   warp 9      TMEM allocator; its lane 0 issues the MMAs of query tile 0
//   warp 10     lane 0 issues the MMAs of query tile 1
//   warp 11     scheduler: fetches the next item, builds its run list into the
//               second of two item slots
// The launch gives every thread 168 registers (three warps share a
// sub-partition's 16K); the third warpgroup then hands registers back
// (setmaxnreg.dec to 56) and the softmax warpgroups take them (224), enough to
// hold a whole 128-column row of S without spilling.
// TMEM (512 columns): S_a at [128a, 128a+128); P_a (f16, two per column) is
// written over the first 64 columns of S_a and is the A operand of O_a += P_a V
// (B: an f16 copy of V, made before the launch; both operands of one MMA are
// of one type);
// O_a at [256 + a*D, 256 + (a+1)*D).  The tensor pipe takes
//   PV_0(t), S_0(t+1), PV_1(t), S_1(t+1), PV_0(t+1), ...
// so while one warpgroup turns S into P the tensor core works for the other.
// The two issuing threads take turns in that order (a barrier hands the turn
// over): the pipe queues about one MMA, so a lone issuing thread runs in lock
// step with it and its own barrier waits and commits between bursts would
// leave the pipe idle; with two, each passes its waits during the other's
// turn.  A thread hands the turn over right after its last MMA of the turn
// (and the S-ready commit its own softmax waits for); the release, Q-free and
// O-ready commits, which only later consumers wait for, come after.  The P
// barriers take one arrival per softmax warp.
// P reaches the tensor core in two halves of 64 keys, each behind its own
// barrier, so PV_a(t) on the first half runs while the second half is still
// being exponentiated.
// Online softmax in fp32, exp2 domain, one ex2.approx per element (the
// scale-and-shift and the row sums on packed f32x2 FMA / add); O is rescaled
// whenever a warp's running max grows (two rounds of two 32-column TMEM slices
// with packed multiplies), so that the largest weight of a row is exactly 1.
#include "common.cuh"
#include "launchers.h"

namespace dhsa {
namespace {

constexpr int kBM = 128;
constexpr int kBN = 128;
constexpr int kThreads = 384;
constexpr uint32_t kRegsSoftmax = 224;  // 8 warps x 224 + 4 warps x 56 = 384 x 168
constexpr uint32_t kRegsOther = 56;
// P is handed to the tensor core in two halves of 64 keys: the PV product of
// the first half runs while the softmax exponentiates the second.
constexpr bool kSplitP = true;
// Scale-and-shift of the logits and the row sums on packed f32x2 FMA / add.
constexpr bool kPackedF32 = true;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kSchedWarp = 11;
constexpr uint32_t kTmemCols = 512;
constexpr int kRangeCap = 96;  // runs cached per item slot in shared memory; more continue from the plan
constexpr int kItemUsers = 11;  // item-slot releases: producer, two MMA threads, eight softmax warps
constexpr int kVStages = 3;     // V ring depth (K uses 2)
// O is rescaled whenever a warp's running max grows (threshold 0 in log2
// units): the row's largest weight is then exp2(0) = 1, exact.  A lazy
// threshold (2^8) let the running max lag, so the largest weight was rounded
// (to bf16 then, up to 2^-8 relative) and that rounding reached O directly: 0.026 of error
// at |O| = 4.4 at 128K, against 0.017 with every growth rescaled, for about
// 4 % of attention time.
constexpr float kRescaleLog2 = 0.0f;

template <int D>
struct PairCfg {
  static constexpr int kQSub = kBM * 128;   // one 64-column slice of a Q tile
  static constexpr int kKVSub = kBN * 128;  // one 64-column slice of a K/V tile
  static constexpr int kQBytes = kBM * D * 2;
  static constexpr int kKVBytes = kBN * D * 2;
  static constexpr int kOffQ = 0;  // tile a at kOffQ + a * kQBytes
  static constexpr int kOffK = 2 * kQBytes;
  static constexpr int kOffV = kOffK + 2 * kKVBytes;
  static constexpr int kOffRanges = kOffV + kVStages * kKVBytes;  // two item slots
  static constexpr int kOffItems = kOffRanges + 2 * kRangeCap * 8;  // two item descriptors
  static constexpr int kOffBar = kOffItems + 2 * 64;
  static constexpr int kSmemBytes = kOffBar + 256 + 1024;
  static constexpr uint32_t kColS = 0;    // + 128 a
  static constexpr uint32_t kColO = 256;  // + D a
  static_assert(256 + 2 * D <= 512, "TMEM budget");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

enum {
  kBarQ = 0,
  kBarKFull = 1,    // + K stage (2)
  kBarVFull = 3,    // + V stage (3)
  kBarRel = 6,      // + (j & 3): MMAs through S(j) done, so K(j+2) and V(j+2) may load
  kBarSFull = 10,   // + query tile
  kBarPFull = 12,   // + query tile
  kBarOReady = 14,  // + query tile: the last PV done (epilogue)
  kBarPHalf = 16,   // + query tile: first 64 keys of P written
  kBarDrain = 18,   // + query tile
  kBarTurn = 20,    // + query tile: that tile's MMA thread ended a turn
  kBarQFree = 22,   // both MMA threads' last S of the item done: Q may be reloaded
  kBarItemReady = 23,  // + slot: the scheduler wrote the slot's next item
  kBarItemFree = 25,   // + slot: every role is done with the slot's item
  kNumBars = 27
};

// One work item (a CTA's unit of work before it became persistent): query
// chunk ci, one or two 128-row query tiles, their key tiles.  Written by the
// scheduler warp into one of two slots, with the slot's run list.
struct Item {
  int done;  // 1: no work left
  int ci;
  int h, h1;  // heads of query tile 0 and tile 1
  int q0_0, q0_1, q_end0, q_end1;
  int valid1;
  int cap;     // last key + 1 of the item's diagonal run
  int p1;      // end of the plan row
  int resume;  // plan position where the runs past the cached list continue
  int ncached;
  int nt, nt0;  // key tiles of the item, and the prefix of them that tile 0 takes
  int pad;
};
static_assert(sizeof(Item) == 64, "item slot size");

// A plan entry read from the caller's plan, clamped into [0, num_chunks) so
// that a malformed plan never indexes the chunk bounds out of range (the
// scheduler reports such an entry; every role clamps it the same way).
__device__ __forceinline__ int plan_chunk(const int* __restrict__ col, int p, int num_chunks) {
  const int c = col[p];
  return min(max(c, 0), num_chunks - 1);
}

__device__ __forceinline__ bool chunk_in_range(int c, int num_chunks) {
  return static_cast<unsigned>(c) < static_cast<unsigned>(num_chunks);
}

// Key tiles of one work item: cached runs first, then (if the run list
// overflowed) runs merged on the fly from the plan in global memory.
struct TileWalk {
  const int2* ranges;
  int ncached, r;
  const int* col;
  const int* bounds;
  int p, pend, nch;
  int k0, re, cap;
  __device__ __forceinline__ void init(const int2* ranges_, int ncached_, const int* col_, const int* bounds_, int resume,
                       int p1, int cap_, int num_chunks) {
    ranges = ranges_;
    ncached = ncached_;
    r = 0;
    col = col_;
    bounds = bounds_;
    p = resume;
    pend = p1;
    nch = num_chunks;
    k0 = 0;
    re = 0;
    cap = cap_;
  }
  __device__ __forceinline__ bool next(int& tk0, int& tke) {
    if (k0 + kBN < re) {
      k0 += kBN;
    } else if (r < ncached) {
      const int2 g = ranges[r++];
      k0 = g.x;
      re = min(g.y, cap);
    } else {
      if (p >= pend) return false;
      int c = plan_chunk(col, p++, nch);
      const int rs = bounds[c];
      int e = bounds[c + 1];
      while (p < pend && plan_chunk(col, p, nch) == c + 1) {
        c = plan_chunk(col, p++, nch);
        e = bounds[c + 1];
      }
      k0 = rs;
      re = min(e, cap);
    }
    tk0 = k0;
    tke = re;
    return true;
  }
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attention_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, __nv_bfloat16* __restrict__ out,
                          const int* __restrict__ bounds, const int* __restrict__ row_ptr,
                          const int* __restrict__ col, int nnz, int num_chunks, int num_q_heads, int group,
                          int plan_group, int head_pair, int tiles, int total_items, float scale_log2,
                          uint32_t* status, int* item_counter) {
  using C = PairCfg<D>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::kOffBar;
  auto bar = [&](int idx) { return bar0 + 8u * static_cast<uint32_t>(idx); };
  int2* ranges_all = reinterpret_cast<int2*>(smem + C::kOffRanges);
  Item* items = reinterpret_cast<Item*>(smem + C::kOffItems);
  int* misc = reinterpret_cast<int*>(smem + C::kOffBar + 8 * kNumBars);
  // misc[0] TMEM base, misc[1] abort flag
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bar(kBarQ), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(kBarKFull + s), 1);
      mbar_init(bar(kBarSFull + s), 1);
      mbar_init(bar(kBarPFull + s), 4);  // one arrival per softmax warp
      mbar_init(bar(kBarOReady + s), 1);
      mbar_init(bar(kBarPHalf + s), 4);
      mbar_init(bar(kBarDrain + s), 1);
      mbar_init(bar(kBarTurn + s), 1);
      mbar_init(bar(kBarItemReady + s), 1);
      mbar_init(bar(kBarItemFree + s), kItemUsers);
    }
    for (int s = 0; s < kVStages; ++s) mbar_init(bar(kBarVFull + s), 1);
    for (int s = 0; s < 4; ++s) mbar_init(bar(kBarRel + s), 2);  // one commit per MMA thread
    mbar_init(bar(kBarQFree), 2);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(misc), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = static_cast<uint32_t>(misc[0]);

  // Persistent: the CTA takes work items (query chunk, heads, pair of query
  // tiles) from a global counter until none are left, in the order
  // i = x + tiles * (y + H * z): chunk n-1-z (longest plan rows first), head
  // (pair) y, tile pair x.  Every barrier phase and ring position below runs
  // on across items, so one item's Q and K/V loads and first QK^T overlap the
  // previous item's last softmax and epilogue.
  if (warp >= 8) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsOther));
  if (warp == kSchedWarp) {
    // ------------------------------------------------------- scheduler
    const int H = head_pair ? num_q_heads / 2 : num_q_heads;
    const unsigned lt = (1u << lane) - 1u;
    for (int k = 0;; ++k) {
      const int s = k & 1;
      // every lane waits; the warp leaves together if any lane gave up
      const bool free_ok = k < 2 || mbar_wait(bar(kBarItemFree + s), ((k - 2) >> 1) & 1, abort_flag, status);
      if (!__all_sync(0xffffffffu, free_ok)) break;
      Item* d = items + s;
      int2* ranges = ranges_all + s * kRangeCap;
      // next non-empty item (chunks shorter than the longest have fewer tiles)
      int ci = 0, hh = 0, q00 = 0, c_end = 0;
      bool done = false;
      while (true) {
        int i = 0;
        if (lane == 0) i = atomicAdd(item_counter, 1);
        i = __shfl_sync(0xffffffffu, i, 0);
        if (i >= total_items) {
          done = true;
          break;
        }
        const int x = i % tiles, r = i / tiles;
        const int y = r % H, z = r / H;
        ci = num_chunks - 1 - z;
        const int c_start = bounds[ci];
        c_end = bounds[ci + 1];
        hh = head_pair ? 2 * y : y;
        q00 = c_start + x * (head_pair ? 1 : 2) * kBM;
        if (q00 < c_end) break;
      }
      if (done) {
        if (lane == 0) d->done = 1;
      } else {
        // Two query tiles: consecutive 128-row tiles of one head, or, with
        // head_pair (a plan row per KV group, even group size), the same 128
        // rows of two heads 2m and 2m+1 of one group, sharing one key list.
        const int q01 = head_pair ? q00 : q00 + kBM;
        const bool valid1 = head_pair || q01 < c_end;
        const int q_end0 = min(q00 + kBM, c_end);
        const int q_end1 = valid1 ? min(q01 + kBM, c_end) : q01;
        const int cap = valid1 ? q_end1 : q_end0;
        const int row_id = (hh / plan_group) * num_chunks + ci;
        int p0 = row_ptr[row_id], p1 = row_ptr[row_id + 1];
        if (p0 < 0 || p1 < p0 || p1 > nnz) {
          // a malformed plan row: reported, and walked as an empty row
          if (lane == 0) report(status, kDevCheck);
          p0 = p1 = 0;
        }
        // merge the row's kept chunks into runs of consecutive chunks
        if (lane == 0) d->resume = p1;
        __syncwarp();
        int nstart = 0, nend = 0;
        for (int base = p0; base < p1; base += 32) {
          const int p = base + lane;
          const bool valid = p < p1;
          const int c = valid ? plan_chunk(col, p, num_chunks) : 0;
          if (valid && !chunk_in_range(col[p], num_chunks)) report(status, kDevCheck);
          int cprev = __shfl_up_sync(0xffffffffu, c, 1);
          int cnext = __shfl_down_sync(0xffffffffu, c, 1);
          if (lane == 0) cprev = (p > p0) ? plan_chunk(col, p - 1, num_chunks) : -2;
          if (lane == 31) cnext = (p + 1 < p1) ? plan_chunk(col, p + 1, num_chunks) : -2;
          const bool is_start = valid && (p == p0 || c != cprev + 1);
          const bool is_end = valid && (p == p1 - 1 || cnext != c + 1);
          const unsigned sm = __ballot_sync(0xffffffffu, is_start);
          const unsigned em = __ballot_sync(0xffffffffu, is_end);
          if (is_start) {
            const int idx = nstart + __popc(sm & lt);
            if (idx < kRangeCap) ranges[idx].x = bounds[c];
            else if (idx == kRangeCap) d->resume = p;
          }
          if (is_end) {
            const int idx = nend + __popc(em & lt);
            if (idx < kRangeCap) ranges[idx].y = bounds[c + 1];
          }
          nstart += __popc(sm);
          nend += __popc(em);
        }
        __syncwarp();
        if (lane == 0) {
          const int ncached = min(nstart, kRangeCap);
          // key tiles of the item (tile 1, or the only tile) and tile 0's prefix
          int nt = 0, nt0 = 0;
          TileWalk w;
          w.init(ranges, ncached, col, bounds, d->resume, p1, cap, num_chunks);
          int k0, ke;
          while (w.next(k0, ke)) {
            ++nt;
            if (k0 < q_end0) ++nt0;
          }
          d->done = 0;
          d->ci = ci;
          d->h = hh;
          d->h1 = head_pair ? hh + 1 : hh;
          d->q0_0 = q00;
          d->q0_1 = q01;
          d->q_end0 = q_end0;
          d->q_end1 = q_end1;
          d->valid1 = valid1 ? 1 : 0;
          d->cap = cap;
          d->p1 = p1;
          d->ncached = ncached;
          d->nt = nt;
          d->nt0 = nt0;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kBarItemReady + s));
      if (done) break;
    }
  } else if (warp == kProducerWarp) {
    // -------------------------------------------------------- producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int T = 0, issued = 0, qloads = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int s = k & 1;
        if (!mbar_wait(bar(kBarItemReady + s), (k >> 1) & 1, abort_flag, status)) break;
        const Item d = items[s];
        if (d.done) break;
        // Q of the previous item is free once both MMA threads' last S is done
        if (k >= 1 && !mbar_wait(bar(kBarQFree), (k - 1) & 1, abort_flag, status)) break;
        mbar_arrive_expect_tx(bar(kBarQ), (d.valid1 ? 2 : 1) * C::kQBytes);
#pragma unroll
        for (int a = 0; a < D / 64; ++a)
          tma_load_3d(sbase + C::kOffQ + a * C::kQSub, &tm_q, bar(kBarQ), a * 64, d.h, d.q0_0);
        if (d.valid1) {
#pragma unroll
          for (int a = 0; a < D / 64; ++a)
            tma_load_3d(sbase + C::kOffQ + C::kQBytes + a * C::kQSub, &tm_q, bar(kBarQ), a * 64, d.h1, d.q0_1);
        }
        qloads = k + 1;
        const int g = d.h / group;
        TileWalk w;
        w.init(ranges_all + s * kRangeCap, d.ncached, col, bounds, d.resume, d.p1, d.cap, num_chunks);
        int k0, ke;
        for (int t = 0; w.next(k0, ke); ++t) {
          const int tg = T + t;  // key tile counted across items
          const int st = tg & 1;
          // K(tg) replaces K(tg-2), read by S(tg-2); V(tg) replaces V(tg-3),
          // read by PV(tg-3), which each MMA thread issued before S(tg-2):
          // both are free once the release commits that follow S(tg-2) land.
          if (tg >= 2 && !mbar_wait(bar(kBarRel + ((tg - 2) & 3)), ((tg - 2) >> 2) & 1, abort_flag, status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(kBarKFull + st), C::kKVBytes);
#pragma unroll
          for (int a = 0; a < D / 64; ++a)
            tma_load_3d(sbase + C::kOffK + st * C::kKVBytes + a * C::kKVSub, &tm_k, bar(kBarKFull + st), a * 64, g,
                        k0);
          const int sv = tg % kVStages;
          mbar_arrive_expect_tx(bar(kBarVFull + sv), C::kKVBytes);
#pragma unroll
          for (int a = 0; a < D / 64; ++a)
            tma_load_3d(sbase + C::kOffV + sv * C::kKVBytes + a * C::kKVSub, &tm_v, bar(kBarVFull + sv), a * 64, g,
                        k0);
          issued = tg + 1;
        }
        T += d.nt;
        mbar_arrive(bar(kBarItemFree + s));
      }
      if (*abort_flag) {
        // let copies already in flight land before the CTA exits (bounded)
        volatile int never = 0;
        if (qloads > 0) mbar_wait(bar(kBarQ), (qloads - 1) & 1, &never, nullptr, 10000000ull);
        for (int t = max(0, issued - 2); t < issued; ++t)
          mbar_wait(bar(kBarKFull + (t & 1)), (t >> 1) & 1, &never, nullptr, 10000000ull);
        for (int t = max(0, issued - kVStages); t < issued; ++t)
          mbar_wait(bar(kBarVFull + t % kVStages), (t / kVStages) & 1, &never, nullptr, 10000000ull);
      }
    }
  } else {
    // ----------------------------------------------------------- MMA
    // One MMA-issuing thread per query tile, taking turns: tile 0's thread
    // issues PV_0(t) and S_0(t+1), hands over, tile 1's thread issues PV_1(t)
    // and S_1(t+1), hands back.  The turns keep the two softmax warpgroups
    // half a period apart (so they do not share the exponential unit); two
    // threads let each one pass its own waits and commits while the other's
    // MMAs run, instead of leaving the tensor pipe idle meanwhile.  Both
    // threads take every turn, also on items with one query tile.
    const int a = warp - kMmaWarp;
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(kBM, kBN, 0);
      constexpr uint32_t idesc_o = idesc_f16_f32(kBM, D, 1);  // P and V in f16
      const uint32_t qbase = sbase + C::kOffQ + a * C::kQBytes;
      auto issue_s = [&](int tg) {
        const uint32_t kbase = sbase + C::kOffK + (tg & 1) * C::kKVBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t ad = smem_desc_sw128(qbase + (kk >> 2) * C::kQSub + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(kbase + (kk >> 2) * C::kKVSub + (kk & 3) * 32, 16, 1024);
          umma_f16_ss(tmem + C::kColS + a * 128, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(bar(kBarSFull + a));
      };
      // turn kt (counted across items): tile 1's thread waits for tile 0's
      // turn kt, tile 0's thread for tile 1's turn kt - 1
      auto wait_turn = [&](int kt) -> bool {
        if (a == 1) return mbar_wait_spin(bar(kBarTurn + 0), kt & 1, abort_flag, status);
        if (kt == 0) return true;
        return mbar_wait_spin(bar(kBarTurn + 1), (kt - 1) & 1, abort_flag, status);
      };
      auto end_turn = [&]() { mbar_arrive(bar(kBarTurn + a)); };
      int T = 0, kt = 0, np = 0;  // key tiles, turns, P tiles of this query tile: all across items
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int s = k & 1;
        if (!mbar_wait(bar(kBarItemReady + s), (k >> 1) & 1, abort_flag, status)) break;
        const Item d = items[s];
        if (d.done) break;
        const int nt = d.nt;
        const int nta = a == 0 ? d.nt0 : (d.valid1 ? d.nt : 0);
        ok = mbar_wait(bar(kBarQ), k & 1, abort_flag, status);
        if (ok) ok = mbar_wait(bar(kBarKFull + (T & 1)), (T >> 1) & 1, abort_flag, status);
        if (ok) ok = wait_turn(kt);
        if (!ok) break;
        tc_fence_after();
        if (nta > 0) issue_s(T);
        // hand the turn over first: the other thread's MMAs wait for it, the
        // commits below only for later consumers
        end_turn();
        ++kt;
        if (nta <= 1) umma_commit(bar(kBarQFree));  // this thread's last S of the item (if any) is issued
        umma_commit(bar(kBarRel + (T & 3)));         // key tile T: S(T) done
        for (int t = 0; t < nt; ++t) {
          const int tg = T + t;
          if (t < nta) {
            const int sv = tg % kVStages;
            if (!mbar_wait_spin(bar(kBarVFull + sv), (tg / kVStages) & 1, abort_flag, status)) { ok = false; break; }
            const uint32_t vbase = sbase + C::kOffV + sv * C::kKVBytes;
            auto issue_pv = [&](int kk0, int kk1) {
#pragma unroll
              for (int kk = kk0; kk < kk1; ++kk) {
                const uint64_t bd = smem_desc_sw128(vbase + kk * 16 * 128, C::kKVSub, 1024);
                umma_f16_ts(tmem + C::kColO + a * D, tmem + C::kColS + a * 128 + kk * 8, bd, idesc_o,
                            (t > 0 || kk > 0) ? 1u : 0u);
              }
            };
            if (!mbar_wait_spin(bar(kBarPHalf + a), np & 1, abort_flag, status)) { ok = false; break; }
            if (t + 1 < nta &&
                !mbar_wait_spin(bar(kBarKFull + ((tg + 1) & 1)), ((tg + 1) >> 1) & 1, abort_flag, status)) {
              ok = false;
              break;
            }
            if (!wait_turn(kt)) { ok = false; break; }
            tc_fence_after();
            issue_pv(0, kBN / 32);
            if (!mbar_wait_spin(bar(kBarPFull + a), np & 1, abort_flag, status)) { ok = false; break; }
            tc_fence_after();
            issue_pv(kBN / 32, kBN / 16);
            ++np;
            if (t + 1 < nta) issue_s(tg + 1);
            end_turn();
            ++kt;
            // only the epilogue waits for O: S(t+1), issued after PV(t), tells
            // the softmax that PV(t) is done before it rescales O
            if (t + 1 == nta) umma_commit(bar(kBarOReady + a));
            if (t + 2 == nta) umma_commit(bar(kBarQFree));  // S(t+1) was the item's last
          } else {
            if (!wait_turn(kt)) {
              ok = false;
              break;
            }
            end_turn();
            ++kt;
          }
          if (t + 1 < nt) umma_commit(bar(kBarRel + ((tg + 1) & 3)));  // key tile tg + 1: S(tg+1) done
        }
        T += nt;
        mbar_arrive(bar(kBarItemFree + s));
      }
      // every MMA issued above completes before TMEM is released
      umma_commit(bar(kBarDrain + a));
      volatile int never = 0;
      mbar_wait(bar(kBarDrain + a), 0, &never, nullptr);
    }
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    // ------------------------------------------------ softmax warpgroups
    const int a = warp >> 2;  // query tile of this warpgroup
    const int row = threadIdx.x & 127;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + C::kColS + a * 128;
    const uint32_t tO = tmem + lane_base + C::kColO + a * D;
    int ns = 0, no = 0;  // S tiles and epilogues of this query tile, across items
    bool ok = true;
    for (int k = 0; ok; ++k) {
    const int slot = k & 1;
    if (!mbar_wait(bar(kBarItemReady + slot), (k >> 1) & 1, abort_flag, status)) break;
    const Item d = items[slot];
    if (d.done) break;
    const int nta = a == 0 ? d.nt0 : (d.valid1 ? d.nt : 0);
    const int q0 = a == 0 ? d.q0_0 : d.q0_1;
    const int q_end = a == 0 ? d.q_end0 : d.q_end1;
    const int t_row = q0 + row;
    float m_run = -INFINITY;  // running max of logits * scale * log2(e)
    float l_run = 0.f;
    TileWalk w;
    w.init(ranges_all + slot * kRangeCap, d.ncached, col, bounds, d.resume, d.p1, d.cap, num_chunks);
    int k0, ke;
    for (int t = 0; t < nta && w.next(k0, ke); ++t) {
      if (!mbar_wait(bar(kBarSFull + a), ns & 1, abort_flag, status)) {
        ok = false;
        break;
      }
      ++ns;
      tc_fence_after();
      // S row -> registers in two halves: the second half is still loading
      // while the first half is masked and max-reduced.
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
          // only 32-column blocks that reach past the row's last valid column
#pragma unroll
          for (int blk = base; blk < base + kBN / 2; blk += 32) {
            if (lim < blk + 32) {
#pragma unroll
              for (int c = blk; c < blk + 32; ++c)
                if (c >= lim) s[c] = -INFINITY;
            }
          }
        }
        // row max as a tree of 3-input maxima (short dependency chains)
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
      float ps[4] = {0.f, 0.f, 0.f, 0.f};
      uint64_t ps2[2] = {0ull, 0ull};  // packed (lo, hi) partial sums
      const uint64_t scale2 = f2_pack(scale_log2, scale_log2);
      const uint64_t shift2 = f2_pack(-m_use, -m_use);
      uint32_t pk[kBN / 2];
      // P = exp2(s * scale - m) for columns [cb, cb + 64), packed to f16 pairs
      auto exp_cols = [&](int cb) {
#pragma unroll
        for (int c = cb; c < cb + kBN / 2; c += 2) {
          float x0, x1;
          if (kPackedF32) {
            f2_unpack(f2_fma(f2_pack(s[c], s[c + 1]), scale2, shift2), x0, x1);
          } else {
            x0 = fmaf(s[c], scale_log2, -m_use);
            x1 = fmaf(s[c + 1], scale_log2, -m_use);
          }
          const float e0 = ex2_approx(x0);
          const float e1 = ex2_approx(x1);
          if (kPackedF32)
            ps2[(c / 2) & 1] = f2_add(ps2[(c / 2) & 1], f2_pack(e0, e1));
          else
            ps[(c / 2) & 3] += e0 + e1;
          pk[c / 2] = pack_f16(e0, e1);
        }
      };
      // O is rescaled before PV(t) accumulates into it; PV(t-1) is done, since
      // S(t), waited for above, was issued after it
      // two 32-column slices per round: both loads in flight, one wait, packed
      // multiplies, both stores (the next round's loads touch other columns)
      auto rescale_o = [&]() -> bool {
        const uint64_t alpha2 = f2_pack(alpha, alpha);
#pragma unroll 1
        for (int c = 0; c < D / 32; c += 2) {
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
        return true;
      };
      exp_cols(0);
      // P over the first 64 columns of S (the S values are already in registers)
      tmem_st32p(tS + 0, pk);
      if (kSplitP) {
        if (any && t > 0 && !rescale_o()) {
          ok = false;
          break;
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kBarPHalf + a));
      }
      exp_cols(kBN / 2);
      tmem_st32p(tS + 32, pk + 32);
      if (kPackedF32) {
        float a0, a1, b0, b1;
        f2_unpack(ps2[0], a0, a1);
        f2_unpack(ps2[1], b0, b1);
        l_run = l_run * alpha + ((a0 + a1) + (b0 + b1));
      } else {
        l_run = l_run * alpha + ((ps[0] + ps[1]) + (ps[2] + ps[3]));
      }
      if (!kSplitP && any && t > 0 && !rescale_o()) {
        ok = false;
        break;
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kBarPFull + a));
    }
    // done with the slot's run list; the epilogue needs registers only
    __syncwarp();
    if (lane == 0) mbar_arrive(bar(kBarItemFree + slot));
    if (!ok) break;
    if (nta > 0) {
      if (!mbar_wait(bar(kBarOReady + a), no & 1, abort_flag, status)) break;
      ++no;
      tc_fence_after();
      const float inv_l = 1.f / l_run;
      const bool valid = t_row < q_end;
      __nv_bfloat16* orow = out + (static_cast<size_t>(t_row) * num_q_heads + (a == 0 ? d.h : d.h1)) * D;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + 32 * c, o);
        tmem_wait_ld();
        reg_dep32(o);
        if (valid) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 wv;
            wv.x = pack_bf16(__uint_as_float(o[e + 0]) * inv_l, __uint_as_float(o[e + 1]) * inv_l);
            wv.y = pack_bf16(__uint_as_float(o[e + 2]) * inv_l, __uint_as_float(o[e + 3]) * inv_l);
            wv.z = pack_bf16(__uint_as_float(o[e + 4]) * inv_l, __uint_as_float(o[e + 5]) * inv_l);
            wv.w = pack_bf16(__uint_as_float(o[e + 6]) * inv_l, __uint_as_float(o[e + 7]) * inv_l);
            *reinterpret_cast<uint4*>(orow + 32 * c + e) = wv;
          }
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

template <int D>
cudaError_t launch_attention_pair_dim(const AttnBf16Args& a, cudaStream_t stream) {
  using C = PairCfg<D>;
  CUtensorMap mq, mk, mv;
  if (encode_qkv_map(&mq, a.q, a.num_q_heads, D, a.total_tokens, kBM) != CUDA_SUCCESS ||
      encode_qkv_map(&mk, a.k, a.num_kv_heads, D, a.total_tokens, kBN) != CUDA_SUCCESS ||
      encode_qkv_map(&mv, a.v16, a.num_kv_heads, D, a.total_tokens, kBN, true) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  auto kern = attention_pair_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  // a plan row per KV group of even size: pair two heads of the group on the same rows
  const int head_pair = (a.plan_group >= 2 && a.plan_group % 2 == 0) ? 1 : 0;
  const int tiles = head_pair ? (a.max_chunk_len + kBM - 1) / kBM : (a.max_chunk_len + 2 * kBM - 1) / (2 * kBM);
  const int heads = head_pair ? a.num_q_heads / 2 : a.num_q_heads;
  const long long total = static_cast<long long>(tiles) * heads * a.num_chunks;
  if (total <= 0) return cudaSuccess;
  if (total > 0x7fffffffLL - 2 * 65536) return cudaErrorInvalidValue;
  int dev = 0, sms = 0;
  e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  // one persistent CTA per SM (its shared memory and TMEM fill the SM)
  const int grid = static_cast<int>(total < sms ? total : sms);
  const float scale_log2 = a.scale * 1.4426950408889634f;
  kern<<<grid, kThreads, C::kSmemBytes, stream>>>(mq, mk, mv, static_cast<__nv_bfloat16*>(a.out), a.bounds,
                                                  a.row_ptr, a.col, a.nnz, a.num_chunks, a.num_q_heads,
                                                  a.num_q_heads / a.num_kv_heads, a.plan_group, head_pair, tiles,
                                                  static_cast<int>(total), scale_log2, a.status,
                                                  reinterpret_cast<int*>(a.status + 1));
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention_pair(const AttnBf16Args& a, cudaStream_t stream) {
  if (a.head_dim == 128) return launch_attention_pair_dim<128>(a, stream);
  if (a.head_dim == 64) return launch_attention_pair_dim<64>(a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace dhsa
