// select_compact.cu -- one fused kernel per eviction round: score, select the
// top positions of every (request, layer, KV head) segment and compact the
// survivors in place.
//
// What it computes (Random Attention article, "Random Attention：不判断重要性，
// 只随机保留" and "发现四"): the protected slots [0, P) are never candidates;
// the N = L - P candidate slots are ranked by (score desc, original position
// asc), the best M stay and are compacted into slots [P, P + M); K rows, V
// rows and the position map move together.  The score is the Philox draw of
// the (position / block, head, layer, request) counter for the random
// selectors (block = 1: one draw per position; larger blocks keep contiguous
// runs, "发现二"), or the precomputed beacon score.
//
// Design (B200): one CTA per segment, everything between score and copy in
// shared memory.
//   1. score: each thread draws the 32-bit keys of a strided set of slots
//      (the random path reads only the 4-byte position map, never K/V);
//   2. select: 4-pass MSB radix select (8-bit digits, shared-memory
//      histogram) finds the M-th largest key tau, how many keys equal tau and
//      how many of those stay.  When slots are in position order (always, as
//      long as no round filled holes) the tied keys that stay are the lowest
//      slots; otherwise a second radix select over the tied candidates on the
//      complemented position picks the lowest positions exactly;
//   3. ranks: tile-wise block scans with warp ballots give every survivor
//      its rank (order-preserving compaction) or list the holes and the
//      survivors past the new length (hole filling);
//   4. copy, order-preserving: survivors from the first evicted slot on move
//      to slot P + rank.  Each chunk of ranks (8 rows per thread group,
//      64-128 KB of K and V in flight per CTA) is read with 16-byte vector
//      loads into registers, the CTA synchronises, then writes.  A chunk only
//      writes slots below its own highest source slot and the next chunk only
//      reads slots above it, so one barrier per chunk makes the in-place move
//      safe while loads of chunk c+1 overlap stores of chunk c;
//   4'. copy, hole filling: the i-th survivor at or past the new length moves
//      into the i-th evicted slot below it; sources and destinations are
//      disjoint, so the copies need no barrier.
// Rows of the same segment are never touched by another CTA.
#include "kvc_internal.h"
#include "philox.cuh"

namespace kvc {
namespace {

#ifndef KVC_SC_UNROLL_SMALL
#define KVC_SC_UNROLL_SMALL 8
#endif
#ifndef KVC_SC_UNROLL_LARGE
#define KVC_SC_UNROLL_LARGE 8
#endif
// Segments with at most this many candidates run with 256 threads per CTA
// (two CTAs per SM, so one CTA's select phase overlaps the other's copy);
// larger ones with 512.
#ifndef KVC_SC_NT256_MAX_N
#define KVC_SC_NT256_MAX_N 4096
#endif
#ifndef KVC_SC_UNROLL_HOLE
#define KVC_SC_UNROLL_HOLE 2
#endif

// copy / tie variants of the kernel
constexpr int kOrderedSlotTie = 0;  // order-preserving, ties by slot (slots in position order)
constexpr int kOrderedPosTie = 1;   // order-preserving, ties by position
constexpr int kHoleFill = 2;        // hole filling, ties by position

__device__ __forceinline__ uint32_t float_order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// k_in-th largest key (1-based) among the candidates for which keyfn(j, key)
// returns true; also how many keys equal it (count_eq) and how many of those
// belong to the top k_in (need).  MSB radix select with 8-bit digits; once
// the bucket holding the answer has at most kFinish keys (for random 32-bit
// keys that is after the first digit), those keys are gathered and one warp
// finishes by counting, so the remaining passes over all keys are skipped.
// first_ready: hist already holds the top-byte counts of every key (built
// while the keys were drawn), so the first digit needs no pass.
constexpr int kFinish = 64;

template <int NT, class KeyFn>
__device__ __forceinline__ void block_radix_select(int n, int k_in, KeyFn keyfn, uint32_t *hist,
                                                   uint32_t *bcast, uint32_t *cand, uint32_t &tau,
                                                   int &need, int &count_eq, bool first_ready = false) {
  uint32_t prefix = 0, mask = 0;
  int k = k_in;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
#pragma unroll 1
  for (int shift = 24; shift >= 0; shift -= 8) {
    if (!(first_ready && shift == 24)) {
      for (int i = tid; i < 256; i += NT) hist[i] = 0;
      __syncthreads();
      for (int j = tid; j < n; j += NT) {
        uint32_t key;
        if (keyfn(j, key) && (key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
      }
      __syncthreads();
    }
    if (warp == 0) {
      // lane l owns digits 255-8l .. 248-8l (descending)
      uint32_t c[8];
      uint32_t sum = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        c[i] = hist[255 - 8 * lane - i];
        sum += c[i];
      }
      uint32_t incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const uint32_t excl = incl - sum;
      const unsigned hit = __ballot_sync(0xffffffffu, incl >= (uint32_t)k);
      const int first = __ffs(hit) - 1;
      if (lane == first) {
        uint32_t cum = excl;
        int digit = 0;
        uint32_t cnt = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (cum + c[i] >= (uint32_t)k) {
            digit = 255 - 8 * lane - i;
            cnt = c[i];
            break;
          }
          cum += c[i];
        }
        bcast[0] = (uint32_t)digit;
        bcast[1] = (uint32_t)k - cum;
        bcast[2] = cnt;
        bcast[3] = 0;
      }
    }
    __syncthreads();
    prefix |= bcast[0] << shift;
    mask |= 255u << shift;
    k = (int)bcast[1];
    count_eq = (int)bcast[2];
    if (shift > 0 && count_eq <= kFinish) {
      // gather the bucket, then one warp counts: the k-th largest x has
      // #{y > x} < k <= #{y >= x}
      for (int j = tid; j < n; j += NT) {
        uint32_t key;
        if (keyfn(j, key) && (key & mask) == prefix) cand[atomicAdd(&bcast[3], 1u)] = key;
      }
      __syncthreads();
      if (warp == 0) {
        const int m = count_eq;
#pragma unroll
        for (int h = 0; h < kFinish / 32; ++h) {
          const int i = h * 32 + lane;
          if (i < m) {
            const uint32_t x = cand[i];
            int gt = 0, ge = 0;
            for (int t = 0; t < m; ++t) {
              const uint32_t y = cand[t];
              gt += y > x;
              ge += y >= x;
            }
            if (gt < k && k <= ge) {  // every lane holding the answer writes the same values
              bcast[0] = x;
              bcast[1] = (uint32_t)(k - gt);
              bcast[2] = (uint32_t)(ge - gt);
            }
          }
        }
      }
      __syncthreads();
      tau = bcast[0];
      need = (int)bcast[1];
      count_eq = (int)bcast[2];
      __syncthreads();  // bcast and cand are reused by the caller's next select
      return;
    }
    __syncthreads();
  }
  tau = prefix;
  need = k;
}

// Exclusive scan of a per-candidate predicate over [lo, hi) in candidate
// order; calls fn(j, index) for every j with pred(j) true, index = number of
// earlier candidates with pred true.  Returns the total.  Each warp owns a
// contiguous range (whole 32-candidate chunks): it counts its range with
// ballots, one block barrier exchanges the warp totals, and a second sweep
// hands out the indices, so the block synchronises once per scan instead of
// once per chunk.
template <int NT, class Pred, class Fn>
__device__ __forceinline__ int block_scan_each(int lo, int hi, Pred pred, Fn fn, uint32_t *warp_cnt) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int n = hi - lo;
  const int per = ((n + NW * 32 - 1) / (NW * 32)) * 32;  // candidates per warp
  const int w0 = lo + warp * per, w1 = min(hi, w0 + per);
  int cnt = 0;
  for (int base = w0; base < w1; base += 32) {
    const int j = base + lane;
    cnt += __popc(__ballot_sync(0xffffffffu, j < w1 && pred(j)));
  }
  if (lane == 0) warp_cnt[warp] = cnt;
  __syncthreads();
  int off = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    const int c = warp_cnt[w];
    if (w < warp) off += c;
    tot += c;
  }
  for (int base = w0; base < w1; base += 32) {
    const int j = base + lane;
    const bool f = j < w1 && pred(j);
    const unsigned m = __ballot_sync(0xffffffffu, f);
    if (f) fn(j, off + __popc(m & ((1u << lane) - 1u)));
    off += __popc(m);
  }
  __syncthreads();  // warp_cnt reuse
  return tot;
}

// One (request, layer, KV head) segment of a launch: item i of the launch is
// request segs[i / (hkv * layers)], layer (i / hkv) % layers, head i % hkv.
struct ScSeg {
  int h, l, r, P, M, N;
  const int32_t *bt;
  int64_t layer_page0, seg_flat;
};

__device__ __forceinline__ ScSeg sc_seg(const SelectCompactParams &p, int item) {
  ScSeg g;
  g.h = item % p.hkv;
  g.l = (item / p.hkv) % p.layers;
  const SegDesc sd = p.segs[item / (p.hkv * p.layers)];
  g.r = sd.req;
  g.P = sd.P;
  g.M = sd.M;
  g.N = sd.L - sd.P;
  g.bt = p.block_table + (int64_t)g.r * p.bt_stride;
  g.layer_page0 = (int64_t)g.l * p.num_pages;
  g.seg_flat = ((int64_t)g.r * p.layers + g.l) * p.hkv + g.h;
  return g;
}

// global row index (also the position-map index) of slot s of the segment
__device__ __forceinline__ int64_t sc_row(const SelectCompactParams &p, const ScSeg &g, int s) {
  return ((g.layer_page0 + g.bt[s >> 4]) * p.hkv + g.h) * kPage + (s & (kPage - 1));
}

// 32-bit ranking key of candidate j (slot P + j): the order key of the beacon
// score, or the high word of the Philox draw of (position / block, head,
// layer, request) under (seed, round)
template <int MODE>
__device__ __forceinline__ uint32_t sc_key(const SelectCompactParams &p, const ScSeg &g, int j) {
  if (MODE == kModeScores) return float_order_key(p.scores[g.seg_flat * p.max_seq + j]);
  const uint64_t head_field = (MODE == kModeRandomShared) ? ~0ull : (uint64_t)g.h;
  const int pos = p.pos_map[sc_row(p, g, g.P + j)];
  const uint32_t key = philox4x64_10_word0_hi32((uint64_t)(int64_t)(pos / p.block), head_field, (uint64_t)g.l,
                                                (uint64_t)g.r, p.seed, p.round);
  if (p.debug) p.debug[g.seg_flat * p.max_seq + j] = key;
  return key;
}

// Shared scratch of the select and rank steps.
template <int NT>
struct ScScratch {
  uint32_t hist[256];
  uint32_t bcast[4];
  uint32_t cand[kFinish];
  uint32_t warp_cnt[NT / 32], warp_eq[NT / 32];
  int first_evicted;
  int next;  // persistent form: the next work item
};

// The survivors' threshold: keys above tau stay; of the count_eq keys equal
// to tau, `need` stay -- the lowest slots, or (split_by_pos) the lowest
// positions, those whose complemented position is at least ptau.
struct ScThreshold {
  uint32_t tau, ptau;
  int need, count_eq;
  bool split_by_pos;
};

template <int NT, int VAR>
__device__ __forceinline__ ScThreshold sc_threshold(const SelectCompactParams &p, const ScSeg &g,
                                                    const uint32_t *keys, ScScratch<NT> &sh,
                                                    bool hist_ready = false) {
  ScThreshold t;
  block_radix_select<NT>(
      g.N, g.M, [&](int j, uint32_t &k) { k = keys[j]; return true; }, sh.hist, sh.bcast, sh.cand, t.tau, t.need,
      t.count_eq, hist_ready);
  // with ties split and slots possibly out of position order: the `need`
  // lowest positions among the tied keys (positions are distinct)
  t.ptau = 0;
  t.split_by_pos = VAR != kOrderedSlotTie && t.need < t.count_eq;
  if (t.split_by_pos) {
    int need2, cnt2;
    const uint32_t tau = t.tau;
    block_radix_select<NT>(
        g.N, t.need,
        [&](int j, uint32_t &k) {
          if (keys[j] != tau) return false;
          k = ~(uint32_t)p.pos_map[sc_row(p, g, g.P + j)];
          return true;
        },
        sh.hist, sh.bcast, sh.cand, t.ptau, need2, cnt2);
  }
  return t;
}

// kept flag of candidate j when ties go by position
__device__ __forceinline__ bool sc_kept_pos(const SelectCompactParams &p, const ScSeg &g, const uint32_t *keys,
                                            const ScThreshold &t, int j) {
  const uint32_t key = keys[j];
  if (key != t.tau) return key > t.tau;
  if (!t.split_by_pos) return true;
  return ~(uint32_t)p.pos_map[sc_row(p, g, g.P + j)] >= t.ptau;
}

// Ranks of an order-preserving round: src_of_rank[q] = the candidate that
// becomes the q-th survivor, for q < M, and the first evicted candidate in
// sh.first_evicted (N if none).  Ends with a block barrier.
template <int NT, int VAR>
__device__ __forceinline__ void sc_ordered_ranks(const SelectCompactParams &p, const ScSeg &g, const uint32_t *keys,
                                                 const ScThreshold &t, uint16_t *src_of_rank, ScScratch<NT> &sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int N = g.N;
  if (VAR == kOrderedSlotTie) {
    // kept = key > tau, or key == tau among the first `need` such slots:
    // two counts per candidate (greater, equal) scanned over warp ranges
    constexpr int NW = NT / 32;
    const uint32_t tau = t.tau;
    const int need = t.need;
    const int per = ((N + NW * 32 - 1) / (NW * 32)) * 32;
    const int w0 = warp * per, w1 = min(N, w0 + per);
    int cgt = 0, ceq = 0;
    for (int base = w0; base < w1; base += 32) {
      const int j = base + lane;
      const uint32_t key = j < w1 ? keys[j] : 0u;
      cgt += __popc(__ballot_sync(0xffffffffu, j < w1 && key > tau));
      ceq += __popc(__ballot_sync(0xffffffffu, j < w1 && key == tau));
    }
    if (lane == 0) {
      sh.warp_cnt[warp] = cgt;
      sh.warp_eq[warp] = ceq;
    }
    __syncthreads();
    int off_gt = 0, off_eq = 0;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      if (w < warp) {
        off_gt += sh.warp_cnt[w];
        off_eq += sh.warp_eq[w];
      }
    }
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int base = w0; base < w1; base += 32) {
      const int j = base + lane;
      const bool valid = j < w1;
      const uint32_t key = valid ? keys[j] : 0u;
      const bool gt = valid && key > tau;
      const bool eq = valid && key == tau;
      const unsigned mgt = __ballot_sync(0xffffffffu, gt);
      const unsigned meq = __ballot_sync(0xffffffffu, eq);
      const int gt_before = off_gt + __popc(mgt & lt_mask);
      const int eq_before = off_eq + __popc(meq & lt_mask);
      const bool kept = gt || (eq && eq_before < need);
      if (kept) {
        src_of_rank[gt_before + min(eq_before, need)] = (uint16_t)j;
      } else if (valid) {
        atomicMin(&sh.first_evicted, j);
      }
      off_gt += __popc(mgt);
      off_eq += __popc(meq);
    }
  } else {
    block_scan_each<NT>(
        0, N, [&](int j) { return sc_kept_pos(p, g, keys, t, j); },
        [&](int j, int rank) { src_of_rank[rank] = (uint16_t)j; }, sh.warp_cnt);
    for (int j = threadIdx.x; j < N; j += NT)
      if (!sc_kept_pos(p, g, keys, t, j)) atomicMin(&sh.first_evicted, j);
  }
  __syncthreads();
}

template <int NT, int MODE, int kUnroll, int VAR>
__global__ void __launch_bounds__(NT) select_compact_kernel(SelectCompactParams p, int keys_cap) {
  extern __shared__ __align__(16) uint8_t smem[];
  uint32_t *keys = reinterpret_cast<uint32_t *>(smem);                  // [keys_cap]
  uint16_t *src_of_rank = reinterpret_cast<uint16_t *>(keys + keys_cap);  // [keys_cap]
  __shared__ ScScratch<NT> sh;

  const int tid = threadIdx.x;
  const ScSeg g = sc_seg(p, blockIdx.x);
  const int P = g.P, M = g.M, N = g.N;

  // 1. keys
  if (tid == 0) sh.first_evicted = N;
  for (int j = tid; j < N; j += NT) keys[j] = sc_key<MODE>(p, g, j);
  __syncthreads();

  // 2. threshold
  const ScThreshold t = sc_threshold<NT, VAR>(p, g, keys, sh);

  const int vpr = p.row_bytes >> 4;  // 16-byte vectors per row
  const int rows_per_pass = NT / vpr;
  const int my_row = tid / vpr, my_vec = tid - (tid / vpr) * vpr;
  const bool active = my_row < rows_per_pass;
  const int64_t rb = p.row_bytes;

  if (VAR != kHoleFill) {
    // 3. ranks in slot order
    sc_ordered_ranks<NT, VAR>(p, g, keys, t, src_of_rank, sh);

    // 4. in-place, order-preserving copy of ranks [first_evicted, M)
    const int q0 = sh.first_evicted;
#pragma unroll 1
    for (int base = q0; base < M; base += rows_per_pass * kUnroll) {
      uint4 kr[kUnroll], vr[kUnroll];
      int pr[kUnroll];
      int64_t drow[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int q = base + u * rows_per_pass + my_row;
        drow[u] = -1;
        if (active && q < M) {
          const int64_t srow = sc_row(p, g, P + src_of_rank[q]);
          drow[u] = sc_row(p, g, P + q);
          kr[u] = *reinterpret_cast<const uint4 *>(p.k_pool + srow * rb + my_vec * 16);
          vr[u] = *reinterpret_cast<const uint4 *>(p.v_pool + srow * rb + my_vec * 16);
          if (my_vec == 0) pr[u] = p.pos_map[srow];
        }
      }
      __syncthreads();
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        if (drow[u] >= 0) {
          *reinterpret_cast<uint4 *>(p.k_pool + drow[u] * rb + my_vec * 16) = kr[u];
          *reinterpret_cast<uint4 *>(p.v_pool + drow[u] * rb + my_vec * 16) = vr[u];
          if (my_vec == 0) p.pos_map[drow[u]] = pr[u];
        }
      }
    }
    if (tid == 0 && M > q0) atomicAdd(p.counters, (unsigned long long)(M - q0));
  } else {
    // 3'. holes (evicted candidates below M) and movers (kept at or past M),
    // each listed in candidate order: holes at src_of_rank[0..), movers at
    // src_of_rank[M..)
    const int n_holes = block_scan_each<NT>(
        0, M, [&](int j) { return !sc_kept_pos(p, g, keys, t, j); },
        [&](int j, int i) { src_of_rank[i] = (uint16_t)j; }, sh.warp_cnt);
    block_scan_each<NT>(
        M, N, [&](int j) { return sc_kept_pos(p, g, keys, t, j); },
        [&](int j, int i) { src_of_rank[M + i] = (uint16_t)j; }, sh.warp_cnt);
    __syncthreads();
    // 4'. the i-th mover goes to the i-th hole; all copies are independent
#pragma unroll 1
    for (int base = 0; base < n_holes; base += rows_per_pass * kUnroll) {
      uint4 kr[kUnroll], vr[kUnroll];
      int pr[kUnroll];
      int64_t drow[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int i = base + u * rows_per_pass + my_row;
        drow[u] = -1;
        if (active && i < n_holes) {
          const int64_t srow = sc_row(p, g, P + src_of_rank[M + i]);
          drow[u] = sc_row(p, g, P + src_of_rank[i]);
          kr[u] = *reinterpret_cast<const uint4 *>(p.k_pool + srow * rb + my_vec * 16);
          vr[u] = *reinterpret_cast<const uint4 *>(p.v_pool + srow * rb + my_vec * 16);
          if (my_vec == 0) pr[u] = p.pos_map[srow];
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        if (drow[u] >= 0) {
          *reinterpret_cast<uint4 *>(p.k_pool + drow[u] * rb + my_vec * 16) = kr[u];
          *reinterpret_cast<uint4 *>(p.v_pool + drow[u] * rb + my_vec * 16) = vr[u];
          if (my_vec == 0) p.pos_map[drow[u]] = pr[u];
        }
      }
    }
    if (tid == 0 && n_holes > 0) atomicAdd(p.counters, (unsigned long long)n_holes);
  }
}

// Asynchronous 4-byte global -> shared copies (no register destination):
// each thread waits only for the copies it issued itself.
__device__ __forceinline__ void cp_async4(void *smem_dst, const void *gsrc) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"((uint32_t)__cvta_generic_to_shared(smem_dst)),
               "l"(gsrc)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// The key of candidate j from the raw word fetched for it: the score's bits
// (kModeScores) or its position (random selectors).
template <int MODE>
__device__ __forceinline__ uint32_t sc_key_from(const SelectCompactParams &p, const ScSeg &g, int j, uint32_t raw) {
  if (MODE == kModeScores) return float_order_key(__uint_as_float(raw));
  const uint64_t head_field = (MODE == kModeRandomShared) ? ~0ull : (uint64_t)g.h;
  const uint32_t key = philox4x64_10_word0_hi32((uint64_t)(int64_t)((int)raw / p.block), head_field, (uint64_t)g.l,
                                                (uint64_t)g.r, p.seed, p.round);
  if (p.debug) p.debug[g.seg_flat * p.max_seq + j] = key;
  return key;
}

// The persistent form's work counter: an int in the context's 256-byte
// counter block, past the moved-row counter (zeroed before each launch).
__host__ __device__ __forceinline__ int *sc_work_counter(const SelectCompactParams &p) {
  return reinterpret_cast<int *>(p.counters + 24);
}

// Persistent form of the order-preserving round for segments with more than
// 4096 candidates (one 512-thread CTA per SM, shared memory for up to 32768
// candidates and two block-table rows).  Each CTA takes its segments from a
// work counter, the list being ordered by decreasing candidate count
// (longest first), and prepares the keys of its next segment during the copy
// of the current one, so that the key draws (bound by the integer
// multiplier) overlap the copy (bound by HBM) and only the threshold and the
// ranks stay between two segments' copies:
//   - before chunk 0, cp.async brings the next segment's block-table row
//     (and, for beacon scores, the scores themselves) into shared memory;
//   - after chunk 0's barrier has made that row visible, cp.async brings the
//     position of every candidate (random selectors) into the keys buffer;
//   - from the next chunk on, between issuing the chunk's loads and its
//     barrier, each thread turns a share of the words it fetched itself into
//     keys (Philox draws, or the scores' order keys) and counts their top
//     bytes, so the threshold's first radix digit needs no pass of its own.
// No dependent global load sits between a chunk's loads and its stores, so
// the draws never wait behind the copy's loads in flight.  The keys buffer is
// free during the copy (the copy reads only src_of_rank), and the next
// segment's rows are disjoint from the current one's.  The block-table rows
// in shared memory also serve every row address of the copy.
template <int MODE, int kUnroll, int VAR>
__global__ void __launch_bounds__(512, 1)
    select_compact_pipe_kernel(SelectCompactParams p, int n_items, int keys_cap, int m_cap) {
  constexpr int NT = 512;
  // draws start at this chunk: scores arrive with the block-table row, the
  // positions of the random selectors one chunk later
  constexpr int kFirst = MODE == kModeScores ? 1 : 2;
  extern __shared__ __align__(16) uint8_t smem[];
  uint32_t *keys = reinterpret_cast<uint32_t *>(smem);                      // [keys_cap]
  uint16_t *src_of_rank = reinterpret_cast<uint16_t *>(keys + keys_cap);      // [m_cap]
  int32_t *bt_buf = reinterpret_cast<int32_t *>(src_of_rank + m_cap);         // [2][bt_stride]
  __shared__ ScScratch<NT> sh;

  const int tid = threadIdx.x;
  int *work = sc_work_counter(p);
  if (tid == 0) sh.next = atomicAdd(work, 1);
  __syncthreads();
  int cur = sh.next;
  if (cur >= n_items) return;
  ScSeg g = sc_seg(p, cur);
  int buf = 0;
  {
    const int pages = (g.P + g.N + kPage - 1) / kPage;
    for (int i = tid; i < pages; i += NT) bt_buf[i] = g.bt[i];
    for (int i = tid; i < 256; i += NT) sh.hist[i] = 0;
    g.bt = bt_buf;
    __syncthreads();
    for (int j = tid; j < g.N; j += NT) {
      const uint32_t key = sc_key<MODE>(p, g, j);
      keys[j] = key;
      atomicAdd(&sh.hist[key >> 24], 1u);
    }
  }

  const int vpr = p.row_bytes >> 4;  // 16-byte vectors per row
  const int rows_per_pass = NT / vpr;
  const int rows_per_chunk = rows_per_pass * kUnroll;
  const int my_row = tid / vpr, my_vec = tid - (tid / vpr) * vpr;
  const bool active = my_row < rows_per_pass;
  const int64_t rb = p.row_bytes;

#pragma unroll 1
  while (true) {
    if (tid == 0) sh.first_evicted = g.N;
    __syncthreads();  // the keys of g are complete
    const ScThreshold t = sc_threshold<NT, VAR>(p, g, keys, sh, true);
    sc_ordered_ranks<NT, VAR>(p, g, keys, t, src_of_rank, sh);
    const int q0 = sh.first_evicted;
    // the next item; every thread has read sh.next of the previous one and
    // sh.first_evicted of this one before the barrier.  The histogram is
    // free again: the next segment's draws count their top bytes into it
    if (tid == 0) sh.next = atomicAdd(work, 1);
    for (int i = tid; i < 256; i += NT) sh.hist[i] = 0;
    __syncthreads();
    const int nxt = sh.next;
    const bool more = nxt < n_items;
    ScSeg gn{};
    int nn = 0;
    int32_t *bt_next = bt_buf + (buf ^ 1) * p.bt_stride;
    if (more) {
      gn = sc_seg(p, nxt);
      nn = gn.N;
      const int pages = (gn.P + nn + kPage - 1) / kPage;
      for (int i = tid; i < pages; i += NT) cp_async4(bt_next + i, gn.bt + i);
      if (MODE == kModeScores) {
        const float *src = p.scores + gn.seg_flat * p.max_seq;
        for (int j = tid; j < nn; j += NT) cp_async4(keys + j, src + j);
      }
      cp_async_commit();
      gn.bt = bt_next;  // read only once chunk 0's barrier (or the tail's) has made it visible
    }
    // positions of the next segment's candidates (random selectors)
    auto fetch_positions = [&]() {
      if (MODE != kModeScores) {
        for (int j = tid; j < nn; j += NT) cp_async4(keys + j, p.pos_map + sc_row(p, gn, gn.P + j));
        cp_async_commit();
      }
    };
    const int M = g.M, P = g.P;
    const int nchunks = M > q0 ? (M - q0 + rows_per_chunk - 1) / rows_per_chunk : 0;
    const int per = nchunks > kFirst ? (nn + NT * (nchunks - kFirst) - 1) / (NT * (nchunks - kFirst)) : 0;
    int jn = tid;  // this thread's next key of the next segment
#pragma unroll 1
    for (int c = 0, base = q0; base < M; ++c, base += rows_per_chunk) {
      uint4 kr[kUnroll], vr[kUnroll];
      int pr[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int q = base + u * rows_per_pass + my_row;
        if (active && q < M) {
          const int64_t srow = sc_row(p, g, P + src_of_rank[q]);
          kr[u] = *reinterpret_cast<const uint4 *>(p.k_pool + srow * rb + my_vec * 16);
          vr[u] = *reinterpret_cast<const uint4 *>(p.v_pool + srow * rb + my_vec * 16);
          if (my_vec == 0) pr[u] = p.pos_map[srow];
        }
      }
      if (c == 0) {
        cp_async_wait_all();  // this thread's share of the row (and scores)
      } else if (c == 1) {
        fetch_positions();
      }
      if (c >= kFirst) {
        if (c == kFirst && MODE != kModeScores) cp_async_wait_all();
#pragma unroll 1
        for (int i = 0; i < per && jn < nn; ++i, jn += NT) {
          const uint32_t key = sc_key_from<MODE>(p, gn, jn, keys[jn]);
          keys[jn] = key;
          atomicAdd(&sh.hist[key >> 24], 1u);
        }
      }
      __syncthreads();  // every load of the chunk has landed before any store
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int q = base + u * rows_per_pass + my_row;
        if (active && q < M) {
          const int64_t drow = sc_row(p, g, P + q);
          *reinterpret_cast<uint4 *>(p.k_pool + drow * rb + my_vec * 16) = kr[u];
          *reinterpret_cast<uint4 *>(p.v_pool + drow * rb + my_vec * 16) = vr[u];
          if (my_vec == 0) p.pos_map[drow] = pr[u];
        }
      }
    }
    if (tid == 0 && M > q0) atomicAdd(p.counters, (unsigned long long)(M - q0));
    if (!more) break;
    // copies that the loop was too short to cover
    if (MODE != kModeScores && nchunks < 2) {
      if (nchunks == 0) {
        cp_async_wait_all();
        __syncthreads();  // the row is visible
      }
      fetch_positions();
    }
    cp_async_wait_all();
    for (; jn < nn; jn += NT) {
      const uint32_t key = sc_key_from<MODE>(p, gn, jn, keys[jn]);
      keys[jn] = key;
      atomicAdd(&sh.hist[key >> 24], 1u);
    }
    g = gn;
    buf ^= 1;
  }
}

template <int NT, int U, int MODE, int VAR>
cudaError_t launch_one(const SelectCompactParams &p, int n_seg_req, int keys_cap, size_t smem,
                       cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(select_compact_kernel<NT, MODE, U, VAR>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  select_compact_kernel<NT, MODE, U, VAR><<<(unsigned)(n_seg_req * p.layers * p.hkv), NT, smem, s>>>(
      p, keys_cap);
  return cudaGetLastError();
}

// Shared memory of the persistent form: keys, the rank map (sized by the
// launch's largest M) and two block-table rows.
inline size_t pipe_smem(const SelectCompactParams &p, int keys_cap, int m_cap) {
  return (size_t)keys_cap * sizeof(uint32_t) + (size_t)m_cap * sizeof(uint16_t) +
         (size_t)2 * p.bt_stride * sizeof(int32_t);
}
// The copy's loads in flight are staged in L1, which shares its storage with
// shared memory: past the 196 KB carve-out (this much dynamic shared memory,
// plus the static scratch and the 1 KB the runtime reserves per CTA) only
// 28 KB of L1 remain and the copy slows by about 15 % against the 60 KB that
// 196 KB leaves (measured), so larger launches take the one-CTA-per-segment
// kernel instead.
constexpr size_t kPipeSmemMax = 192 * 1024;

template <int MODE, int VAR>
cudaError_t launch_pipe(const SelectCompactParams &p, int n_seg_req, int keys_cap, int m_cap, cudaStream_t s) {
  auto kernel = select_compact_pipe_kernel<MODE, KVC_SC_UNROLL_LARGE, VAR>;
  const size_t smem = pipe_smem(p, keys_cap, m_cap);
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148, per_sm = 1;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, 512, smem)) != cudaSuccess) return e;
  const int n_items = n_seg_req * p.layers * p.hkv;
  const int grid = std::min(n_items, sms * std::max(per_sm, 1));
  if ((e = cudaMemsetAsync(sc_work_counter(p), 0, sizeof(int), s)) != cudaSuccess) return e;
  kernel<<<grid, 512, smem, s>>>(p, n_items, keys_cap, m_cap);
  return cudaGetLastError();
}

template <int NT, int U, int MODE>
cudaError_t launch_var(const SelectCompactParams &p, int var, int n_seg_req, int keys_cap, int m_cap,
                       size_t smem, cudaStream_t s) {
  // order-preserving rounds with more than 4096 candidates: the persistent
  // form where its shared memory leaves the copy enough L1
  const bool pipe = NT == 512 && pipe_smem(p, keys_cap, m_cap) <= kPipeSmemMax;
  switch (var) {
    case kOrderedSlotTie:
      if constexpr (NT == 512)
        if (pipe) return launch_pipe<MODE, kOrderedSlotTie>(p, n_seg_req, keys_cap, m_cap, s);
      return launch_one<NT, U, MODE, kOrderedSlotTie>(p, n_seg_req, keys_cap, smem, s);
    case kOrderedPosTie:
      if constexpr (NT == 512)
        if (pipe) return launch_pipe<MODE, kOrderedPosTie>(p, n_seg_req, keys_cap, m_cap, s);
      return launch_one<NT, U, MODE, kOrderedPosTie>(p, n_seg_req, keys_cap, smem, s);
    // hole filling moves few rows: a short copy chunk keeps registers low and
    // lets more CTAs per SM hide the latency of the select phase
    default: return launch_one<NT, KVC_SC_UNROLL_HOLE, MODE, kHoleFill>(p, n_seg_req, keys_cap, smem, s);
  }
}

template <int NT, int U>
cudaError_t launch_nt(const SelectCompactParams &p, int mode, int var, int n_seg_req, int max_n, int max_m,
                      cudaStream_t s) {
  const int keys_cap = (max_n + 7) & ~7;
  const int m_cap = (max_m + 7) & ~7;
  const size_t smem = (size_t)keys_cap * (sizeof(uint32_t) + sizeof(uint16_t));
  switch (mode) {
    case kModeRandom: return launch_var<NT, U, kModeRandom>(p, var, n_seg_req, keys_cap, m_cap, smem, s);
    case kModeRandomShared:
      return launch_var<NT, U, kModeRandomShared>(p, var, n_seg_req, keys_cap, m_cap, smem, s);
    default: return launch_var<NT, U, kModeScores>(p, var, n_seg_req, keys_cap, m_cap, smem, s);
  }
}

}  // namespace

cudaError_t launch_select_compact(const SelectCompactParams &p, int mode, int n_seg_req,
                                  int max_n, int max_m, cudaStream_t s) {
  if (n_seg_req <= 0) return cudaSuccess;
  const int var = (p.flags & kScHoleFill) ? kHoleFill : (p.flags & kScTieByPos) ? kOrderedPosTie : kOrderedSlotTie;
  if (max_n <= KVC_SC_NT256_MAX_N)
    return launch_nt<256, KVC_SC_UNROLL_SMALL>(p, mode, var, n_seg_req, max_n, max_m, s);
  return launch_nt<512, KVC_SC_UNROLL_LARGE>(p, mode, var, n_seg_req, max_n, max_m, s);
}

}  // namespace kvc
