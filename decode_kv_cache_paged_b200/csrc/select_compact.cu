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
constexpr int kFinish = 64;

template <int NT, class KeyFn>
__device__ __forceinline__ void block_radix_select(int n, int k_in, KeyFn keyfn, uint32_t *hist,
                                                   uint32_t *bcast, uint32_t *cand, uint32_t &tau,
                                                   int &need, int &count_eq) {
  uint32_t prefix = 0, mask = 0;
  int k = k_in;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
#pragma unroll 1
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += NT) hist[i] = 0;
    __syncthreads();
    for (int j = tid; j < n; j += NT) {
      uint32_t key;
      if (keyfn(j, key) && (key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
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

template <int NT, int MODE, int kUnroll, int VAR>
__global__ void __launch_bounds__(NT) select_compact_kernel(SelectCompactParams p, int keys_cap) {
  extern __shared__ __align__(16) uint8_t smem[];
  uint32_t *keys = reinterpret_cast<uint32_t *>(smem);                  // [keys_cap]
  uint16_t *src_of_rank = reinterpret_cast<uint16_t *>(keys + keys_cap);  // [keys_cap]
  __shared__ uint32_t hist[256];
  __shared__ uint32_t bcast[4];
  __shared__ uint32_t cand[kFinish];
  __shared__ uint32_t warp_cnt[NT / 32], warp_eq[NT / 32];
  __shared__ int first_evicted;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int h = blockIdx.x % p.hkv;
  const int l = (blockIdx.x / p.hkv) % p.layers;
  const SegDesc sd = p.segs[blockIdx.x / (p.hkv * p.layers)];
  const int r = sd.req, P = sd.P, M = sd.M;
  const int N = sd.L - P;
  const int32_t *bt = p.block_table + (int64_t)r * p.bt_stride;
  const int64_t layer_page0 = (int64_t)l * p.num_pages;
  const int64_t seg_flat = ((int64_t)r * p.layers + l) * p.hkv + h;
  // global row index (also the position-map index) of slot s of this segment
  auto row_of = [&](int s) -> int64_t {
    return ((layer_page0 + bt[s >> 4]) * p.hkv + h) * kPage + (s & (kPage - 1));
  };

  // 1. keys
  if (tid == 0) first_evicted = N;
  const uint64_t head_field = (MODE == kModeRandomShared) ? ~0ull : (uint64_t)h;
  for (int j = tid; j < N; j += NT) {
    uint32_t key;
    if (MODE == kModeScores) {
      key = float_order_key(p.scores[seg_flat * p.max_seq + j]);
    } else {
      const int pos = p.pos_map[row_of(P + j)];
      key = philox4x64_10_word0_hi32((uint64_t)(int64_t)(pos / p.block), head_field, (uint64_t)l,
                                     (uint64_t)r, p.seed, p.round);
      if (p.debug) p.debug[seg_flat * p.max_seq + j] = key;
    }
    keys[j] = key;
  }
  __syncthreads();

  // 2. threshold
  uint32_t tau;
  int need, count_eq;
  block_radix_select<NT>(
      N, M, [&](int j, uint32_t &k) { k = keys[j]; return true; }, hist, bcast, cand, tau, need, count_eq);
  // with ties split and slots possibly out of position order: the `need`
  // lowest positions among the tied keys (positions are distinct)
  uint32_t ptau = 0;
  const bool split_by_pos = VAR != kOrderedSlotTie && need < count_eq;
  if (split_by_pos) {
    int need2, cnt2;
    block_radix_select<NT>(
        N, need,
        [&](int j, uint32_t &k) {
          if (keys[j] != tau) return false;
          k = ~(uint32_t)p.pos_map[row_of(P + j)];
          return true;
        },
        hist, bcast, cand, ptau, need2, cnt2);
  }
  auto kept_pos = [&](int j) -> bool {  // kept flag when ties go by position
    const uint32_t key = keys[j];
    if (key != tau) return key > tau;
    if (!split_by_pos) return true;
    return ~(uint32_t)p.pos_map[row_of(P + j)] >= ptau;
  };

  const int vpr = p.row_bytes >> 4;  // 16-byte vectors per row
  const int rows_per_pass = NT / vpr;
  const int my_row = tid / vpr, my_vec = tid - (tid / vpr) * vpr;
  const bool active = my_row < rows_per_pass;
  const int64_t rb = p.row_bytes;

  if (VAR != kHoleFill) {
    // 3. ranks in slot order
    if (VAR == kOrderedSlotTie) {
      // kept = key > tau, or key == tau among the first `need` such slots:
      // two counts per candidate (greater, equal) scanned over warp ranges
      constexpr int NW = NT / 32;
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
        warp_cnt[warp] = cgt;
        warp_eq[warp] = ceq;
      }
      __syncthreads();
      int off_gt = 0, off_eq = 0;
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        if (w < warp) {
          off_gt += warp_cnt[w];
          off_eq += warp_eq[w];
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
          atomicMin(&first_evicted, j);
        }
        off_gt += __popc(mgt);
        off_eq += __popc(meq);
      }
    } else {
      block_scan_each<NT>(
          0, N, [&](int j) { return kept_pos(j); },
          [&](int j, int rank) { src_of_rank[rank] = (uint16_t)j; }, warp_cnt);
      for (int j = tid; j < N; j += NT)
        if (!kept_pos(j)) atomicMin(&first_evicted, j);
    }
    __syncthreads();

    // 4. in-place, order-preserving copy of ranks [first_evicted, M)
    const int q0 = first_evicted;
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
          const int64_t srow = row_of(P + src_of_rank[q]);
          drow[u] = row_of(P + q);
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
        0, M, [&](int j) { return !kept_pos(j); },
        [&](int j, int i) { src_of_rank[i] = (uint16_t)j; }, warp_cnt);
    block_scan_each<NT>(
        M, N, [&](int j) { return kept_pos(j); },
        [&](int j, int i) { src_of_rank[M + i] = (uint16_t)j; }, warp_cnt);
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
          const int64_t srow = row_of(P + src_of_rank[M + i]);
          drow[u] = row_of(P + src_of_rank[i]);
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

template <int NT, int U, int MODE>
cudaError_t launch_var(const SelectCompactParams &p, int var, int n_seg_req, int keys_cap, size_t smem,
                       cudaStream_t s) {
  switch (var) {
    case kOrderedSlotTie: return launch_one<NT, U, MODE, kOrderedSlotTie>(p, n_seg_req, keys_cap, smem, s);
    case kOrderedPosTie: return launch_one<NT, U, MODE, kOrderedPosTie>(p, n_seg_req, keys_cap, smem, s);
    // hole filling moves few rows: a short copy chunk keeps registers low and
    // lets more CTAs per SM hide the latency of the select phase
    default: return launch_one<NT, KVC_SC_UNROLL_HOLE, MODE, kHoleFill>(p, n_seg_req, keys_cap, smem, s);
  }
}

template <int NT, int U>
cudaError_t launch_nt(const SelectCompactParams &p, int mode, int var, int n_seg_req, int max_n,
                      cudaStream_t s) {
  const int keys_cap = (max_n + 7) & ~7;
  const size_t smem = (size_t)keys_cap * (sizeof(uint32_t) + sizeof(uint16_t));
  switch (mode) {
    case kModeRandom: return launch_var<NT, U, kModeRandom>(p, var, n_seg_req, keys_cap, smem, s);
    case kModeRandomShared: return launch_var<NT, U, kModeRandomShared>(p, var, n_seg_req, keys_cap, smem, s);
    default: return launch_var<NT, U, kModeScores>(p, var, n_seg_req, keys_cap, smem, s);
  }
}

}  // namespace

cudaError_t launch_select_compact(const SelectCompactParams &p, int mode, int n_seg_req,
                                  int max_n, int max_m, cudaStream_t s) {
  (void)max_m;
  if (n_seg_req <= 0) return cudaSuccess;
  const int var = (p.flags & kScHoleFill) ? kHoleFill : (p.flags & kScTieByPos) ? kOrderedPosTie : kOrderedSlotTie;
  if (max_n <= KVC_SC_NT256_MAX_N) return launch_nt<256, KVC_SC_UNROLL_SMALL>(p, mode, var, n_seg_req, max_n, s);
  return launch_nt<512, KVC_SC_UNROLL_LARGE>(p, mode, var, n_seg_req, max_n, s);
}

}  // namespace kvc
