// select_compact.cu -- one fused kernel per eviction round: score, select the
// top positions of every (request, layer, KV head) segment and compact the
// survivors in place.
//
// What it computes (Random Attention article, "Random Attention：不判断重要性，
// 只随机保留" and "发现四"): the prompt slots [0, P) are never candidates; the
// N = L - P generated slots are ranked by (score desc, original position asc),
// the best M stay and are packed, in their original order, into slots P,
// P+1, ...; K rows, V rows and the position map move together.  The score is
// the Philox draw of the (position, head, layer, request) counter for the
// random selectors, or the precomputed beacon score.
//
// Design (B200): one CTA per segment, everything between score and copy in
// shared memory.
//   1. score: each thread draws the 32-bit keys of a strided set of slots
//      (the random path reads only the 4-byte position map, never K/V);
//   2. select: 4-pass MSB radix select (8-bit digits, shared-memory
//      histogram) finds the M-th largest key tau and how many keys equal to
//      tau stay (the lowest slots among them, which hold the lowest
//      positions because slots are kept in position order);
//   3. ranks: tile-wise block scan of (key > tau, key == tau) with warp
//      ballots gives every survivor its destination rank; the inverse map
//      rank -> source slot is kept as uint16 in shared memory;
//   4. copy: survivors from the first evicted slot on move to slot P + rank.
//      Each chunk of ranks (8 rows per thread group, 64-128 KB of K and V in
//      flight per CTA) is read (16-byte vector loads, K and V rows plus
//      the position entry) into registers, the CTA synchronises, then writes.
//      A chunk only writes slots below its own highest source slot, and the
//      next chunk only reads slots above it, so one barrier per chunk makes
//      the in-place move safe while loads of chunk c+1 overlap stores of c.
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

__device__ __forceinline__ uint32_t float_order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <int NT>
__device__ __forceinline__ void block_radix_select(const uint32_t *keys, int n, int k_in,
                                                   uint32_t *hist, uint32_t *bcast,
                                                   uint32_t &tau, int &need) {
  // Finds the k_in-th largest key (1-based) and how many keys equal to it
  // belong to the top k_in.
  uint32_t prefix = 0, mask = 0;
  int k = k_in;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
#pragma unroll 1
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += NT) hist[i] = 0;
    __syncthreads();
    for (int j = tid; j < n; j += NT) {
      const uint32_t key = keys[j];
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
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
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (cum + c[i] >= (uint32_t)k) {
            digit = 255 - 8 * lane - i;
            break;
          }
          cum += c[i];
        }
        bcast[0] = (uint32_t)digit;
        bcast[1] = (uint32_t)k - cum;
      }
    }
    __syncthreads();
    prefix |= bcast[0] << shift;
    mask |= 255u << shift;
    k = (int)bcast[1];
    __syncthreads();
  }
  tau = prefix;
  need = k;
}

template <int NT, int MODE, int kUnroll>
__global__ void __launch_bounds__(NT) select_compact_kernel(SelectCompactParams p, int keys_cap) {
  extern __shared__ __align__(16) uint8_t smem[];
  uint32_t *keys = reinterpret_cast<uint32_t *>(smem);                  // [keys_cap]
  uint16_t *src_of_rank = reinterpret_cast<uint16_t *>(keys + keys_cap);  // [keys_cap]
  __shared__ uint32_t hist[256];
  __shared__ uint32_t bcast[2];
  __shared__ uint32_t warp_gt[NT / 32], warp_eq[NT / 32];
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
      key = philox4x64_10_word0_hi32((uint64_t)(int64_t)pos, head_field, (uint64_t)l,
                                     (uint64_t)r, p.seed, p.round);
      if (p.debug) p.debug[seg_flat * p.max_seq + j] = key;
    }
    keys[j] = key;
  }
  __syncthreads();

  // 2. threshold
  uint32_t tau;
  int need;
  block_radix_select<NT>(keys, N, M, hist, bcast, tau, need);

  // 3. ranks (tiles of NT slots in slot order)
  int carry_gt = 0, carry_eq = 0;
#pragma unroll 1
  for (int base = 0; base < N; base += NT) {
    const int j = base + tid;
    const bool valid = j < N;
    const uint32_t key = valid ? keys[j] : 0u;
    const bool gt = valid && key > tau;
    const bool eq = valid && key == tau;
    const unsigned mgt = __ballot_sync(0xffffffffu, gt);
    const unsigned meq = __ballot_sync(0xffffffffu, eq);
    const unsigned lt_mask = (1u << lane) - 1u;
    if (lane == 0) {
      warp_gt[warp] = __popc(mgt);
      warp_eq[warp] = __popc(meq);
    }
    __syncthreads();
    int off_gt = carry_gt, off_eq = carry_eq, tot_gt = 0, tot_eq = 0;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) {
      const int g = warp_gt[w], e = warp_eq[w];
      if (w < warp) {
        off_gt += g;
        off_eq += e;
      }
      tot_gt += g;
      tot_eq += e;
    }
    const int gt_before = off_gt + __popc(mgt & lt_mask);
    const int eq_before = off_eq + __popc(meq & lt_mask);
    const bool kept = gt || (eq && eq_before < need);
    if (kept) {
      const int rank = gt_before + min(eq_before, need);
      src_of_rank[rank] = (uint16_t)j;
    } else if (valid) {
      atomicMin(&first_evicted, j);
    }
    carry_gt += tot_gt;
    carry_eq += tot_eq;
    __syncthreads();  // warp_gt/warp_eq reuse
  }
  __syncthreads();

  // 4. in-place, order-preserving copy of ranks [first_evicted, M)
  const int q0 = first_evicted;
  const int vpr = p.row_bytes >> 4;  // 16-byte vectors per row
  const int rows_per_pass = NT / vpr;
  const int my_row = tid / vpr, my_vec = tid - (tid / vpr) * vpr;
  const bool active = my_row < rows_per_pass;
  const int64_t rb = p.row_bytes;
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
}

template <int NT, int U>
cudaError_t launch_nt(const SelectCompactParams &p, int mode, int n_seg_req, int max_n,
                      cudaStream_t s) {
  const int keys_cap = (max_n + 7) & ~7;
  const size_t smem = (size_t)keys_cap * (sizeof(uint32_t) + sizeof(uint16_t));
  const dim3 grid((unsigned)(n_seg_req * p.layers * p.hkv));
  cudaError_t e = cudaSuccess;
  switch (mode) {
    case kModeRandom:
      e = cudaFuncSetAttribute(select_compact_kernel<NT, kModeRandom, U>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e == cudaSuccess)
        select_compact_kernel<NT, kModeRandom, U><<<grid, NT, smem, s>>>(p, keys_cap);
      break;
    case kModeRandomShared:
      e = cudaFuncSetAttribute(select_compact_kernel<NT, kModeRandomShared, U>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e == cudaSuccess)
        select_compact_kernel<NT, kModeRandomShared, U><<<grid, NT, smem, s>>>(p, keys_cap);
      break;
    default:
      e = cudaFuncSetAttribute(select_compact_kernel<NT, kModeScores, U>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e == cudaSuccess)
        select_compact_kernel<NT, kModeScores, U><<<grid, NT, smem, s>>>(p, keys_cap);
      break;
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_select_compact(const SelectCompactParams &p, int mode, int n_seg_req,
                                  int max_n, int max_m, cudaStream_t s) {
  (void)max_m;
  if (n_seg_req <= 0) return cudaSuccess;
  if (max_n <= 4096) return launch_nt<256, KVC_SC_UNROLL_SMALL>(p, mode, n_seg_req, max_n, s);
  return launch_nt<512, KVC_SC_UNROLL_LARGE>(p, mode, n_seg_req, max_n, s);
}

}  // namespace kvc
