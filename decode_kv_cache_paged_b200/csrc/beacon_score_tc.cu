// beacon_score_tc.cu -- BeaconKV beacon score on the 5th-generation tensor
// cores (tcgen05) for bf16 caches with head_dim 128.
//
// Score (the library's definition; the BeaconKV explainer, §3.2, leaves the
// importance rule open): z_bj = c_b.k_j/sqrt(d), lse_b = log sum_j exp(z_bj)
// over every cached key j < L, score_j = max_b exp(z_bj - lse_b) for the
// generated keys j in [P, L).  The contraction c_b.k_j is bf16 x bf16 with
// fp32 accumulation; with 64+ beacons it carries 64+ flop per key byte, above
// what the SIMT pipes sustain at HBM speed, so it runs on tcgen05.mma with
// the accumulators in tensor memory (TMEM).
//
// Structure: a persistent kernel, one CTA per SM, walking its segments
// (request, layer, KV head) and, per segment, the 128-key tiles of the key
// sequence twice:
//   pass 1 (all tiles): D1[b, j] = C K^T with the beacons on TMEM lanes
//          (A = beacons, M = 128 rows per MMA, two MMAs for B > 128) and 128
//          keys on columns; each epilogue thread owns one beacon row and keeps
//          an online (max, sum of 2^u) over its columns;
//   pass 2 (tiles holding generated keys): D2[j, b] = K C^T with the keys on
//          lanes (A = keys, M = 128, N = B); each epilogue thread owns one key
//          and takes the max over beacon columns of u_bj - lse2_b.
// Work in base 2: u = z_raw * log2(e)/sqrt(d), lse2 = log2 sum 2^u, score =
// 2^(max_b u_bj - lse2_b).
// Warp roles: warp 0 allocates TMEM and issues the TMA loads (128-byte
// swizzle, page ids loaded one tile ahead): a tile whose 8 page ids are
// consecutive comes in as two 4-D boxes (64 columns x 16 rows x 8 pages of
// one head, the pool seen as columns, rows, heads, layer * pages); any other
// tile as one 2-D box per (page, 64-column half), lane q of the warp taking
// page q (a page holds 16 keys x 256 B contiguous; that map covers the pool
// as rows of 128 bf16).  The number of boxes, not their bytes, limited the
// key stream; warp 1 issues the MMAs (one elected lane) and commits them to
// mbarriers; warps 2-9 run the epilogue in two groups of four, group g taking
// the tiles whose accumulator is in TMEM buffers of parity g (tcgen05.ld of
// 64 columns at a time; sums and maxima in 8 independent partials; the
// per-beacon partial (max, sum) of the groups merged once per segment).
// Pass 1 adds a full 64-column chunk as sum 2^(u - m) against the running
// reference m with no max pass first; only a chunk whose sum would pass
// 2^64 (a new maximum far above m) or a partial chunk takes the max-then-
// rescale step.  Key tiles rotate through 4 shared-memory stages; the
// accumulators through four 128-column TMEM buffers (at most 128 beacons)
// or two of 256.  No load uses cluster multicast.
// Every mbarrier wait is bounded (2 s of %globaltimer): on expiry the kernel
// records KVC_ERR_DEVICE_TIMEOUT in the status word, the other roles see the
// abort flag and leave, and TMEM is released before the CTA exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "kvc_internal.h"
#include "tc_ptx.cuh"

#ifndef KVC_TC_NCB_SMALL
#define KVC_TC_NCB_SMALL 2
#endif
#ifndef KVC_TC_STAGES_SMALL
#define KVC_TC_STAGES_SMALL 4
#endif

namespace kvc {
namespace {

constexpr int kTileKeys = 128;
constexpr int kEpiWarps = 8;   // two groups of 4: group g drains accumulator buffer g
constexpr int kThreads = 64 + 32 * kEpiWarps;  // warp 0 TMA, warp 1 MMA, warps 2-9 epilogue
constexpr uint32_t kTmemCols = 512;

struct TcParams {
  const int32_t *block_table;
  const SegDesc *segs;
  float *scores;
  float *lse_out;
  const float *trig;  // cluster-trigger shares [seg][B], or null for the max rule
  int32_t *status;
  int64_t num_pages;
  int32_t bt_stride, layers, hkv, B, max_seq, n_segs;
  float alpha;  // log2(e) / sqrt(d)
};

// Per-segment geometry shared by every role.
struct SegGeom {
  int r, l, h, L, P;
  int64_t seg_flat;
  int n1, t2, n2;  // pass-1 tiles, first pass-2 tile, pass-2 tiles
  int nres;        // pass-2 tiles still resident in their pass-1 stages
  // tile index of item t of the segment's sequence: pass 1 in order, then
  // pass 2 starting with the resident tiles (the last nres of pass 1), then
  // the remaining generated tiles from the last down, so that the tiles pass
  // 1 loaded most recently, the likeliest to still be in L2, come first
  __device__ __forceinline__ int tile_of(int t) const {
    if (t < n1) return t;
    const int u = t - n1;
    return u < nres ? n1 - nres + u : n1 - 1 - u;
  }
};
template <int S>
__device__ __forceinline__ SegGeom seg_geom(const TcParams &p, int s) {
  SegGeom g;
  g.h = s % p.hkv;
  g.l = (s / p.hkv) % p.layers;
  const SegDesc sd = p.segs[s / (p.hkv * p.layers)];
  g.r = sd.req;
  g.L = sd.L;
  g.P = sd.P;
  g.seg_flat = ((int64_t)g.r * p.layers + g.l) * p.hkv + g.h;
  g.n1 = (g.L + kTileKeys - 1) / kTileKeys;
  g.t2 = g.P / kTileKeys;
  g.n2 = g.n1 - g.t2;
  // item n1 + k lands in the stage that held pass-1 item n1 + k - S, i.e. the
  // tile n1 - S + k, exactly when S pass-2 items reuse the last S pass-1 tiles
  g.nres = (g.n1 >= S && g.n2 >= S) ? S : 0;
  return g;
}

// 4-D tiled load (no multicast): the key pool seen as (128 columns, 16 rows,
// KV heads, layer * pages + page), so one box brings the same 64 columns of 8
// consecutive page ids' 16 rows of one head
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap *map, int x, int y, int z, int w,
                                            uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z), "r"(w)
      : "memory");
}

template <int CROWS, int NCB, int kStages>
__global__ void __launch_bounds__(kThreads, 1)
    beacon_score_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap cmap,
                           const __grid_constant__ CUtensorMap kmap4, TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_align<1024>(smem_raw);
  constexpr uint32_t kCBytes = CROWS * 256;          // beacon tile: CROWS rows x 128 bf16
  constexpr uint32_t kTileBytes = kTileKeys * 256;   // 32 KB
  // TMEM accumulator buffers: 4 of 128 columns when a tile's products fit in
  // 128 columns (at most 128 beacons), else 2 of 256; the epilogue group g
  // drains the buffers b with b % 2 == g
  constexpr int NACC = CROWS <= 128 ? 4 : 2;
  constexpr uint32_t ACOLS = kTmemCols / NACC;
  uint8_t *cbuf = smem;                              // [NCB][2 K-halves][CROWS][128 B]
  uint8_t *kbuf = smem + NCB * kCBytes;              // [kStages][2][128][128 B]
  uint64_t *bars = reinterpret_cast<uint64_t *>(kbuf + kStages * kTileBytes);
  uint64_t *full = bars, *empty = bars + kStages;
  uint64_t *acc_full = bars + 2 * kStages, *acc_empty = acc_full + NACC;
  uint64_t *c_full = acc_empty + NACC, *c_empty = c_full + 2, *mma_done = c_empty + 2;
  uint64_t *epi_bar = mma_done + 1;  // the 4 epilogue warps, once per segment
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(epi_bar + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  float *lse2 = reinterpret_cast<float *>(tmem_slot + 4);  // [2][256]
  float *part = lse2 + 512;                                 // [4][2][256] partial (m, sum)
  float *wts2 = part + 4 * 2 * 256;                         // [2][256] trigger shares

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < NACC; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&c_full[i], 1);
      mbar_init(&c_empty[i], 1);
    }
    mbar_init(mma_done, 1);
    mbar_init(epi_bar, kEpiWarps);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tmem_fence_before();
  __syncthreads();
  tmem_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int B = p.B;
  // With 64 beacons or fewer the tile holds two copies of them (rows 0-63 and
  // 64-127) so that all four epilogue warps share pass 1, each copy taking
  // half of the key columns.
  const bool dup = B <= 64;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    // The whole warp walks the tile sequence in step (waits by lane 0,
    // results and the abort flag broadcast); lane q issues the two loads of
    // page q of each tile, so a tile's 16 loads leave in one instruction.
    constexpr int kTP = kTileKeys / kPage;
    auto uniform_abort = [&]() { return __shfl_sync(0xffffffffu, lane == 0 ? *abort_flag : 0, 0) != 0; };
    uint32_t it = 0;  // key-tile counter across segments
    int si = 0;       // local segment counter
    for (int s = blockIdx.x; s < p.n_segs; s += gridDim.x, ++si) {
      if (uniform_abort()) break;
      const SegGeom g = seg_geom<kStages>(p, s);
      const int cb = si % NCB;
      if (!warp_wait(&c_empty[cb], ((si / NCB) & 1) ^ 1, abort_flag, p.status)) break;
      if (lane == 0) {
        mbar_expect_tx(&c_full[cb], (uint32_t)B * 256u * (dup ? 2u : 1u));
        const int crow = (int)(g.seg_flat * B);
        for (int copy = 0; copy < (dup ? 2 : 1); ++copy) {
          uint8_t *cdst = cbuf + cb * kCBytes + copy * 64 * 128;
          tma_load_2d(smem_u32(cdst), &cmap, 0, crow, &c_full[cb]);
          tma_load_2d(smem_u32(cdst + CROWS * 128), &cmap, 64, crow, &c_full[cb]);
        }
      }
      const int32_t *bt = p.block_table + (int64_t)g.r * p.bt_stride;
      const int pages = (g.L + kPage - 1) / kPage;
      // this lane's page id of a tile (lanes >= 8 idle), loaded one tile ahead
      auto page_of = [&](int tile) { const int pg = tile * kTP + lane; return (lane < kTP && pg < pages) ? __ldg(bt + pg) : 0; };
      int pg_cur = page_of(g.tile_of(0));
      const int n_items = g.n1 + g.n2;
      bool ok = true;
      for (int t = 0; t < n_items; ++t, ++it) {
        if (uniform_abort()) {
          ok = false;
          break;
        }
        const int tile = g.tile_of(t);
        const int pg_next = (t + 1 < n_items) ? page_of(g.tile_of(t + 1)) : 0;
        const int st = it % kStages;
        if (!warp_wait(&empty[st], ((it / kStages) & 1) ^ 1, abort_flag, p.status)) {
          ok = false;
          break;
        }
        if (t >= g.n1 && t - g.n1 < g.nres) {
          if (lane == 0) mbar_arrive(&full[st]);  // the tile is still in this stage from pass 1
        } else {
          const int npg = min(kTP, pages - tile * kTP);
          if (lane == 0) mbar_expect_tx(&full[st], (uint32_t)npg * 2u * 2048u);
          __syncwarp();
          // a full tile whose 8 page ids are consecutive: two 4-D boxes (8
          // pages x 16 rows x 64 columns, the same 16 KB layout) instead of
          // 16 page boxes
          const int pg_first = __shfl_sync(0xffffffffu, pg_cur, 0);
          const bool run = npg == kTP && __all_sync(0xffffffffu, lane >= kTP || pg_cur == pg_first + lane);
          if (run) {
            if (lane < 2)
              tma_load_4d(smem_u32(kbuf + st * kTileBytes + lane * kTileKeys * 128), &kmap4, lane * 64, 0, g.h,
                          (int)(g.l * p.num_pages) + pg_first, &full[st]);
          } else if (lane < npg) {
            uint8_t *dst = kbuf + st * kTileBytes;
            const int64_t row = (((int64_t)g.l * p.num_pages + pg_cur) * p.hkv + g.h) * kPage;
            tma_load_2d(smem_u32(dst + lane * 2048), &kmap, 0, (int)row, &full[st]);
            tma_load_2d(smem_u32(dst + kTileKeys * 128 + lane * 2048), &kmap, 64, (int)row, &full[st]);
          }
        }
        __syncwarp();
        pg_cur = pg_next;
      }
      if (!ok) break;
    }
    if (lane == 0 && *abort_flag) {
      // let loads already issued land before the CTA's shared memory goes away
      for (int i = 0; i < kStages && it > 0; ++i) {
        const uint32_t k = it - 1 - i;
        mbar_wait(&full[k % kStages], (k / kStages) & 1, abort_flag, p.status, false);
        if (k == 0) break;
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------- MMA issuer
    if (lane == 0) {
      uint32_t it = 0, acc_it = 0;
      int si = 0;
      const uint32_t idesc1 = idesc_bf16_f32(128, kTileKeys);
      const uint32_t idesc2 = idesc_bf16_f32(128, B);
      bool ok = true;
      for (int s = blockIdx.x; s < p.n_segs && ok; s += gridDim.x, ++si) {
        const SegGeom g = seg_geom<kStages>(p, s);
        const int cb = si % NCB;
        ok = mbar_wait(&c_full[cb], (si / NCB) & 1, abort_flag, p.status);
        if (!ok) break;
        const uint32_t c_addr = smem_u32(cbuf + cb * kCBytes);
        for (int t = 0; t < g.n1 + g.n2; ++t, ++it, ++acc_it) {
          const int st = it % kStages, buf = acc_it % NACC;
          ok = mbar_wait(&full[st], (it / kStages) & 1, abort_flag, p.status) &&
               mbar_wait(&acc_empty[buf], ((acc_it / NACC) & 1) ^ 1, abort_flag, p.status);
          if (!ok) break;
          tmem_fence_after();
          const uint32_t k_addr = smem_u32(kbuf + st * kTileBytes);
          const uint32_t d = tmem_base + buf * ACOLS;
          if (t < g.n1) {
            for (int half = 0; half * 128 < B; ++half)
              for (int kb = 0; kb < 2; ++kb)
                for (int ks = 0; ks < 4; ++ks) {
                  const uint64_t a = sw128_desc(c_addr + kb * CROWS * 128 + half * 128 * 128 + ks * 32);
                  const uint64_t b = sw128_desc(k_addr + kb * kTileKeys * 128 + ks * 32);
                  umma(d + half * 128, a, b, idesc1, (kb | ks) != 0);
                }
          } else {
            for (int kb = 0; kb < 2; ++kb)
              for (int ks = 0; ks < 4; ++ks) {
                const uint64_t a = sw128_desc(k_addr + kb * kTileKeys * 128 + ks * 32);
                const uint64_t b = sw128_desc(c_addr + kb * CROWS * 128 + ks * 32);
                umma(d, a, b, idesc2, (kb | ks) != 0);
              }
          }
          umma_commit(&empty[st]);
          umma_commit(&acc_full[buf]);
        }
        if (!ok) break;
        umma_commit(&c_empty[cb]);
      }
      umma_commit(mma_done);
      mbar_wait(mma_done, 0, abort_flag, p.status, false);
    }
  } else {
    // ---------------------------------------------------------- epilogue
    // Group grp (warps 2-5 or 6-9) handles the tiles whose accumulator sits
    // in buffer grp, i.e. every other tile; each warp reads the TMEM lane
    // quarter (warp % 4) it may access.
    const int ew = warp - 2, grp = ew >> 2;
    const int q = warp & 3;                 // TMEM lane quarter of this warp
    const int row = q * 32 + lane;          // TMEM lane = D row
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    const int copy = dup ? (row >> 6) : 0;  // warp-uniform
    const int col_lo = dup ? copy * 64 : 0, ncols = dup ? 64 : kTileKeys;
    const int nslot = dup ? 4 : 2;          // partials per beacon: groups x copies
    const int slot = grp * (dup ? 2 : 1) + copy;
    const float alpha = p.alpha;
    uint32_t acc_it = 0, epi_ph = 0;
    int si = 0;
    bool ok = true;
    for (int s = blockIdx.x; s < p.n_segs && ok; s += gridDim.x, ++si) {
      const SegGeom g = seg_geom<kStages>(p, s);
      float *lse_buf = lse2 + (si & 1) * 256;
      float *w_buf = wts2 + (si & 1) * 256;
      // pass 1: per-beacon online log2-sum-exp2 over this group's tiles
      float m0 = -INFINITY, s0 = 0.f, m1 = -INFINITY, s1 = 0.f;
      for (int t = 0; t < g.n1; ++t, ++acc_it) {
        const int buf = acc_it % NACC;
        if ((buf & 1) != grp) continue;
        ok = warp_wait(&acc_full[buf], (acc_it / NACC) & 1, abort_flag, p.status);
        if (!ok) break;
        tmem_fence_after();
        const int nvalid = min(kTileKeys, g.L - t * kTileKeys);
        const int nhalf = (B + 127) / 128;
        for (int half = 0; half < nhalf; ++half) {
          const int b = half * 128 + (dup ? (row & 63) : row);
          const bool mine = b < B;
          float &m = half ? m1 : m0;
          float &sum = half ? s1 : s0;
          for (int c0 = col_lo; c0 < col_lo + ncols; c0 += 64) {
            float v[64];
            tmem_ld64(tmem_base + lane_addr + buf * ACOLS + half * 128 + c0, v);
            if (half == nhalf - 1 && c0 + 64 >= col_lo + ncols) {
              // the tile's last load has landed in registers: hand the
              // buffer back to the MMA warp before the arithmetic
              tmem_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&acc_empty[buf]);
            }
            const int nv = min(64, nvalid - c0);
            if (!mine || nv <= 0) continue;
            if (nv == 64 && m != -INFINITY) {
              // full chunk against the running reference m, with no max
              // pass: sum stays sum_j 2^(u_j - m) whether or not u_j <= m,
              // and a chunk sum within 2^64 cannot lose the total to
              // overflow; a larger one (a new maximum far above m, or a
              // NaN) takes the exact path below
              // (two-wide packed FMA and add: the rounding of two scalar ops)
              float2 ps[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) ps[i] = make_float2(0.f, 0.f);
              const float2 a2 = make_float2(alpha, alpha), nm2 = make_float2(-m, -m);
#pragma unroll
              for (int i = 0; i < 64; i += 2) {
                const float2 t = __ffma2_rn(make_float2(v[i], v[i + 1]), a2, nm2);
                ps[(i >> 1) & 3] = __fadd2_rn(ps[(i >> 1) & 3], make_float2(exp2f(t.x), exp2f(t.y)));
              }
              const float cs = ((ps[0].x + ps[0].y) + (ps[1].x + ps[1].y)) + ((ps[2].x + ps[2].y) + (ps[3].x + ps[3].y));
              if (cs <= 0x1p64f) {
                sum += cs;
                continue;
              }
            }
            float mx[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) mx[i] = -INFINITY;
#pragma unroll
            for (int i = 0; i < 64; ++i)
              if (i < nv) mx[i & 7] = fmaxf(mx[i & 7], v[i]);
            const float cm = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                   fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) * alpha;
            if (cm > m) {
              sum *= exp2f(m - cm);
              m = cm;
            }
            float ps[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) ps[i] = 0.f;
#pragma unroll
            for (int i = 0; i < 64; ++i)
              if (i < nv) ps[i & 7] += exp2f(fmaf(v[i], alpha, -m));
            sum += ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
          }
        }
      }
      if (!ok) break;
      // merge the partial (max, sum) of each beacon over groups and copies
      for (int half = 0; half * 128 < B; ++half) {
        const int b = half * 128 + (dup ? (row & 63) : row);
        if (b < B) {
          part[(slot * 2 + 0) * 256 + b] = half ? m1 : m0;
          part[(slot * 2 + 1) * 256 + b] = half ? s1 : s0;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(epi_bar);
      ok = warp_wait(epi_bar, epi_ph & 1, abort_flag, p.status);
      ++epi_ph;
      if (!ok) break;
      if (slot == 0) {
        for (int half = 0; half * 128 < B; ++half) {
          const int b = half * 128 + row;
          if (b < B) {
            float mm = -INFINITY;
            for (int k = 0; k < nslot; ++k) mm = fmaxf(mm, part[(k * 2) * 256 + b]);
            float ss = 0.f;
            for (int k = 0; k < nslot; ++k) {
              const float pm = part[(k * 2) * 256 + b];
              if (pm != -INFINITY) ss += part[(k * 2 + 1) * 256 + b] * exp2f(pm - mm);
            }
            const float l2 = mm + log2f(ss);
            lse_buf[b] = -l2;  // negated: pass 2 adds it in one packed FMA
            if (p.trig) w_buf[b] = p.trig[g.seg_flat * B + b];
            if (p.lse_out) p.lse_out[g.seg_flat * B + b] = l2 * 0.69314718055994531f;
            if (l2 != l2) atomicCAS(p.status, kDevOk, kDevNaN);
          }
        }
      }
      // every beacon's lse is in shared memory before any thread reads it
      __syncwarp();
      if (lane == 0) mbar_arrive(epi_bar);
      ok = warp_wait(epi_bar, epi_ph & 1, abort_flag, p.status);
      ++epi_ph;
      if (!ok) break;
      // pass 2: per-key max over beacons of u - lse2 (this group's tiles)
      for (int t = 0; t < g.n2; ++t, ++acc_it) {
        const int buf = acc_it % NACC;
        if ((buf & 1) != grp) continue;
        ok = warp_wait(&acc_full[buf], (acc_it / NACC) & 1, abort_flag, p.status);
        if (!ok) break;
        tmem_fence_after();
        float bm[8];
        const bool trig = p.trig != nullptr;
        const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
        for (int i = 0; i < 8; ++i) bm[i] = trig ? 0.f : -INFINITY;
        for (int c0 = 0; c0 < B; c0 += 64) {
          float v[64];
          tmem_ld64(tmem_base + lane_addr + buf * ACOLS + c0, v);
          if (c0 + 64 >= B) {  // the tile's last load: hand the buffer back
            tmem_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[buf]);
          }
          const float4 *l4 = reinterpret_cast<const float4 *>(lse_buf + c0);
          if (trig) {
            // cluster trigger: sum over beacons of share_b * 2^(u_bj - lse2_b)
            const float4 *w4 = reinterpret_cast<const float4 *>(w_buf + c0);
#pragma unroll
            for (int i4 = 0; i4 < 16; ++i4) {
              const float4 L4 = l4[i4], W4 = w4[i4];
              const float2 t01 = __ffma2_rn(make_float2(v[4 * i4], v[4 * i4 + 1]), a2, make_float2(L4.x, L4.y));
              const float2 t23 = __ffma2_rn(make_float2(v[4 * i4 + 2], v[4 * i4 + 3]), a2, make_float2(L4.z, L4.w));
              bm[(4 * i4) & 7] = fmaf(W4.x, exp2f(t01.x), bm[(4 * i4) & 7]);
              bm[(4 * i4 + 1) & 7] = fmaf(W4.y, exp2f(t01.y), bm[(4 * i4 + 1) & 7]);
              bm[(4 * i4 + 2) & 7] = fmaf(W4.z, exp2f(t23.x), bm[(4 * i4 + 2) & 7]);
              bm[(4 * i4 + 3) & 7] = fmaf(W4.w, exp2f(t23.y), bm[(4 * i4 + 3) & 7]);
            }
          } else {
#pragma unroll
            for (int i4 = 0; i4 < 16; ++i4) {
              const float4 L4 = l4[i4];
              const float2 t01 = __ffma2_rn(make_float2(v[4 * i4], v[4 * i4 + 1]), a2, make_float2(L4.x, L4.y));
              const float2 t23 = __ffma2_rn(make_float2(v[4 * i4 + 2], v[4 * i4 + 3]), a2, make_float2(L4.z, L4.w));
              bm[(4 * i4) & 7] = fmaxf(bm[(4 * i4) & 7], t01.x);
              bm[(4 * i4 + 1) & 7] = fmaxf(bm[(4 * i4 + 1) & 7], t01.y);
              bm[(4 * i4 + 2) & 7] = fmaxf(bm[(4 * i4 + 2) & 7], t23.x);
              bm[(4 * i4 + 3) & 7] = fmaxf(bm[(4 * i4 + 3) & 7], t23.y);
            }
          }
        }
        const int j = g.tile_of(g.n1 + t) * kTileKeys + row;
        if (j >= g.P && j < g.L) {
          const float sc =
              trig ? ((bm[0] + bm[1]) + (bm[2] + bm[3])) + ((bm[4] + bm[5]) + (bm[6] + bm[7]))
                   : exp2f(fmaxf(fmaxf(fmaxf(bm[0], bm[1]), fmaxf(bm[2], bm[3])),
                                 fmaxf(fmaxf(bm[4], bm[5]), fmaxf(bm[6], bm[7]))));
          if (sc != sc) atomicCAS(p.status, kDevOk, kDevNaN);
          p.scores[g.seg_flat * p.max_seq + (j - g.P)] = sc;
        }
      }
    }
  }
  tmem_fence_before();
  __syncthreads();
  if (warp == 0) {
    tmem_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols));
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// rows x 128 bf16, row stride 256 B, box (64 columns, box_rows rows), 128-byte swizzle
bool make_map(CUtensorMap *m, const void *base, uint64_t rows, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {128, rows};
  cuuint64_t strides[1] = {256};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// the same pool as (128 columns, 16 rows, hkv heads, layers * pages), box
// (64 columns, 16 rows, 1 head, 8 pages), 128-byte swizzle
bool make_map4(CUtensorMap *m, const void *base, uint64_t layer_pages, uint32_t hkv) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {128, kPage, hkv, layer_pages};
  cuuint64_t strides[3] = {256, (cuuint64_t)kPage * 256, (cuuint64_t)hkv * kPage * 256};
  cuuint32_t box[4] = {64, kPage, 1, kTileKeys / kPage};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int CROWS, int NCB, int kStages>
cudaError_t launch(const CUtensorMap &km, const CUtensorMap &cm, const CUtensorMap &km4, const TcParams &tp,
                   cudaStream_t s) {
  const size_t smem = 1024 + (size_t)NCB * CROWS * 256 + (size_t)kStages * kTileKeys * 256 + 256 +
                      2 * 256 * 4 + 4 * 2 * 256 * 4 + 2 * 256 * 4;
  cudaError_t e = cudaFuncSetAttribute(beacon_score_tc_kernel<CROWS, NCB, kStages>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = tp.n_segs < sms ? tp.n_segs : sms;
  beacon_score_tc_kernel<CROWS, NCB, kStages><<<grid, kThreads, smem, s>>>(km, cm, km4, tp);
  return cudaGetLastError();
}

}  // namespace

bool beacon_score_tc_supported(int d, int B, int dtype) {
  return dtype == KVC_BF16 && d == 128 && B >= 64 && B <= 256 && B % 64 == 0 && encode_fn() != nullptr;
}

cudaError_t launch_beacon_score_tc(const BeaconScoreParams &p, int n_req, int max_l, cudaStream_t s) {
  (void)max_l;
  if (!beacon_score_tc_supported(p.d, p.B, p.dtype)) return cudaErrorNotSupported;
  if (n_req <= 0) return cudaSuccess;
  CUtensorMap km, cm, km4;
  const uint64_t krows = (uint64_t)p.layers * (uint64_t)p.num_pages * (uint64_t)p.hkv * kPage;
  // the beacon map spans every (request, layer, head) segment's B rows
  const uint64_t crows = (uint64_t)p.total_segs * (uint64_t)p.B;
  if (krows >= (1ull << 31) || crows >= (1ull << 31)) return cudaErrorInvalidValue;
  if (!make_map(&km, p.k_pool, krows, kPage) || !make_map(&cm, p.beacons_s, crows, (uint32_t)p.B) ||
      !make_map4(&km4, p.k_pool, (uint64_t)p.layers * (uint64_t)p.num_pages, (uint32_t)p.hkv))
    return cudaErrorInvalidValue;
  TcParams tp{};
  tp.block_table = p.block_table;
  tp.segs = p.segs;
  tp.scores = p.scores;
  tp.lse_out = p.lse_out;
  tp.trig = p.trig;
  tp.status = p.status;
  tp.num_pages = p.num_pages;
  tp.bt_stride = p.bt_stride;
  tp.layers = p.layers;
  tp.hkv = p.hkv;
  tp.B = p.B;
  tp.max_seq = p.max_seq;
  tp.n_segs = n_req * p.layers * p.hkv;
  tp.alpha = 1.4426950408889634f / sqrtf(128.0f);
  if (p.B <= 128) return launch<128, KVC_TC_NCB_SMALL, KVC_TC_STAGES_SMALL>(km, cm, km4, tp, s);
  return launch<256, 1, 4>(km, cm, km4, tp, s);
}

}  // namespace kvc
