// beacon_update_tc.cu -- BeaconKV periodic beacon update with the nearest-
// beacon assignment on the tensor cores (bf16 query ring, head_dim 128).
//
// What it computes (BeaconKV explainer §3.2: a query goes to its nearest
// beacon; beacons are updated periodically and incrementally): every point
// (a query of one of the G query heads of the KV head, over the steps since
// the previous update) is assigned to the beacon with the smallest squared
// distance, ties to the lower index, against the beacons as they were before
// this update; each beacon with m new points becomes (n c + sum)/(n + m).
//
// Assignment as a product: |x - c|^2 = |x|^2 + |c|^2 - 2 x.c and |x|^2 does
// not depend on the beacon, so the argmin is that of |c|^2 - 2 x.c.  The
// points are bf16 (exact as MMA operands); the fp32 beacons enter as two bf16
// terms, c = c_hi + c_lo + r with |r_k| <= 2^-18 |c_k|, so x.c is computed
// as x.c_hi + x.c_lo with one fp32 accumulation in TMEM and an error of at
// most 2^-18 sum_k |x_k c_k| beyond fp32 rounding.  |c|^2 is the fp32 norm of
// the fp32 beacon.  The per-beacon sums are a second tensor-core product of
// one-hot assignment tiles with the same point tile (kernel comment below).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "kvc_internal.h"
#include "tc_ptx.cuh"

namespace kvc {
namespace {

constexpr int kUT = 128;  // threads: one point of the 128-point tile each

// Byte offset of bf16 element k (0..63) of `row` inside one 64-element
// K-block of a K-major tile in the 128-byte-swizzled canonical layout.
__device__ __forceinline__ uint32_t sw128_off(int row, int k) {
  return (uint32_t)row * 128u + ((uint32_t)((k >> 3) ^ (row & 7)) << 4) + (uint32_t)(k & 7) * 2u;
}

// One CTA of 128 threads per (request, layer, KV head).  Per tile of 128
// points (TMEM lane = point):
//   1. assignment: X (C_hi + C_lo)^T into TMEM columns [0, A) (N = B), the
//      argmin over |c|^2 - 2 x.c per lane;
//   2. sums: for each half of up to 128 beacons, the one-hot tile
//      A_h^T [beacon rows x points] holds a 1 at (a_p, p) for the points of
//      that half, and D_h += A_h^T X (M = 128 beacon rows, N = 128 dims,
//      K = 128 points) accumulates the per-beacon sums in fp32 in TMEM,
//      with X read as an MN-major operand: its 128-byte-swizzled K-major
//      layout is the canonical MN-major one with 64-dimension blocks 16 KB
//      apart (LBO) and 8-point groups 1 KB apart (SBO).
// No point is read twice from global memory.  Then thread b updates beacon b
// (and b + 128) from its TMEM lane: (n c + sum) / (n + m).
__global__ void __launch_bounds__(kUT) beacon_update_tc_kernel(BeaconUpdateParams p, uint32_t tmem_cols) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_align<1024>(smem_raw);
  constexpr int D = 128;
  const int B = p.B, NP = p.W * p.G;
  const int nh = (B + 127) / 128;        // halves of 128 beacons
  const bool dup = B <= 64;              // one-hot rows written twice (see below)
  const uint32_t acol = B <= 128 ? 128u : 256u;  // sums of half h at columns acol + 128 h
  uint8_t *xs = smem;                    // [2 K-blocks][128 points][128 B]
  uint8_t *chi = xs + 32768;             // [2][B][128 B]
  uint8_t *clo = chi + B * 256;          // [2][B][128 B]
  uint8_t *asum = clo + B * 256;         // [2 point blocks][128 beacon rows][128 B], one-hot^T of a half
  float *cn = reinterpret_cast<float *>(asum + 32768);  // [B]
  float *cpart = cn + B;                                 // [4][B]
  int32_t *cnt = reinterpret_cast<int32_t *>(cpart + 4 * B);  // [B]
  uint64_t *mbar = smem_align<16>(reinterpret_cast<uint64_t *>(cnt + B));
  uint32_t *tslot = reinterpret_cast<uint32_t *>(mbar + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tslot + 1);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int h = blockIdx.x % p.hkv;
  const int l = (blockIdx.x / p.hkv) % p.layers;
  const UpdateDesc ud = p.descs[blockIdx.x / (p.hkv * p.layers)];
  const int r = ud.req;
  const int n_pts = ud.n_steps * p.G;
  const int64_t seg = ((int64_t)r * p.layers + l) * p.hkv + h;
  float *gbeac = p.beacons + seg * B * D;
  int32_t *gcnt = p.counts + seg * B;
  const __nv_bfloat16 *ring = reinterpret_cast<const __nv_bfloat16 *>(p.qring);
  auto point_base = [&](int pt) -> int64_t {
    const int step = pt / p.G, g = pt - step * p.G;
    const int slot = (ud.ring_start + step) % p.W;
    return ((((int64_t)r * p.layers + l) * p.W + slot) * p.hq + (h * p.G + g)) * D;
  };
  // beacon b's value before this update, element k (first update: a point)
  auto c_old = [&](int b, int k) -> float {
    if (ud.init) return __bfloat162float(ring[point_base((int)(((int64_t)b * n_pts) / B)) + k]);
    return gbeac[b * D + k];
  };

  if (tid == 0) {
    mbar_init(mbar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tslot)),
                 "r"(tmem_cols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  // this thread's point of the next tile, loaded into registers one tile
  // ahead (the first before the beacon preparation) so the global latency
  // overlaps the work on the current tile
  uint4 xw[16];
  auto load_point = [&](int p0) {
    const int pt = p0 + tid;
    if (pt < n_pts) {
      const uint4 *src = reinterpret_cast<const uint4 *>(ring + point_base(pt));
#pragma unroll
      for (int c = 0; c < 16; ++c) xw[c] = src[c];
    } else {
#pragma unroll
      for (int c = 0; c < 16; ++c) xw[c] = make_uint4(0, 0, 0, 0);
    }
  };
  load_point(0);
  // the one-hot tile starts at zero; counts at zero
  for (int i = tid; i < 32768 / 16; i += kUT) reinterpret_cast<uint4 *>(asum)[i] = make_uint4(0, 0, 0, 0);
  for (int b = tid; b < B; b += kUT) cnt[b] = 0;
  // beacons: bf16 hi/lo terms in the swizzled layout, fp32 squared norms;
  // 32 beacons' loads in flight at once, the next 32 issued before this
  // batch is split and stored
  float cnext[32];
  auto load_batch = [&](int b0) {
    if (ud.init) {
#pragma unroll
      for (int u = 0; u < 32; ++u) cnext[u] = c_old(b0 + u, tid);
    } else {
      // no branch between the loads, so all 32 are in flight together
#pragma unroll
      for (int u = 0; u < 32; ++u) cnext[u] = gbeac[(b0 + u) * D + tid];
    }
  };
  load_batch(0);
#pragma unroll 1
  for (int b0 = 0; b0 < B; b0 += 32) {  // B is a multiple of 32
    float c[32];
#pragma unroll
    for (int u = 0; u < 32; ++u) c[u] = cnext[u];
    if (b0 + 32 < B) load_batch(b0 + 32);
    const int kb = tid >> 6, k = tid & 63;
#pragma unroll
    for (int u8 = 0; u8 < 32; u8 += 8) {
      float sq[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float cv = c[u8 + u];
        const __nv_bfloat16 hi = __float2bfloat16_rn(cv);
        const __nv_bfloat16 lo = __float2bfloat16_rn(cv - __bfloat162float(hi));
        *reinterpret_cast<__nv_bfloat16 *>(chi + kb * B * 128 + sw128_off(b0 + u8 + u, k)) = hi;
        *reinterpret_cast<__nv_bfloat16 *>(clo + kb * B * 128 + sw128_off(b0 + u8 + u, k)) = lo;
        sq[u] = cv * cv;
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1)
#pragma unroll
        for (int u = 0; u < 8; ++u) sq[u] += __shfl_xor_sync(0xffffffffu, sq[u], o);
      if (lane == 0)
#pragma unroll
        for (int u = 0; u < 8; ++u) cpart[warp * B + b0 + u8 + u] = sq[u];
    }
  }
  tmem_fence_before();
  __syncthreads();
  tmem_fence_after();
  const uint32_t tmem_base = *tslot;
  for (int b = tid; b < B; b += kUT) cn[b] = ((cpart[b] + cpart[B + b]) + cpart[2 * B + b]) + cpart[3 * B + b];

  const uint32_t idesc_asg = idesc_bf16_f32(128, B);
  // sums: A = one-hot^T (K-major), B operand = X (MN-major, transpose bit 16)
  const uint32_t idesc_sum = idesc_bf16_f32(128, D) | (1u << 16);
  const uint32_t lane_addr = (uint32_t)(warp * 32) << 16;
  // the running mean's first 64 old values and old count of this thread's
  // first beacon (mapping as in the running mean below), loaded now so that
  // they arrive while the point tiles run
  const int b_first = dup ? (tid & 63) : tid;
  float4 ov0[16];
  int n_first = 0;
  if (!ud.init && b_first < B) {
    const float4 *src = reinterpret_cast<const float4 *>(gbeac + (int64_t)b_first * D + (dup ? (tid >> 6) * (D / 2) : 0));
#pragma unroll
    for (int q = 0; q < 16; ++q) ov0[q] = src[q];
    n_first = gcnt[b_first];
  }
  bool nan = false;
  int phase = 0;
  for (int p0 = 0; p0 < n_pts; p0 += 128) {
    const int pt = p0 + tid;
#pragma unroll
    for (int c = 0; c < 16; ++c)
      *reinterpret_cast<uint4 *>(xs + (c >> 3) * 16384 + tid * 128 + (((c & 7) ^ (tid & 7)) << 4)) = xw[c];
    if (p0 + 128 < n_pts) load_point(p0 + 128);  // in flight during this tile
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    tmem_fence_before();
    __syncthreads();
    if (tid == 0) {
      tmem_fence_after();
      const uint32_t xa = smem_u32(xs), ha = smem_u32(chi), la = smem_u32(clo);
      for (int term = 0; term < 2; ++term)
        for (int kb = 0; kb < 2; ++kb)
          for (int ks = 0; ks < 4; ++ks) {
            const uint64_t a = sw128_desc(xa + kb * 16384 + ks * 32);
            const uint64_t bd = sw128_desc((term ? la : ha) + kb * B * 128 + ks * 32);
            umma(tmem_base, a, bd, idesc_asg, (term | kb | ks) != 0);
          }
      umma_commit(mbar);
      if (!mbar_wait(mbar, phase & 1, abort_flag, p.status)) *abort_flag = 1;
    }
    ++phase;
    __syncthreads();
    if (*abort_flag) break;
    tmem_fence_after();
    float best = __int_as_float(0x7f800000);
    int besti = 0;
    for (int c0 = 0; c0 < B; c0 += 32) {
      float v[32];
      tmem_ld32(tmem_base + lane_addr + c0, v);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float dist = fmaf(-2.f, v[i], cn[c0 + i]);
        nan |= (dist != dist);
        if (dist < best) {
          best = dist;
          besti = c0 + i;
        }
      }
    }
    const bool valid = pt < n_pts;
    if (valid) {
      if (p.assign_out) p.assign_out[seg * (int64_t)NP + pt] = besti;
      atomicAdd(&cnt[besti], 1);
    }
    // this point's entry of the one-hot tile (row = beacon within its half);
    // with at most 64 beacons every row is written twice (rows b and b + 64),
    // so the sums of beacon b sit in TMEM lanes b and b + 64 and all four
    // warps take part in the running mean
    const uint32_t oh_off = (uint32_t)(tid >> 6) * 16384u + sw128_off(besti & 127, tid & 63);
    const uint32_t oh_dup = dup ? (uint32_t)(tid >> 6) * 16384u + sw128_off(besti + 64, tid & 63) : oh_off;
    for (int hh = 0; hh < nh; ++hh) {
      const bool here = valid && (besti >> 7) == hh;
      if (here) {
        *reinterpret_cast<__nv_bfloat16 *>(asum + oh_off) = __float2bfloat16_rn(1.f);
        *reinterpret_cast<__nv_bfloat16 *>(asum + oh_dup) = __float2bfloat16_rn(1.f);
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tmem_fence_before();
      __syncthreads();
      if (tid == 0) {
        tmem_fence_after();
        const uint32_t aa = smem_u32(asum), xa = smem_u32(xs);
        for (int ks = 0; ks < 8; ++ks) {
          const uint64_t a = sw128_desc(aa + (ks >> 2) * 16384 + (ks & 3) * 32);
          // X as MN-major: start at the 16-point group, LBO 16 KB, SBO 1 KB
          uint64_t bd = sw128_desc(xa + ks * 2048);
          bd = (bd & ~(uint64_t)(0x3FFFull << 16)) | ((uint64_t)(16384 >> 4) << 16);
          umma(tmem_base + acol + 128u * hh, a, bd, idesc_sum, (p0 > 0 || ks > 0) ? 1u : 0u);
        }
        umma_commit(mbar);
        if (!mbar_wait(mbar, phase & 1, abort_flag, p.status)) *abort_flag = 1;
      }
      ++phase;
      __syncthreads();  // the product has read the one-hot tile
      if (*abort_flag) break;
      if (here) {
        *reinterpret_cast<__nv_bfloat16 *>(asum + oh_off) = __float2bfloat16_rn(0.f);
        *reinterpret_cast<__nv_bfloat16 *>(asum + oh_dup) = __float2bfloat16_rn(0.f);
      }
    }
    if (*abort_flag) break;
    tmem_fence_before();
    __syncthreads();  // xs and the assignment columns are reused by the next tile
  }
  if (nan) atomicCAS(p.status, kDevOk, kDevNaN);

  if (!*abort_flag) {
    // running mean: thread t updates beacons t and t + 128 from TMEM lane t of
    // each half's sums (columns = dims), 32 dimensions at a time with the old
    // values loaded together
    tmem_fence_after();
    for (int hh = 0; hh < nh; ++hh) {
      // thread t: beacon 128 hh + t, all dimensions; or, with the duplicated
      // rows, beacon t % 64 and the dimension half t / 64
      const int b = dup ? (tid & 63) : 128 * hh + tid;
      const int dlo = dup ? (tid >> 6) * (D / 2) : 0;
      const int nchunk = dup ? 2 : 4;  // 32-dimension chunks of this thread (CTA-uniform)
      const bool mine = b < B;
      const int m = mine ? cnt[b] : 0;
      const int n = hh == 0 ? n_first : ((mine && !ud.init) ? gcnt[b] : 0);
      __syncthreads();  // every thread has read the old count before any is rewritten
      float4 *g4 = reinterpret_cast<float4 *>(gbeac + (int64_t)b * D);
      __nv_bfloat162 *s2 = reinterpret_cast<__nv_bfloat162 *>(reinterpret_cast<__nv_bfloat16 *>(p.beacons_s) +
                                                               (seg * B + b) * D);
      // old values of the chunks past the first two of the first half: the
      // next chunk's loads in flight while this chunk is combined and stored
      float4 ov[8];
      auto load_old = [&](int c0) {
        if (mine && !ud.init)
#pragma unroll
          for (int q = 0; q < 8; ++q) ov[q] = g4[c0 / 4 + q];
      };
      if (hh > 0) load_old(dlo);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (k >= nchunk) break;
        const int c0 = dlo + 32 * k;
        const bool early = hh == 0 && k < 2;  // loaded before the tiles
        float sm[32];
        tmem_ld32(tmem_base + lane_addr + acol + 128u * hh + c0, sm);  // warp-collective
        float v[32];
        if (mine) {
          if (ud.init) {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = c_old(b, c0 + i);
          } else {
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float4 o = early ? ov0[8 * (k & 1) + q] : ov[q];
              v[4 * q] = o.x; v[4 * q + 1] = o.y; v[4 * q + 2] = o.z; v[4 * q + 3] = o.w;
            }
          }
        }
        if (k + 1 < nchunk && !(hh == 0 && k + 1 < 2)) load_old(c0 + 32);
        if (mine) {
          if (m > 0)
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = ((float)n * v[i] + sm[i]) / (float)(n + m);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            g4[c0 / 4 + q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
            s2[c0 / 2 + 2 * q] = __floats2bfloat162_rn(v[4 * q], v[4 * q + 1]);
            s2[c0 / 2 + 2 * q + 1] = __floats2bfloat162_rn(v[4 * q + 2], v[4 * q + 3]);
          }
        }
      }
      if (mine && dlo == 0) {
        gcnt[b] = n + m;
        p.trig[seg * B + b] = (float)m / (float)n_pts;
      }
    }
  }
  tmem_fence_before();
  __syncthreads();
  if (warp == 0) {
    tmem_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(tmem_cols));
  }
}


// ---------------------------------------------------------------------------
// Pipelined form (a CTA pair per segment above 128 beacons, below).  One
// persistent CTA per SM walks its segments; the work is split by role so that the point loads, the beacon
// preparation, the products, the argmins and the running means of
// neighbouring tiles and segments overlap instead of running as one serial
// chain per segment:
//   warp 0      TMEM allocation and the MMA issuer (one lane); within a
//               segment the assignment product of tile g+1 is issued before
//               the sums of tile g, and a segment's last sums before the next
//               segment's first assignment;
//   warps 1-4   point warps: one point per thread: the argmin over its TMEM
//               lane of the assignment product (four interleaved compare
//               chains, merged by value then index), its one-hot entry and
//               its count;
//   warps 5-8   preparation, one beacon per thread: the next segment's
//               beacons as bf16 hi/lo terms (swizzled, the B operand of the
//               assignment) and their fp32 squared norms;
//   warps 9-12  running mean: one dimension per thread, over every beacon,
//               (n c + sum) * (1 / (n + m)) with the reciprocal taken once
//               per beacon;
//   warp 13     the point producer: one TMA box per 64-dimension half of a
//               128-point tile into one of NXS stages (128-byte swizzle, the
//               K-major A operand of the assignment).
// The tiles walk the segment's query ring in physical slot order: tile t
// holds slots [t S, t S + S) with S = 128 / G steps of G query heads, so a
// tile is always one box and never wraps.  A point belongs to this update
// when its slot's step lies in the update's window (the last n_steps steps,
// starting at slot ring_start); the others (older queries, slots past W,
// which read the next ring or the box's zero fill) are neither assigned nor
// counted and leave a zero one-hot column, so their finite values add
// nothing to the sums.  The ring is zeroed when the context is created.
// The sums are D[dim][beacon] = X^T OH, with the point tile read as an
// MN-major A operand (dimensions on M, its 64-dimension blocks 16 KB apart)
// and the one-hot tile OH [beacon rows x point columns] as a K-major B
// operand: a segment's sums take B TMEM columns, and the running mean reads
// and writes each beacon row with one coalesced access per warp.
// TMEM columns: two assignment buffers of BM, then two sums buffers of BM
// (sums of neighbouring segments alternate).  NOH one-hot tiles: two, or one
// where shared memory is better spent on a third point stage.  The counts of
// three segments rotate in shared memory so that the preparation never waits
// for a mean, and the squared norms through NCB + 2 buffers so that it waits
// only for the MMA's last read of the beacon terms.  Every role loads the
// next segment's descriptor a segment ahead.
// More than 128 beacons: a cluster of two CTAs per segment (CL = 2), CTA r
// holding beacons [128 r, 128 r + nb) with the layout above.  Both load the
// same point tiles; each point thread takes the argmin over its CTA's
// beacons and the two CTAs swap (distance, index) through distributed shared
// memory (asynchronous stores completing on the peer's barriers, receipted
// the same way), the lower half winning ties, so both hold the argmin over
// every beacon.  Each CTA then writes the one-hot entries and counts of its
// own beacons and runs their sums and means.  The pair prefetches its next
// segment's beacons and point tiles into L2 while the current one runs.
// Every wait is bounded.
constexpr int kPipeWarps = 14;
constexpr int kPipeThreads = 32 * kPipeWarps;

__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Every lane of the warp waits (bounded); the warp takes one decision.
__device__ __forceinline__ bool lanes_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                           int32_t *status) {
  const bool ok = mbar_wait(bar, parity, abort_flag, status);
  return __all_sync(0xffffffffu, ok);
}

struct PipeSeg {
  int r, l, h, n_pts, T, init, ring_start;
  int64_t seg;
};
__device__ __forceinline__ PipeSeg pipe_seg(const BeaconUpdateParams &p, int s) {
  PipeSeg g;
  g.h = s % p.hkv;
  g.l = (s / p.hkv) % p.layers;
  const UpdateDesc ud = p.descs[s / (p.hkv * p.layers)];
  g.r = ud.req;
  g.n_pts = ud.n_steps * p.G;
  g.T = (p.W * p.G + 127) / 128;  // tiles over every slot of the ring
  g.init = ud.init;
  g.ring_start = ud.ring_start;
  g.seg = ((int64_t)g.r * p.layers + g.l) * p.hkv + g.h;
  return g;
}
// Element offset in the query ring of point pt of the segment (step pt / G,
// query head h*G + pt % G of the step's ring slot).
__device__ __forceinline__ int64_t pipe_point(const BeaconUpdateParams &p, const PipeSeg &g, int pt) {
  const int step = pt / p.G, gq = pt - step * p.G;
  int slot = g.ring_start + step;
  if (slot >= p.W) slot -= p.W;
  return ((((int64_t)g.r * p.layers + g.l) * p.W + slot) * p.hq + (g.h * p.G + gq)) * 128;
}

// Distributed shared memory between the two CTAs of a cluster.
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// The same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_peer(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
// Every thread of both CTAs of the cluster arrives; neither goes on before
// all have.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
// Asynchronous stores into the peer CTA's shared memory, each completing as
// transaction bytes on a barrier of the peer (whose complete-tx releases the
// bytes at cluster scope): no fence on the sending side.
__device__ __forceinline__ void st_async_v2(uint32_t caddr, float a, int32_t b, uint32_t cbar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.b32 [%0], {%1, %2}, [%3];" ::"r"(caddr),
               "r"(__float_as_int(a)), "r"(b), "r"(cbar)
               : "memory");
}
__device__ __forceinline__ void st_async_b32(uint32_t caddr, int32_t a, uint32_t cbar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(caddr), "r"(a),
               "r"(cbar)
               : "memory");
}
// Bounded wait whose acquire covers stores made by the peer CTA.
__device__ __forceinline__ bool mbar_wait_cl(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                             int32_t *status, bool honor_abort = true) {
  auto try_once = [&]() {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(1000000u)
        : "memory");
    return ok != 0;
  };
  if (try_once()) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
    if (try_once()) return true;
    if (honor_abort && *abort_flag) return false;
    if (global_ns() - t0 > kWaitNs) {
      atomicCAS(status, kDevOk, kDevTimeout);
      *abort_flag = 1;
      return false;
    }
  }
}

// L2 prefetches: `bytes` contiguous bytes (16-byte aligned, a multiple of
// 16), and one box of a tensor map.  Neither writes shared memory.
__device__ __forceinline__ void prefetch_l2(const void *src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ void prefetch_box_3d(const CUtensorMap *map, int x, int y, int z) {
  asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y), "r"(z)
               : "memory");
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, int x, int y, int z,
                                            uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

template <int BM, int NXS, int NCB, int NOH, int CL>
__global__ void __launch_bounds__(kPipeThreads, 1)
    beacon_update_pipe_kernel(const __grid_constant__ CUtensorMap qmap, BeaconUpdateParams p, int n_segs) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_align<1024>(smem_raw);
  constexpr int D = 128;
  constexpr uint32_t kXBytes = 32768;    // 128 points x 128 bf16
  constexpr uint32_t kCBytes = BM * 256;  // one term of one beacon buffer (B rows x 128 bf16)
  // a beacon buffer holds, per 64-dimension block, the B hi rows followed by
  // the B lo rows: [2 K-blocks][hi B rows | lo B rows][128 B], 128-byte
  // swizzle; one assignment product per term
  constexpr uint32_t kAsgCols = BM;          // TMEM columns of one assignment buffer
  constexpr uint32_t kSumCol0 = 2 * kAsgCols;  // first sums column
  constexpr uint32_t kTmemAlloc = 4u * BM;
  constexpr uint32_t kOHBytes = BM * 256; // one one-hot tile: [2 point blocks][B rows][128 B]
  // this CTA's beacons: [b_lo, b_lo + B) of the segment's Bg
  const int Bg = p.B;
  const uint32_t rank = CL > 1 ? cluster_rank() : 0u;
  const int b_lo = (int)rank * 128;
  const int B = CL > 1 ? (rank ? Bg - 128 : 128) : Bg;
  const int seg0 = blockIdx.x / CL, seg_step = gridDim.x / CL;
  uint8_t *xs = smem;
  uint8_t *cterm = xs + NXS * kXBytes;  // [NCB][2 K-blocks][2 B rows][128 B]
  uint8_t *oh = cterm + NCB * 2 * kCBytes;
  // squared norms: a ring of NCB + 2, so that the preparation of segment
  // si + NCB (which starts once the MMA has read segment si's terms) never
  // overwrites the norms of a segment the point warps may still scan
  constexpr int NCN = NCB + 2;
  float *cn = reinterpret_cast<float *>(oh + NOH * kOHBytes);   // [NCN][BM] squared norms
  int32_t *cnt = reinterpret_cast<int32_t *>(cn + NCN * BM);     // [3][BM] this update's counts
  int32_t *nold = cnt + 3 * BM;                                   // [3][BM] counts before the update
  float *mfac = reinterpret_cast<float *>(nold + 3 * BM);         // [2][2][BM] old count n, 1/(n+m) or 0
  uint64_t *bars = reinterpret_cast<uint64_t *>(mfac + 4 * BM);
  uint64_t *x_full = bars, *x_empty = x_full + NXS;
  uint64_t *prep_full = x_empty + NXS, *prep_empty = prep_full + NCB;
  uint64_t *cnt_full = prep_empty + NCB, *cnt_empty = cnt_full + 3;
  uint64_t *acc_full = cnt_empty + 3, *acc_empty = acc_full + 2;
  uint64_t *oh_full = acc_empty + 2, *oh_empty = oh_full + 2;
  uint64_t *sum_full = oh_empty + 2, *sum_empty = sum_full + 2;
  uint64_t *mean_sync = sum_empty + 2, *mma_done = mean_sync + 1;
  uint64_t *xch_full = mma_done + 1, *xch_empty = xch_full + 2;  // the argmin swap (CL = 2)
  float2 *xch = reinterpret_cast<float2 *>(xch_empty + 2);          // [2][128] the peer's (distance, index)
  int32_t *ack = reinterpret_cast<int32_t *>(xch + (CL > 1 ? 256 : 0));  // [2][128] the peer's receipts
  uint32_t *tslot = reinterpret_cast<uint32_t *>(ack + (CL > 1 ? 256 : 0));
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tslot + 1);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  if (tid == 0) {
    for (int i = 0; i < NXS; ++i) {
      mbar_init(&x_full[i], 1);  // the producer's expect_tx arrival; the box bytes complete it
      mbar_init(&x_empty[i], 1);
    }
    for (int i = 0; i < NCB; ++i) {
      mbar_init(&prep_full[i], 128);
      mbar_init(&prep_empty[i], 1);  // MMA commit after the segment's last assignment
    }
    for (int i = 0; i < 3; ++i) {
      mbar_init(&cnt_full[i], 128);   // point warps: the segment's counts are complete
      mbar_init(&cnt_empty[i], 128);  // mean warps: counts read and zeroed again
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 128);
      mbar_init(&oh_full[i], 128);
      mbar_init(&oh_empty[i], 1);
      mbar_init(&sum_full[i], 1);
      mbar_init(&sum_empty[i], 128);
    }
    mbar_init(mean_sync, 128);
    mbar_init(mma_done, 1);
    for (int i = 0; i < 2; ++i) {
      // completed by the peer's stores: its 128 argmins in xch (8 bytes each),
      // its 128 receipts for ours (4 bytes each); each phase is armed by this
      // CTA's point thread 0 one phase ahead, the first ones here
      mbar_init(&xch_full[i], 1);
      mbar_init(&xch_empty[i], 1);
      if (CL > 1) {
        mbar_expect_tx(&xch_full[i], 128 * 8);
        mbar_expect_tx(&xch_empty[i], 128 * 4);
      }
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // the one-hot tiles start at zero (each point clears its own entry later),
  // and so do the count buffers (the mean warps zero each after reading it)
  for (int i = tid; i < (int)(NOH * kOHBytes / 16); i += kPipeThreads)
    reinterpret_cast<uint4 *>(oh)[i] = make_uint4(0, 0, 0, 0);
  for (int i = tid; i < 3 * BM; i += kPipeThreads) cnt[i] = 0;
  fence_proxy_async();
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tslot)),
                 "r"(kTmemAlloc));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tmem_fence_before();
  __syncthreads();
  if constexpr (CL > 1) cluster_sync_all();  // the peer's barriers are initialised
  tmem_fence_after();
  const uint32_t tmem_base = *tslot;
  const __nv_bfloat16 *ring = reinterpret_cast<const __nv_bfloat16 *>(p.qring);

  if (warp == 0) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc_asg = idesc_bf16_f32(128, B);
      const uint32_t idesc_sum = idesc_bf16_f32(128, B) | (1u << 15);  // A (the point tile) MN-major
      bool ok = true;
      auto assign = [&](uint32_t gi, int si, int t, int T) {
        const int cb = si % NCB;
        if (t == 0) ok = ok && mbar_wait(&prep_full[cb], (si / NCB) & 1, abort_flag, p.status);
        ok = ok && mbar_wait(&x_full[gi % NXS], (gi / NXS) & 1, abort_flag, p.status) &&
             mbar_wait(&acc_empty[gi & 1], ((gi >> 1) & 1) ^ 1, abort_flag, p.status);
        if (!ok) return;
        tmem_fence_after();
        const uint32_t xa = smem_u32(xs + (gi % NXS) * kXBytes);
        const uint32_t ca = smem_u32(cterm + cb * 2 * kCBytes);
        for (int term = 0; term < 2; ++term)
          for (int kb = 0; kb < 2; ++kb)
            for (int ks = 0; ks < 4; ++ks) {
              const uint64_t a = sw128_desc(xa + kb * 16384 + ks * 32);
              const uint64_t bd = sw128_desc(ca + kb * 2 * B * 128 + term * B * 128 + ks * 32);
              umma(tmem_base + (gi & 1) * kAsgCols, a, bd, idesc_asg, (term | kb | ks) != 0);
            }
        umma_commit(&acc_full[gi & 1]);
        if (t == T - 1) umma_commit(&prep_empty[cb]);  // the beacon terms have been read
      };
      auto sums = [&](uint32_t gi, int si, int t, int T) {
        const int sb = si & 1;
        ok = ok && mbar_wait(&oh_full[gi % NOH], (gi / NOH) & 1, abort_flag, p.status);
        if (t == 0) ok = ok && mbar_wait(&sum_empty[sb], ((si >> 1) & 1) ^ 1, abort_flag, p.status);
        if (!ok) return;
        tmem_fence_after();
        const uint32_t xa = smem_u32(xs + (gi % NXS) * kXBytes), oa = smem_u32(oh + (gi % NOH) * kOHBytes);
        for (int ks = 0; ks < 8; ++ks) {
          // X^T: 16 points from point group ks, 64-dimension blocks 16 KB apart (LBO), 8-point groups 1 KB
          // apart (SBO)
          uint64_t a = sw128_desc(xa + ks * 2048);
          a = (a & ~(uint64_t)(0x3FFFull << 16)) | ((uint64_t)(16384 >> 4) << 16);
          const uint64_t bd = sw128_desc(oa + (ks >> 2) * B * 128 + (ks & 3) * 32);
          umma(tmem_base + kSumCol0 + sb * BM, a, bd, idesc_sum, (t > 0 || ks > 0) ? 1u : 0u);
        }
        umma_commit(&x_empty[gi % NXS]);
        umma_commit(&oh_empty[gi % NOH]);
        if (t == T - 1) umma_commit(&sum_full[sb]);
      };
      // tile stream; the assignment runs one tile ahead of the sums
      uint32_t gi = 0;
      int si = 0;
      bool have_prev = false;
      uint32_t pg = 0;
      int ps = 0, pt = 0, pT = 0;
      // within a segment; at a segment boundary the last sums go first, so
      // that the running mean of a segment never waits for the next
      // segment's beacon preparation
      // each segment's descriptor is loaded a segment ahead (its latency hidden)
      PipeSeg g_next = seg0 < n_segs ? pipe_seg(p, seg0) : PipeSeg{};
      for (int s = seg0; s < n_segs && ok; s += seg_step, ++si) {
        const PipeSeg g = g_next;
        if (s + seg_step < n_segs) g_next = pipe_seg(p, s + seg_step);
        for (int t = 0; t < g.T && ok; ++t, ++gi) {
          if (have_prev && t == 0) sums(pg, ps, pt, pT);
          assign(gi, si, t, g.T);
          if (have_prev && t > 0) sums(pg, ps, pt, pT);
          have_prev = true;
          pg = gi;
          ps = si;
          pt = t;
          pT = g.T;
        }
      }
      if (have_prev && ok) sums(pg, ps, pt, pT);
      umma_commit(mma_done);
      mbar_wait(mma_done, 0, abort_flag, p.status, false);
    }
    __syncwarp();
  } else if (warp < 5) {
    // --------------------------------------------------------- point warps
    const int q = warp & 3, row = q * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    const int NP = p.W * p.G;
    uint32_t gi = 0;
    int si = 0;
    bool ok = true, nan = false;
    uint32_t last_off0 = 0xffffffffu, last_off1 = 0xffffffffu;  // this point's entry in each one-hot tile
    const int S = 128 / p.G;                 // ring slots per tile
    const int slot_in_tile = row / p.G, gq = row - (row / p.G) * p.G;
    uint32_t peer_xch = 0, peer_ack = 0, peer_full = 0, peer_empty = 0;
    if constexpr (CL > 1) {
      peer_xch = map_peer(smem_u32(xch), rank ^ 1u);
      peer_ack = map_peer(smem_u32(ack), rank ^ 1u);
      peer_full = map_peer(smem_u32(xch_full), rank ^ 1u);
      peer_empty = map_peer(smem_u32(xch_empty), rank ^ 1u);
    }
    // each segment's descriptor is loaded a segment ahead (its latency hidden)
    PipeSeg g_next = seg0 < n_segs ? pipe_seg(p, seg0) : PipeSeg{};
    for (int s = seg0; s < n_segs && ok; s += seg_step, ++si) {
      const PipeSeg g = g_next;
      if (s + seg_step < n_segs) g_next = pipe_seg(p, s + seg_step);
      const int cb = si % NCB, kb3 = si % 3;
      ok = lanes_wait(&prep_full[cb], (si / NCB) & 1, abort_flag, p.status) &&
           lanes_wait(&cnt_empty[kb3], ((si / 3) & 1) ^ 1, abort_flag, p.status);
      if (!ok) break;
      const float *cnb = cn + (si % NCN) * BM;
      int32_t *cntb = cnt + kb3 * BM;
      for (int t = 0; t < g.T; ++t, ++gi) {
        // this row's slot; its step in the update's window, if it is in it
        const int slot = t * S + slot_in_tile;
        const int step = slot - g.ring_start + (slot < g.ring_start ? p.W : 0);
        const bool valid = slot < p.W && step < g.n_pts / p.G;
        const int pt = step * p.G + gq;
        const int ab = gi & 1;
        ok = lanes_wait(&acc_full[ab], (gi >> 1) & 1, abort_flag, p.status);
        if (!ok) break;
        tmem_fence_after();
        // four interleaved chains (column i in chain i % 4), each keeping its
        // first minimum; merged by value, then by the lower index, which is
        // the first minimum of one pass over every column
        float bst[4];
        int bix[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          bst[j] = __int_as_float(0x7f800000);
          bix[j] = 0;
        }
        constexpr int kChunk = 32;
        for (int c0 = 0; c0 < B; c0 += kChunk) {
          float v[kChunk];
          tmem_ld32(tmem_base + lane_addr + ab * kAsgCols + c0, v);
#pragma unroll
          for (int i = 0; i < kChunk; i += 2) {
            // two distances per packed FMA (each rounded as one fmaf)
            const float2 cc = *reinterpret_cast<const float2 *>(cnb + c0 + i);
            const float2 d2 = __ffma2_rn(make_float2(-2.f, -2.f), make_float2(v[i], v[i + 1]), cc);
            nan |= valid && (d2.x != d2.x || d2.y != d2.y);
            if (d2.x < bst[i & 3]) {
              bst[i & 3] = d2.x;
              bix[i & 3] = c0 + i;
            }
            if (d2.y < bst[(i + 1) & 3]) {
              bst[(i + 1) & 3] = d2.y;
              bix[(i + 1) & 3] = c0 + i + 1;
            }
          }
        }
        float best = bst[0];
        int besti = bix[0];
#pragma unroll
        for (int j = 1; j < 4; ++j)
          if (bst[j] < best || (bst[j] == best && bix[j] < besti)) {
            best = bst[j];
            besti = bix[j];
          }
        tmem_fence_before();
        mbar_arrive(&acc_empty[ab]);
        int fin = besti + b_lo;  // the argmin over the segment's beacons
        if constexpr (CL > 1) {
          // swap with the peer: wait until it has receipted what this thread
          // put in its slot two tiles ago, send, then read the peer's entry
          // here and receipt it (the receipt carries the value read)
          ok = __all_sync(0xffffffffu, mbar_wait_cl(&xch_empty[ab], ((gi >> 1) & 1) ^ 1, abort_flag, p.status));
          if (!ok) break;
          if (row == 0 && gi >= 2) mbar_expect_tx(&xch_empty[ab], 128 * 4);  // receipts for this tile's entries
          st_async_v2(peer_xch + (ab * 128 + row) * 8, best, fin, peer_full + ab * 8);
          ok = __all_sync(0xffffffffu, mbar_wait_cl(&xch_full[ab], (gi >> 1) & 1, abort_flag, p.status));
          if (!ok) break;
          const float2 o = xch[ab * 128 + row];
          if (row == 0) mbar_expect_tx(&xch_full[ab], 128 * 8);  // the peer's argmins of tile gi + 2
          st_async_b32(peer_ack + (ab * 128 + row) * 4, __float_as_int(o.y), peer_empty + ab * 8);
          // lower beacon indices win ties, as in one pass over every beacon
          if (rank == 0 ? (o.x < best) : !(best < o.x)) fin = __float_as_int(o.y);
        }
        const bool mine = valid && fin >= b_lo && fin < b_lo + B;
        if (valid) {
          if (p.assign_out && rank == 0) p.assign_out[g.seg * (int64_t)NP + pt] = fin;
          if (mine) atomicAdd(&cntb[fin - b_lo], 1);
        }
        const int ob = gi % NOH;
        ok = lanes_wait(&oh_empty[ob], ((gi / NOH) & 1) ^ 1, abort_flag, p.status);
        if (!ok) break;
        uint8_t *ohb = oh + ob * kOHBytes;
        const uint32_t prev = ob ? last_off1 : last_off0;
        if (prev != 0xffffffffu) *reinterpret_cast<uint16_t *>(ohb + prev) = 0;
        uint32_t off = 0xffffffffu;
        if (mine) {
          off = (uint32_t)(row >> 6) * (uint32_t)B * 128u + sw128_off(fin - b_lo, row & 63);
          *reinterpret_cast<uint16_t *>(ohb + off) = 0x3F80;  // bf16 1.0
        }
        if (ob) last_off1 = off;
        else last_off0 = off;
        fence_proxy_async();
        mbar_arrive(&oh_full[ob]);
      }
      if (!ok) break;
      mbar_arrive(&cnt_full[kb3]);
    }
    if constexpr (CL > 1) {
      // the peer's receipts for the last two tiles land before this CTA may
      // leave (bounded by time alone, also after an abort)
      for (uint32_t gt = gi >= 2 ? gi - 2 : 0; gt < gi; ++gt)
        mbar_wait_cl(&xch_empty[gt & 1], (((gt + 2) >> 1) & 1) ^ 1, abort_flag, p.status, false);
    }
    if (nan) atomicCAS(p.status, kDevOk, kDevNaN);
  } else if (warp < 9) {
    // --------------------------------------------------------- preparation
    // thread b: beacon b of this CTA's share, its 128 dimensions in four
    // quarters of 32 (the next quarter's loads in flight): bf16 hi/lo terms
    // written as 16-byte chunks of the swizzled layout, and the squared norm
    // as one running fp32 sum over the dimensions
    const int b = (warp - 5) * 32 + lane;
    int si = 0;
    bool ok = true;
    // each segment's descriptor is loaded a segment ahead (its latency hidden)
    PipeSeg g_next = seg0 < n_segs ? pipe_seg(p, seg0) : PipeSeg{};
    for (int s = seg0; s < n_segs && ok; s += seg_step, ++si) {
      const PipeSeg g = g_next;
      if (s + seg_step < n_segs) g_next = pipe_seg(p, s + seg_step);
      const int cb = si % NCB;
      const bool have = b < B;
      uint8_t *hb = cterm + cb * 2 * kCBytes, *lb = hb + B * 128;  // lo rows follow the hi rows
      const float *frow = p.beacons + (g.seg * Bg + b_lo + b) * D;
      const __nv_bfloat16 *irow =
          ring + pipe_point(p, g, (int)(((int64_t)(b_lo + (have ? b : 0)) * g.n_pts) / Bg));
      float4 qn[8];
      auto load_q = [&](int kq) {
        if (!have) return;
        if (g.init) {
          const uint4 *src = reinterpret_cast<const uint4 *>(irow + kq * 32);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint4 w = src[j];  // 8 bf16, the lower element in the lower half
            qn[2 * j] = make_float4(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xffff0000u),
                                    __uint_as_float(w.y << 16), __uint_as_float(w.y & 0xffff0000u));
            qn[2 * j + 1] = make_float4(__uint_as_float(w.z << 16), __uint_as_float(w.z & 0xffff0000u),
                                        __uint_as_float(w.w << 16), __uint_as_float(w.w & 0xffff0000u));
          }
        } else {
          const float4 *src = reinterpret_cast<const float4 *>(frow + kq * 32);
#pragma unroll
          for (int j = 0; j < 8; ++j) qn[j] = src[j];
        }
      };
      load_q(0);  // in flight while the buffer is still in use
      // the pair form: this CTA's beacons of its next segment into L2
      if (CL > 1 && b == 0 && s + seg_step < n_segs) {
        const PipeSeg &gn = g_next;
        prefetch_l2(p.beacons + (gn.seg * Bg + b_lo) * D, (uint32_t)(B * D * sizeof(float)));
      }
      // the old count, for the running mean a segment or two later
      const int n_old = (have && !g.init) ? p.counts[g.seg * Bg + b_lo + b] : 0;
      ok = lanes_wait(&prep_empty[cb], ((si / NCB) & 1) ^ 1, abort_flag, p.status);
      if (!ok) break;
      float nrm = 0.f;
#pragma unroll 1
      for (int kq = 0; kq < 4; ++kq) {
        float c[32];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          c[4 * j] = qn[j].x;
          c[4 * j + 1] = qn[j].y;
          c[4 * j + 2] = qn[j].z;
          c[4 * j + 3] = qn[j].w;
        }
        if (kq < 3) load_q(kq + 1);
        if (!have) continue;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t h[4], l[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float x0 = c[ch * 8 + 2 * e], x1 = c[ch * 8 + 2 * e + 1];
            const __nv_bfloat162 hh = __floats2bfloat162_rn(x0, x1);
            const float2 hf = __bfloat1622float2(hh);
            const __nv_bfloat162 ll = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
            h[e] = *reinterpret_cast<const uint32_t *>(&hh);
            l[e] = *reinterpret_cast<const uint32_t *>(&ll);
          }
          const int kk = kq * 32 + ch * 8;  // the chunk's first dimension
          const uint32_t off = (uint32_t)(kk >> 6) * 2u * (uint32_t)B * 128u + sw128_off(b, kk & 63);
          *reinterpret_cast<uint4 *>(hb + off) = make_uint4(h[0], h[1], h[2], h[3]);
          *reinterpret_cast<uint4 *>(lb + off) = make_uint4(l[0], l[1], l[2], l[3]);
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) nrm = fmaf(c[i], c[i], nrm);
      }
      if (have) cn[(si % NCN) * BM + b] = nrm;
      fence_proxy_async();  // the beacon terms, for the MMA
      // the count slot of this segment is free once the mean of segment si - 3 is done with it
      ok = lanes_wait(&cnt_empty[si % 3], ((si / 3) & 1) ^ 1, abort_flag, p.status);
      if (!ok) break;
      if (have) nold[(si % 3) * BM + b] = n_old;
      mbar_arrive(&prep_full[cb]);
    }
  } else if (warp == 13) {
    // ------------------------------------------------------ point producer
    if (lane == 0) {
      uint32_t gl = 0;
      bool ok = true;
      const int S = 128 / p.G;
      // each segment's descriptor is loaded a segment ahead (its latency hidden)
      PipeSeg g_next = seg0 < n_segs ? pipe_seg(p, seg0) : PipeSeg{};
      for (int s = seg0; s < n_segs && ok; s += seg_step) {
        const PipeSeg g = g_next;
        if (s + seg_step < n_segs) g_next = pipe_seg(p, s + seg_step);
        const int z0 = (g.r * p.layers + g.l) * p.W;  // ring row of slot 0 of this (request, layer)
        // the pair form: the next segment's point tiles into L2 (one CTA)
        if (CL > 1 && rank == 0 && s + seg_step < n_segs) {
          const PipeSeg &gn = g_next;
          const int zn = (gn.r * p.layers + gn.l) * p.W;
          for (int t = 0; t < gn.T; ++t)
            for (int kb = 0; kb < 2; ++kb) prefetch_box_3d(&qmap, kb * 64, gn.h * p.G, zn + t * S);
        }
        for (int t = 0; t < g.T; ++t, ++gl) {
          const int st = gl % NXS;
          ok = mbar_wait(&x_empty[st], ((gl / NXS) & 1) ^ 1, abort_flag, p.status);
          if (!ok) break;
          mbar_expect_tx(&x_full[st], kXBytes);
          for (int kb = 0; kb < 2; ++kb)
            tma_load_3d(smem_u32(xs + st * kXBytes + kb * 16384), &qmap, kb * 64, g.h * p.G, z0 + t * S,
                        &x_full[st]);
        }
      }
      if (*abort_flag && gl > 0) {
        // let the boxes already issued land before the shared memory goes away
        for (int i = 0; i < NXS; ++i) {
          const uint32_t k = gl - 1 - i;
          mbar_wait(&x_full[k % NXS], (k / NXS) & 1, abort_flag, p.status, false);
          if (k == 0) break;
        }
      }
    }
    __syncwarp();
  } else {
    // -------------------------------------------------------- running mean
    const int q = warp & 3, k = q * 32 + lane;  // this thread's dimension = its TMEM lane
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    int si = 0;
    uint32_t ph = 0;
    bool ok = true;
    // each segment's descriptor is loaded a segment ahead (its latency hidden)
    PipeSeg g_next = seg0 < n_segs ? pipe_seg(p, seg0) : PipeSeg{};
    for (int s = seg0; s < n_segs && ok; s += seg_step, ++si) {
      const PipeSeg g = g_next;
      if (s + seg_step < n_segs) g_next = pipe_seg(p, s + seg_step);
      const int kb3 = si % 3, sb = si & 1;
      int32_t *cntb = cnt + kb3 * BM;
      float *gbeac = p.beacons + (g.seg * Bg + b_lo) * D;
      int32_t *gcnt = p.counts + g.seg * Bg + b_lo;
      __nv_bfloat16 *gs = reinterpret_cast<__nv_bfloat16 *>(p.beacons_s) + (g.seg * Bg + b_lo) * D;
      float *nf = mfac + sb * 2 * BM, *inv = nf + BM;
      // the first old values do not depend on this update's points: their
      // loads fly while the sums are still being produced
      float onext[32];
      auto load_old = [&](int b0) {
        if (g.init) {
#pragma unroll
          for (int u = 0; u < 32; ++u)
            onext[u] =
                __bfloat162float(ring[pipe_point(p, g, (int)(((int64_t)(b_lo + b0 + u) * g.n_pts) / Bg)) + k]);
        } else {
#pragma unroll
          for (int u = 0; u < 32; ++u) onext[u] = gbeac[(b0 + u) * D + k];
        }
      };
      load_old(0);
      ok = lanes_wait(&cnt_full[kb3], (si / 3) & 1, abort_flag, p.status) &&
           lanes_wait(&sum_full[sb], (si >> 1) & 1, abort_flag, p.status);
      if (!ok) break;
      tmem_fence_after();
      // per beacon: n and 1/(n + m), or 0 when no point joined it (unchanged);
      // thread k is the only reader of count k, so it clears it at once and
      // the count slot goes back to the point and preparation warps
      int m = 0, n_old = 0;
      if (k < B) {
        m = cntb[k];
        n_old = nold[kb3 * BM + k];
        cntb[k] = 0;
        nf[k] = (float)n_old;
        inv[k] = m > 0 ? 1.f / (float)(n_old + m) : 0.f;
      }
      mbar_arrive(&cnt_empty[kb3]);
      mbar_arrive(mean_sync);
      ok = lanes_wait(mean_sync, ph & 1, abort_flag, p.status);
      ++ph;
      if (!ok) break;
      for (int b0 = 0; b0 < B; b0 += 32) {
        float sm[32], v[32];
        tmem_ld32(tmem_base + lane_addr + kSumCol0 + sb * BM + b0, sm);
#pragma unroll
        for (int u = 0; u < 32; ++u) v[u] = onext[u];
        if (b0 + 32 < B) load_old(b0 + 32);
#pragma unroll
        for (int u = 0; u < 32; ++u) {
          const int b = b0 + u;
          const float iv = inv[b];
          const float x = iv != 0.f ? fmaf(nf[b], v[u], sm[u]) * iv : v[u];
          gbeac[b * D + k] = x;
          gs[b * D + k] = __float2bfloat16_rn(x);
        }
      }
      tmem_fence_before();
      mbar_arrive(&sum_empty[sb]);
      if (k < B) {
        gcnt[k] = n_old + m;
        p.trig[g.seg * Bg + b_lo + k] = (float)m / (float)g.n_pts;
      }
    }
  }
  tmem_fence_before();
  __syncthreads();
  // neither CTA leaves while the other may still write into its shared memory
  if constexpr (CL > 1) cluster_sync_all();
  if (warp == 0) {
    tmem_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemAlloc));
  }
}

PFN_cuTensorMapEncodeTiled_v12000 tma_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// The query ring as (128 dimensions, Hq heads, R * layers * W slots) of bf16;
// box (64 dimensions, G heads, 128 / G slots) = one 16 KB half of a point
// tile in the 128-byte-swizzled K-major layout (row = slot * G + head).
bool make_ring_map(CUtensorMap *m, const BeaconUpdateParams &p, int n_rows) {
  auto fn = tma_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {128, (cuuint64_t)p.hq, (cuuint64_t)n_rows};
  cuuint64_t strides[2] = {256, (cuuint64_t)p.hq * 256};
  cuuint32_t box[3] = {64, (cuuint32_t)p.G, (cuuint32_t)(128 / p.G)};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint8_t *>(p.qring), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BM, int NXS, int NCB, int NOH, int CL>
cudaError_t launch_pipe(const BeaconUpdateParams &p, int n_segs, int n_rows, cudaStream_t s) {
  CUtensorMap qmap;
  if (!make_ring_map(&qmap, p, n_rows)) return cudaErrorInvalidValue;
  const size_t smem = 1024 + (size_t)NXS * 32768 + 2 * (size_t)NCB * BM * 256 + (size_t)NOH * BM * 256 +
                      sizeof(float) * ((size_t)(NCB + 2) * BM + 4 * BM) + sizeof(int32_t) * 6 * (size_t)BM +
                      8 * (2 * NXS + 2 * NCB + 6 + 12 + 2 + 4) + (CL > 1 ? 256 * 12 : 0) +
                      16;  // barriers, swap slots, TMEM slot, abort flag
  auto kernel = beacon_update_pipe_kernel<BM, NXS, NCB, NOH, CL>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (CL == 1) {
    const int grid = n_segs < sms ? n_segs : sms;
    kernel<<<grid, kPipeThreads, smem, s>>>(qmap, p, n_segs);
    return cudaGetLastError();
  }
  // one cluster per segment at a time, as many clusters as fit at once
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(kPipeThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3((unsigned)(CL * (sms / CL)));
  int clusters = 0;
  e = cudaOccupancyMaxActiveClusters(&clusters, kernel, &cfg);
  if (e != cudaSuccess) return e;
  if (clusters <= 0) return cudaErrorNotSupported;
  if (clusters > n_segs) clusters = n_segs;
  cfg.gridDim = dim3((unsigned)(CL * clusters));
  return cudaLaunchKernelEx(&cfg, kernel, qmap, p, n_segs);
}

}  // namespace

bool beacon_update_tc_supported(int d, int B, int dtype) {
  return dtype == KVC_BF16 && d == 128 && B >= 32 && B <= 256 && B % 32 == 0;
}

cudaError_t launch_beacon_update_tc(const BeaconUpdateParams &p, int n_req, cudaStream_t s) {
  if (!beacon_update_tc_supported(p.d, p.B, p.dtype)) return cudaErrorNotSupported;
  if (n_req <= 0) return cudaSuccess;
  // point tile, c_hi/c_lo tiles, one-hot tile, cn + cpart[4] + cnt (6 words per
  // beacon), barrier/slot/flag; TMEM: assignment columns then 128 per half
  const size_t smem = 1024 + 32768 + (size_t)p.B * 512 + 32768 + (size_t)p.B * 4 * 6 + 64;
  const int n_segs = n_req * p.layers * p.hkv;
  // the pipelined form: G dividing 128 (a tile is whole ring slots), the ring
  // addressable by the map's 32-bit slot coordinate
  const int64_t ring_rows = (int64_t)p.n_ring * p.layers * p.W;
  if (p.B <= 128 && 128 % p.G == 0 && ring_rows < (1ll << 31) && tma_encode_fn()) {
    if (p.B <= 64) return launch_pipe<64, 3, 2, 2, 1>(p, n_segs, (int)ring_rows, s);
    return launch_pipe<128, 2, 1, 2, 1>(p, n_segs, (int)ring_rows, s);
  }
  if (128 % p.G == 0 && ring_rows < (1ll << 31) && tma_encode_fn()) {
    // more than 128 beacons: a CTA pair per segment, 128 beacons in the first;
    // one one-hot buffer buys a third point stage
    const cudaError_t e = launch_pipe<128, 3, 1, 1, 2>(p, n_segs, (int)ring_rows, s);
    if (e != cudaErrorNotSupported) return e;
  }
  const uint32_t cols = p.B <= 128 ? 256u : 512u;
  cudaError_t e = cudaFuncSetAttribute(beacon_update_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  beacon_update_tc_kernel<<<(unsigned)(n_req * p.layers * p.hkv), kUT, smem, s>>>(p, cols);
  return cudaGetLastError();
}

}  // namespace kvc
