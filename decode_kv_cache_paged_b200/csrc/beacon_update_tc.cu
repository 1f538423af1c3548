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
// the fp32 beacon.  One CTA of 128 threads per (request, layer, KV head):
// tiles of 128 points (TMEM lane = point) against all B beacons (N = B).
// Then a stable counting sort of the points by beacon (warp match) and one
// warp per beacon summing its points in point order.
#include <cuda_bf16.h>

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

__global__ void __launch_bounds__(kUT) beacon_update_tc_kernel(BeaconUpdateParams p, uint32_t tmem_cols) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_align<1024>(smem_raw);
  constexpr int D = 128;
  const int B = p.B, NP = p.W * p.G;
  uint8_t *xs = smem;                    // [2 K-blocks][128 rows][128 B]
  uint8_t *chi = xs + 32768;             // [2][B][128 B]
  uint8_t *clo = chi + B * 256;          // [2][B][128 B]
  float *cn = reinterpret_cast<float *>(clo + B * 256);  // [B]
  float *cpart = cn + B;                                  // [4][B]
  int32_t *assign = reinterpret_cast<int32_t *>(cpart + 4 * B);  // [NP]
  int32_t *order = assign + NP;                                   // [NP]
  int32_t *offs = order + NP;                                     // [B + 1]
  int32_t *cursor = offs + B + 1;                                 // [B]
  uint64_t *mbar = smem_align<16>(reinterpret_cast<uint64_t *>(cursor + B));
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

  // beacons: bf16 hi/lo terms in the swizzled layout, fp32 squared norms
  for (int b0 = 0; b0 < B; b0 += 4) {  // B is a multiple of 32
    float c[4], sq[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) c[u] = c_old(b0 + u, tid);
    const int kb = tid >> 6, k = tid & 63;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const __nv_bfloat16 hi = __float2bfloat16_rn(c[u]);
      const __nv_bfloat16 lo = __float2bfloat16_rn(c[u] - __bfloat162float(hi));
      *reinterpret_cast<__nv_bfloat16 *>(chi + kb * B * 128 + sw128_off(b0 + u, k)) = hi;
      *reinterpret_cast<__nv_bfloat16 *>(clo + kb * B * 128 + sw128_off(b0 + u, k)) = lo;
      sq[u] = c[u] * c[u];
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1)
#pragma unroll
      for (int u = 0; u < 4; ++u) sq[u] += __shfl_xor_sync(0xffffffffu, sq[u], o);
    if (lane == 0)
#pragma unroll
      for (int u = 0; u < 4; ++u) cpart[warp * B + b0 + u] = sq[u];
  }
  tmem_fence_before();
  __syncthreads();
  tmem_fence_after();
  const uint32_t tmem_base = *tslot;
  for (int b = tid; b < B; b += kUT) cn[b] = ((cpart[b] + cpart[B + b]) + cpart[2 * B + b]) + cpart[3 * B + b];

  // assignment, 128 points per tile
  const uint32_t idesc = idesc_bf16_f32(128, B);
  const uint32_t lane_addr = (uint32_t)(warp * 32) << 16;
  bool nan = false;
  int tile = 0;
  for (int p0 = 0; p0 < n_pts; p0 += 128, ++tile) {
    const int pt = p0 + tid;
    if (pt < n_pts) {
      const uint4 *src = reinterpret_cast<const uint4 *>(ring + point_base(pt));
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const uint4 w = src[c];
        *reinterpret_cast<uint4 *>(xs + (c >> 3) * 16384 + tid * 128 + (((c & 7) ^ (tid & 7)) << 4)) = w;
      }
    } else {
#pragma unroll
      for (int c = 0; c < 16; ++c)
        *reinterpret_cast<uint4 *>(xs + (c >> 3) * 16384 + tid * 128 + (((c & 7) ^ (tid & 7)) << 4)) =
            make_uint4(0, 0, 0, 0);
    }
    // the tensor core reads shared memory through the async proxy
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
            umma(tmem_base, a, bd, idesc, (term | kb | ks) != 0);
          }
      umma_commit(mbar);
      if (!mbar_wait(mbar, tile & 1, abort_flag, p.status)) *abort_flag = 1;
    }
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
    if (pt < n_pts) {
      assign[pt] = besti;
      if (p.assign_out) p.assign_out[seg * (int64_t)NP + pt] = besti;
    }
    tmem_fence_before();
    __syncthreads();  // xs and the accumulator are rewritten by the next tile
  }
  if (nan) atomicCAS(p.status, kDevOk, kDevNaN);

  if (!*abort_flag) {
    // stable counting sort of the points by beacon
    for (int b = tid; b <= B; b += kUT) offs[b] = 0;
    __syncthreads();
    for (int pt = tid; pt < n_pts; pt += kUT) atomicAdd(&offs[assign[pt] + 1], 1);
    __syncthreads();
    if (warp == 0) {
      int carry = 0;
      for (int b0 = 0; b0 <= B; b0 += 32) {
        const int b = b0 + lane;
        int v = b <= B ? offs[b] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int u = __shfl_up_sync(0xffffffffu, v, o);
          if (lane >= o) v += u;
        }
        if (b <= B) offs[b] = v + carry;
        carry += __shfl_sync(0xffffffffu, v, 31);
      }
      __syncwarp();
      for (int b = lane; b < B; b += 32) cursor[b] = offs[b];
      __syncwarp();
      for (int c0 = 0; c0 < n_pts; c0 += 32) {
        const int pt = c0 + lane;
        const int a = pt < n_pts ? assign[pt] : -1 - lane;  // distinct for lanes past the end
        const unsigned peers = __match_any_sync(0xffffffffu, a);
        const int leader = __ffs(peers) - 1;
        const int rank = __popc(peers & ((1u << lane) - 1u));
        int base = (lane == leader && a >= 0) ? cursor[a] : 0;
        base = __shfl_sync(0xffffffffu, base, leader);
        if (a >= 0) order[base + rank] = pt;
        __syncwarp();
        if (lane == leader && a >= 0) cursor[a] = base + __popc(peers);
        __syncwarp();
      }
    }
    __syncthreads();
    // running mean, one warp per beacon, its points in point order
    for (int b = warp; b < B; b += kUT / 32) {
      float sum[4] = {0.f, 0.f, 0.f, 0.f};
      const int o0 = offs[b], m = offs[b + 1] - o0;
      int i = 0;
      for (; i + 4 <= m; i += 4) {
        float x[4][4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int64_t pb = point_base(order[o0 + i + u]);
#pragma unroll
          for (int j = 0; j < 4; ++j) x[u][j] = __bfloat162float(ring[pb + lane + 32 * j]);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int j = 0; j < 4; ++j) sum[j] += x[u][j];
      }
      for (; i < m; ++i) {
        const int64_t pb = point_base(order[o0 + i]);
#pragma unroll
        for (int j = 0; j < 4; ++j) sum[j] += __bfloat162float(ring[pb + lane + 32 * j]);
      }
      const int n = ud.init ? 0 : gcnt[b];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int k = lane + 32 * j;
        float v = c_old(b, k);
        if (m > 0) v = ((float)n * v + sum[j]) / (float)(n + m);
        gbeac[b * D + k] = v;
        reinterpret_cast<__nv_bfloat16 *>(p.beacons_s)[seg * B * D + b * D + k] = __float2bfloat16_rn(v);
      }
      if (lane == 0) {
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

// B <= 128: the per-beacon sums are a second product.  After the argmin of a
// tile, A^T [beacons x points] holds a 1 at (a_p, p) and the tile's points X
// are summed per beacon by D_sum += A^T X (M = 128 beacon rows, N = 128 dims,
// K = 128 points), with X read as an MN-major operand: its 128-byte-swizzled
// K-major layout is the canonical MN-major one with 64-dimension blocks 16 KB
// apart (LBO) and 8-point groups 1 KB apart (SBO).  The sums of bf16 values
// accumulate in fp32 in TMEM across the segment's tiles; no point is read
// twice from global memory.
__global__ void __launch_bounds__(kUT) beacon_update_tc_scatter_kernel(BeaconUpdateParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_align<1024>(smem_raw);
  constexpr int D = 128;
  constexpr uint32_t kCols = 256;        // [0, 128) assignment product, [128, 256) sums
  const int B = p.B, NP = p.W * p.G;
  uint8_t *xs = smem;                    // [2 K-blocks][128 points][128 B]
  uint8_t *chi = xs + 32768;             // [2][B][128 B]
  uint8_t *clo = chi + B * 256;          // [2][B][128 B]
  uint8_t *asum = clo + B * 256;         // [2 point blocks][128 beacon rows][128 B], one-hot^T
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
                 "r"(kCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  // the one-hot tile starts at zero; counts at zero
  for (int i = tid; i < 32768 / 16; i += kUT) reinterpret_cast<uint4 *>(asum)[i] = make_uint4(0, 0, 0, 0);
  for (int b = tid; b < B; b += kUT) cnt[b] = 0;
  // beacons: bf16 hi/lo terms in the swizzled layout, fp32 squared norms
  for (int b0 = 0; b0 < B; b0 += 8) {  // B is a multiple of 32
    float c[8], sq[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) c[u] = c_old(b0 + u, tid);
    const int kb = tid >> 6, k = tid & 63;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const __nv_bfloat16 hi = __float2bfloat16_rn(c[u]);
      const __nv_bfloat16 lo = __float2bfloat16_rn(c[u] - __bfloat162float(hi));
      *reinterpret_cast<__nv_bfloat16 *>(chi + kb * B * 128 + sw128_off(b0 + u, k)) = hi;
      *reinterpret_cast<__nv_bfloat16 *>(clo + kb * B * 128 + sw128_off(b0 + u, k)) = lo;
      sq[u] = c[u] * c[u];
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1)
#pragma unroll
      for (int u = 0; u < 8; ++u) sq[u] += __shfl_xor_sync(0xffffffffu, sq[u], o);
    if (lane == 0)
#pragma unroll
      for (int u = 0; u < 8; ++u) cpart[warp * B + b0 + u] = sq[u];
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
  bool nan = false;
  int phase = 0;
  uint32_t prev_off = 0xffffffffu;  // where this thread's one-hot 1 of the previous tile sits
  for (int p0 = 0; p0 < n_pts; p0 += 128) {
    const int pt = p0 + tid;
    if (pt < n_pts) {
      const uint4 *src = reinterpret_cast<const uint4 *>(ring + point_base(pt));
      uint4 w[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) w[c] = src[c];
#pragma unroll
      for (int c = 0; c < 16; ++c)
        *reinterpret_cast<uint4 *>(xs + (c >> 3) * 16384 + tid * 128 + (((c & 7) ^ (tid & 7)) << 4)) = w[c];
    } else {
#pragma unroll
      for (int c = 0; c < 16; ++c)
        *reinterpret_cast<uint4 *>(xs + (c >> 3) * 16384 + tid * 128 + (((c & 7) ^ (tid & 7)) << 4)) =
            make_uint4(0, 0, 0, 0);
    }
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
    // one-hot column of this point: clear last tile's 1, set this one
    if (prev_off != 0xffffffffu) *reinterpret_cast<__nv_bfloat16 *>(asum + prev_off) = __float2bfloat16_rn(0.f);
    prev_off = 0xffffffffu;
    if (pt < n_pts) {
      if (p.assign_out) p.assign_out[seg * (int64_t)NP + pt] = besti;
      atomicAdd(&cnt[besti], 1);
      prev_off = (uint32_t)(tid >> 6) * 16384u + sw128_off(besti, tid & 63);
      *reinterpret_cast<__nv_bfloat16 *>(asum + prev_off) = __float2bfloat16_rn(1.f);
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
        umma(tmem_base + 128, a, bd, idesc_sum, (p0 > 0 || ks > 0) ? 1u : 0u);
      }
      umma_commit(mbar);
      if (!mbar_wait(mbar, phase & 1, abort_flag, p.status)) *abort_flag = 1;
    }
    ++phase;
    __syncthreads();  // xs, asum and the accumulators are reused by the next tile
    if (*abort_flag) break;
  }
  if (nan) atomicCAS(p.status, kDevOk, kDevNaN);

  if (!*abort_flag) {
    // running mean: thread b reads beacon b's sums (TMEM lane b, columns = dims)
    tmem_fence_after();
    float sum[D];
#pragma unroll
    for (int c0 = 0; c0 < D; c0 += 32) {
      float v[32];
      tmem_ld32(tmem_base + lane_addr + 128 + c0, v);
#pragma unroll
      for (int i = 0; i < 32; ++i) sum[c0 + i] = v[i];
    }
    const int b = tid;
    if (b < B) {
      const int m = cnt[b];
      const int n = ud.init ? 0 : gcnt[b];
      float4 *g4 = reinterpret_cast<float4 *>(gbeac + b * D);
      __nv_bfloat162 *s2 = reinterpret_cast<__nv_bfloat162 *>(reinterpret_cast<__nv_bfloat16 *>(p.beacons_s) +
                                                               seg * B * D + b * D);
#pragma unroll
      for (int k4 = 0; k4 < D / 4; ++k4) {
        float v[4];
        if (ud.init) {
#pragma unroll
          for (int e = 0; e < 4; ++e) v[e] = c_old(b, 4 * k4 + e);
        } else {
          const float4 o = g4[k4];
          v[0] = o.x; v[1] = o.y; v[2] = o.z; v[3] = o.w;
        }
        if (m > 0)
#pragma unroll
          for (int e = 0; e < 4; ++e) v[e] = ((float)n * v[e] + sum[4 * k4 + e]) / (float)(n + m);
        g4[k4] = make_float4(v[0], v[1], v[2], v[3]);
        s2[2 * k4] = __floats2bfloat162_rn(v[0], v[1]);
        s2[2 * k4 + 1] = __floats2bfloat162_rn(v[2], v[3]);
      }
      gcnt[b] = n + m;
      p.trig[seg * B + b] = (float)m / (float)n_pts;
    }
  }
  tmem_fence_before();
  __syncthreads();
  if (warp == 0) {
    tmem_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kCols));
  }
}

}  // namespace

bool beacon_update_tc_supported(int d, int B, int dtype) {
  return dtype == KVC_BF16 && d == 128 && B >= 32 && B <= 256 && B % 32 == 0;
}

cudaError_t launch_beacon_update_tc(const BeaconUpdateParams &p, int n_req, cudaStream_t s) {
  if (!beacon_update_tc_supported(p.d, p.B, p.dtype)) return cudaErrorNotSupported;
  if (n_req <= 0) return cudaSuccess;
  const int NP = p.W * p.G;
  if (p.B <= 128) {
    const size_t smem = 1024 + 32768 + (size_t)p.B * 512 + 32768 + (size_t)p.B * 4 * 6 + 64;
    cudaError_t e = cudaFuncSetAttribute(beacon_update_tc_scatter_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    beacon_update_tc_scatter_kernel<<<(unsigned)(n_req * p.layers * p.hkv), kUT, smem, s>>>(p);
    return cudaGetLastError();
  }
  // x tile, c_hi/c_lo tiles, cn + cpart[4] + cursor (6 floats/ints per beacon),
  // assign + order (2 ints per point), offs (B + 1), barrier/slot/flag
  const size_t smem = 1024 + 32768 + (size_t)p.B * 512 + (size_t)p.B * 4 * 6 + (size_t)NP * 8 +
                      (size_t)(p.B + 1) * 4 + 64;
  uint32_t cols = 32;
  while ((int)cols < p.B) cols <<= 1;
  cudaError_t e = cudaFuncSetAttribute(beacon_update_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  beacon_update_tc_kernel<<<(unsigned)(n_req * p.layers * p.hkv), kUT, smem, s>>>(p, cols);
  return cudaGetLastError();
}

}  // namespace kvc
