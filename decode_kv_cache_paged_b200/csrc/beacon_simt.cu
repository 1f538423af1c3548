// beacon_simt.cu -- BeaconKV beacon maintenance and the SIMT (fp32 FMA)
// beacon score.
//
// Update (BeaconKV explainer §3.2 "on_new_query": project, nearest beacon,
// periodic incremental update; BeaconKV abstract: beacons are compact
// representatives of global query clusters).  project() is the identity.  One
// CTA per (request, layer, KV head): the beacons sit in shared memory as
// fp32; the points are assigned in blocks of 64 with a register-tiled
// product (each thread 4 points x B/16 beacons, float4 operands, 8 FMAs per
// shared-memory load) on the expanded distance |c|^2 - 2 x.c, which has the
// same argmin; ties go to the lower beacon.  Then one warp per beacon gathers
// its points in point order with ballots and applies the running mean
// (n*c + sum)/(n + m).
//
// Score (the library's definition; the pages leave the importance rule open):
// z_bj = c_b.k_j/sqrt(d), lse_b = log sum_j exp(z_bj) over every cached key,
// score_j = max_b exp(z_bj - lse_b) over the generated keys.  Two passes over
// the segment's paged keys: pass 1 keeps an online (max, sum) per beacon,
// pass 2 recomputes z for the candidates.  Dot products are fp32 FMA chains
// over shared-memory tiles (keys padded to avoid bank conflicts, beacons read
// as broadcasts).  This kernel serves fp32 caches and is the baseline the
// tcgen05 kernel replaces for bf16.
#include <cuda_bf16.h>

#include "kvc_internal.h"

namespace kvc {
namespace {

template <int DT>
__device__ __forceinline__ float load_elem(const uint8_t *base, int64_t idx) {
  if (DT == KVC_BF16)
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(base)[idx]);
  else
    return reinterpret_cast<const float *>(base)[idx];
}

template <int DT>
__device__ __forceinline__ void store_scoring(uint8_t *base, int64_t idx, float v) {
  if (DT == KVC_BF16)
    reinterpret_cast<__nv_bfloat16 *>(base)[idx] = __float2bfloat16_rn(v);
  else
    reinterpret_cast<float *>(base)[idx] = v;
}

__device__ __forceinline__ void set_status(int32_t *status, int code) {
  atomicCAS(status, kDevOk, code);
}

constexpr int kUpdNT = 256;
constexpr int kPB = 64;  // points per assignment block

// One (request, layer, KV head) segment per CTA.  Shared memory: the beacons
// as fp32 rows padded to D+4 floats, a block of kPB points likewise, the
// beacons' squared norms and the assignment of every point.
template <int D, int DT>
__global__ void __launch_bounds__(kUpdNT) beacon_update_kernel(BeaconUpdateParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  constexpr int RS = D + 4;  // padded row stride (floats)
  float *cs = reinterpret_cast<float *>(smem);  // [B][RS]
  float *xs = cs + p.B * RS;                     // [kPB][RS]
  float *cn = xs + kPB * RS;                     // [B]
  int32_t *assign = reinterpret_cast<int32_t *>(cn + p.B);  // [W*G]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int h = blockIdx.x % p.hkv;
  const int l = (blockIdx.x / p.hkv) % p.layers;
  const UpdateDesc ud = p.descs[blockIdx.x / (p.hkv * p.layers)];
  const int r = ud.req;
  const int n_pts = ud.n_steps * p.G;
  const int64_t seg = ((int64_t)r * p.layers + l) * p.hkv + h;
  float *gbeac = p.beacons + seg * p.B * D;
  int32_t *gcnt = p.counts + seg * p.B;
  // element index of point pt's first coordinate in the ring
  auto point_base = [&](int pt) -> int64_t {
    const int step = pt / p.G, g = pt - step * p.G;
    const int ring = (ud.ring_start + step) % p.W;
    return ((((int64_t)r * p.layers + l) * p.W + ring) * p.hq + (h * p.G + g)) * D;
  };

  // beacons before this update (first update: points floor(i*n_pts/B))
  for (int e = tid; e < p.B * D; e += kUpdNT) {
    const int b = e / D, k = e - b * D;
    if (ud.init) {
      const int src = (int)(((int64_t)b * n_pts) / p.B);
      cs[b * RS + k] = load_elem<DT>(p.qring, point_base(src) + k);
    } else {
      cs[b * RS + k] = gbeac[e];
    }
  }
  __syncthreads();
  // squared norms of the beacons, for the expanded distance |c|^2 - 2 x.c
  // (|x|^2 is the same for every beacon of a point and does not move the argmin)
  for (int b = tid; b < p.B; b += kUpdNT) {
    float a = 0.f;
    for (int k = 0; k < D; ++k) a = fmaf(cs[b * RS + k], cs[b * RS + k], a);
    cn[b] = a;
  }

  // assignment, kPB points at a time: thread (ty, tx) owns points 4ty..4ty+3
  // of the block and beacons tx, tx+16, ...; dot products accumulate in k order
  constexpr int kMaxNB = kMaxBeacons / 16;
  const int ty = tid >> 4, tx = tid & 15;
  const int NB = (p.B + 15) >> 4;  // beacons tx + 16 j, j < NB, that are < B
  bool nan = false;
  for (int p0 = 0; p0 < n_pts; p0 += kPB) {
    __syncthreads();  // xs reuse
    constexpr int kVec = (DT == KVC_BF16) ? 8 : 4;  // elements per 16-byte load
    constexpr int kChunks = D / kVec;
    for (int e = tid; e < kPB * kChunks; e += kUpdNT) {
      const int pi = e / kChunks, c = e - pi * kChunks;
      const int pt = p0 + pi;
      float4 lo = make_float4(0.f, 0.f, 0.f, 0.f), hi = lo;
      if (pt < n_pts) {
        const uint8_t *src = p.qring + (point_base(pt) + c * kVec) * (DT == KVC_BF16 ? 2 : 4);
        const uint4 w = *reinterpret_cast<const uint4 *>(src);
        if (DT == KVC_BF16) {
          lo = make_float4(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xffff0000u),
                           __uint_as_float(w.y << 16), __uint_as_float(w.y & 0xffff0000u));
          hi = make_float4(__uint_as_float(w.z << 16), __uint_as_float(w.z & 0xffff0000u),
                           __uint_as_float(w.w << 16), __uint_as_float(w.w & 0xffff0000u));
        } else {
          lo = make_float4(__uint_as_float(w.x), __uint_as_float(w.y), __uint_as_float(w.z),
                           __uint_as_float(w.w));
        }
      }
      float4 *dst = reinterpret_cast<float4 *>(xs + pi * RS + c * kVec);
      dst[0] = lo;
      if (DT == KVC_BF16) dst[1] = hi;
    }
    __syncthreads();
    float acc[4][kMaxNB];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < kMaxNB; ++j) acc[i][j] = 0.f;
    const float4 *x4 = reinterpret_cast<const float4 *>(xs) + (ty * 4) * (RS / 4);
    const float4 *c4 = reinterpret_cast<const float4 *>(cs) + tx * (RS / 4);
#pragma unroll 2
    for (int k4 = 0; k4 < D / 4; ++k4) {
      float4 xv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) xv[i] = x4[i * (RS / 4) + k4];
#pragma unroll
      for (int j = 0; j < kMaxNB; ++j) {
        if (j < NB) {
          const float4 cv = c4[j * 16 * (RS / 4) + k4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float a = acc[i][j];
            a = fmaf(xv[i].x, cv.x, a);
            a = fmaf(xv[i].y, cv.y, a);
            a = fmaf(xv[i].z, cv.z, a);
            a = fmaf(xv[i].w, cv.w, a);
            acc[i][j] = a;
          }
        }
      }
    }
    // argmin over this thread's beacons, then over the 16 threads of the row
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float best = __int_as_float(0x7f800000);
      int besti = 0x7fffffff;
#pragma unroll
      for (int j = 0; j < kMaxNB; ++j) {
        const int b = tx + 16 * j;
        if (j < NB && b < p.B) {
          const float dist = fmaf(-2.f, acc[i][j], cn[b]);
          nan |= (dist != dist);
          if (dist < best) {
            best = dist;
            besti = b;
          }
        }
      }
#pragma unroll
      for (int o = 8; o >= 1; o >>= 1) {
        const float ob = __shfl_xor_sync(0xffffffffu, best, o);
        const int oi = __shfl_xor_sync(0xffffffffu, besti, o);
        if (ob < best || (ob == best && oi < besti)) {
          best = ob;
          besti = oi;
        }
      }
      const int pt = p0 + ty * 4 + i;
      if (tx == 0 && pt < n_pts) {
        const int a = besti == 0x7fffffff ? 0 : besti;  // all distances NaN: flagged below
        assign[pt] = a;
        if (p.assign_out) p.assign_out[seg * (int64_t)(p.W * p.G) + pt] = a;
      }
    }
  }
  if (nan) set_status(p.status, kDevNaN);
  __syncthreads();

  // running mean, one warp per beacon, points in order
  constexpr int kPer = D / 32;
  for (int b = warp; b < p.B; b += kUpdNT / 32) {
    float sum[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) sum[i] = 0.f;
    int m = 0;
    for (int c0 = 0; c0 < n_pts; c0 += 32) {
      const int pt = c0 + lane;
      unsigned mask = __ballot_sync(0xffffffffu, pt < n_pts && assign[pt] == b);
      while (mask) {
        const int i = __ffs(mask) - 1;
        mask &= mask - 1;
        const int64_t pb = point_base(c0 + i);
#pragma unroll
        for (int k = 0; k < kPer; ++k) sum[k] += load_elem<DT>(p.qring, pb + lane + 32 * k);
        ++m;
      }
    }
    const int n = ud.init ? 0 : gcnt[b];
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      const int e = b * D + lane + 32 * k;
      float v = cs[b * RS + lane + 32 * k];
      if (m > 0) v = ((float)n * v + sum[k]) / (float)(n + m);
      gbeac[e] = v;
      store_scoring<DT>(p.beacons_s, seg * p.B * D + e, v);
    }
    if (lane == 0) {
      gcnt[b] = n + m;
      p.trig[seg * p.B + b] = (float)m / (float)n_pts;
    }
  }
}

// ---------------------------------------------------------------- score --

constexpr int kScNT = 256;
constexpr int kTK = 32;  // keys per tile
constexpr int kNG = kScNT / kTK;

template <int D, int DT>
__global__ void __launch_bounds__(kScNT) beacon_score_simt_kernel(BeaconScoreParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  float *cs = reinterpret_cast<float *>(smem);  // [B][D]
  float *ks = cs + p.B * D;                      // [kTK][D+1]
  float *zs = ks + kTK * (D + 1);                // [B][kTK+1]
  float *lse = zs + p.B * (kTK + 1);             // [B]
  float *red = lse + p.B;                        // [kNG][kTK]
  float *wts = red + kNG * kTK;                   // [B] trigger shares (cluster-trigger mode)
  const int tid = threadIdx.x;
  const int h = blockIdx.x % p.hkv;
  const int l = (blockIdx.x / p.hkv) % p.layers;
  const SegDesc sd = p.segs[blockIdx.x / (p.hkv * p.layers)];
  const int r = sd.req, L = sd.L, P = sd.P;
  const int64_t seg = ((int64_t)r * p.layers + l) * p.hkv + h;
  const int32_t *bt = p.block_table + (int64_t)r * p.bt_stride;
  const float inv_sqrt_d = 1.0f / sqrtf((float)D);

  for (int e = tid; e < p.B * D; e += kScNT)
    cs[e] = load_elem<DT>(p.beacons_s, seg * p.B * D + e);
  if (p.trig)
    for (int e = tid; e < p.B; e += kScNT) wts[e] = p.trig[seg * p.B + e];

  const int jj = tid % kTK, bg = tid / kTK;
  auto load_tile = [&](int j0) {
    for (int e = tid; e < kTK * D; e += kScNT) {
      const int t = e / D, k = e - t * D;
      const int s = j0 + t;
      float v = 0.f;
      if (s < L) {
        const int64_t row = (((int64_t)l * p.num_pages + bt[s >> 4]) * p.hkv + h) * kPage + (s & 15);
        v = load_elem<DT>(p.k_pool, row * D + k);
      }
      ks[t * (D + 1) + k] = v;
    }
  };
  auto dots = [&]() {
    for (int b = bg; b < p.B; b += kNG) {
      const float *c = cs + b * D;
      const float *k = ks + jj * (D + 1);
      float acc = 0.f;
#pragma unroll 8
      for (int i = 0; i < D; ++i) acc = fmaf(c[i], k[i], acc);
      zs[b * (kTK + 1) + jj] = acc * inv_sqrt_d;
    }
  };

  // pass 1: online log-sum-exp per beacon over all L keys
  float run_m = __int_as_float(0xff800000), run_s = 0.f;  // thread b < B owns beacon b
#pragma unroll 1
  for (int j0 = 0; j0 < L; j0 += kTK) {
    __syncthreads();
    load_tile(j0);
    __syncthreads();
    dots();
    __syncthreads();
    if (tid < p.B) {
      const int nv = min(kTK, L - j0);
      const float *z = zs + tid * (kTK + 1);
      float tm = z[0];
      for (int t = 1; t < nv; ++t) tm = fmaxf(tm, z[t]);
      if (tm > run_m) {
        run_s *= expf(run_m - tm);
        run_m = tm;
      }
      for (int t = 0; t < nv; ++t) run_s += expf(z[t] - run_m);
    }
  }
  if (tid < p.B) {
    const float v = run_m + logf(run_s);
    lse[tid] = v;
    if (p.lse_out) p.lse_out[seg * p.B + tid] = v;
    if (v != v) set_status(p.status, kDevNaN);
  }

  // pass 2: per candidate key, max over beacons of z - lse (or the
  // trigger-weighted sum of the beacons' attention on it)
#pragma unroll 1
  for (int j0 = P; j0 < L; j0 += kTK) {
    __syncthreads();
    load_tile(j0);
    __syncthreads();
    dots();
    __syncthreads();
    if (p.trig) {
      // cluster trigger: sum over beacons of share_b * exp(z - lse_b)
      float acc = 0.f;
      for (int b = bg; b < p.B; b += kNG) acc = fmaf(wts[b], expf(zs[b * (kTK + 1) + jj] - lse[b]), acc);
      red[bg * kTK + jj] = acc;
    } else {
      float mx = __int_as_float(0xff800000);
      for (int b = bg; b < p.B; b += kNG) mx = fmaxf(mx, zs[b * (kTK + 1) + jj] - lse[b]);
      red[bg * kTK + jj] = mx;
    }
    __syncthreads();
    if (tid < kTK && j0 + tid < L) {
      float m = red[tid];
      float sc;
      if (p.trig) {
        for (int g = 1; g < kNG; ++g) m += red[g * kTK + tid];
        sc = m;
      } else {
        for (int g = 1; g < kNG; ++g) m = fmaxf(m, red[g * kTK + tid]);
        sc = expf(m);
      }
      if (sc != sc) set_status(p.status, kDevNaN);
      p.scores[seg * p.max_seq + (j0 + tid - P)] = sc;
    }
  }
}

}  // namespace

cudaError_t launch_beacon_update(const BeaconUpdateParams &p, int n_req, cudaStream_t s) {
  if (n_req <= 0) return cudaSuccess;
  const unsigned grid = (unsigned)(n_req * p.layers * p.hkv);
  const size_t smem = sizeof(float) * ((size_t)p.B * (p.d + 4) + (size_t)kPB * (p.d + 4) + p.B) +
                      (size_t)p.W * p.G * sizeof(int32_t);
  cudaError_t e = cudaErrorInvalidValue;
#define KVC_UPD(DV, DTV)                                                                      \
  if (p.d == DV && p.dtype == DTV) {                                                          \
    e = cudaFuncSetAttribute(beacon_update_kernel<DV, DTV>,                                   \
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);         \
    if (e == cudaSuccess) beacon_update_kernel<DV, DTV><<<grid, kUpdNT, smem, s>>>(p);        \
  }
  KVC_UPD(64, KVC_BF16)
  KVC_UPD(128, KVC_BF16)
  KVC_UPD(64, KVC_F32)
  KVC_UPD(128, KVC_F32)
#undef KVC_UPD
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_beacon_score_simt(const BeaconScoreParams &p, int n_req, cudaStream_t s) {
  if (n_req <= 0) return cudaSuccess;
  const unsigned grid = (unsigned)(n_req * p.layers * p.hkv);
  const size_t smem = sizeof(float) * ((size_t)p.B * p.d + (size_t)kTK * (p.d + 1) +
                                       (size_t)p.B * (kTK + 1) + p.B + kNG * kTK + p.B);
  cudaError_t e = cudaErrorInvalidValue;
#define KVC_SC(DV, DTV)                                                                       \
  if (p.d == DV && p.dtype == DTV) {                                                          \
    e = cudaFuncSetAttribute(beacon_score_simt_kernel<DV, DTV>,                               \
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);         \
    if (e == cudaSuccess) beacon_score_simt_kernel<DV, DTV><<<grid, kScNT, smem, s>>>(p);     \
  }
  KVC_SC(64, KVC_BF16)
  KVC_SC(128, KVC_BF16)
  KVC_SC(64, KVC_F32)
  KVC_SC(128, KVC_F32)
#undef KVC_SC
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace kvc
