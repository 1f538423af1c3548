// decode_attention.cu -- one decode step of grouped-query attention over the
// compacted paged cache: for every (layer, request, query head) the softmax
// attention of the step's query over the request's cached rows [0, length).
//
// What it computes (Random Attention article, "发现四": every selector runs
// on the same paged attention kernels; eviction only changes which rows they
// read): s_j = scale * q . k_j, out = sum_j softmax(s)_j v_j and
// lse = log sum_j exp(s_j), with query head hq reading KV head hq / G.  The
// rows of a segment may sit in any slot order (hole-filling compaction):
// attention does not depend on it.
//
// Design (B200): the kernel is HBM-bound (each K and V byte is used by the
// G query heads of its KV head only, 2G flop per element), so it runs on the
// CUDA cores and spends its effort on keeping HBM busy.
//   * Work unit = (layer, request, KV head, split of the pages); one CTA of
//     128 threads each.  Splits give short batches enough CTAs; a second
//     kernel merges the per-split (max, sum, output) partials.
//   * Tiles of 4 pages (64 rows): the K and V rows of a page are 16
//     consecutive pool rows, fetched by one elected thread as 2-D TMA tiles
//     (128-byte boxes, 128-byte swizzle) into a ring of stages with
//     transaction-count mbarriers, so loads of later tiles overlap compute.
//   * Scores: two threads per row, each half the dimensions; with the
//     swizzle, the 8 lanes of a quarter-warp read 8 different rows' chunks
//     from 8 different bank groups while reading the same query chunk
//     (broadcast).  Online softmax in base 2 with the scale folded into q.
//   * P.V: each thread owns 8 bytes of a row (4 bf16 dimensions) for all G
//     heads and walks a quarter of the tile's rows; the row groups are added
//     at the end.
// Every mbarrier wait is bounded: on timeout the kernel records
// kDevTimeout in the status word, lets its own copies land (bounded) and
// leaves, all threads of the CTA together.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include "kvc_internal.h"
#include "tc_ptx.cuh"

namespace kvc {
namespace {

constexpr int kThreads = 128;
constexpr int kTilePages = 4;
constexpr int kTileRows = kTilePages * kPage;  // 64
constexpr int kBox = 128;                      // bytes per TMA box row (the swizzle span)
constexpr float kLn2 = 0.6931471805599453f;

template <typename T>
__device__ __forceinline__ void load_chunk(const uint8_t *p, float (&x)[16 / sizeof(T)]);
template <>
__device__ __forceinline__ void load_chunk<__nv_bfloat16>(const uint8_t *p, float (&x)[8]) {
  const uint4 u = *reinterpret_cast<const uint4 *>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}
template <>
__device__ __forceinline__ void load_chunk<float>(const uint8_t *p, float (&x)[4]) {
  const float4 u = *reinterpret_cast<const float4 *>(p);
  x[0] = u.x;
  x[1] = u.y;
  x[2] = u.z;
  x[3] = u.w;
}
template <typename T>
__device__ __forceinline__ void load_pair8(const uint8_t *p, float (&x)[8 / sizeof(T)]);
template <>
__device__ __forceinline__ void load_pair8<__nv_bfloat16>(const uint8_t *p, float (&x)[4]) {
  const uint2 u = *reinterpret_cast<const uint2 *>(p);
  x[0] = __uint_as_float(u.x << 16);
  x[1] = __uint_as_float(u.x & 0xffff0000u);
  x[2] = __uint_as_float(u.y << 16);
  x[3] = __uint_as_float(u.y & 0xffff0000u);
}
template <>
__device__ __forceinline__ void load_pair8<float>(const uint8_t *p, float (&x)[2]) {
  const float2 u = *reinterpret_cast<const float2 *>(p);
  x[0] = u.x;
  x[1] = u.y;
}
__device__ __forceinline__ float to_float(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ float to_float(float v) { return v; }

template <typename T, int D, int G>
struct AttnShape {
  static constexpr int kRowBytes = D * (int)sizeof(T);
  static constexpr int kBoxes = kRowBytes / kBox;           // boxes per row (>= 1)
  static constexpr int kChunks = kRowBytes / 16;            // 16-byte chunks per row
  static constexpr int kHalfChunks = kChunks / 2;
  static constexpr int kEpc = 16 / (int)sizeof(T);          // elements per chunk
  static constexpr int kPageBox = kPage * kBox;             // 2 KB: one page, one box
  static constexpr int kPageBytes = kBoxes * kPageBox;      // one page of K (or V)
  static constexpr int kStageBytes = 2 * kTilePages * kPageBytes;
  static constexpr int kStages = kStageBytes <= 32768 ? 3 : 2;
  static constexpr int kVt = 8 / (int)sizeof(T);            // V elements per thread per row
  static constexpr int kVThreadsPerRow = kRowBytes / 8;
  static constexpr int kVGroups = kThreads / kVThreadsPerRow;
  static constexpr int kRedBytes = kVGroups * G * D * 4;
  static constexpr size_t kSmem = 1024 + (size_t)kStages * kStageBytes + 1024;
  static_assert(kRowBytes % kBox == 0, "rows must be whole 128-byte boxes");
  static_assert(kVGroups >= 1 && kThreads % kVThreadsPerRow == 0, "V mapping");
  static_assert(kRedBytes <= kStages * kStageBytes, "reduction buffer reuses the stages");
};

// byte offset, inside a page's K (or V) block, of 16-byte chunk c of row rr
template <int kBoxes>
__device__ __forceinline__ uint32_t chunk_off(int rr, int c) {
  return (uint32_t)((c >> 3) * (kPage * kBox) + rr * kBox + (((c & 7) ^ (rr & 7)) << 4));
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads) decode_attention_kernel(const __grid_constant__ CUtensorMap kmap,
                                                                   const __grid_constant__ CUtensorMap vmap,
                                                                   DecodeAttnParams p) {
  using S = AttnShape<T, D, G>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(16) float q_s[G][D];
  __shared__ __align__(16) float p_s[kTileRows][G];
  __shared__ float wmax[4][G];
  __shared__ float wsum[4][G];
  __shared__ __align__(8) uint64_t full[S::kStages];
  __shared__ int abort_flag_s;
  volatile int *abort_flag = &abort_flag_s;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int unit = blockIdx.x;
  const int split = unit % p.nsplit;
  const int h = (unit / p.nsplit) % p.hkv;
  const int r = (unit / (p.nsplit * p.hkv)) % p.R;
  const int lc = unit / (p.nsplit * p.hkv * p.R);
  const int l = p.layer_begin + lc;
  const int len = p.lengths[r];
  const int n_pages = (len + kPage - 1) / kPage;
  const int pg0 = split * p.pages_per_split;
  const int pg1 = min(n_pages, pg0 + p.pages_per_split);
  const int n_tiles = pg1 > pg0 ? (pg1 - pg0 + kTilePages - 1) / kTilePages : 0;
  const int32_t *bt = p.block_table + (int64_t)r * p.bt_stride;

  if (tid == 0) {
    for (int i = 0; i < S::kStages; ++i) mbar_init(&full[i], 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // this CTA's G query rows, pre-scaled into base 2
  {
    const T *q = reinterpret_cast<const T *>(p.q) + (((int64_t)lc * p.R + r) * p.hq + (int64_t)h * G) * D;
    for (int i = tid; i < G * D; i += kThreads) (&q_s[0][0])[i] = to_float(q[i]) * p.qscale;
  }
  __syncthreads();

  auto issue_tile = [&](int t) {  // one elected thread
    const int st = t % S::kStages;
    uint8_t *kd = smem + st * S::kStageBytes;
    uint8_t *vd = kd + kTilePages * S::kPageBytes;
    const int a = pg0 + t * kTilePages;
    const int np = min(kTilePages, pg1 - a);
    mbar_expect_tx(&full[st], (uint32_t)(np * S::kPageBytes * 2));
    for (int i = 0; i < np; ++i) {
      const int64_t row0 = (((int64_t)l * p.num_pages + bt[a + i]) * p.hkv + h) * kPage;
#pragma unroll
      for (int b = 0; b < S::kBoxes; ++b) {
        const int x = b * (kBox / (int)sizeof(T));
        tma_load_2d(smem_u32(kd + i * S::kPageBytes + b * S::kPageBox), &kmap, x, (int)row0, &full[st]);
        tma_load_2d(smem_u32(vd + i * S::kPageBytes + b * S::kPageBox), &vmap, x, (int)row0, &full[st]);
      }
    }
  };
  if (tid == 0)
    for (int t = 0; t < min(n_tiles, S::kStages); ++t) issue_tile(t);

  float m_run[G], l_w[G], acc[G][S::kVt];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m_run[g] = -INFINITY;
    l_w[g] = 0.f;
#pragma unroll
    for (int e = 0; e < S::kVt; ++e) acc[g][e] = 0.f;
  }
  // score mapping: warp w takes page w of the tile; lanes l and l^8 share a row
  const int half = (lane >> 3) & 1;
  const int rr = (lane & 7) + 8 * (lane >> 4);
  // V mapping
  const int vg = tid / S::kVThreadsPerRow;
  const int vslot = tid % S::kVThreadsPerRow;

  int t = 0;
  for (; t < n_tiles; ++t) {
    const int st = t % S::kStages;
    // every thread waits for the tile (acquiring the TMA's writes); the
    // decision to leave on a timeout is made block-wide below
    const bool landed = mbar_wait(&full[st], (uint32_t)((t / S::kStages) & 1), abort_flag, p.status);
    const uint8_t *kt = smem + st * S::kStageBytes;
    const uint8_t *vt = kt + kTilePages * S::kPageBytes;
    const int row0 = (pg0 + t * kTilePages) * kPage;  // slot of the tile's first row
    const int valid = min(kTileRows, len - row0);

    // 1. scores of row (warp, rr)
    float s[G];
#pragma unroll
    for (int g = 0; g < G; ++g) s[g] = 0.f;
    const uint8_t *kp = kt + warp * S::kPageBytes;
#pragma unroll
    for (int i = 0; i < S::kHalfChunks; ++i) {
      const int c = half * S::kHalfChunks + i;
      float x[S::kEpc];
      load_chunk<T>(kp + chunk_off<S::kBoxes>(rr, c), x);
#pragma unroll
      for (int g = 0; g < G; ++g) {
#pragma unroll
        for (int e = 0; e < S::kEpc; e += 4) {
          const float4 qv = *reinterpret_cast<const float4 *>(&q_s[g][c * S::kEpc + e]);
          s[g] = fmaf(qv.x, x[e], s[g]);
          s[g] = fmaf(qv.y, x[e + 1], s[g]);
          s[g] = fmaf(qv.z, x[e + 2], s[g]);
          s[g] = fmaf(qv.w, x[e + 3], s[g]);
        }
      }
    }
    const int row = warp * kPage + rr;
    const bool ok = row < valid;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      s[g] += __shfl_xor_sync(0xffffffffu, s[g], 8);
      s[g] = ok ? s[g] : -INFINITY;
      float mx = s[g];
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      if (lane == 0) wmax[warp][g] = mx;
    }
    if (__syncthreads_or(!landed)) break;
    // 2. running max, weights, per-warp sums
    float alpha[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float tmax = fmaxf(fmaxf(wmax[0][g], wmax[1][g]), fmaxf(wmax[2][g], wmax[3][g]));
      const float m_new = fmaxf(m_run[g], tmax);
      alpha[g] = exp2f(m_run[g] - m_new);
      m_run[g] = m_new;
      const float pw = ok ? exp2f(s[g] - m_new) : 0.f;
      if (half == 0) p_s[row][g] = pw;
      float sum = half == 0 ? pw : 0.f;
      sum += __shfl_xor_sync(0xffffffffu, sum, 1);
      sum += __shfl_xor_sync(0xffffffffu, sum, 2);
      sum += __shfl_xor_sync(0xffffffffu, sum, 4);
      sum += __shfl_xor_sync(0xffffffffu, sum, 8);
      sum += __shfl_xor_sync(0xffffffffu, sum, 16);
      l_w[g] = l_w[g] * alpha[g] + sum;
    }
    __syncthreads();
    // 3. acc = acc * alpha + P.V over this thread's rows
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int e = 0; e < S::kVt; ++e) acc[g][e] *= alpha[g];
    {
      const int c = vslot >> 1;
      const int sub = (vslot & 1) * 8;
#pragma unroll 4
      for (int vr = vg; vr < valid; vr += S::kVGroups) {
        const int pg = vr >> 4, vrr = vr & 15;
        float x[S::kVt];
        load_pair8<T>(vt + pg * S::kPageBytes + chunk_off<S::kBoxes>(vrr, c) + sub, x);
        float pw[G];
        if constexpr (G % 4 == 0) {
#pragma unroll
          for (int g = 0; g < G; g += 4) {
            const float4 w4 = *reinterpret_cast<const float4 *>(&p_s[vr][g]);
            pw[g] = w4.x;
            pw[g + 1] = w4.y;
            pw[g + 2] = w4.z;
            pw[g + 3] = w4.w;
          }
        } else {
#pragma unroll
          for (int g = 0; g < G; ++g) pw[g] = p_s[vr][g];
        }
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
          for (int e = 0; e < S::kVt; ++e) acc[g][e] = fmaf(pw[g], x[e], acc[g][e]);
      }
    }
    __syncthreads();  // stage st and p_s are free again
    if (tid == 0 && t + S::kStages < n_tiles) issue_tile(t + S::kStages);
  }
  if (t < n_tiles) {
    // a wait ran out: let this CTA's copies land (bounded) and leave
    if (tid == 0)
      for (int k = t; k < min(n_tiles, t + S::kStages); ++k)
        mbar_wait(&full[k % S::kStages], (uint32_t)((k / S::kStages) & 1), abort_flag, p.status, false);
    return;
  }

  // 4. combine the row groups and the warps' sums
  float *red = reinterpret_cast<float *>(smem);  // [kVGroups][G][D]
  {
    const int d0 = vslot * S::kVt;
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int e = 0; e < S::kVt; ++e) red[(vg * G + g) * D + d0 + e] = acc[g][e];
  }
  if (lane == 0)
#pragma unroll
    for (int g = 0; g < G; ++g) wsum[warp][g] = l_w[g];
  __syncthreads();
  const int64_t head0 = ((int64_t)lc * p.R + r) * p.hq + (int64_t)h * G;  // first query head row
  for (int i = tid; i < G * D; i += kThreads) {
    const int g = i / D;
    float o = 0.f;
#pragma unroll
    for (int k = 0; k < S::kVGroups; ++k) o += red[k * G * D + i];
    const float lsum = wsum[0][g] + wsum[1][g] + wsum[2][g] + wsum[3][g];
    if (p.nsplit == 1) {
      p.out[head0 * D + i] = lsum > 0.f ? o / lsum : 0.f;
      if (p.lse && (i % D) == 0)
        p.lse[head0 + g] = lsum > 0.f ? (m_run[g] + log2f(lsum)) * kLn2 : -INFINITY;
    } else {
      const int64_t pu = (head0 + g) * p.nsplit + split;  // partial row of (query head, split)
      p.part_o[pu * D + (i % D)] = o;
      if ((i % D) == 0) {
        p.part_ml[pu * 2] = n_tiles > 0 ? m_run[g] : -INFINITY;
        p.part_ml[pu * 2 + 1] = lsum;
      }
    }
  }
}

// merge the splits of one (layer, request, KV head): G*D outputs
__global__ void __launch_bounds__(kThreads) decode_attention_merge_kernel(DecodeAttnParams p, int G, int D) {
  const int64_t head0 = (int64_t)blockIdx.x * G;
  for (int i = threadIdx.x; i < G * D; i += kThreads) {
    const int g = i / D, c = i % D;
    const int64_t pu0 = (head0 + g) * p.nsplit;
    float m = -INFINITY;
    for (int s = 0; s < p.nsplit; ++s) m = fmaxf(m, p.part_ml[(pu0 + s) * 2]);
    float o = 0.f, l = 0.f;
    if (m != -INFINITY) {
      for (int s = 0; s < p.nsplit; ++s) {
        const float ms = p.part_ml[(pu0 + s) * 2];
        if (ms == -INFINITY) continue;
        const float w = exp2f(ms - m);
        l = fmaf(p.part_ml[(pu0 + s) * 2 + 1], w, l);
        o = fmaf(p.part_o[(pu0 + s) * D + c], w, o);
      }
    }
    p.out[(head0 + g) * D + c] = l > 0.f ? o / l : 0.f;
    if (p.lse && c == 0) p.lse[head0 + g] = l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void *q = nullptr;
    cudaDriverEntryPointQueryResult res;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &q, cudaEnableDefault, &res) == cudaSuccess &&
        res == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(q);
  }
  return fn;
}

// pool viewed as [rows][D] of dtype, box (128 bytes of a row, 16 rows), 128-byte swizzle
bool make_pool_map(CUtensorMap *m, const void *base, uint64_t rows, int D, int dtype) {
  auto fn = encode_fn();
  if (!fn) return false;
  const int es = dtype == KVC_BF16 ? 2 : 4;
  cuuint64_t dims[2] = {(cuuint64_t)D, rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * es};
  cuuint32_t box[2] = {(cuuint32_t)(kBox / es), (cuuint32_t)kPage};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, dtype == KVC_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
            const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T, int D, int G>
cudaError_t launch_typed(const CUtensorMap &km, const CUtensorMap &vm, const DecodeAttnParams &p, int units,
                         cudaStream_t s) {
  using S = AttnShape<T, D, G>;
  cudaError_t e = cudaFuncSetAttribute(decode_attention_kernel<T, D, G>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)S::kSmem);
  if (e != cudaSuccess) return e;
  decode_attention_kernel<T, D, G><<<units, kThreads, S::kSmem, s>>>(km, vm, p);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_g(const CUtensorMap &km, const CUtensorMap &vm, const DecodeAttnParams &p, int G, int units,
                     cudaStream_t s) {
  switch (G) {
    case 1: return launch_typed<T, D, 1>(km, vm, p, units, s);
    case 2: return launch_typed<T, D, 2>(km, vm, p, units, s);
    case 4: return launch_typed<T, D, 4>(km, vm, p, units, s);
    default: return launch_typed<T, D, 8>(km, vm, p, units, s);
  }
}

}  // namespace

bool decode_attention_supported(int dtype, int head_dim, int G) {
  return (dtype == KVC_BF16 || dtype == KVC_F32) && (head_dim == 64 || head_dim == 128) &&
         (G == 1 || G == 2 || G == 4 || G == 8) && encode_fn() != nullptr;
}

cudaError_t launch_decode_attention(const DecodeAttnParams &p, const void *k_pool, const void *v_pool,
                                    int64_t pool_rows, int head_dim, int dtype, int G, int *launches,
                                    cudaStream_t s) {
  *launches = 0;
  CUtensorMap km, vm;
  if (!make_pool_map(&km, k_pool, (uint64_t)pool_rows, head_dim, dtype) ||
      !make_pool_map(&vm, v_pool, (uint64_t)pool_rows, head_dim, dtype))
    return cudaErrorInvalidValue;
  const int units = p.layer_count * p.R * p.hkv * p.nsplit;
  if (units <= 0) return cudaSuccess;
  cudaError_t e;
  if (dtype == KVC_BF16)
    e = head_dim == 128 ? launch_g<__nv_bfloat16, 128>(km, vm, p, G, units, s)
                        : launch_g<__nv_bfloat16, 64>(km, vm, p, G, units, s);
  else
    e = head_dim == 128 ? launch_g<float, 128>(km, vm, p, G, units, s) : launch_g<float, 64>(km, vm, p, G, units, s);
  if (e != cudaSuccess) return e;
  *launches = 1;
  if (p.nsplit > 1) {
    decode_attention_merge_kernel<<<p.layer_count * p.R * p.hkv, kThreads, 0, s>>>(p, G, head_dim);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    *launches = 2;
  }
  return cudaSuccess;
}

}  // namespace kvc
