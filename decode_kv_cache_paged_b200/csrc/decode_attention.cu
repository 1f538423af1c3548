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
//     4 warps each.  Splits give short batches enough CTAs; a second kernel
//     merges the per-split (max, sum, output) partials.
//   * Each warp walks every 4th page of the unit on its own: the K rows and
//     the V rows of a page are each 16 consecutive pool rows, so one bulk
//     copy apiece (a contiguous 4 KB at bf16 d = 128) brings them into the
//     warp's 2-slot ring, completing on a transaction-count mbarrier.  Warps
//     keep their own running max and sums, so no block-wide barrier is taken
//     until the four warps' states are merged at the end.
//   * Scores: every lane owns one 16-byte chunk of the row (the same chunk
//     for every row it scores) and keeps that chunk of the G query rows in
//     registers, so the only shared-memory reads of the score step are the
//     K rows themselves, a quarter-warp reading 128 consecutive bytes.  The
//     lanes of a row then sum their partial dot products with a butterfly
//     reduce-scatter (each exchange halves the sums a lane holds), ending
//     with each lane holding whole scores of one row for a few heads; each
//     lane stores its partial sums in a lane-dependent order so that the
//     exchanges need no selects.  The
//     query used to be re-read from shared memory for every chunk, which
//     made the shared-memory data pipe the limit.  Online softmax in base 2
//     with the scale folded into q.
//   * P.V: each lane owns 8-byte segments of a row for all G heads.
//   * Products and sums use the packed two-wide fp32 FMA of sm_100 (the
//     same rounding as two scalar FMAs, half the instructions).
// Every mbarrier wait is bounded: on timeout the kernel records
// kDevTimeout in the status word, lets its own copies land (bounded) and
// leaves, all threads of the CTA together.
#include <cuda_bf16.h>

#include "kvc_internal.h"
#include "tc_ptx.cuh"

namespace kvc {
namespace {

#ifndef KVC_ATTN_STAGES
#define KVC_ATTN_STAGES 2
#endif

constexpr int kThreads = 128;
constexpr float kLn2 = 0.6931471805599453f;

// bf16 pair / fp32 pair of a 32-bit or 64-bit word as a float2
__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// 16-byte chunk as float2 pairs
template <typename T>
__device__ __forceinline__ void load_chunk2(const uint8_t *p, float2 (&x)[16 / sizeof(T) / 2]);
template <>
__device__ __forceinline__ void load_chunk2<__nv_bfloat16>(const uint8_t *p, float2 (&x)[4]) {
  const uint4 u = *reinterpret_cast<const uint4 *>(p);
  x[0] = bf16x2_to_float2(u.x);
  x[1] = bf16x2_to_float2(u.y);
  x[2] = bf16x2_to_float2(u.z);
  x[3] = bf16x2_to_float2(u.w);
}
template <>
__device__ __forceinline__ void load_chunk2<float>(const uint8_t *p, float2 (&x)[2]) {
  const float4 u = *reinterpret_cast<const float4 *>(p);
  x[0] = make_float2(u.x, u.y);
  x[1] = make_float2(u.z, u.w);
}
// 8 bytes as float2 pairs
template <typename T>
__device__ __forceinline__ void load_8b2(const uint8_t *p, float2 (&x)[8 / sizeof(T) / 2]);
template <>
__device__ __forceinline__ void load_8b2<__nv_bfloat16>(const uint8_t *p, float2 (&x)[2]) {
  const uint2 u = *reinterpret_cast<const uint2 *>(p);
  x[0] = bf16x2_to_float2(u.x);
  x[1] = bf16x2_to_float2(u.y);
}
template <>
__device__ __forceinline__ void load_8b2<float>(const uint8_t *p, float2 (&x)[1]) {
  x[0] = *reinterpret_cast<const float2 *>(p);
}
__device__ __forceinline__ float to_float(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ float to_float(float v) { return v; }

template <typename T, int D, int G>
struct AttnShape {
  static constexpr int kRowBytes = D * (int)sizeof(T);
  static constexpr int kChunks = kRowBytes / 16;           // 16-byte chunks per row
  static constexpr int kPairs = 16 / (int)sizeof(T) / 2;   // element pairs per chunk
  static constexpr int kEpc = 2 * kPairs;                  // elements per chunk
  static constexpr int kPageBytes = kPage * kRowBytes;     // one page of K (or V): 16 rows, contiguous
  static constexpr int kSlotBytes = 2 * kPageBytes;        // K and V of one page
  static constexpr int kWarpStages = KVC_ATTN_STAGES;      // page slots per warp
  static constexpr int kWarps = kThreads / 32;
  static constexpr size_t kSmem = 128 + (size_t)kWarps * kWarpStages * kSlotBytes;
  // P.V: each lane owns 8-byte segments of a row; short rows are walked
  // kRowPar at a time by lane groups
  static constexpr int kSeg = kRowBytes >= 256 ? kRowBytes / 256 : 1;
  static constexpr int kRowPar = kRowBytes >= 256 ? 1 : 256 / kRowBytes;
  static constexpr int kVp = 8 / (int)sizeof(T) / 2;       // element pairs per 8-byte segment
  static constexpr int kAccPairs = kSeg * kVp;             // accumulator pairs per head per lane
  // scores: kLpr lanes per row, one chunk each; a warp scores kRowGroups rows
  // at once; a lane's partial sums are reduced kRb rows (kNv sums) at a time
  static constexpr int kLpr = kChunks;
  static constexpr int kRowGroups = 32 / kLpr;
  static constexpr int kRowsPerGroup = kPage / kRowGroups;
  static constexpr int kRb = kRowsPerGroup < 32 / G ? kRowsPerGroup : 32 / G;
  static constexpr int kBatches = kRowsPerGroup / kRb;
  static constexpr int kNv = kRb * G;
  // after the reduce-scatter a lane holds kKeep whole scores (consecutive
  // heads of one row); kDup lanes hold each score when kNv < kLpr
  static constexpr int kKeep = kNv >= kLpr ? kNv / kLpr : 1;
  static constexpr int kDup = kNv >= kLpr ? 1 : kLpr / kNv;
  // lanes xor-apart by at least kHeadMask hold the same heads (other rows)
  static constexpr int kHeadMask = kLpr / kRb;
  static_assert(kRowBytes >= 128 && kRowBytes <= 512, "row size");
  static_assert(kKeep < G || G == 1, "a lane keeps part of the heads of one row");
  static_assert(kHeadMask >= 2 && kHeadMask <= 32 && kDup <= kHeadMask, "lane classes");
  static_assert((size_t)kWarps * G * D * 4 <= (size_t)kWarps * kWarpStages * kSlotBytes,
                "the merge buffer reuses the page slots");
};

// Reduce-scatter of N partial sums over the lanes xor M, M/2, ..., 1 apart:
// each exchange keeps the lower half of the sums still held and adds the
// partner's upper half; once a lane holds one sum the remaining exchanges add
// the partner's copy of it.  The lanes store their partial sums permuted (see
// the kernel) so that at every exchange the lower half holds the entries this
// lane keeps and the upper half those its partner keeps: no selects.
// Afterwards, with M = the lanes of a row / 2, lane c of the row holds the
// whole sums of entries c * N / (2M) + k, k < max(1, N / (2M)), in v[k].
template <int N, int M, int NV>
__device__ __forceinline__ void reduce_scatter(float (&v)[NV]) {
  if constexpr (M >= 1) {
    if constexpr (N > 1) {
#pragma unroll
      for (int k = 0; k < N / 2; ++k) v[k] += __shfl_xor_sync(0xffffffffu, v[k + N / 2], M);
      reduce_scatter<N / 2, M / 2>(v);
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], M);
      reduce_scatter<1, M / 2>(v);
    }
  }
}

constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x / 2); }

// Each of the 4 warps walks every 4th page of the CTA's split through its own
// 2-slot ring (K and V of one page per slot), with its own running max and
// sums; no block-wide barrier is taken until the warps' states are merged.
template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads) decode_attention_kernel(DecodeAttnParams p) {
  using S = AttnShape<T, D, G>;
  constexpr int W = S::kWarps, NS = S::kWarpStages, KEEP = S::kKeep;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_align<128>(smem_raw);
  __shared__ __align__(16) float p_s[W][kPage][G];  // the page's softmax weights
  __shared__ __align__(16) float a_s[W][G];         // the page's rescale factors
  __shared__ float m_s[W][G], l_s[W][G];
  __shared__ __align__(8) uint64_t full[W][NS];
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
  const int n_my = pg1 - pg0 > warp ? (pg1 - pg0 - warp + W - 1) / W : 0;  // pages of this warp
  const int32_t *bt = p.block_table + (int64_t)r * p.bt_stride;
  uint8_t *ring = smem + warp * NS * S::kSlotBytes;

  if (tid == 0) {
    for (int w = 0; w < W; ++w)
      for (int i = 0; i < NS; ++i) mbar_init(&full[w][i], 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  // lanes 0 and 1 copy page k's K and V rows (each one contiguous block of
  // 16 rows) into the warp's slot
  auto issue_page = [&](int k) {
    const int slot = k % NS;
    const int page = pg0 + warp + k * W;
    if (lane == 0) mbar_expect_tx(&full[warp][slot], (uint32_t)S::kSlotBytes);
    __syncwarp();
    if (lane < 2) {
      const int64_t row0 = (((int64_t)l * p.num_pages + bt[page]) * p.hkv + h) * kPage;
      const uint8_t *src = (lane ? p.v_pool : p.k_pool) + row0 * S::kRowBytes;
      bulk_load(smem_u32(ring + slot * S::kSlotBytes + lane * S::kPageBytes), src, (uint32_t)S::kPageBytes,
                &full[warp][slot]);
    }
  };
  for (int k = 0; k < min(n_my, NS); ++k) issue_page(k);

  // scoring lanes: chunk c of the rows of row group grp; the whole scores a
  // lane ends with are of entries e0 + k (row e0 / G of a batch, heads g0 + k)
  const int c = lane % S::kLpr;
  const int grp = lane / S::kLpr;
  const int e0 = (c / S::kDup) * KEEP;
  const int g0 = e0 % G;
  const bool writer = (c % S::kDup) == 0;  // one lane of each set of copies stores

  // The lane stores partial sum (i, g) of a batch in slot (i ^ p_row, g ^
  // p_head): its lane bit of the exchange at mask kLpr/2 >> st flips slot bit
  // log2(kNv) - 1 - st, for the exchanges that split.  Then at every exchange
  // the entries this lane keeps sit in the lower half of its array and the
  // ones its partner keeps in the upper half.
  int perm = 0;
  {
    constexpr int kLogNv = ilog2(S::kNv), kSplit = ilog2(S::kLpr) < kLogNv ? ilog2(S::kLpr) : kLogNv;
#pragma unroll
    for (int st = 0; st < kSplit; ++st)
      if (lane & ((S::kLpr / 2) >> st)) perm |= 1 << (kLogNv - 1 - st);
  }
  const int p_row = perm >> ilog2(G), p_head = perm & (G - 1);

  // chunk c of this KV head's G query rows (head g ^ p_head in slot g), scaled
  // into base 2, in registers
  float2 qr[G][S::kPairs];
  {
    const T *q = reinterpret_cast<const T *>(p.q) + (((int64_t)lc * p.R + r) * p.hq + (int64_t)h * G) * D;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const T *qg = q + (g ^ p_head) * D + c * S::kEpc;
#pragma unroll
      for (int e = 0; e < S::kPairs; ++e)
        qr[g][e] = make_float2(to_float(qg[2 * e]) * p.qscale, to_float(qg[2 * e + 1]) * p.qscale);
    }
  }

  float m_run[KEEP], l_lane[KEEP];
  float2 acc[G][S::kAccPairs];
#pragma unroll
  for (int k = 0; k < KEEP; ++k) {
    m_run[k] = -INFINITY;
    l_lane[k] = 0.f;
  }
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < S::kAccPairs; ++e) acc[g][e] = make_float2(0.f, 0.f);
  // P.V: row group and 8-byte segment of this lane
  const int vgrp = lane / (32 / S::kRowPar);
  const int vlane = lane % (32 / S::kRowPar);

  int k = 0;
  for (; k < n_my; ++k) {
    const int slot = k % NS;
    const bool landed = mbar_wait(&full[warp][slot], (uint32_t)((k / NS) & 1), abort_flag, p.status);
    if (__any_sync(0xffffffffu, !landed)) break;
    const uint8_t *kp = ring + slot * S::kSlotBytes;
    const uint8_t *vp = kp + S::kPageBytes;
    const int valid = min(kPage, len - (pg0 + warp + k * W) * kPage);

    // 1. scores: partial dot products of chunk c, reduced across the row's lanes
    float sv[S::kBatches][KEEP];
#pragma unroll
    for (int b = 0; b < S::kBatches; ++b) {
      float part[S::kNv];  // slot i * G + g: row i ^ p_row of the batch, head g ^ p_head
#pragma unroll
      for (int i = 0; i < S::kRb; ++i) {
        const int row = grp * S::kRowsPerGroup + b * S::kRb + (i ^ p_row);
        float2 x[S::kPairs];
        load_chunk2<T>(kp + row * S::kRowBytes + c * 16, x);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          float2 t = __fmul2_rn(qr[g][0], x[0]);
#pragma unroll
          for (int e = 1; e < S::kPairs; ++e) t = __ffma2_rn(qr[g][e], x[e], t);
          part[i * G + g] = t.x + t.y;
        }
      }
      reduce_scatter<S::kNv, S::kLpr / 2>(part);
      const int row = grp * S::kRowsPerGroup + b * S::kRb + e0 / G;
#pragma unroll
      for (int kk = 0; kk < KEEP; ++kk) sv[b][kk] = row < valid ? part[kk] : -INFINITY;
    }

    // 2. online softmax per head: the max over the lanes holding that head
    float alpha[KEEP];
#pragma unroll
    for (int kk = 0; kk < KEEP; ++kk) {
      float mx = sv[0][kk];
#pragma unroll
      for (int b = 1; b < S::kBatches; ++b) mx = fmaxf(mx, sv[b][kk]);
#pragma unroll
      for (int m = S::kHeadMask; m < 32; m <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m));
      const float m_new = fmaxf(m_run[kk], mx);  // finite: a page has a valid row
      alpha[kk] = exp2f(m_run[kk] - m_new);
      m_run[kk] = m_new;
      float ps = 0.f;
#pragma unroll
      for (int b = 0; b < S::kBatches; ++b) {
        sv[b][kk] = exp2f(sv[b][kk] - m_new);  // 0 for rows past the end
        ps += sv[b][kk];
      }
      l_lane[kk] = fmaf(l_lane[kk], alpha[kk], ps);
    }
    if (writer) {
#pragma unroll
      for (int b = 0; b < S::kBatches; ++b) {
        float *dst = &p_s[warp][grp * S::kRowsPerGroup + b * S::kRb + e0 / G][g0];
        if constexpr (KEEP == 4)
          *reinterpret_cast<float4 *>(dst) = make_float4(sv[b][0], sv[b][1], sv[b][2], sv[b][3]);
        else if constexpr (KEEP == 2)
          *reinterpret_cast<float2 *>(dst) = make_float2(sv[b][0], sv[b][1]);
        else
#pragma unroll
          for (int kk = 0; kk < KEEP; ++kk) dst[kk] = sv[b][kk];
      }
      if (lane < S::kHeadMask)  // lanes below kHeadMask hold every head once
#pragma unroll
        for (int kk = 0; kk < KEEP; ++kk) a_s[warp][g0 + kk] = alpha[kk];
    }
    __syncwarp();

    // 3. acc = acc * alpha + P.V over the page's valid rows
    auto read_g = [&](const float *src, float (&w)[G]) {
      if constexpr (G % 4 == 0) {
#pragma unroll
        for (int g = 0; g < G; g += 4) {
          const float4 w4 = *reinterpret_cast<const float4 *>(src + g);
          w[g] = w4.x;
          w[g + 1] = w4.y;
          w[g + 2] = w4.z;
          w[g + 3] = w4.w;
        }
      } else {
#pragma unroll
        for (int g = 0; g < G; ++g) w[g] = src[g];
      }
    };
    {
      float a[G];
      read_g(a_s[warp], a);
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int e = 0; e < S::kAccPairs; ++e) acc[g][e] = __fmul2_rn(acc[g][e], make_float2(a[g], a[g]));
    }
    auto pv_row = [&](int vr) {
      float w[G];
      read_g(p_s[warp][vr], w);
#pragma unroll
      for (int sg = 0; sg < S::kSeg; ++sg) {
        const int byte = sg * 256 + vlane * 8;  // 8-byte segment within the row
        float2 x[S::kVp];
        load_8b2<T>(vp + vr * S::kRowBytes + byte, x);
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
          for (int e = 0; e < S::kVp; ++e)
            acc[g][sg * S::kVp + e] = __ffma2_rn(make_float2(w[g], w[g]), x[e], acc[g][sg * S::kVp + e]);
      }
    };
    if (valid == kPage) {
      // full page (all but a segment's last): rows known at compile time
#pragma unroll
      for (int i = 0; i < kPage / S::kRowPar; ++i) pv_row(i * S::kRowPar + vgrp);
    } else {
#pragma unroll 1
      for (int vr = vgrp; vr < valid; vr += S::kRowPar) pv_row(vr);
    }
    __syncwarp();  // the slot, p_s and a_s are free again
    if (k + NS < n_my) issue_page(k + NS);
  }
  if (k < n_my) {
    *abort_flag = 1;
    // let this warp's copies land (bounded) before the CTA may leave
    if (lane == 0)
      for (int j = k; j < min(n_my, k + NS); ++j)
        mbar_wait(&full[warp][j % NS], (uint32_t)((j / NS) & 1), abort_flag, p.status, false);
  }

  // 4. merge the warps: each writes (max, sum, accumulators)
#pragma unroll
  for (int kk = 0; kk < KEEP; ++kk) {
    float ls = l_lane[kk];
#pragma unroll
    for (int m = S::kHeadMask; m < 32; m <<= 1) ls += __shfl_xor_sync(0xffffffffu, ls, m);
    if (writer && lane < S::kHeadMask) {
      m_s[warp][g0 + kk] = m_run[kk];
      l_s[warp][g0 + kk] = ls;
    }
  }
  if constexpr (S::kRowPar > 1) {
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int e = 0; e < S::kAccPairs; ++e) {
        acc[g][e].x += __shfl_xor_sync(0xffffffffu, acc[g][e].x, 16);
        acc[g][e].y += __shfl_xor_sync(0xffffffffu, acc[g][e].y, 16);
      }
  }
  __syncthreads();  // every warp is past its loop: the page slots are free
  if (*abort_flag) return;
  float *red = reinterpret_cast<float *>(smem);  // [W][G][D]
  if (vgrp == 0) {
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int sg = 0; sg < S::kSeg; ++sg) {
        const int d0 = (sg * 256 + vlane * 8) / (int)sizeof(T);
#pragma unroll
        for (int e = 0; e < S::kVp; ++e)
          *reinterpret_cast<float2 *>(&red[(warp * G + g) * D + d0 + 2 * e]) = acc[g][sg * S::kVp + e];
      }
  }
  __syncthreads();
  const int64_t head0 = ((int64_t)lc * p.R + r) * p.hq + (int64_t)h * G;  // first query head row
  for (int i = tid; i < G * D; i += kThreads) {
    const int g = i / D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < W; ++w) M = fmaxf(M, m_s[w][g]);
    float o = 0.f, lsum = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < W; ++w) {
        if (m_s[w][g] == -INFINITY) continue;
        const float sc = exp2f(m_s[w][g] - M);
        o = fmaf(red[(w * G + g) * D + (i % D)], sc, o);
        lsum = fmaf(l_s[w][g], sc, lsum);
      }
    }
    if (p.nsplit == 1) {
      p.out[head0 * D + i] = lsum > 0.f ? o / lsum : 0.f;
      if (p.lse && (i % D) == 0) p.lse[head0 + g] = lsum > 0.f ? (M + log2f(lsum)) * kLn2 : -INFINITY;
    } else {
      const int64_t pu = (head0 + g) * p.nsplit + split;  // partial row of (query head, split)
      p.part_o[pu * D + (i % D)] = o;
      if ((i % D) == 0) {
        p.part_ml[pu * 2] = M;
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

template <typename T, int D, int G>
cudaError_t launch_typed(const DecodeAttnParams &p, int units, cudaStream_t s) {
  using S = AttnShape<T, D, G>;
  cudaError_t e = cudaFuncSetAttribute(decode_attention_kernel<T, D, G>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)S::kSmem);
  if (e != cudaSuccess) return e;
  decode_attention_kernel<T, D, G><<<units, kThreads, S::kSmem, s>>>(p);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_g(const DecodeAttnParams &p, int G, int units, cudaStream_t s) {
  switch (G) {
    case 1: return launch_typed<T, D, 1>(p, units, s);
    case 2: return launch_typed<T, D, 2>(p, units, s);
    case 4: return launch_typed<T, D, 4>(p, units, s);
    default: return launch_typed<T, D, 8>(p, units, s);
  }
}

}  // namespace

bool decode_attention_supported(int dtype, int head_dim, int G) {
  return (dtype == KVC_BF16 || dtype == KVC_F32) && (head_dim == 64 || head_dim == 128) &&
         (G == 1 || G == 2 || G == 4 || G == 8);
}

cudaError_t launch_decode_attention(const DecodeAttnParams &p, int head_dim, int dtype, int G, int *launches,
                                    cudaStream_t s) {
  *launches = 0;
  const int units = p.layer_count * p.R * p.hkv * p.nsplit;
  if (units <= 0) return cudaSuccess;
  cudaError_t e;
  if (dtype == KVC_BF16)
    e = head_dim == 128 ? launch_g<__nv_bfloat16, 128>(p, G, units, s) : launch_g<__nv_bfloat16, 64>(p, G, units, s);
  else
    e = head_dim == 128 ? launch_g<float, 128>(p, G, units, s) : launch_g<float, 64>(p, G, units, s);
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
