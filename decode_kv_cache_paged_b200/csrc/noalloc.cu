// noalloc.cu -- kvc_beacon_select_noalloc: beacon scores and top-K selection
// of dense segments without allocating any device memory.
//
// Some callers cannot allocate device memory.  Code that runs while a CUDA
// graph is being captured may not call cudaMalloc.  A plug-in that lives
// inside another engine's fixed memory arena, or an embedded host without a
// device allocator, has no way to hand the library a workspace.  This entry
// point needs only the caller's inputs and outputs.  The one buffer it needs
// in between, the per-candidate scores that the selection kernel reads back,
// lives in a fixed array in the library's own device memory (below), which
// every GPU that loads the library holds until the process exits.
//
// The kernels are variants of the context path's SIMT beacon score and of the
// select kernel, for dense key rows instead of paged ones; the arithmetic and
// its order are the same, so the results match kvc_compress(KVC_SEL_BEACON).
#include <cuda_bf16.h>

#include <memory>
#include <mutex>
#include <string>

#include "kvc_internal.h"

namespace kvc {
void set_thread_error(const std::string &msg);  // kvc_api.cu
}

using namespace kvc;

// Scratch for the scores: at most S*(L-P) floats per call.
constexpr size_t kNoAllocScratchFloats = size_t(1) << 20;  // 4 MiB per device
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
float *g_scratch_addr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on `dev` (which must be current).  The
// symbol's name in host code is only a host-side stand-in; kernels must get
// this address.  Looked up once per device, on the first call there.
cudaError_t scratch_address(int dev, float **out) {
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void *p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = static_cast<float *>(p);
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

template <int DT>
__device__ __forceinline__ float na_load(const uint8_t *base, int64_t idx) {
  if (DT == KVC_BF16)
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(base)[idx]);
  else
    return reinterpret_cast<const float *>(base)[idx];
}

// Elements of one 16-byte chunk: 8 bf16 or 4 fp32.
template <int DT>
struct NaChunk {
  static constexpr int kElems = DT == KVC_BF16 ? 8 : 4;
};

// Loads the 16-byte chunk that starts at element idx (16-byte aligned) and
// widens it to fp32.
template <int DT>
__device__ __forceinline__ void na_load_chunk(const uint8_t *base, int64_t idx, float *out) {
  if (DT == KVC_BF16) {
    const uint4 u = __ldg(reinterpret_cast<const uint4 *>(base + idx * 2));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      out[2 * i] = __uint_as_float(w[i] << 16);
      out[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  } else {
    const float4 f = __ldg(reinterpret_cast<const float4 *>(base + idx * 4));
    out[0] = f.x;
    out[1] = f.y;
    out[2] = f.z;
    out[3] = f.w;
  }
}

constexpr int kNT = 256;
constexpr int kTK = 32;
constexpr int kNG = kNT / kTK;

// Scores of dense segment blockIdx.x into scratch[s*N + j - P].
template <int D, int DT>
__global__ void __launch_bounds__(kNT)
    na_score_kernel(const uint8_t *keys, const uint8_t *beacons, int L, int P, int B, float *scratch) {
  extern __shared__ __align__(16) uint8_t smem[];
  float *cs = reinterpret_cast<float *>(smem);
  float *ks = cs + B * D;
  float *zs = ks + kTK * (D + 1);
  float *lse = zs + B * (kTK + 1);
  float *red = lse + B;
  __shared__ int seg_nan;  // a beacon's log-sum-exp is NaN: every score of the segment is NaN
  const int tid = threadIdx.x, s = blockIdx.x;
  const int N = L - P;
  const float inv_sqrt_d = 1.0f / sqrtf((float)D);
  if (tid == 0) seg_nan = 0;
  // 16-byte loads when both inputs start on a 16-byte boundary (a row is
  // D * sizeof(dtype) bytes, a multiple of 16, so every row chunk is then
  // aligned too); element loads otherwise.  Same values either way.
  constexpr int CE = NaChunk<DT>::kElems;
  constexpr int CPR = D / CE;  // chunks per row
  const bool vec = (((uintptr_t)keys | (uintptr_t)beacons) & 15) == 0;
  if (vec) {
    for (int c = tid; c < B * CPR; c += kNT) {
      float v[CE];
      na_load_chunk<DT>(beacons, (int64_t)s * B * D + (int64_t)c * CE, v);
#pragma unroll
      for (int i = 0; i < CE; ++i) cs[c * CE + i] = v[i];
    }
  } else {
    for (int e = tid; e < B * D; e += kNT) cs[e] = na_load<DT>(beacons, (int64_t)s * B * D + e);
  }
  const int jj = tid % kTK, bg = tid / kTK;
  auto load_tile = [&](int j0) {
    if (vec) {
      for (int c = tid; c < kTK * CPR; c += kNT) {
        const int t = c / CPR, k = (c - t * CPR) * CE;
        const int j = j0 + t;
        float v[CE];
        if (j < L) {
          na_load_chunk<DT>(keys, ((int64_t)s * L + j) * D + k, v);
        } else {
#pragma unroll
          for (int i = 0; i < CE; ++i) v[i] = 0.f;
        }
#pragma unroll
        for (int i = 0; i < CE; ++i) ks[t * (D + 1) + k + i] = v[i];
      }
    } else {
      for (int e = tid; e < kTK * D; e += kNT) {
        const int t = e / D, k = e - t * D;
        const int j = j0 + t;
        ks[t * (D + 1) + k] = j < L ? na_load<DT>(keys, ((int64_t)s * L + j) * D + k) : 0.f;
      }
    }
  };
  auto dots = [&]() {
    for (int b = bg; b < B; b += kNG) {
      const float *c = cs + b * D;
      const float *k = ks + jj * (D + 1);
      float acc = 0.f;
#pragma unroll 8
      for (int i = 0; i < D; ++i) acc = fmaf(c[i], k[i], acc);
      zs[b * (kTK + 1) + jj] = acc * inv_sqrt_d;
    }
  };
  float run_m = __int_as_float(0xff800000), run_s = 0.f;
#pragma unroll 1
  for (int j0 = 0; j0 < L; j0 += kTK) {
    __syncthreads();
    load_tile(j0);
    __syncthreads();
    dots();
    __syncthreads();
    if (tid < B) {
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
  if (tid < B) {
    const float v = run_m + logf(run_s);
    lse[tid] = v;
    if (v != v) seg_nan = 1;  // a NaN key or beacon (fmaxf below would drop it)
  }
#pragma unroll 1
  for (int j0 = P; j0 < L; j0 += kTK) {
    __syncthreads();
    load_tile(j0);
    __syncthreads();
    dots();
    __syncthreads();
    float mx = __int_as_float(0xff800000);
    for (int b = bg; b < B; b += kNG) mx = fmaxf(mx, zs[b * (kTK + 1) + jj] - lse[b]);
    red[bg * kTK + jj] = mx;
    __syncthreads();
    if (tid < kTK && j0 + tid < L) {
      float m = red[tid];
      for (int g = 1; g < kNG; ++g) m = fmaxf(m, red[g * kTK + tid]);
      scratch[(int64_t)s * N + (j0 + tid - P)] = seg_nan ? __int_as_float(0x7fffffff) : expf(m);
    }
  }
}

// Order-preserving map of a score to an unsigned key.  A NaN score (one NaN
// key or beacon makes every score of its segment NaN) maps to 0, below every
// other score, so NaN candidates are the first to go and ties among them keep
// the lowest slots.  This call does not
// synchronise, so unlike kvc_compress it reports no KVC_ERR_NAN; callers that
// need to detect NaN inputs read scores_out.
__device__ __forceinline__ uint32_t na_order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  if (f != f) return 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Kept slots of dense segment blockIdx.x: [0, P) then the M best candidates
// by (score desc, slot asc), ascending, into kept[s*R ...].
__global__ void __launch_bounds__(kNT)
    na_select_kernel(const float *scratch, int L, int P, int M, int R, int32_t *kept, float *scores_out) {
  extern __shared__ __align__(16) uint8_t smem[];
  uint32_t *keys = reinterpret_cast<uint32_t *>(smem);
  __shared__ uint32_t hist[256];
  __shared__ uint32_t bcast[2];
  __shared__ uint32_t warp_gt[kNT / 32], warp_eq[kNT / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, s = blockIdx.x;
  const int N = L - P;
  int32_t *out = kept + (int64_t)s * R;
  for (int i = tid; i < P; i += kNT) out[i] = i;
  if (M >= N) {  // nothing evicted
    for (int j = tid; j < N; j += kNT) out[P + j] = P + j;
    return;
  }
  if (M == 0) return;  // only the prompt stays
  for (int j = tid; j < N; j += kNT) {
    const float v = scratch[(int64_t)s * N + j];
    if (scores_out) scores_out[(int64_t)s * N + j] = v;
    keys[j] = na_order_key(v);
  }
  __syncthreads();
  // M-th largest key (MSB radix select, 8-bit digits)
  uint32_t prefix = 0, mask = 0;
  int k = M;
#pragma unroll 1
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kNT) hist[i] = 0;
    __syncthreads();
    for (int j = tid; j < N; j += kNT) {
      const uint32_t key = keys[j];
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (warp == 0) {
      uint32_t c[8], sum = 0;
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
      const unsigned hit = __ballot_sync(0xffffffffu, incl >= (uint32_t)k);
      if (lane == __ffs(hit) - 1) {
        uint32_t cum = incl - sum;
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
  const uint32_t tau = prefix;
  const int need = k;
  int carry_gt = 0, carry_eq = 0;
#pragma unroll 1
  for (int base = 0; base < N; base += kNT) {
    const int j = base + tid;
    const bool valid = j < N;
    const uint32_t key = valid ? keys[j] : 0u;
    const bool gt = valid && key > tau, eq = valid && key == tau;
    const unsigned mgt = __ballot_sync(0xffffffffu, gt), meq = __ballot_sync(0xffffffffu, eq);
    const unsigned lt = (1u << lane) - 1u;
    if (lane == 0) {
      warp_gt[warp] = __popc(mgt);
      warp_eq[warp] = __popc(meq);
    }
    __syncthreads();
    int off_gt = carry_gt, off_eq = carry_eq, tot_gt = 0, tot_eq = 0;
#pragma unroll
    for (int w = 0; w < kNT / 32; ++w) {
      if (w < warp) {
        off_gt += warp_gt[w];
        off_eq += warp_eq[w];
      }
      tot_gt += warp_gt[w];
      tot_eq += warp_eq[w];
    }
    const int gb = off_gt + __popc(mgt & lt), eb = off_eq + __popc(meq & lt);
    if (gt || (eq && eb < need)) out[P + gb + min(eb, need)] = P + j;
    carry_gt += tot_gt;
    carry_eq += tot_eq;
    __syncthreads();
  }
}

}  // namespace

extern "C" kvc_status kvc_beacon_select_noalloc(const void *keys, const void *beacons, int32_t S,
                                                int32_t L, int32_t P, int32_t K, int32_t B,
                                                int32_t head_dim, int32_t dtype, int32_t *kept_out,
                                                float *scores_out, void *cuda_stream) {
  auto bad = [](const std::string &m) {
    set_thread_error("kvc_beacon_select_noalloc: " + m);
    return KVC_ERR_INVALID_ARG;
  };
  if (!keys || !beacons || !kept_out) return bad("keys, beacons and kept_out are required");
  if (S < 1 || L < 1 || L > kMaxSeqLen) return bad("need S >= 1 and 1 <= L <= 32768");
  if (P < 0 || P > L || K < 0) return bad("need 0 <= P <= L and K >= 0");
  if (B < 1 || B > kMaxBeacons) return bad("B must be in [1, 256]");
  if (head_dim != 64 && head_dim != 128) return bad("head_dim must be 64 or 128");
  if (dtype != KVC_BF16 && dtype != KVC_F32) return bad("dtype must be KVC_BF16 or KVC_F32");
  const int es = dtype == KVC_BF16 ? 2 : 4;
  if (((uintptr_t)keys | (uintptr_t)beacons) % es || ((uintptr_t)kept_out | (uintptr_t)scores_out) & 3)
    return bad("misaligned pointer");
  const int64_t N = L - P;
  if ((int64_t)S * N > (int64_t)kNoAllocScratchFloats)
    return bad("S*(L-P) = " + std::to_string((int64_t)S * N) + " exceeds the scratch limit of " +
               std::to_string(kNoAllocScratchFloats) + " scores per call");
  cudaPointerAttributes a{};
  if (cudaPointerGetAttributes(&a, keys) != cudaSuccess || a.type != cudaMemoryTypeDevice) {
    cudaGetLastError();
    return bad("keys must be device memory");
  }
  const int dev = a.device;
  if (dev < 0 || dev >= kMaxDevices) return bad("device index out of range");
  for (const void *p : {beacons, static_cast<const void *>(kept_out), static_cast<const void *>(scores_out)}) {
    if (!p) continue;
    cudaPointerAttributes b{};
    if (cudaPointerGetAttributes(&b, p) != cudaSuccess || b.type != cudaMemoryTypeDevice || b.device != dev) {
      cudaGetLastError();
      return bad("beacons, kept_out and scores_out must be device memory of the keys' device");
    }
  }
  auto cuda_err = [](cudaError_t e, const char *what) {
    set_thread_error(std::string("kvc_beacon_select_noalloc: ") + what + ": " + cudaGetErrorString(e));
    return KVC_ERR_CUDA;
  };
  // The launches go to the keys' device; the caller's current device is put
  // back on every return path.
  int prev_dev = -1;
  cudaError_t e = cudaGetDevice(&prev_dev);
  if (e != cudaSuccess) return cuda_err(e, "cudaGetDevice");
  struct RestoreDevice {
    int dev;
    ~RestoreDevice() { cudaSetDevice(dev); }
  };
  std::unique_ptr<RestoreDevice> restore;
  if (prev_dev != dev) {
    if ((e = cudaSetDevice(dev)) != cudaSuccess) return cuda_err(e, "cudaSetDevice");
    restore.reset(new RestoreDevice{prev_dev});
  }
  float *scratch = nullptr;
  if ((e = scratch_address(dev, &scratch)) != cudaSuccess) return cuda_err(e, "cudaGetSymbolAddress");
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  const int M = L <= K ? (int)N : (K > P ? K - P : 0);
  const int R = P + M;
  if (N > 0 && M > 0 && M < N) {
    const size_t smem = sizeof(float) * ((size_t)B * head_dim + (size_t)kTK * (head_dim + 1) +
                                         (size_t)B * (kTK + 1) + B + kNG * kTK);
    const uint8_t *kp = static_cast<const uint8_t *>(keys), *bp = static_cast<const uint8_t *>(beacons);
#define KVC_NA(DV, DTV)                                                                            \
  if (head_dim == DV && dtype == DTV) {                                                            \
    e = cudaFuncSetAttribute(na_score_kernel<DV, DTV>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                             (int)smem);                                                           \
    if (e == cudaSuccess) na_score_kernel<DV, DTV><<<S, kNT, smem, st>>>(kp, bp, L, P, B, scratch); \
  }
    KVC_NA(64, KVC_BF16)
    KVC_NA(128, KVC_BF16)
    KVC_NA(64, KVC_F32)
    KVC_NA(128, KVC_F32)
#undef KVC_NA
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_err(e, "score kernel");
  }
  const size_t sel_smem = (size_t)(N > 0 ? N : 1) * sizeof(uint32_t);
  e = cudaFuncSetAttribute(na_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sel_smem);
  if (e == cudaSuccess) {
    na_select_kernel<<<S, kNT, sel_smem, st>>>(scratch, L, P, M, R, kept_out, scores_out);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) return cuda_err(e, "select kernel");
  return KVC_OK;
}
