// kvc_api.cu -- the C ABI of libkvc.so and its host-side orchestration:
// configuration checks, workspace carving, the page allocator, block tables,
// per-round segment descriptors and kernel launch order.
//
// The pages place the eviction round inside a serving engine: the compression
// trigger fires at a batch sync point and runs the selector, then the cache
// compaction every method needs (Random Attention article, "发现四"); the
// engine keeps a paged KV cache.  This file is that engine-side plumbing for
// one GPU; every byte of K/V and every score is produced by the kernels in the
// other .cu files.
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "kvc_internal.h"

namespace {
// NVTX range for the duration of a scope: the library's calls and the phases
// of a round show up by name in profilers (ncu --nvtx --nvtx-include ...).
// Without an attached tool each push and pop returns at once.
struct NvtxRange {
  explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange &) = delete;
  NvtxRange &operator=(const NvtxRange &) = delete;
};
}  // namespace

using namespace kvc;

namespace {

constexpr int kStageSlots = 4;
thread_local std::string g_create_error;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct Layout {
  size_t bt, len, prompt, pos, qring, beacons, beacons_s, counts, trig, scores, lse, status, counters,
      stage, attn, total, stage_slot;
};

// Split partials of the decode attention: room for this many splits of one layer.
constexpr int kAttnSplits = 16;

int elem_size(int dtype) { return dtype == KVC_BF16 ? 2 : 4; }

// Returns an empty string if cfg is valid for this build, else the reason.
std::string check_config(const kvc_config *c) {
  if (!c) return "config is NULL";
  if (c->num_requests < 1 || c->num_layers < 1 || c->num_kv_heads < 1 || c->head_dim < 1)
    return "num_requests, num_layers, num_kv_heads and head_dim must be >= 1";
  if (c->num_q_heads < c->num_kv_heads || c->num_q_heads % c->num_kv_heads != 0)
    return "num_q_heads must be a positive multiple of num_kv_heads";
  if (c->page_size != kPage) return "page_size must be 16";
  if (c->dtype != KVC_BF16 && c->dtype != KVC_F32) return "dtype must be KVC_BF16 or KVC_F32";
  const int rb = c->head_dim * elem_size(c->dtype);
  if (rb % 16 != 0 || rb > kMaxRowBytes)
    return "head_dim * sizeof(dtype) must be a multiple of 16 bytes and at most 1024";
  if (c->max_seq_len < kPage || c->max_seq_len % kPage != 0 || c->max_seq_len > kMaxSeqLen)
    return "max_seq_len must be a multiple of 16 in [16, 32768]";
  if (c->num_pages < 1 || c->num_pages > (int64_t)0x7fffffff) return "num_pages out of range";
  if (c->num_beacons < 0 || c->num_beacons > kMaxBeacons) return "num_beacons must be in [0, 256]";
  if (c->query_window < 0) return "query_window must be >= 0";
  const int G = c->num_q_heads / c->num_kv_heads;
  if ((int64_t)c->query_window * G > kMaxPoints) return "query_window * G must be <= 4096";
  if (c->num_beacons > 0) {
    if (c->query_window < 1) return "the beacon state needs query_window >= 1";
    if (c->head_dim != 64 && c->head_dim != 128)
      return "the beacon selector supports head_dim 64 or 128";
  }
  return "";
}

Layout make_layout(const kvc_config &c) {
  Layout L{};
  const size_t R = c.num_requests, Ly = c.num_layers, H = c.num_kv_heads, Hq = c.num_q_heads;
  const size_t d = c.head_dim, es = elem_size(c.dtype), B = c.num_beacons, W = c.query_window;
  const size_t maxp = c.max_seq_len / kPage;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, 256);
    return at;
  };
  L.bt = take(R * maxp * 4);
  L.len = take(R * 4);
  L.prompt = take(R * 4);
  L.pos = take(Ly * (size_t)c.num_pages * H * kPage * 4);
  L.qring = take(R * Ly * W * Hq * d * es);
  L.beacons = take(R * Ly * H * B * d * 4);
  L.beacons_s = take(R * Ly * H * B * d * es);
  L.counts = take(R * Ly * H * B * 4);
  L.trig = take(R * Ly * H * B * 4);
  L.scores = take(B > 0 ? R * Ly * H * (size_t)c.max_seq_len * 4 : 0);
  L.lse = take(R * Ly * H * B * 4);
  L.status = take(256);
  L.counters = take(256);
  L.stage_slot = align_up(R * 16 + R * maxp * 8 + R * 8 + 1024, 256);
  L.stage = take(L.stage_slot * kStageSlots);
  L.attn = take(R * Hq * (d + 2) * 4 * (size_t)kAttnSplits);
  L.total = off;
  return L;
}

}  // namespace

namespace kvc {
// Message for kvc_last_error(NULL) from entry points that take no context.
void set_thread_error(const std::string &msg) { g_create_error = msg; }
}  // namespace kvc

struct kvc_ctx {
  kvc_config cfg{};
  Layout lay{};
  int device = 0;
  cudaStream_t stream = nullptr;
  uint8_t *k_pool = nullptr, *v_pool = nullptr, *ws = nullptr;
  int32_t *d_bt = nullptr, *d_len = nullptr, *d_prompt = nullptr, *d_pos = nullptr;
  uint8_t *d_qring = nullptr, *d_beacons_s = nullptr, *d_stage = nullptr;
  float *d_beacons = nullptr, *d_scores = nullptr, *d_lse = nullptr, *d_trig = nullptr;
  int32_t *d_counts = nullptr, *d_status = nullptr;
  unsigned long long *d_counters = nullptr;
  uint8_t *h_stage = nullptr;
  cudaEvent_t stage_ev[kStageSlots] = {};
  int stage_next = 0;
  cudaEvent_t ev[4] = {};
  std::vector<int32_t> h_bt, h_len, h_prompt;
  std::vector<int64_t> h_next_pos, q_total, q_last;
  std::vector<uint8_t> h_binit;
  std::vector<uint8_t> h_unordered;  // a hole-filling round left slots out of position order
  std::vector<int32_t> free_pages;
  int64_t round = 0;
  int score_impl = 0;
  int update_impl = 0;
  int es = 2, row_bytes = 0, G = 1, maxp = 0, num_sms = 148;
  float *d_attn = nullptr;
  std::string err;
};

namespace {

kvc_status fail(kvc_ctx *ctx, kvc_status s, const std::string &msg) {
  if (ctx)
    ctx->err = msg;
  else
    g_create_error = msg;
  return s;
}

kvc_status cuda_fail(kvc_ctx *ctx, cudaError_t e, const char *what) {
  return fail(ctx, KVC_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

#define KVC_CUDA(ctx, call)                                   \
  do {                                                        \
    cudaError_t e_ = (call);                                  \
    if (e_ != cudaSuccess) return cuda_fail((ctx), e_, #call); \
  } while (0)

// A slot of the pinned host staging ring and its device twin.  The event of a
// slot is recorded after the kernels that read its device twin, so the host
// copy is only rewritten once those kernels (and the copy) are done.
struct Stage {
  int slot;
  uint8_t *h;
  uint8_t *d;
};

kvc_status stage_acquire(kvc_ctx *ctx, Stage &st) {
  st.slot = ctx->stage_next;
  ctx->stage_next = (ctx->stage_next + 1) % kStageSlots;
  KVC_CUDA(ctx, cudaEventSynchronize(ctx->stage_ev[st.slot]));
  st.h = ctx->h_stage + (size_t)st.slot * ctx->lay.stage_slot;
  st.d = ctx->d_stage + (size_t)st.slot * ctx->lay.stage_slot;
  return KVC_OK;
}

kvc_status stage_upload(kvc_ctx *ctx, const Stage &st, size_t bytes) {
  if (bytes > ctx->lay.stage_slot) return fail(ctx, KVC_ERR_INVALID_ARG, "staging slot overflow");
  if (bytes) KVC_CUDA(ctx, cudaMemcpyAsync(st.d, st.h, bytes, cudaMemcpyHostToDevice, ctx->stream));
  return KVC_OK;
}

kvc_status stage_release(kvc_ctx *ctx, const Stage &st) {
  KVC_CUDA(ctx, cudaEventRecord(ctx->stage_ev[st.slot], ctx->stream));
  return KVC_OK;
}

// Classifies a pointer the kernels will read: device memory of the context's
// device, or page-locked host memory.
bool readable_by_device(const kvc_ctx *ctx, const void *p) {
  cudaPointerAttributes a{};
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  if (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged)
    return a.device == ctx->device;
  return a.type == cudaMemoryTypeHost;
}

bool device_ptr_on(int device, const void *p) {
  cudaPointerAttributes a{};
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) && a.device == device;
}

// Reads and clears the device status word (the stream must be synchronised).
kvc_status take_device_status(kvc_ctx *ctx) {
  int32_t *h = reinterpret_cast<int32_t *>(ctx->h_stage + (size_t)ctx->stage_next * ctx->lay.stage_slot);
  KVC_CUDA(ctx, cudaEventSynchronize(ctx->stage_ev[ctx->stage_next]));
  KVC_CUDA(ctx, cudaMemcpyAsync(h, ctx->d_status, 4, cudaMemcpyDeviceToHost, ctx->stream));
  KVC_CUDA(ctx, cudaStreamSynchronize(ctx->stream));
  const int32_t dev_status = *h;
  if (dev_status == kDevOk) return KVC_OK;
  KVC_CUDA(ctx, cudaMemsetAsync(ctx->d_status, 0, 4, ctx->stream));
  KVC_CUDA(ctx, cudaStreamSynchronize(ctx->stream));
  return fail(ctx,
              dev_status == kDevNaN       ? KVC_ERR_NAN
              : dev_status == kDevTimeout ? KVC_ERR_DEVICE_TIMEOUT
                                          : KVC_ERR_DEVICE_CHECK,
              "device reported an error (status word " + std::to_string(dev_status) + ")");
}

}  // namespace

extern "C" {

size_t kvc_workspace_bytes(const kvc_config *cfg) {
  if (!check_config(cfg).empty()) return 0;
  return make_layout(*cfg).total;
}

const char *kvc_status_string(kvc_status s) {
  switch (s) {
    case KVC_OK: return "KVC_OK";
    case KVC_ERR_INVALID_ARG: return "KVC_ERR_INVALID_ARG";
    case KVC_ERR_OUT_OF_PAGES: return "KVC_ERR_OUT_OF_PAGES";
    case KVC_ERR_STATE: return "KVC_ERR_STATE";
    case KVC_ERR_CUDA: return "KVC_ERR_CUDA";
    case KVC_ERR_NAN: return "KVC_ERR_NAN";
    case KVC_ERR_DEVICE_CHECK: return "KVC_ERR_DEVICE_CHECK";
    case KVC_ERR_DEVICE_TIMEOUT: return "KVC_ERR_DEVICE_TIMEOUT";
    case KVC_ERR_UNSUPPORTED: return "KVC_ERR_UNSUPPORTED";
  }
  return "KVC_UNKNOWN_STATUS";
}

const char *kvc_last_error(const kvc_ctx *ctx) {
  return ctx ? ctx->err.c_str() : g_create_error.c_str();
}

kvc_status kvc_create(const kvc_config *cfg, void *k_pool, void *v_pool, void *workspace,
                      size_t workspace_bytes, void *cuda_stream, kvc_ctx **out) {
  if (!out) return fail(nullptr, KVC_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  const std::string why = check_config(cfg);
  if (!why.empty()) return fail(nullptr, KVC_ERR_INVALID_ARG, why);
  if (!k_pool || !v_pool || !workspace)
    return fail(nullptr, KVC_ERR_INVALID_ARG, "k_pool, v_pool and workspace are required");
  if (((uintptr_t)k_pool | (uintptr_t)v_pool | (uintptr_t)workspace) & 255)
    return fail(nullptr, KVC_ERR_INVALID_ARG, "pools and workspace must be 256-byte aligned");
  const Layout lay = make_layout(*cfg);
  if (workspace_bytes < lay.total)
    return fail(nullptr, KVC_ERR_INVALID_ARG,
                "workspace too small: need " + std::to_string(lay.total) + " bytes");
  cudaPointerAttributes a{};
  if (cudaPointerGetAttributes(&a, k_pool) != cudaSuccess || a.type != cudaMemoryTypeDevice) {
    cudaGetLastError();
    return fail(nullptr, KVC_ERR_INVALID_ARG, "k_pool is not device memory");
  }
  const int dev = a.device;
  if (!device_ptr_on(dev, v_pool) || !device_ptr_on(dev, workspace))
    return fail(nullptr, KVC_ERR_INVALID_ARG, "v_pool and workspace must be device memory of k_pool's device");
  cudaError_t e = cudaSetDevice(dev);
  if (e != cudaSuccess) return fail(nullptr, KVC_ERR_CUDA, cudaGetErrorString(e));

  kvc_ctx *c = new kvc_ctx();
  c->cfg = *cfg;
  c->lay = lay;
  c->device = dev;
  c->stream = static_cast<cudaStream_t>(cuda_stream);
  c->k_pool = static_cast<uint8_t *>(k_pool);
  c->v_pool = static_cast<uint8_t *>(v_pool);
  c->ws = static_cast<uint8_t *>(workspace);
  c->es = elem_size(cfg->dtype);
  c->row_bytes = cfg->head_dim * c->es;
  c->G = cfg->num_q_heads / cfg->num_kv_heads;
  c->maxp = cfg->max_seq_len / kPage;
  c->d_bt = reinterpret_cast<int32_t *>(c->ws + lay.bt);
  c->d_len = reinterpret_cast<int32_t *>(c->ws + lay.len);
  c->d_prompt = reinterpret_cast<int32_t *>(c->ws + lay.prompt);
  c->d_pos = reinterpret_cast<int32_t *>(c->ws + lay.pos);
  c->d_qring = c->ws + lay.qring;
  c->d_beacons = reinterpret_cast<float *>(c->ws + lay.beacons);
  c->d_beacons_s = c->ws + lay.beacons_s;
  c->d_counts = reinterpret_cast<int32_t *>(c->ws + lay.counts);
  c->d_trig = reinterpret_cast<float *>(c->ws + lay.trig);
  c->d_scores = reinterpret_cast<float *>(c->ws + lay.scores);
  c->d_lse = reinterpret_cast<float *>(c->ws + lay.lse);
  c->d_status = reinterpret_cast<int32_t *>(c->ws + lay.status);
  c->d_counters = reinterpret_cast<unsigned long long *>(c->ws + lay.counters);
  c->d_stage = c->ws + lay.stage;
  c->d_attn = reinterpret_cast<float *>(c->ws + lay.attn);
  if (cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    c->num_sms = 148;
  }
  const int R = cfg->num_requests;
  c->h_bt.assign((size_t)R * c->maxp, -1);
  c->h_len.assign(R, 0);
  c->h_prompt.assign(R, 0);
  c->h_next_pos.assign(R, 0);
  c->q_total.assign(R, 0);
  c->q_last.assign(R, 0);
  c->h_binit.assign(R, 0);
  c->h_unordered.assign(R, 0);
  c->free_pages.resize((size_t)cfg->num_pages);
  for (int64_t i = 0; i < cfg->num_pages; ++i)
    c->free_pages[(size_t)i] = (int32_t)(cfg->num_pages - 1 - i);  // pop_back gives 0, 1, ...

  auto cleanup = [&](cudaError_t err, const char *what) {
    kvc_status s = fail(nullptr, KVC_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(err));
    for (auto &ev : c->stage_ev)
      if (ev) cudaEventDestroy(ev);
    for (auto &ev : c->ev)
      if (ev) cudaEventDestroy(ev);
    if (c->h_stage) cudaFreeHost(c->h_stage);
    delete c;
    return s;
  };
  if ((e = cudaHostAlloc(&c->h_stage, lay.stage_slot * kStageSlots, cudaHostAllocDefault)) != cudaSuccess)
    return cleanup(e, "cudaHostAlloc(staging)");
  for (auto &ev : c->stage_ev)
    if ((e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming)) != cudaSuccess)
      return cleanup(e, "cudaEventCreate");
  for (auto &ev : c->ev)
    if ((e = cudaEventCreate(&ev)) != cudaSuccess) return cleanup(e, "cudaEventCreate");
  // device state: block tables -1, lengths 0, position map -1, query ring 0, beacon counts 0
  if ((e = cudaMemsetAsync(c->d_bt, 0xff, (size_t)R * c->maxp * 4, c->stream)) != cudaSuccess ||
      (e = cudaMemsetAsync(c->d_len, 0, (size_t)R * 4, c->stream)) != cudaSuccess ||
      (e = cudaMemsetAsync(c->d_prompt, 0, (size_t)R * 4, c->stream)) != cudaSuccess ||
      (e = cudaMemsetAsync(c->d_pos, 0xff, lay.qring - lay.pos, c->stream)) != cudaSuccess ||
      (e = cudaMemsetAsync(c->d_qring, 0, lay.beacons - lay.qring, c->stream)) != cudaSuccess ||
      (e = cudaMemsetAsync(c->ws + lay.counts, 0, lay.scores - lay.counts, c->stream)) != cudaSuccess ||
      (e = cudaMemsetAsync(c->ws + lay.status, 0, lay.stage - lay.status, c->stream)) != cudaSuccess)
    return cleanup(e, "cudaMemsetAsync(workspace)");
  *out = c;
  return KVC_OK;
}

kvc_status kvc_destroy(kvc_ctx *ctx) {
  if (!ctx) return KVC_OK;
  cudaSetDevice(ctx->device);
  cudaStreamSynchronize(ctx->stream);
  for (auto &ev : ctx->stage_ev) cudaEventDestroy(ev);
  for (auto &ev : ctx->ev) cudaEventDestroy(ev);
  cudaFreeHost(ctx->h_stage);
  delete ctx;
  return KVC_OK;
}

kvc_status kvc_set_stream(kvc_ctx *ctx, void *cuda_stream) {
  if (!ctx) return KVC_ERR_INVALID_ARG;
  KVC_CUDA(ctx, cudaSetDevice(ctx->device));
  KVC_CUDA(ctx, cudaStreamSynchronize(ctx->stream));
  ctx->stream = static_cast<cudaStream_t>(cuda_stream);
  return KVC_OK;
}

kvc_status kvc_set_option(kvc_ctx *ctx, kvc_option opt, int64_t value) {
  if (!ctx) return KVC_ERR_INVALID_ARG;
  switch (opt) {
    case KVC_OPT_BEACON_SCORE_IMPL:
      if (value < 0 || value > 2) return fail(ctx, KVC_ERR_INVALID_ARG, "impl must be 0, 1 or 2");
      if (value == 2 && !beacon_score_tc_supported(ctx->cfg.head_dim, ctx->cfg.num_beacons, ctx->cfg.dtype))
        return fail(ctx, KVC_ERR_UNSUPPORTED, "tcgen05 beacon score not available for this config");
      ctx->score_impl = (int)value;
      return KVC_OK;
    case KVC_OPT_BEACON_UPDATE_IMPL:
      if (value < 0 || value > 2) return fail(ctx, KVC_ERR_INVALID_ARG, "impl must be 0, 1 or 2");
      if (value == 2 && !beacon_update_tc_supported(ctx->cfg.head_dim, ctx->cfg.num_beacons, ctx->cfg.dtype))
        return fail(ctx, KVC_ERR_UNSUPPORTED, "tcgen05 beacon update not available for this config");
      ctx->update_impl = (int)value;
      return KVC_OK;
  }
  return fail(ctx, KVC_ERR_INVALID_ARG, "unknown option");
}

kvc_status kvc_append(kvc_ctx *ctx, const int32_t *req_ids, int32_t n_req, int32_t n_tokens,
                      const void *k_new, const void *v_new, const void *q_new, int32_t protect) {
  NvtxRange nvtx_range("kvc_append");
  if (!ctx) return KVC_ERR_INVALID_ARG;
  const kvc_config &c = ctx->cfg;
  if (n_req < 0 || n_tokens < 0) return fail(ctx, KVC_ERR_INVALID_ARG, "negative n_req or n_tokens");
  if (n_req == 0 || n_tokens == 0) return KVC_OK;
  if (!req_ids || !k_new || !v_new) return fail(ctx, KVC_ERR_INVALID_ARG, "req_ids, k_new and v_new are required");
  if (n_req > c.num_requests) return fail(ctx, KVC_ERR_INVALID_ARG, "n_req > num_requests");
  if (((uintptr_t)k_new | (uintptr_t)v_new | (uintptr_t)q_new) & 15)
    return fail(ctx, KVC_ERR_INVALID_ARG, "k_new, v_new and q_new must be 16-byte aligned");
  if (q_new && c.query_window == 0) return fail(ctx, KVC_ERR_INVALID_ARG, "q_new given but query_window is 0");
  KVC_CUDA(ctx, cudaSetDevice(ctx->device));
  if (!readable_by_device(ctx, k_new) || !readable_by_device(ctx, v_new) ||
      (q_new && !readable_by_device(ctx, q_new)))
    return fail(ctx, KVC_ERR_INVALID_ARG,
                "k_new/v_new/q_new must be device memory of the context's device or page-locked host memory");
  std::vector<uint8_t> seen(c.num_requests, 0);
  int64_t pages_needed = 0;
  for (int i = 0; i < n_req; ++i) {
    const int r = req_ids[i];
    if (r < 0 || r >= c.num_requests) return fail(ctx, KVC_ERR_INVALID_ARG, "request id out of range");
    if (seen[r]) return fail(ctx, KVC_ERR_INVALID_ARG, "duplicate request id");
    seen[r] = 1;
    if (protect && ctx->h_prompt[r] != ctx->h_len[r])
      return fail(ctx, KVC_ERR_STATE, "protected tokens must precede every generated token of request " + std::to_string(r));
    const int64_t nl = (int64_t)ctx->h_len[r] + n_tokens;
    if (nl > c.max_seq_len)
      return fail(ctx, KVC_ERR_OUT_OF_PAGES, "request " + std::to_string(r) + " would exceed max_seq_len");
    pages_needed += (nl + kPage - 1) / kPage - (ctx->h_len[r] + kPage - 1) / kPage;
  }
  if (pages_needed > (int64_t)ctx->free_pages.size())
    return fail(ctx, KVC_ERR_OUT_OF_PAGES, "page pool exhausted: need " + std::to_string(pages_needed) +
                                               ", free " + std::to_string(ctx->free_pages.size()));
  const size_t need = (size_t)n_req * 32 + (size_t)pages_needed * 8;
  if (need > ctx->lay.stage_slot) return fail(ctx, KVC_ERR_INVALID_ARG, "append too large for the staging ring");

  Stage st;
  if (kvc_status s = stage_acquire(ctx, st)) return s;
  int32_t *kvdesc = reinterpret_cast<int32_t *>(st.h);
  int32_t *qdesc = kvdesc + 4 * n_req;
  int32_t *pairs = qdesc + 4 * n_req;
  int n_pairs = 0;
  const int W = c.query_window;
  const int t0 = (q_new && n_tokens > W) ? n_tokens - W : 0;
  for (int i = 0; i < n_req; ++i) {
    const int r = req_ids[i];
    const int len0 = ctx->h_len[r];
    kvdesc[4 * i + 0] = r;
    kvdesc[4 * i + 1] = len0;
    kvdesc[4 * i + 2] = (int32_t)ctx->h_next_pos[r];
    kvdesc[4 * i + 3] = 0;
    qdesc[4 * i + 0] = r;
    qdesc[4 * i + 1] = W > 0 ? (int32_t)(ctx->q_total[r] % W) : 0;
    qdesc[4 * i + 2] = 0;
    qdesc[4 * i + 3] = 0;
    const int p0 = (len0 + kPage - 1) / kPage, p1 = (len0 + n_tokens + kPage - 1) / kPage;
    for (int pg = p0; pg < p1; ++pg) {
      const int32_t id = ctx->free_pages.back();
      ctx->free_pages.pop_back();
      ctx->h_bt[(size_t)r * ctx->maxp + pg] = id;
      pairs[2 * n_pairs] = r * ctx->maxp + pg;
      pairs[2 * n_pairs + 1] = id;
      ++n_pairs;
    }
  }
  if (kvc_status s = stage_upload(ctx, st, need)) return s;
  cudaError_t e;
  if ((e = launch_bt_scatter(reinterpret_cast<int32_t *>(st.d + (size_t)n_req * 32), n_pairs, ctx->d_bt, ctx->stream)) != cudaSuccess)
    return cuda_fail(ctx, e, "bt_scatter");
  if ((e = launch_append_kv(static_cast<const uint8_t *>(k_new), static_cast<const uint8_t *>(v_new),
                            ctx->k_pool, ctx->v_pool, ctx->d_pos, ctx->d_bt,
                            reinterpret_cast<int32_t *>(st.d), n_req, c.num_layers, n_tokens,
                            c.num_kv_heads, ctx->row_bytes, c.num_pages, ctx->maxp, ctx->stream)) != cudaSuccess)
    return cuda_fail(ctx, e, "append_kv");
  if (q_new) {
    if ((e = launch_append_q(static_cast<const uint8_t *>(q_new), ctx->d_qring,
                             reinterpret_cast<int32_t *>(st.d + (size_t)n_req * 16), n_req,
                             c.num_layers, n_tokens, t0, W, c.num_q_heads, ctx->row_bytes,
                             ctx->stream)) != cudaSuccess)
      return cuda_fail(ctx, e, "append_q");
  }
  for (int i = 0; i < n_req; ++i) {
    const int r = req_ids[i];
    ctx->h_len[r] += n_tokens;
    ctx->h_next_pos[r] += n_tokens;
    if (protect) ctx->h_prompt[r] += n_tokens;
    if (q_new) ctx->q_total[r] += n_tokens;
  }
  // lengths and prompt lengths of every request, after the append
  Stage st2;
  if (kvc_status s = stage_release(ctx, st)) return s;
  if (kvc_status s = stage_acquire(ctx, st2)) return s;
  const int R = c.num_requests;
  std::memcpy(st2.h, ctx->h_len.data(), (size_t)R * 4);
  std::memcpy(st2.h + (size_t)R * 4, ctx->h_prompt.data(), (size_t)R * 4);
  KVC_CUDA(ctx, cudaMemcpyAsync(ctx->d_len, st2.h, (size_t)R * 4, cudaMemcpyHostToDevice, ctx->stream));
  KVC_CUDA(ctx, cudaMemcpyAsync(ctx->d_prompt, st2.h + (size_t)R * 4, (size_t)R * 4, cudaMemcpyHostToDevice, ctx->stream));
  return stage_release(ctx, st2);
}

kvc_status kvc_update_beacons(kvc_ctx *ctx, int32_t *assign_out, float *ms_out) {
  NvtxRange nvtx_range("kvc_update_beacons");
  if (!ctx) return KVC_ERR_INVALID_ARG;
  const kvc_config &c = ctx->cfg;
  if (c.num_beacons == 0) return fail(ctx, KVC_ERR_STATE, "the context has no beacon state (num_beacons = 0)");
  KVC_CUDA(ctx, cudaSetDevice(ctx->device));
  if (assign_out && !device_ptr_on(ctx->device, assign_out))
    return fail(ctx, KVC_ERR_INVALID_ARG, "assign_out must be device memory");
  const int W = c.query_window, B = c.num_beacons;
  std::vector<UpdateDesc> descs;
  for (int r = 0; r < c.num_requests; ++r) {
    const int64_t fresh = ctx->q_total[r] - ctx->q_last[r];
    if (fresh <= 0) continue;
    const int n_steps = (int)std::min<int64_t>(fresh, W);
    const int init = ctx->h_binit[r] ? 0 : 1;
    if (init && (int64_t)n_steps * ctx->G < B)
      return fail(ctx, KVC_ERR_STATE, "request " + std::to_string(r) + ": first beacon update needs at least B points");
    descs.push_back(UpdateDesc{r, (int)((ctx->q_total[r] - n_steps) % W), n_steps, init});
  }
  if (descs.empty()) {
    if (ms_out) *ms_out = 0.f;
    return KVC_OK;
  }
  Stage st;
  if (kvc_status s = stage_acquire(ctx, st)) return s;
  std::memcpy(st.h, descs.data(), descs.size() * sizeof(UpdateDesc));
  if (kvc_status s = stage_upload(ctx, st, descs.size() * sizeof(UpdateDesc))) return s;
  BeaconUpdateParams p{};
  p.qring = ctx->d_qring;
  p.beacons = ctx->d_beacons;
  p.beacons_s = ctx->d_beacons_s;
  p.counts = ctx->d_counts;
  p.trig = ctx->d_trig;
  p.assign_out = assign_out;
  p.descs = reinterpret_cast<const UpdateDesc *>(st.d);
  p.status = ctx->d_status;
  p.layers = c.num_layers;
  p.hkv = c.num_kv_heads;
  p.hq = c.num_q_heads;
  p.G = ctx->G;
  p.W = W;
  p.B = B;
  p.d = c.head_dim;
  p.dtype = c.dtype;
  p.n_ring = c.num_requests;
  if (ms_out) KVC_CUDA(ctx, cudaEventRecord(ctx->ev[0], ctx->stream));
  const bool use_tc = ctx->update_impl == 2 ||
                      (ctx->update_impl == 0 && beacon_update_tc_supported(c.head_dim, B, c.dtype));
  cudaError_t e = use_tc ? launch_beacon_update_tc(p, (int)descs.size(), ctx->stream)
                         : launch_beacon_update(p, (int)descs.size(), ctx->stream);
  if (e != cudaSuccess) return cuda_fail(ctx, e, "beacon_update");
  if (ms_out) KVC_CUDA(ctx, cudaEventRecord(ctx->ev[1], ctx->stream));
  if (kvc_status s = stage_release(ctx, st)) return s;
  for (const auto &d : descs) {
    ctx->q_last[d.req] = ctx->q_total[d.req];
    ctx->h_binit[d.req] = 1;
  }
  if (ms_out) {
    KVC_CUDA(ctx, cudaEventSynchronize(ctx->ev[1]));
    KVC_CUDA(ctx, cudaEventElapsedTime(ms_out, ctx->ev[0], ctx->ev[1]));
  }
  return KVC_OK;
}

kvc_status kvc_compress(kvc_ctx *ctx, kvc_selector selector, const int32_t *budgets,
                        uint64_t seed, void *debug_scores, kvc_round_stats *stats) {
  return kvc_compress_ex(ctx, selector, budgets, seed, nullptr, debug_scores, stats);
}

kvc_status kvc_compress_ex(kvc_ctx *ctx, kvc_selector selector, const int32_t *budgets,
                           uint64_t seed, const kvc_round_options *opts, void *debug_scores,
                           kvc_round_stats *stats) {
  NvtxRange nvtx_range("kvc_compress");
  if (!ctx) return KVC_ERR_INVALID_ARG;
  const kvc_config &c = ctx->cfg;
  if (selector != KVC_SEL_RANDOM && selector != KVC_SEL_RANDOM_SHARED && selector != KVC_SEL_BEACON &&
      selector != KVC_SEL_BEACON_TRIGGER)
    return fail(ctx, KVC_ERR_INVALID_ARG, "unknown selector");
  if (!budgets) return fail(ctx, KVC_ERR_INVALID_ARG, "budgets is NULL");
  const kvc_round_options o = opts ? *opts : kvc_round_options{-1, 1, KVC_COMPACT_ORDERED, 0};
  if (o.block < 1 || o.block > kMaxSeqLen)
    return fail(ctx, KVC_ERR_INVALID_ARG, "block must be in [1, 32768]");
  const bool beacon_sel = selector == KVC_SEL_BEACON || selector == KVC_SEL_BEACON_TRIGGER;
  if (o.block != 1 && beacon_sel)
    return fail(ctx, KVC_ERR_INVALID_ARG, "block-granular draws apply to the random selectors only");
  if (o.compaction != KVC_COMPACT_ORDERED && o.compaction != KVC_COMPACT_HOLE_FILL)
    return fail(ctx, KVC_ERR_INVALID_ARG, "unknown compaction");
  if (o.reserved != 0) return fail(ctx, KVC_ERR_INVALID_ARG, "reserved option field must be 0");
  KVC_CUDA(ctx, cudaSetDevice(ctx->device));
  if (debug_scores && !device_ptr_on(ctx->device, debug_scores))
    return fail(ctx, KVC_ERR_INVALID_ARG, "debug_scores must be device memory");
  if ((uintptr_t)debug_scores & 3) return fail(ctx, KVC_ERR_INVALID_ARG, "debug_scores must be 4-byte aligned");
  const int R = c.num_requests;
  const int64_t per_req_segs = (int64_t)c.num_layers * c.num_kv_heads;
  kvc_round_stats st{};
  st.round = ctx->round;
  st.segments = (int64_t)R * per_req_segs;
  std::vector<SegDesc> segs;
  std::vector<int32_t> new_len(ctx->h_len), new_prompt(ctx->h_prompt);
  bool tie_by_pos = false;
  for (int r = 0; r < R; ++r) {
    const int K = budgets[r];
    if (K < 0) return fail(ctx, KVC_ERR_INVALID_ARG, "negative budget for request " + std::to_string(r));
    const int L = ctx->h_len[r];
    const int P = o.sink_tokens < 0 ? ctx->h_prompt[r] : std::min(ctx->h_prompt[r], o.sink_tokens);
    st.head_positions += (int64_t)L * per_req_segs;
    if (L <= K) {
      st.noop_segments += per_req_segs;
      continue;
    }
    const int M = std::max(0, K - P);
    if (P > K) st.prompt_over_budget_segments += per_req_segs;
    st.candidates += (int64_t)(L - P) * per_req_segs;
    st.evicted += (int64_t)(L - P - M) * per_req_segs;
    new_len[r] = P + M;
    new_prompt[r] = P;
    if (M > 0) {
      if (beacon_sel && !ctx->h_binit[r])
        return fail(ctx, KVC_ERR_STATE, "request " + std::to_string(r) + " has no beacons yet (call kvc_update_beacons)");
      segs.push_back(SegDesc{r, L, P, M});
      tie_by_pos = tie_by_pos || ctx->h_unordered[r];
    }
  }
  if (beacon_sel && c.num_beacons == 0)
    return fail(ctx, KVC_ERR_STATE, "the context has no beacon state (num_beacons = 0)");
  // longest first (the persistent select launch takes its segments in list
  // order), bucketed by candidate count so each launch sizes its shared memory
  std::stable_sort(segs.begin(), segs.end(), [](const SegDesc &a, const SegDesc &b) {
    return (a.L - a.P) > (b.L - b.P);
  });
  const size_t seg_bytes = segs.size() * sizeof(SegDesc);
  Stage sd_stage;
  if (kvc_status s = stage_acquire(ctx, sd_stage)) return s;
  std::memcpy(sd_stage.h, segs.data(), seg_bytes);
  std::memcpy(sd_stage.h + align_up(seg_bytes, 16), new_len.data(), (size_t)R * 4);
  std::memcpy(sd_stage.h + align_up(seg_bytes, 16) + (size_t)R * 4, new_prompt.data(), (size_t)R * 4);
  if (kvc_status s = stage_upload(ctx, sd_stage, align_up(seg_bytes, 16) + (size_t)R * 8)) return s;
  const SegDesc *d_segs = reinterpret_cast<const SegDesc *>(sd_stage.d);
  const bool timed = stats != nullptr;
  if (timed) {
    KVC_CUDA(ctx, cudaMemsetAsync(ctx->d_counters, 0, 64, ctx->stream));
    KVC_CUDA(ctx, cudaEventRecord(ctx->ev[0], ctx->stream));
  }
  cudaError_t e;
  float *score_buf = (debug_scores && beacon_sel) ? static_cast<float *>(debug_scores) : ctx->d_scores;
  if (beacon_sel && !segs.empty()) {
    NvtxRange nvtx_score("score");  // inside kvc_compress: "kvc_compress/score/" to ncu
    BeaconScoreParams bp{};
    bp.k_pool = ctx->k_pool;
    bp.block_table = ctx->d_bt;
    bp.segs = d_segs;
    bp.beacons_s = ctx->d_beacons_s;
    bp.scores = score_buf;
    bp.lse_out = ctx->d_lse;
    bp.trig = selector == KVC_SEL_BEACON_TRIGGER ? ctx->d_trig : nullptr;
    bp.status = ctx->d_status;
    bp.num_pages = c.num_pages;
    bp.total_segs = (int64_t)R * per_req_segs;
    bp.bt_stride = ctx->maxp;
    bp.layers = c.num_layers;
    bp.hkv = c.num_kv_heads;
    bp.B = c.num_beacons;
    bp.d = c.head_dim;
    bp.dtype = c.dtype;
    bp.max_seq = c.max_seq_len;
    int max_l = 0;
    for (const auto &s : segs) max_l = std::max(max_l, s.L);
    const bool use_tc = ctx->score_impl == 2 ||
                        (ctx->score_impl == 0 && beacon_score_tc_supported(c.head_dim, c.num_beacons, c.dtype));
    e = use_tc ? launch_beacon_score_tc(bp, (int)segs.size(), max_l, ctx->stream)
               : launch_beacon_score_simt(bp, (int)segs.size(), ctx->stream);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "beacon_score");
    st.launches += 1;
    st.score_kernel = use_tc ? 2 : 1;
  }
  if (timed) KVC_CUDA(ctx, cudaEventRecord(ctx->ev[1], ctx->stream));
  SelectCompactParams sp{};
  sp.k_pool = ctx->k_pool;
  sp.v_pool = ctx->v_pool;
  sp.pos_map = ctx->d_pos;
  sp.block_table = ctx->d_bt;
  sp.scores = score_buf;
  sp.debug = (debug_scores && !beacon_sel) ? static_cast<uint32_t *>(debug_scores) : nullptr;
  sp.counters = ctx->d_counters;
  sp.status = ctx->d_status;
  sp.num_pages = c.num_pages;
  sp.bt_stride = ctx->maxp;
  sp.layers = c.num_layers;
  sp.hkv = c.num_kv_heads;
  sp.row_bytes = ctx->row_bytes;
  sp.max_seq = c.max_seq_len;
  sp.block = o.block;
  sp.flags = (o.compaction == KVC_COMPACT_HOLE_FILL ? kScHoleFill : 0) | (tie_by_pos ? kScTieByPos : 0);
  sp.seed = seed;
  sp.round = (uint64_t)ctx->round;
  const int mode = selector == KVC_SEL_RANDOM ? kModeRandom
                   : selector == KVC_SEL_RANDOM_SHARED ? kModeRandomShared : kModeScores;
  // launches: every segment with more than kSelectSmallMax candidates in one
  // (the kernel's persistent form, which balances the segments itself), the
  // others in buckets of candidate counts (2^(k-1), 2^k], k >= 10.  The split
  // only sizes the launches: any bucket is computed correctly.
  {
    NvtxRange nvtx_select("select_compact");  // "kvc_compress/select_compact/"
    constexpr int kSelectSmallMax = 4096;
    size_t i0 = 0;
    while (i0 < segs.size()) {
      const int max_n = segs[i0].L - segs[i0].P;
      int lo = kSelectSmallMax;
      if (max_n <= kSelectSmallMax) {
        int cap = 1024;
        while (cap < max_n) cap *= 2;
        lo = cap == 1024 ? 0 : cap / 2;
      }
      size_t i1 = i0;
      int max_m = 0;
      while (i1 < segs.size() && segs[i1].L - segs[i1].P > lo) {
        max_m = std::max(max_m, segs[i1].M);
        ++i1;
      }
      sp.segs = d_segs + i0;
      e = launch_select_compact(sp, mode, (int)(i1 - i0), max_n, max_m, ctx->stream);
      if (e != cudaSuccess) return cuda_fail(ctx, e, "select_compact");
      st.launches += 1;
      i0 = i1;
    }
  }
  if (timed) KVC_CUDA(ctx, cudaEventRecord(ctx->ev[2], ctx->stream));
  KVC_CUDA(ctx, cudaMemcpyAsync(ctx->d_len, sd_stage.d + align_up(seg_bytes, 16), (size_t)R * 4,
                                cudaMemcpyDeviceToDevice, ctx->stream));
  if (new_prompt != ctx->h_prompt)
    KVC_CUDA(ctx, cudaMemcpyAsync(ctx->d_prompt, sd_stage.d + align_up(seg_bytes, 16) + (size_t)R * 4,
                                  (size_t)R * 4, cudaMemcpyDeviceToDevice, ctx->stream));
  if (kvc_status s = stage_release(ctx, sd_stage)) return s;
  // host mirror: lengths and freed pages
  for (int r = 0; r < R; ++r) {
    const int L = ctx->h_len[r], Rn = new_len[r];
    if (Rn == L) continue;
    for (int pg = (Rn + kPage - 1) / kPage; pg < (L + kPage - 1) / kPage; ++pg) {
      int32_t &id = ctx->h_bt[(size_t)r * ctx->maxp + pg];
      ctx->free_pages.push_back(id);
      id = -1;
    }
    ctx->h_len[r] = Rn;
  }
  ctx->h_prompt = new_prompt;
  if (o.compaction == KVC_COMPACT_HOLE_FILL)
    for (const auto &sg : segs) ctx->h_unordered[sg.req] = 1;
  ctx->round += 1;
  if (timed) {
    KVC_CUDA(ctx, cudaStreamSynchronize(ctx->stream));
    unsigned long long moved = 0;
    KVC_CUDA(ctx, cudaMemcpy(&moved, ctx->d_counters, sizeof(moved), cudaMemcpyDeviceToHost));
    st.moved_rows = (int64_t)moved;
    st.compaction_bytes = st.moved_rows * ctx->row_bytes * 2 * 2;
    if (beacon_sel)
      for (const auto &s : segs) st.key_bytes_scored += (int64_t)s.L * ctx->row_bytes * per_req_segs;
    KVC_CUDA(ctx, cudaEventElapsedTime(&st.ms_score, ctx->ev[0], ctx->ev[1]));
    KVC_CUDA(ctx, cudaEventElapsedTime(&st.ms_select_compact, ctx->ev[1], ctx->ev[2]));
    KVC_CUDA(ctx, cudaEventElapsedTime(&st.ms_total, ctx->ev[0], ctx->ev[2]));
    *stats = st;
    return take_device_status(ctx);
  }
  return KVC_OK;
}

kvc_status kvc_gather_view(const kvc_ctx *ctx, kvc_view *out) {
  if (!ctx || !out) return KVC_ERR_INVALID_ARG;
  out->k_pool = ctx->k_pool;
  out->v_pool = ctx->v_pool;
  out->block_table = ctx->d_bt;
  out->lengths = ctx->d_len;
  out->prompt_lengths = ctx->d_prompt;
  out->pos_map = ctx->d_pos;
  out->query_ring = ctx->d_qring;
  out->beacons = ctx->d_beacons;
  out->beacons_scoring = ctx->d_beacons_s;
  out->beacon_counts = ctx->d_counts;
  out->beacon_triggers = ctx->d_trig;
  out->max_pages_per_request = ctx->maxp;
  out->row_bytes = ctx->row_bytes;
  out->round = ctx->round;
  return KVC_OK;
}

kvc_status kvc_get_lengths(const kvc_ctx *ctx, int32_t *lengths, int32_t *prompt_lengths) {
  if (!ctx) return KVC_ERR_INVALID_ARG;
  const size_t R = ctx->cfg.num_requests;
  if (lengths) std::memcpy(lengths, ctx->h_len.data(), R * 4);
  if (prompt_lengths) std::memcpy(prompt_lengths, ctx->h_prompt.data(), R * 4);
  return KVC_OK;
}

kvc_status kvc_gather_dense(kvc_ctx *ctx, int32_t layer, int32_t req_begin, int32_t req_count,
                            int32_t cap, void *k_out, void *v_out, int32_t *pos_out) {
  NvtxRange nvtx_range("kvc_gather_dense");
  if (!ctx) return KVC_ERR_INVALID_ARG;
  const kvc_config &c = ctx->cfg;
  if (layer < 0 || layer >= c.num_layers || req_begin < 0 || req_count < 0 ||
      req_begin + req_count > c.num_requests || cap < 0)
    return fail(ctx, KVC_ERR_INVALID_ARG, "layer / request range / cap out of range");
  KVC_CUDA(ctx, cudaSetDevice(ctx->device));
  for (const void *p : {static_cast<const void *>(k_out), static_cast<const void *>(v_out),
                        static_cast<const void *>(pos_out)})
    if (p && !device_ptr_on(ctx->device, p))
      return fail(ctx, KVC_ERR_INVALID_ARG, "outputs must be device memory");
  if (((uintptr_t)k_out | (uintptr_t)v_out) & 15) return fail(ctx, KVC_ERR_INVALID_ARG, "k_out/v_out must be 16-byte aligned");
  cudaError_t e = launch_gather_dense(ctx->k_pool, ctx->v_pool, ctx->d_pos, ctx->d_bt, ctx->d_len, layer,
                                      req_begin, req_count, cap, c.num_kv_heads, ctx->row_bytes,
                                      c.num_pages, ctx->maxp, static_cast<uint8_t *>(k_out),
                                      static_cast<uint8_t *>(v_out), pos_out, ctx->stream);
  if (e != cudaSuccess) return cuda_fail(ctx, e, "gather_dense");
  return KVC_OK;
}

kvc_status kvc_decode_attention(kvc_ctx *ctx, int32_t layer_begin, int32_t layer_count, const void *q,
                                float scale, float *out, float *lse, float *ms_out) {
  NvtxRange nvtx_range("kvc_decode_attention");
  if (!ctx) return KVC_ERR_INVALID_ARG;
  const kvc_config &c = ctx->cfg;
  if (layer_begin < 0 || layer_count < 1 || layer_begin + layer_count > c.num_layers)
    return fail(ctx, KVC_ERR_INVALID_ARG, "layer range out of bounds");
  if (!q || !out) return fail(ctx, KVC_ERR_INVALID_ARG, "q and out are required");
  if (!(scale >= 0.f) || !std::isfinite(scale)) return fail(ctx, KVC_ERR_INVALID_ARG, "scale must be finite and >= 0");
  KVC_CUDA(ctx, cudaSetDevice(ctx->device));
  if (!device_ptr_on(ctx->device, q) || !device_ptr_on(ctx->device, out) ||
      (lse && !device_ptr_on(ctx->device, lse)))
    return fail(ctx, KVC_ERR_INVALID_ARG, "q, out and lse must be device memory of the context's device");
  if (((uintptr_t)q % ctx->es) || ((uintptr_t)out & 3) || ((uintptr_t)lse & 3))
    return fail(ctx, KVC_ERR_INVALID_ARG, "q, out or lse misaligned");
  const int G = ctx->G;
  if (!decode_attention_supported(c.dtype, c.head_dim, G))
    return fail(ctx, KVC_ERR_UNSUPPORTED,
                "decode attention needs bf16 or f32, head_dim 64 or 128 and 1, 2, 4 or 8 query heads per KV head");
  const int R = c.num_requests;
  int max_len = 0;
  for (int r = 0; r < R; ++r) max_len = std::max(max_len, ctx->h_len[r]);
  const int np_max = (max_len + kPage - 1) / kPage;
  // splits: enough CTAs for two waves of two CTAs per SM, pages of a split a
  // multiple of the 4-page tile, at least two tiles per split
  const int64_t base = (int64_t)layer_count * R * c.num_kv_heads;
  int nsplit = 1;
  if (np_max > 0) {
    const int64_t want = (4LL * ctx->num_sms + base - 1) / base;
    nsplit = (int)std::max<int64_t>(1, std::min<int64_t>({want, kAttnSplits / layer_count, (np_max + 7) / 8}));
  }
  int pps = std::max(1, (np_max + nsplit - 1) / nsplit);
  pps = (pps + 3) & ~3;
  nsplit = std::max(1, (np_max + pps - 1) / pps);
  DecodeAttnParams p{};
  p.k_pool = ctx->k_pool;
  p.v_pool = ctx->v_pool;
  p.q = static_cast<const uint8_t *>(q);
  p.block_table = ctx->d_bt;
  p.lengths = ctx->d_len;
  p.out = out;
  p.lse = lse;
  p.part_o = ctx->d_attn;
  p.part_ml = ctx->d_attn + (size_t)layer_count * R * c.num_q_heads * nsplit * c.head_dim;
  p.status = ctx->d_status;
  p.num_pages = c.num_pages;
  p.bt_stride = ctx->maxp;
  p.layer_begin = layer_begin;
  p.layer_count = layer_count;
  p.R = R;
  p.hkv = c.num_kv_heads;
  p.hq = c.num_q_heads;
  p.nsplit = nsplit;
  p.pages_per_split = pps;
  p.qscale = (scale > 0.f ? scale : 1.0f / std::sqrt((float)c.head_dim)) * 1.4426950408889634f;
  if (ms_out) KVC_CUDA(ctx, cudaEventRecord(ctx->ev[0], ctx->stream));
  int launches = 0;
  cudaError_t e = launch_decode_attention(p, c.head_dim, c.dtype, G, &launches, ctx->stream);
  if (e != cudaSuccess) return cuda_fail(ctx, e, "decode_attention");
  if (ms_out) {
    KVC_CUDA(ctx, cudaEventRecord(ctx->ev[1], ctx->stream));
    KVC_CUDA(ctx, cudaEventSynchronize(ctx->ev[1]));
    KVC_CUDA(ctx, cudaEventElapsedTime(ms_out, ctx->ev[0], ctx->ev[1]));
    return take_device_status(ctx);
  }
  return KVC_OK;
}

kvc_status kvc_check_wait_timeout(kvc_ctx *ctx, uint32_t limit_ms) {
  if (!ctx) return KVC_ERR_INVALID_ARG;
  if (limit_ms < 1 || limit_ms > 2000) return fail(ctx, KVC_ERR_INVALID_ARG, "limit_ms must be in [1, 2000]");
  KVC_CUDA(ctx, cudaSetDevice(ctx->device));
  if (kvc_status st = take_device_status(ctx)) return st;  // an earlier error is reported as such
  cudaError_t e = launch_wait_timeout_probe(ctx->d_status, limit_ms, ctx->stream);
  if (e != cudaSuccess) return cuda_fail(ctx, e, "wait_timeout_probe");
  return take_device_status(ctx);
}

kvc_status kvc_sync(kvc_ctx *ctx) {
  if (!ctx) return KVC_ERR_INVALID_ARG;
  KVC_CUDA(ctx, cudaSetDevice(ctx->device));
  KVC_CUDA(ctx, cudaStreamSynchronize(ctx->stream));
  return take_device_status(ctx);
}

}  // extern "C"
