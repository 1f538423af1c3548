// paged_io.cu -- moving tokens into and out of the paged cache.
//
// append: the decode step writes the new token's K and V into the cache and
// the cache grows by one position per step (BeaconKV abstract; Random
// Attention article, "长推理的显存瓶颈").  The attention backend also hands
// over the step's queries (BeaconKV explainer §7.2), which go to a ring of the
// last W steps for the periodic beacon update.
// gather_dense: a dense copy of one layer, used to check the cache against
// the oracle.
//
// All three kernels move 16-byte vectors, one per thread, with consecutive
// threads on consecutive bytes of the source (coalesced reads; writes are
// contiguous per row).  Sources may be page-locked host memory, read over
// PCIe through the unified address space.
#include "kvc_internal.h"

namespace kvc {
namespace {

__global__ void bt_scatter_kernel(const int32_t *__restrict__ pairs, int n,
                                  int32_t *__restrict__ block_table) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) block_table[pairs[2 * i]] = pairs[2 * i + 1];
}

// source [n_req][layers][T][hkv][row] ; one thread per 16-byte vector
__global__ void append_kv_kernel(const uint8_t *__restrict__ k_src, const uint8_t *__restrict__ v_src,
                                 uint8_t *__restrict__ k_pool, uint8_t *__restrict__ v_pool,
                                 int32_t *__restrict__ pos_map, const int32_t *__restrict__ block_table,
                                 const int4 *__restrict__ desc, int layers, int T, int hkv,
                                 int vpr, int64_t total, int64_t num_pages, int bt_stride) {
  const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (g >= total) return;
  int64_t rest = g;
  const int v = (int)(rest % vpr);
  rest /= vpr;
  const int h = (int)(rest % hkv);
  rest /= hkv;
  const int t = (int)(rest % T);
  rest /= T;
  const int l = (int)(rest % layers);
  const int i = (int)(rest / layers);
  const int4 d = desc[i];  // req, len_before, pos_before
  const int slot = d.y + t;
  const int page = block_table[(int64_t)d.x * bt_stride + (slot >> 4)];
  const int64_t row = (((int64_t)l * num_pages + page) * hkv + h) * kPage + (slot & (kPage - 1));
  const int64_t dst = row * vpr * 16 + (int64_t)v * 16;
  *reinterpret_cast<uint4 *>(k_pool + dst) = *reinterpret_cast<const uint4 *>(k_src + g * 16);
  *reinterpret_cast<uint4 *>(v_pool + dst) = *reinterpret_cast<const uint4 *>(v_src + g * 16);
  if (v == 0) pos_map[row] = d.z + t;
}

// source [n_req][layers][T][hq][row]; only the last W steps are written
__global__ void append_q_kernel(const uint8_t *__restrict__ q_src, uint8_t *__restrict__ qring,
                                const int4 *__restrict__ desc, int layers, int T, int t0, int W,
                                int hq, int vpr, int64_t total) {
  const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (g >= total) return;
  int64_t rest = g;
  const int v = (int)(rest % vpr);
  rest /= vpr;
  const int hh = (int)(rest % hq);
  rest /= hq;
  const int tt = (int)(rest % (T - t0));
  rest /= (T - t0);
  const int l = (int)(rest % layers);
  const int i = (int)(rest / layers);
  const int t = t0 + tt;
  const int4 d = desc[i];  // req, ring slot of step 0
  const int ring = (d.y + t) % W;
  const int64_t src = ((((int64_t)i * layers + l) * T + t) * hq + hh) * vpr + v;
  const int64_t dst = ((((int64_t)d.x * layers + l) * W + ring) * hq + hh) * vpr + v;
  reinterpret_cast<uint4 *>(qring)[dst] = reinterpret_cast<const uint4 *>(q_src)[src];
}

__global__ void gather_dense_kernel(const uint8_t *__restrict__ k_pool, const uint8_t *__restrict__ v_pool,
                                    const int32_t *__restrict__ pos_map,
                                    const int32_t *__restrict__ block_table,
                                    const int32_t *__restrict__ lengths, int layer, int req_begin,
                                    int cap, int hkv, int vpr, int64_t total, int64_t num_pages,
                                    int bt_stride, uint8_t *__restrict__ k_out,
                                    uint8_t *__restrict__ v_out, int32_t *__restrict__ pos_out) {
  const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (g >= total) return;
  int64_t rest = g;
  const int v = (int)(rest % vpr);
  rest /= vpr;
  const int slot = (int)(rest % cap);
  rest /= cap;
  const int h = (int)(rest % hkv);
  const int i = (int)(rest / hkv);
  const int r = req_begin + i;
  uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
  int pos = -1;
  if (slot < lengths[r]) {
    const int page = block_table[(int64_t)r * bt_stride + (slot >> 4)];
    const int64_t row = (((int64_t)layer * num_pages + page) * hkv + h) * kPage + (slot & (kPage - 1));
    kv = *reinterpret_cast<const uint4 *>(k_pool + row * vpr * 16 + (int64_t)v * 16);
    vv = *reinterpret_cast<const uint4 *>(v_pool + row * vpr * 16 + (int64_t)v * 16);
    pos = pos_map[row];
  }
  if (k_out) reinterpret_cast<uint4 *>(k_out)[g] = kv;
  if (v_out) reinterpret_cast<uint4 *>(v_out)[g] = vv;
  if (pos_out && v == 0) pos_out[g / vpr] = pos;
}

inline unsigned blocks_for(int64_t total, int nt) { return (unsigned)((total + nt - 1) / nt); }

}  // namespace

cudaError_t launch_bt_scatter(const int32_t *pairs, int n, int32_t *block_table, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  bt_scatter_kernel<<<blocks_for(n, 256), 256, 0, s>>>(pairs, n, block_table);
  return cudaGetLastError();
}

cudaError_t launch_append_kv(const uint8_t *k_src, const uint8_t *v_src, uint8_t *k_pool,
                             uint8_t *v_pool, int32_t *pos_map, const int32_t *block_table,
                             const int32_t *desc, int n_req, int layers, int T, int hkv,
                             int row_bytes, int64_t num_pages, int bt_stride, cudaStream_t s) {
  const int vpr = row_bytes / 16;
  const int64_t total = (int64_t)n_req * layers * T * hkv * vpr;
  if (total <= 0) return cudaSuccess;
  append_kv_kernel<<<blocks_for(total, 256), 256, 0, s>>>(
      k_src, v_src, k_pool, v_pool, pos_map, block_table, reinterpret_cast<const int4 *>(desc),
      layers, T, hkv, vpr, total, num_pages, bt_stride);
  return cudaGetLastError();
}

cudaError_t launch_append_q(const uint8_t *q_src, uint8_t *qring, const int32_t *desc, int n_req,
                            int layers, int T, int t0, int W, int hq, int row_bytes,
                            cudaStream_t s) {
  const int vpr = row_bytes / 16;
  const int64_t total = (int64_t)n_req * layers * (T - t0) * hq * vpr;
  if (total <= 0) return cudaSuccess;
  append_q_kernel<<<blocks_for(total, 256), 256, 0, s>>>(
      q_src, qring, reinterpret_cast<const int4 *>(desc), layers, T, t0, W, hq, vpr, total);
  return cudaGetLastError();
}

cudaError_t launch_gather_dense(const uint8_t *k_pool, const uint8_t *v_pool,
                                const int32_t *pos_map, const int32_t *block_table,
                                const int32_t *lengths, int layer, int req_begin, int req_count,
                                int cap, int hkv, int row_bytes, int64_t num_pages, int bt_stride,
                                uint8_t *k_out, uint8_t *v_out, int32_t *pos_out, cudaStream_t s) {
  const int vpr = row_bytes / 16;
  const int64_t total = (int64_t)req_count * hkv * cap * vpr;
  if (total <= 0) return cudaSuccess;
  gather_dense_kernel<<<blocks_for(total, 256), 256, 0, s>>>(
      k_pool, v_pool, pos_map, block_table, lengths, layer, req_begin, cap, hkv, vpr, total,
      num_pages, bt_stride, k_out, v_out, pos_out);
  return cudaGetLastError();
}

}  // namespace kvc
