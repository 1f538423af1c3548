// kvc_internal.h -- structures shared by the host orchestration (kvc_api.cu)
// and the sm_100a kernels of libkvc.so.  Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kvc.h"

namespace kvc {

constexpr int kPage = 16;            // tokens per page
constexpr int kMaxSeqLen = 32768;    // per request; bounds the select kernel's shared memory
constexpr int kMaxBeacons = 256;
constexpr int kMaxPoints = 4096;     // query_window * G
constexpr int kMaxRowBytes = 1024;

// Device status word values (first error wins).
constexpr int kDevOk = 0;
constexpr int kDevNaN = 1;
constexpr int kDevIndex = 2;
constexpr int kDevTimeout = 3;  // a bounded device wait ran out

// Score sources of the fused select + compaction kernel.
enum ScoreMode : int { kModeRandom = 0, kModeRandomShared = 1, kModeScores = 2 };

// One evicting request of a round: its pre-round length L, protected prompt
// P and number M of generated positions to keep (0 < M < L - P).
struct SegDesc {
  int32_t req, L, P, M;
};

struct SelectCompactParams {
  uint8_t *k_pool, *v_pool;
  int32_t *pos_map;             // [layers][pages][Hkv][16]
  const int32_t *block_table;   // [R][bt_stride]
  const SegDesc *segs;          // [n_segs_req] one per request in this launch
  const float *scores;          // beacon scores [R][layers][Hkv][max_seq] (kModeScores)
  uint32_t *debug;              // optional: candidate keys, same layout as scores
  unsigned long long *counters; // [0] moved rows
  int32_t *status;
  int64_t num_pages;
  int32_t bt_stride, layers, hkv, row_bytes, max_seq;
  int32_t block;  // positions per Philox draw (random selectors)
  int32_t flags;  // kScTieByPos | kScHoleFill
  uint64_t seed, round;
};

// SelectCompactParams::flags
constexpr int kScTieByPos = 1;  // slots may be out of position order: split ties by position
constexpr int kScHoleFill = 2;  // hole-filling compaction (implies ties by position)

// One decode step of attention over the cache (decode_attention.cu).
struct DecodeAttnParams {
  const uint8_t *k_pool, *v_pool;  // [layers][pages][Hkv][16][d] dtype
  const uint8_t *q;            // [layer_count][R][Hq][d] dtype
  const int32_t *block_table;  // [R][bt_stride]
  const int32_t *lengths;      // [R] device lengths
  float *out;                  // [layer_count][R][Hq][d]
  float *lse;                  // [layer_count][R][Hq] or null
  float *part_o;               // split partials [layer_count][R][Hq][nsplit][d]
  float *part_ml;              // [layer_count][R][Hq][nsplit][2] (max in base 2, sum)
  int32_t *status;
  int64_t num_pages;
  int32_t bt_stride, layer_begin, layer_count, R, hkv, hq, nsplit, pages_per_split;
  float qscale;                // scale * log2(e)
};

// Beacon update over the query ring.
struct UpdateDesc {
  int32_t req, ring_start, n_steps, init;
};

struct BeaconUpdateParams {
  const uint8_t *qring;       // [R][layers][W][Hq][d] dtype
  float *beacons;             // [R][layers][Hkv][B][d]
  uint8_t *beacons_s;         // scoring copy, dtype
  int32_t *counts;            // [R][layers][Hkv][B]
  int32_t *assign_out;        // optional [R][layers][Hkv][W*G]
  float *trig;                // [R][layers][Hkv][B]: share of this update's points per beacon
  const UpdateDesc *descs;
  int32_t *status;
  int32_t layers, hkv, hq, G, W, B, d, dtype;
  int32_t n_ring;             // requests in the query ring (R)
};

// Beacon score over the paged keys of a segment.
struct BeaconScoreParams {
  const uint8_t *k_pool;
  const int32_t *block_table;
  const SegDesc *segs;
  const uint8_t *beacons_s;   // [R][layers][Hkv][B][d] dtype
  float *scores;              // [R][layers][Hkv][max_seq]
  float *lse_out;             // optional [R][layers][Hkv][B]
  const float *trig;          // cluster-trigger mode: [R][layers][Hkv][B] shares; null = max mode
  int32_t *status;
  int64_t num_pages;
  int64_t total_segs;         // R * layers * Hkv (rows of the beacon arrays / B)
  int32_t bt_stride, layers, hkv, B, d, dtype, max_seq;
};

// Kernel launchers (each returns the launch error, if any).
cudaError_t launch_bt_scatter(const int32_t *pairs, int n, int32_t *block_table, cudaStream_t s);
cudaError_t launch_append_kv(const uint8_t *k_src, const uint8_t *v_src, uint8_t *k_pool,
                             uint8_t *v_pool, int32_t *pos_map, const int32_t *block_table,
                             const int32_t *desc /* [n_req][4]: req, len_before, pos_before, - */,
                             int n_req, int layers, int T, int hkv, int row_bytes,
                             int64_t num_pages, int bt_stride, cudaStream_t s);
cudaError_t launch_append_q(const uint8_t *q_src, uint8_t *qring,
                            const int32_t *desc /* [n_req][4]: req, ring slot of step 0, t0, - */,
                            int n_req, int layers, int T, int t0_global, int W, int hq,
                            int row_bytes, cudaStream_t s);
cudaError_t launch_gather_dense(const uint8_t *k_pool, const uint8_t *v_pool,
                                const int32_t *pos_map, const int32_t *block_table,
                                const int32_t *lengths, int layer, int req_begin, int req_count,
                                int cap, int hkv, int row_bytes, int64_t num_pages, int bt_stride,
                                uint8_t *k_out, uint8_t *v_out, int32_t *pos_out, cudaStream_t s);
cudaError_t launch_wait_timeout_probe(int32_t *status, uint32_t limit_ms, cudaStream_t s);
bool decode_attention_supported(int dtype, int head_dim, int G);
cudaError_t launch_decode_attention(const DecodeAttnParams &p, int head_dim, int dtype, int G, int *launches,
                                    cudaStream_t s);
cudaError_t launch_select_compact(const SelectCompactParams &p, int mode, int n_seg_req,
                                  int max_n, int max_m, cudaStream_t s);
cudaError_t launch_beacon_update(const BeaconUpdateParams &p, int n_req, cudaStream_t s);
cudaError_t launch_beacon_score_simt(const BeaconScoreParams &p, int n_req, cudaStream_t s);
cudaError_t launch_beacon_score_tc(const BeaconScoreParams &p, int n_req, int max_l,
                                   cudaStream_t s);
bool beacon_score_tc_supported(int d, int B, int dtype);
cudaError_t launch_beacon_update_tc(const BeaconUpdateParams &p, int n_req, cudaStream_t s);
bool beacon_update_tc_supported(int d, int B, int dtype);

}  // namespace kvc
