/*
 * kvc.h -- C ABI of libkvc.so, a B200 (sm_100a) library for the batched
 * decode-time KV-cache eviction round over a paged KV cache.
 *
 * The round, for every segment s = (request r, layer l, KV head h):
 *   (a) scores the generated positions with the Random-Attention selector (a
 *       counter-based Philox score per head and position) or with the BeaconKV
 *       selector (maximum softmax mass over the segment's beacons);
 *   (b) never evicts the protected prompt;
 *   (c) keeps the top positions by (score desc, original position asc)
 *       against the request's budget K;
 *   (d) compacts the surviving K/V rows in place, in their original order.
 *
 * Passages that define the operations (web pages, by title and section):
 *   [RA] Random Attention article, "随机保留 KV Cache 竟不输精心设计的 eviction
 *        策略？..." (aiinking.com/article/67532): "长推理的显存瓶颈" (fixed
 *        budget K), "Random Attention：不判断重要性，只随机保留" (full prompt
 *        protection; independent random Top-K per head; one RNG call plus one
 *        Top-K), "发现二" (one random set shared by all heads), "发现四" (the
 *        compression trigger at a batch sync point; cache compaction, which
 *        every method needs; content selectors traverse the paged KV state).
 *   [BX] BeaconKV explainer (papers.ananclaw.com/promo/explainers__2609-04971)
 *        §3.2: a query goes to its nearest beacon; beacons are updated
 *        periodically and incrementally; §7.2: the attention backend must
 *        expose the queries.
 *   [BA] BeaconKV abstract (chatpaper.ai): beacon queries are compact
 *        representatives of global query clusters.
 *
 * Conventions for every call:
 *  - Status codes only; nothing throws across the ABI.  On error the context
 *    is unchanged unless stated, and kvc_last_error() describes the failure.
 *  - Ownership: all device memory (the two K/V pools and the workspace) is
 *    allocated by the caller and borrowed for the life of the context; the
 *    library never frees device memory.  It owns only host metadata (and a
 *    small pinned host staging ring), released by kvc_destroy().
 *  - Ordering: every call is enqueued on the context's CUDA stream and is
 *    asynchronous unless stated.  Host arrays passed in are consumed before
 *    the call returns.  A context is not thread-safe.
 *  - Device-detected errors (KVC_ERR_NAN, KVC_ERR_DEVICE_TIMEOUT) are latched
 *    in a device status word and reported by the next synchronising call
 *    (kvc_sync, or a call given a stats pointer).  Page ids, slots and
 *    lengths reach the kernels only from the library's own bookkeeping
 *    (kvc_append allocates the pages; kvc_compress frees them), which the
 *    host validates, so the kernels do not range-check them; a caller that
 *    writes into the state through kvc_gather_view takes that on itself.
 *
 * Data layout (all row-major, C order):
 *   k_pool, v_pool  [num_layers][num_pages][num_kv_heads][16][head_dim] dtype
 *                   (page size 16; a page id addresses the same page in every
 *                   layer; the 16 rows of one (page, head) are contiguous)
 *   block table     [num_requests][max_seq_len/16] int32 page ids, shared by
 *                   all layers and heads of a request
 *   position map    [num_layers][num_pages][num_kv_heads][16] int32: the
 *                   original absolute position held by each slot
 *   query ring      [num_requests][num_layers][query_window][num_q_heads][head_dim] dtype
 *   beacons         [num_requests][num_layers][num_kv_heads][num_beacons][head_dim]
 *                   fp32 state + counts int32 + a scoring copy in dtype
 * Slots hold positions in increasing order at all times (appends add
 * increasing positions; compaction preserves order), so the tie-break by
 * lower original position is the tie-break by lower slot.
 */
#ifndef KVC_H
#define KVC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KVC_OK = 0,
  KVC_ERR_INVALID_ARG = 1,    /* bad pointer, size, alignment or enum value */
  KVC_ERR_OUT_OF_PAGES = 2,   /* the page pool cannot hold the append */
  KVC_ERR_STATE = 3,          /* call not valid in the current state */
  KVC_ERR_CUDA = 4,           /* a CUDA runtime/driver call failed */
  KVC_ERR_NAN = 5,            /* a NaN reached a beacon distance or score */
  KVC_ERR_DEVICE_CHECK = 6,   /* reserved, never returned by this build: the value is kept for a
                                 build whose kernels range-check page ids and slots */
  KVC_ERR_DEVICE_TIMEOUT = 7, /* a bounded device wait ran out (see kvc_check_wait_timeout) */
  KVC_ERR_UNSUPPORTED = 8     /* valid request this build does not support */
} kvc_status;

typedef enum { KVC_BF16 = 0, KVC_F32 = 1 } kvc_dtype;

typedef enum {
  KVC_SEL_RANDOM = 0,        /* [RA]: independent Philox score per head and position */
  KVC_SEL_RANDOM_SHARED = 1, /* [RA "发现二"]: one score per (request, layer, position) */
  KVC_SEL_BEACON = 2,        /* [BX]/[BA]: max over beacons of softmax(c.K^T/sqrt(d)) */
  KVC_SEL_BEACON_TRIGGER = 3 /* [BX] §3.2 cluster-level trigger: sum over beacons of the latest
                                update's share of points in the beacon's cluster times the
                                beacon's softmax (see kvc_compress) */
} kvc_selector;

/* Limits of this build (checked by kvc_create):
 *   page_size == 16; head_dim * sizeof(dtype) a multiple of 16 bytes and
 *   <= 1024 bytes; max_seq_len a multiple of 16 and <= 32768;
 *   num_beacons in [0, 256]; query_window * (num_q_heads / num_kv_heads)
 *   <= 4096; num_q_heads a multiple of num_kv_heads. */
typedef struct {
  int32_t num_requests;
  int32_t num_layers;
  int32_t num_kv_heads;
  int32_t num_q_heads;   /* query heads; GQA group G = num_q_heads / num_kv_heads */
  int32_t head_dim;
  int32_t page_size;     /* must be 16 */
  int32_t dtype;         /* kvc_dtype of K, V, queries and the beacon scoring copy */
  int32_t num_beacons;   /* B per (request, layer, KV head); 0 = no beacon state */
  int32_t query_window;  /* W decode steps kept per request; 0 = no query ring */
  int32_t max_seq_len;   /* cache length limit per request (block table width x 16) */
  int64_t num_pages;     /* pages in each layer's pool */
} kvc_config;

/* Per-round counters, filled by kvc_compress when given a stats pointer. */
typedef struct {
  int64_t round;                 /* index of this round, from 0 */
  int64_t segments;              /* (request, layer, KV head) segments in the round */
  int64_t noop_segments;         /* segments with L <= K (nothing evicted) */
  int64_t prompt_over_budget_segments; /* segments with P > K < L */
  int64_t head_positions;        /* sum over segments of the pre-round length L */
  int64_t candidates;            /* sum of N = L - P over evicting segments */
  int64_t evicted;               /* sum of evicted positions */
  int64_t moved_rows;            /* rows moved by compaction (each: one K and one V row) */
  int64_t compaction_bytes;      /* moved_rows * 2 * row_bytes * 2 (read + write K and V) */
  int64_t key_bytes_scored;      /* beacon selector: key bytes of all cached keys, once */
  float ms_score;                /* device time of the beacon scoring kernel(s) */
  float ms_select_compact;       /* device time of the fused select + compaction kernel */
  float ms_total;                /* device time of the whole call */
  int32_t launches;              /* kernels this call launched */
  int32_t score_kernel;          /* beacon score kernel used: 0 none, 1 SIMT fp32, 2 tcgen05 */
  int32_t reserved;
} kvc_round_stats;

/* Zero-copy view of the context's device state (pointers into the pools and
 * the workspace; valid until kvc_destroy). */
typedef struct {
  void *k_pool;
  void *v_pool;
  int32_t *block_table;       /* [num_requests][max_pages_per_request] */
  int32_t *lengths;           /* [num_requests] current cache lengths */
  int32_t *prompt_lengths;    /* [num_requests] protected prefix lengths */
  int32_t *pos_map;           /* [num_layers][num_pages][num_kv_heads][16] */
  void *query_ring;           /* [num_requests][num_layers][W][num_q_heads][head_dim] */
  float *beacons;             /* [num_requests][num_layers][num_kv_heads][B][head_dim] */
  void *beacons_scoring;      /* same shape, dtype */
  int32_t *beacon_counts;     /* [num_requests][num_layers][num_kv_heads][B] */
  float *beacon_triggers;     /* [num_requests][num_layers][num_kv_heads][B]: share of the latest
                                 update's points assigned to each beacon */
  int32_t max_pages_per_request;
  int32_t row_bytes;          /* head_dim * sizeof(dtype) */
  int64_t round;              /* rounds completed */
} kvc_view;

typedef enum {
  KVC_OPT_BEACON_SCORE_IMPL = 0, /* 0 auto, 1 SIMT fp32 kernel, 2 tcgen05 (bf16, head_dim 128) */
  KVC_OPT_BEACON_UPDATE_IMPL = 1 /* 0 auto, 1 SIMT fp32 kernel, 2 tcgen05 assignment (bf16, head_dim 128,
                                    B a multiple of 32): x.c as x.c_hi + x.c_lo with bf16 terms of the
                                    fp32 beacons, error <= 2^-18 sum_k |x_k c_k| beyond fp32 rounding */
} kvc_option;

typedef struct kvc_ctx kvc_ctx;

/* Bytes of device workspace kvc_create needs for cfg (0 if cfg is invalid).
 * The workspace holds the block tables, lengths, position map, query ring,
 * beacon state, per-candidate score scratch ([R][layers][Hkv][max_seq_len]
 * fp32, used by the beacon selector) and round descriptors. */
size_t kvc_workspace_bytes(const kvc_config *cfg);

/* Creates a context over caller-allocated device memory.
 *   k_pool, v_pool: device, 256-byte aligned, each
 *     num_layers*num_pages*num_kv_heads*16*head_dim*sizeof(dtype) bytes.
 *   workspace: device, 256-byte aligned, >= kvc_workspace_bytes(cfg) bytes;
 *     its contents are initialised here (enqueued on the stream).
 *   cuda_stream: cudaStream_t on the pools' device (NULL = legacy stream).
 * All requests start empty; every page is free. */
kvc_status kvc_create(const kvc_config *cfg, void *k_pool, void *v_pool, void *workspace,
                      size_t workspace_bytes, void *cuda_stream, kvc_ctx **out);

/* Releases host metadata.  Synchronises the stream first.  NULL is a no-op. */
kvc_status kvc_destroy(kvc_ctx *ctx);

/* Makes later calls enqueue on another stream of the same device. */
kvc_status kvc_set_stream(kvc_ctx *ctx, void *cuda_stream);

kvc_status kvc_set_option(kvc_ctx *ctx, kvc_option opt, int64_t value);

/* Appends n_tokens decode (or prompt) tokens to each listed request.
 *   req_ids: host int32[n_req], distinct, in [0, num_requests).
 *   k_new, v_new: [n_req][num_layers][n_tokens][num_kv_heads][head_dim] dtype,
 *     device memory or page-locked host memory (read over PCIe by the kernel).
 *   q_new: [n_req][num_layers][n_tokens][num_q_heads][head_dim] dtype, same
 *     memory rules, or NULL.  The queries of the last query_window steps are
 *     kept in the ring for kvc_update_beacons ([BX §7.2]: the backend exposes
 *     the queries).
 *   protect: 1 = the tokens belong to the protected prompt [RA]; only valid
 *     while the request holds no generated token (else KVC_ERR_STATE).
 * Token t of request i takes position (its length before the call) + t.
 * Errors (nothing enqueued): KVC_ERR_INVALID_ARG, KVC_ERR_STATE,
 * KVC_ERR_OUT_OF_PAGES (max_seq_len or the pool would overflow). */
kvc_status kvc_append(kvc_ctx *ctx, const int32_t *req_ids, int32_t n_req, int32_t n_tokens,
                      const void *k_new, const void *v_new, const void *q_new, int32_t protect);

/* BeaconKV periodic beacon update [BX §3.2], for every request with queries
 * appended since its previous update (at most the last query_window steps).
 * Points of segment (r, l, h): the queries of the G query heads h*G..h*G+G-1
 * of each of those steps, ordered by (step, head).  First update of a
 * request: beacon i of each segment starts as point floor(i*n_pts/B) with
 * count 0 (KVC_ERR_STATE if n_pts < B).  Then each point goes to the beacon
 * at the smallest squared L2 distance (beacons as before this update; ties to
 * the lowest index) and each beacon with m new points becomes the running
 * mean (n*c + sum)/(n + m), n += m; the scoring copy is the new beacon
 * rounded to dtype (round to nearest even).
 *   assign_out: device int32 [R][num_layers][num_kv_heads][W*G] or NULL;
 *     receives each point's beacon (entries past n_pts untouched).
 *   ms_out: host float or NULL; if given, the call synchronises and writes
 *     the device time of the update kernel. */
kvc_status kvc_update_beacons(kvc_ctx *ctx, int32_t *assign_out, float *ms_out);

/* One eviction round over all requests ([RA] "Random Attention：...", "发现四").
 *   budgets: host int32[num_requests], K_r >= 0 per request.
 *   seed: Philox key word 0 (word 1 is the round counter).
 * Per segment with cached length L, prompt P, budget K:
 *   L <= K: unchanged; else the prompt stays and the best max(0, K-P)
 *   generated positions by (score desc, original position asc) are packed in
 *   order to slots P, P+1, ...; the new length is max(P, K); pages past it
 *   return to the free pool.  Random score = high 32 bits of word 0 of
 *   Philox4x64-10(counter = (pos, h, l, r), key = (seed, round)); the shared
 *   variant uses h = 2^64-1.  Beacon score (needs initialised beacons) =
 *   max_b exp(z_bj - logsumexp_j' z_bj') with z_bj = c_b.k_j/sqrt(d) over all
 *   cached keys j (prompt included) and c_b the scoring copy.  Cluster-trigger
 *   score (KVC_SEL_BEACON_TRIGGER; the explainer's "query -> cluster -> KV",
 *   [BX] §3.2 mark_important, read as: each query of the latest update raises
 *   the keys its cluster's beacon attends to) = sum_b w_b exp(z_bj - lse_b)
 *   with w_b the share of the latest update's points assigned to beacon b.
 *   debug_scores: device, NULL or [R][num_layers][num_kv_heads][max_seq_len]
 *     32-bit; receives each candidate's score at index j - P (uint32 for the
 *     random selectors, float for the beacon selector).
 *   stats: host, NULL or filled after synchronising the stream.
 * The round counter advances by one on success. */
kvc_status kvc_compress(kvc_ctx *ctx, kvc_selector selector, const int32_t *budgets,
                        uint64_t seed, void *debug_scores, kvc_round_stats *stats);

/* Options of one eviction round (kvc_compress_ex).  The all-default value,
 * {-1, 1, KVC_COMPACT_ORDERED, 0}, is the round of kvc_compress.
 *   sink_tokens: < 0 protects the whole prompt.  S >= 0 protects only the
 *     first min(P, S) positions, the attention sinks, as the SnapKV-style
 *     baselines of the Random Attention article do ("发现一", on protection
 *     regimes); the rest of the prompt competes with the generated
 *     positions, and the request's protected length becomes min(P, S) for
 *     later rounds once a round evicts from it.
 *   block: random selectors only (must be 1 for the beacon selector),
 *     1 <= block <= 32768: the positions of one block, pos / block, share one
 *     Philox draw (counter word 0 = pos / block), so whole blocks are kept in
 *     order of their draw and at most one block is split, at its lowest
 *     positions ("发现二": contiguous blocks of 1 to 256 tokens).
 *   compaction: KVC_COMPACT_ORDERED packs the survivors in slot order;
 *     KVC_COMPACT_HOLE_FILL leaves every survivor below the new length in
 *     place and moves the i-th survivor at or past it into the i-th evicted
 *     slot below it (ascending), copying only as many rows as there are
 *     holes.  Slots then no longer follow position order; later rounds still
 *     rank ties by original position and keep slot order among survivors.
 *   reserved: 0. */
typedef enum kvc_compaction { KVC_COMPACT_ORDERED = 0, KVC_COMPACT_HOLE_FILL = 1 } kvc_compaction;

typedef struct kvc_round_options {
  int32_t sink_tokens;
  int32_t block;
  int32_t compaction;
  int32_t reserved;
} kvc_round_options;

/* kvc_compress with round options; opts NULL means the defaults.  Invalid
 * options return KVC_ERR_INVALID_ARG with nothing enqueued. */
kvc_status kvc_compress_ex(kvc_ctx *ctx, kvc_selector selector, const int32_t *budgets,
                           uint64_t seed, const kvc_round_options *opts, void *debug_scores,
                           kvc_round_stats *stats);

/* One decode step of attention over the cache as it stands (after any
 * eviction round), for layers [layer_begin, layer_begin + layer_count): the
 * attention kernels every selector shares in the Random Attention article's
 * serving setup ("发现四"; eviction only changes which rows they read).  For
 * request r, layer l and query head hq, with h = hq / G the KV head it reads
 * (G = num_q_heads / num_kv_heads, as in the beacon update):
 *     s_j = scale * q . k_j over the request's cached rows j < length(r),
 *     out = sum_j exp(s_j - lse) v_j,   lse = log sum_j exp(s_j).
 * Slot order does not matter (rows after hole filling included).  A request
 * with no rows gets out = 0 and lse = -inf.
 *   q:   device [layer_count][num_requests][num_q_heads][head_dim] in the
 *        cache dtype, element-aligned; read only.
 *   scale: > 0, or 0 for 1/sqrt(head_dim).
 *   out: device float [layer_count][num_requests][num_q_heads][head_dim].
 *   lse: device float [layer_count][num_requests][num_q_heads] or NULL
 *        (natural log).
 *   ms_out: host float or NULL; if given, the call synchronises and writes
 *     the device time of its kernels, and reports latched device errors.
 * Enqueued on the context's stream; uses the context's workspace for split
 * partials, so calls on one context must not overlap.  Errors (nothing
 * enqueued): KVC_ERR_INVALID_ARG; KVC_ERR_UNSUPPORTED unless the cache is
 * bf16 or f32 with head_dim 64 or 128 and G in {1, 2, 4, 8}. */
kvc_status kvc_decode_attention(kvc_ctx *ctx, int32_t layer_begin, int32_t layer_count, const void *q,
                                float scale, float *out, float *lse, float *ms_out);

/* Fills *out with device pointers to the live state (no copy, no sync). */
kvc_status kvc_gather_view(const kvc_ctx *ctx, kvc_view *out);

/* Host copies of the current lengths and prompt lengths (int32[R] each;
 * either may be NULL).  Reads the host mirror; no sync. */
kvc_status kvc_get_lengths(const kvc_ctx *ctx, int32_t *lengths, int32_t *prompt_lengths);

/* Dense copy of one layer for requests [req_begin, req_begin+req_count):
 *   k_out, v_out: device [req_count][num_kv_heads][cap][head_dim] dtype
 *   pos_out:      device [req_count][num_kv_heads][cap] int32
 * Slot j < min(length, cap) receives the row in slot j; the rest is zero
 * (pos -1).  Any output may be NULL. */
kvc_status kvc_gather_dense(kvc_ctx *ctx, int32_t layer, int32_t req_begin, int32_t req_count,
                            int32_t cap, void *k_out, void *v_out, int32_t *pos_out);

/* Failure-detection self-test (no counterpart in the pages).  Every wait of
 * the library's kernels on a device-side event is bounded; when the bound
 * runs out the kernel records a timeout in the status word and returns,
 * leaving the context usable, and the next synchronising call returns
 * KVC_ERR_DEVICE_TIMEOUT.  This call exercises that path: it enqueues a
 * one-thread kernel that waits, with a bound of limit_ms (1..2000), on an
 * mbarrier nothing arrives on, synchronises, and returns
 * KVC_ERR_DEVICE_TIMEOUT (status cleared) when detection works.  A device
 * error latched before the call is returned first, as itself. */
kvc_status kvc_check_wait_timeout(kvc_ctx *ctx, uint32_t limit_ms);

/* Waits for the stream and reports any latched device error (then clears it). */
kvc_status kvc_sync(kvc_ctx *ctx);

const char *kvc_status_string(kvc_status s);
const char *kvc_last_error(const kvc_ctx *ctx);

/* Allocation-free beacon score and top-K selection of S dense segments.
 * The pages have no counterpart: this entry point exists for callers that
 * cannot allocate device memory, such as code running while a CUDA graph is
 * captured (cudaMalloc is not allowed there), plug-ins confined to another
 * engine's fixed memory arena, or hosts with no device allocator, and which
 * therefore cannot give kvc_create a workspace.  It needs no context.
 *   keys:    device [S][L][head_dim] dtype, each segment's cached keys in
 *            position order (the prompt first).
 *   beacons: device [S][B][head_dim] dtype, each segment's beacon scoring copies.
 *   P, K:    protected prompt length and budget, shared by the S segments.
 *   kept_out:   device int32 [S][R], R = L if L <= K, else max(P, K): the kept
 *               slots of each segment, ascending (the prompt, then the best
 *               max(0, K-P) candidates by (score desc, slot asc)).
 *   scores_out: device float [S][L-P] or NULL; when the round evicts some but
 *               not all candidates it receives each candidate's score, else it
 *               is left untouched.
 *   cuda_stream: cudaStream_t on the inputs' device (NULL = legacy stream).
 * The scores and the selection are those of kvc_compress(KVC_SEL_BEACON)
 * for the same keys and beacons.  NaN: this call does not synchronise and
 * reports no KVC_ERR_NAN; a NaN score (one NaN key or beacon makes every
 * score of its segment NaN) ranks below every other score, ties among NaN
 * scores keep the lowest slots, and scores_out shows the NaN.  The kernels
 * run on the keys' device; the calling thread's current device is the same
 * after the call as before it.  Scratch: the scores pass between the two
 * kernels through a fixed array of 1,048,576 floats (4 MiB) in the library's
 * device memory, held on every GPU that loads the library until the process
 * exits; S*(L-P) above 1,048,576 is rejected with KVC_ERR_INVALID_ARG.  No
 * part of the array needs to start at zero: each call writes every score it
 * reads.  All calls on a device share that device's array, which keeps the
 * last call's contents, so calls that overlap on the same GPU (for example on
 * two streams) race on it: serialise them.  The first
 * call on a device looks up the array's device address (cudaGetSymbolAddress,
 * which may load the library's kernels); make that first call before any
 * stream capture.  The call allocates nothing: no cudaMalloc, cudaFree or
 * allocating library routine.  Limits: L <= 32768, B in [1, 256], head_dim 64
 * or 128.  Errors: KVC_ERR_INVALID_ARG (message in kvc_last_error(NULL)),
 * KVC_ERR_CUDA. */
kvc_status kvc_beacon_select_noalloc(const void *keys, const void *beacons, int32_t S, int32_t L,
                                     int32_t P, int32_t K, int32_t B, int32_t head_dim,
                                     int32_t dtype, int32_t *kept_out, float *scores_out,
                                     void *cuda_stream);

#ifdef __cplusplus
}
#endif

#endif /* KVC_H */
