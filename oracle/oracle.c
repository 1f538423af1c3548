/*
 * oracle.c -- plain, single-threaded CPU oracle for the decode-time KV-cache
 * eviction round (Random-Attention and BeaconKV selectors).
 *
 * TEST INFRASTRUCTURE.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline leg of bench.py may load this library.  The product path
 * (decode_kv_cache_paged_b200) never links, imports or calls it, and shares
 * no code, header, table or constant with it.
 *
 * Everything here is the plain definition written out: every score is
 * computed, candidates are fully sorted, the first M are kept and packed in
 * their original order.  Floating point is double.  There is no blocking,
 * fusion or reordering beyond what the definitions state.
 *
 * Sources (web pages; section names as printed on them):
 *  [RA]  "随机保留 KV Cache 竟不输精心设计的 eviction 策略？新研究重新审视推理
 *        中的显存压缩" (aiinking.com/article/67532), sections
 *        "长推理的显存瓶颈" (fixed budget K), "Random Attention：不判断重要性，
 *        只随机保留" (prompt protection, per-head random Top-K, geometric
 *        survival), "发现二" (all heads sharing one random set) and
 *        "发现四" (cache compaction needed by every method; the paged
 *        attention kernels every selector shares).
 *  [BX]  "BeaconKV: 用"信标查询"指导 KV cache 压缩 ..." explainer
 *        (papers.ananclaw.com/promo/explainers__2609-04971), §3.2 (nearest
 *        beacon assignment, periodic incremental beacon update).
 *  [BA]  BeaconKV abstract (chatpaper.ai): beacon queries are compact
 *        representatives of global query clusters.
 *  Philox4x64-10: Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as
 *        easy as 1, 2, 3", SC'11 (the Philox bijection and its key
 *        schedule).
 * Where the pages leave a step open, the reading used is the one stated in
 * the comment of the function concerned.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ */
/* Philox4x64-10 (Salmon et al. 2011).                                 */
/* ------------------------------------------------------------------ */

/* Multipliers and Weyl key increments as published for Philox4x64. */
#define ORC_PHILOX_M0 0xD2E7470EE14C6C93ULL
#define ORC_PHILOX_M1 0xCA5A826395121157ULL
#define ORC_PHILOX_W0 0x9E3779B97F4A7C15ULL /* golden ratio */
#define ORC_PHILOX_W1 0xBB67AE8584CAA73BULL /* sqrt(3) - 1   */

static void orc_mulhilo64(uint64_t a, uint64_t b, uint64_t *hi, uint64_t *lo) {
  unsigned __int128 p = (unsigned __int128)a * (unsigned __int128)b;
  *hi = (uint64_t)(p >> 64);
  *lo = (uint64_t)p;
}

/* One block of Philox4x64 with 10 rounds.  Round i (i = 0..9) uses the key
 * bumped i times by the Weyl increments.  Each round multiplies words 0 and 2
 * by the two multipliers; the new word 0 is hi(M1*x2) ^ x1 ^ k0, word 1 is
 * lo(M1*x2), word 2 is hi(M0*x0) ^ x3 ^ k1 and word 3 is lo(M0*x0). */
void orc_philox4x64_10(const uint64_t ctr[4], const uint64_t key[2], uint64_t out[4]) {
  uint64_t x0 = ctr[0], x1 = ctr[1], x2 = ctr[2], x3 = ctr[3];
  uint64_t k0 = key[0], k1 = key[1];
  for (int i = 0; i < 10; ++i) {
    if (i > 0) {
      k0 += ORC_PHILOX_W0;
      k1 += ORC_PHILOX_W1;
    }
    uint64_t hi0, lo0, hi1, lo1;
    orc_mulhilo64(ORC_PHILOX_M0, x0, &hi0, &lo0);
    orc_mulhilo64(ORC_PHILOX_M1, x2, &hi1, &lo1);
    uint64_t y0 = hi1 ^ x1 ^ k0;
    uint64_t y1 = lo1;
    uint64_t y2 = hi0 ^ x3 ^ k1;
    uint64_t y3 = lo0;
    x0 = y0;
    x1 = y1;
    x2 = y2;
    x3 = y3;
  }
  out[0] = x0;
  out[1] = x1;
  out[2] = x2;
  out[3] = x3;
}

/* Random-Attention score of one (request r, layer l, KV head h, original
 * position pos) in eviction round `round` [RA, "Random Attention：..."]:
 * counter = (pos, h, l, r), key = (seed, round); the score is the high 32
 * bits of output word 0.  The shared-across-heads variant [RA, "发现二"] uses
 * h = 2^64 - 1 so every head of (r, l) draws the same value.
 * Readings: the pages only say "random"; Philox is the generator, redrawn
 * every round (the geometric survival needs independent rounds), keyed by the
 * original absolute position so the shared variant stays aligned. */
uint32_t orc_random_score(uint64_t seed, uint64_t round, int64_t r, int64_t l, int64_t h,
                          int64_t pos, int32_t shared) {
  uint64_t ctr[4], key[2], out[4];
  ctr[0] = (uint64_t)pos;
  ctr[1] = shared ? ~(uint64_t)0 : (uint64_t)h;
  ctr[2] = (uint64_t)l;
  ctr[3] = (uint64_t)r;
  key[0] = seed;
  key[1] = round;
  orc_philox4x64_10(ctr, key, out);
  return (uint32_t)(out[0] >> 32);
}

/* Block-granular variant [RA, "发现二": retaining contiguous blocks of 1 to
 * 256 tokens instead of scattered ones]: every original position of a block
 * of `block` consecutive positions (block index pos / block) shares one draw,
 * so Top-K keeps whole blocks in order of their draw; ties, i.e. positions of
 * one block, go to the lower position, so at most one block is split.
 * Reading: blocks are aligned to multiples of `block` in original-position
 * space; block = 1 is the per-token score. */
uint32_t orc_random_score_block(uint64_t seed, uint64_t round, int64_t r, int64_t l, int64_t h,
                                int64_t pos, int32_t shared, int64_t block) {
  return orc_random_score(seed, round, r, l, h, pos / (block > 0 ? block : 1), shared);
}

/* ------------------------------------------------------------------ */
/* Retention rule [RA, "长推理的显存瓶颈" and "Random Attention：..."]. */
/* ------------------------------------------------------------------ */

/* L = cached length, P = protected prompt length, K = budget.
 *  - L <= K: nothing is evicted (no-op round for this segment).
 *  - otherwise the prompt [0, P) is always kept and the best
 *    M = max(0, K - P) generated positions are kept.
 * Reading where the pages are silent: if P > K the prompt still wins (it is
 * never evicted), zero generated positions stay and the segment is flagged
 * prompt-over-budget.
 * Outputs: *M_out generated kept, *R_out new length, *flags bit0 = no-op,
 * bit1 = prompt over budget.  Returns 0, or -1 on invalid sizes. */
int32_t orc_retention(int64_t L, int64_t P, int64_t K, int64_t *M_out, int64_t *R_out,
                      int32_t *flags) {
  if (L < 0 || P < 0 || K < 0 || P > L) return -1;
  *flags = 0;
  if (L <= K) {
    *M_out = L - P;
    *R_out = L;
    *flags |= 1;
    return 0;
  }
  int64_t M = K - P;
  if (M < 0) M = 0;
  if (P > K) *flags |= 2;
  *M_out = M;
  *R_out = P + M;
  return 0;
}

/* ------------------------------------------------------------------ */
/* Top-K selection by full sort [RA: "一次随机数生成和一次 Top-K"].       */
/* ------------------------------------------------------------------ */

typedef struct {
  double score;
  int64_t pos;  /* original position: the tie-breaker */
  int64_t slot; /* where the candidate sits in the cache */
} orc_cand;

/* Larger score first; equal scores go to the lower original position. */
static int orc_cmp_rank(const void *a, const void *b) {
  const orc_cand *x = (const orc_cand *)a, *y = (const orc_cand *)b;
  if (x->score > y->score) return -1;
  if (x->score < y->score) return 1;
  if (x->pos < y->pos) return -1;
  if (x->pos > y->pos) return 1;
  return 0;
}

static int orc_cmp_slot(const void *a, const void *b) {
  const orc_cand *x = (const orc_cand *)a, *y = (const orc_cand *)b;
  return (x->slot > y->slot) - (x->slot < y->slot);
}

/* Keeps the M best of N candidates by (score desc, pos asc), then writes the
 * kept slots in ascending slot order to kept_slots[0..M).  Returns M, or -1
 * on bad arguments / allocation failure. */
int64_t orc_select_topk(int64_t N, const double *score, const int64_t *pos, const int64_t *slot,
                        int64_t M, int64_t *kept_slots) {
  if (N < 0 || M < 0 || M > N) return -1;
  if (M == 0) return 0;
  orc_cand *c = (orc_cand *)malloc((size_t)N * sizeof(orc_cand));
  if (!c) return -1;
  for (int64_t j = 0; j < N; ++j) {
    c[j].score = score[j];
    c[j].pos = pos[j];
    c[j].slot = slot[j];
  }
  qsort(c, (size_t)N, sizeof(orc_cand), orc_cmp_rank);
  qsort(c, (size_t)M, sizeof(orc_cand), orc_cmp_slot);
  for (int64_t i = 0; i < M; ++i) kept_slots[i] = c[i].slot;
  free(c);
  return M;
}

/* ------------------------------------------------------------------ */
/* Order-preserving compaction [RA, "发现四": cache compaction].        */
/* ------------------------------------------------------------------ */

/* rows_in holds L rows of row_bytes bytes.  rows_out receives the prompt
 * rows [0, P) unchanged, then the M kept rows in ascending slot order. */
void orc_compact_rows(int64_t P, int64_t row_bytes, const uint8_t *rows_in, int64_t M,
                      const int64_t *kept_slots, uint8_t *rows_out) {
  memcpy(rows_out, rows_in, (size_t)(P * row_bytes));
  for (int64_t i = 0; i < M; ++i)
    memcpy(rows_out + (P + i) * row_bytes, rows_in + kept_slots[i] * row_bytes,
           (size_t)row_bytes);
}

/* ------------------------------------------------------------------ */
/* One Random-Attention round on one segment (r, l, h).                */
/* ------------------------------------------------------------------ */

/* pos_in[0..L) is the original position held by each slot.  Computes the
 * retention rule, scores every generated candidate, selects by full sort and
 * writes the kept slots (prompt slots first, then the kept generated slots,
 * ascending) to kept_slots[0..R) and the new position map to pos_out[0..R).
 * Returns R, or -1 on error. */
int64_t orc_random_round_segment(uint64_t seed, uint64_t round, int64_t r, int64_t l, int64_t h,
                                 int32_t shared, int64_t L, int64_t P, int64_t K,
                                 const int32_t *pos_in, int32_t *pos_out, int64_t *kept_slots) {
  int64_t M, R;
  int32_t flags;
  if (orc_retention(L, P, K, &M, &R, &flags) != 0) return -1;
  for (int64_t s = 0; s < P; ++s) kept_slots[s] = s;
  if (flags & 1) {
    for (int64_t s = P; s < L; ++s) kept_slots[s] = s;
  } else if (M > 0) {
    int64_t N = L - P;
    double *score = (double *)malloc((size_t)N * sizeof(double));
    int64_t *pos = (int64_t *)malloc((size_t)N * sizeof(int64_t));
    int64_t *slot = (int64_t *)malloc((size_t)N * sizeof(int64_t));
    if (!score || !pos || !slot) {
      free(score);
      free(pos);
      free(slot);
      return -1;
    }
    for (int64_t j = 0; j < N; ++j) {
      slot[j] = P + j;
      pos[j] = pos_in[P + j];
      score[j] = (double)orc_random_score(seed, round, r, l, h, pos[j], shared);
    }
    int64_t got = orc_select_topk(N, score, pos, slot, M, kept_slots + P);
    free(score);
    free(pos);
    free(slot);
    if (got != M) return -1;
  }
  for (int64_t i = 0; i < R; ++i) pos_out[i] = pos_in[kept_slots[i]];
  return R;
}

/* Hole-filling compaction (the build's option; the pages only require
 * "cache compaction"): the kept slots below the new length R stay where they
 * are, and the kept slots at or above R fill the evicted slots below R, the
 * i-th such hole (ascending) taking the i-th such survivor (ascending).
 * kept_slots[0..R) ascending on input; slot_out[0..R) receives, for each new
 * slot s, the old slot whose row it holds.  Returns the number of moves. */
int64_t orc_hole_fill(int64_t R, const int64_t *kept_slots, int64_t *slot_out) {
  int64_t n_hole = 0, n_move = 0, next_hole_search = 0;
  for (int64_t s = 0; s < R; ++s) slot_out[s] = -1;
  for (int64_t i = 0; i < R; ++i)
    if (kept_slots[i] < R) slot_out[kept_slots[i]] = kept_slots[i];
  for (int64_t i = 0; i < R; ++i) {
    if (kept_slots[i] < R) continue;
    while (next_hole_search < R && slot_out[next_hole_search] >= 0) ++next_hole_search;
    slot_out[next_hole_search] = kept_slots[i];
    ++n_move;
  }
  for (int64_t s = 0; s < R; ++s)
    if (slot_out[s] < 0) ++n_hole;
  return n_hole == 0 ? n_move : -1;
}

/* One random round with the options of the extended round: protection of
 * the first `protect` positions only (sink tokens) instead of the whole
 * prompt, block-granular draws, hole-filling compaction.  pos_in[0..L);
 * writes pos_out[0..R) and returns R (or -1). */
int64_t orc_random_round_segment_ex(uint64_t seed, uint64_t round, int64_t r, int64_t l, int64_t h,
                                    int32_t shared, int64_t block, int32_t hole_fill, int64_t L,
                                    int64_t P, int64_t K, const int32_t *pos_in, int32_t *pos_out) {
  int64_t M, R;
  int32_t flags;
  if (orc_retention(L, P, K, &M, &R, &flags) != 0) return -1;
  int64_t *kept = (int64_t *)malloc((size_t)(L > 0 ? L : 1) * sizeof(int64_t));
  if (!kept) return -1;
  for (int64_t s = 0; s < P; ++s) kept[s] = s;
  if (flags & 1) {
    for (int64_t s = P; s < L; ++s) kept[s] = s;
  } else if (M > 0) {
    int64_t N = L - P;
    double *score = (double *)malloc((size_t)N * sizeof(double));
    int64_t *pos = (int64_t *)malloc((size_t)N * sizeof(int64_t));
    int64_t *slot = (int64_t *)malloc((size_t)N * sizeof(int64_t));
    if (!score || !pos || !slot) {
      free(score);
      free(pos);
      free(slot);
      free(kept);
      return -1;
    }
    for (int64_t j = 0; j < N; ++j) {
      slot[j] = P + j;
      pos[j] = pos_in[P + j];
      score[j] = (double)orc_random_score_block(seed, round, r, l, h, pos[j], shared, block);
    }
    int64_t got = orc_select_topk(N, score, pos, slot, M, kept + P);
    free(score);
    free(pos);
    free(slot);
    if (got != M) {
      free(kept);
      return -1;
    }
  }
  if (hole_fill && !(flags & 1)) {
    int64_t *src = (int64_t *)malloc((size_t)(R > 0 ? R : 1) * sizeof(int64_t));
    if (!src || orc_hole_fill(R, kept, src) < 0) {
      free(src);
      free(kept);
      return -1;
    }
    for (int64_t i = 0; i < R; ++i) pos_out[i] = pos_in[src[i]];
    free(src);
  } else {
    for (int64_t i = 0; i < R; ++i) pos_out[i] = pos_in[kept[i]];
  }
  free(kept);
  return R;
}

/* Batched form of orc_random_round_segment over n segments, for speed of the
 * test harness only (each segment is still processed by the plain routine).
 * rlh[3*s..] = (r, l, h); lpk[3*s..] = (L, P, K); pos_in/pos_out are
 * [n][stride] int32.  R_out[s] receives the new length.  Returns 0 or the
 * 1-based index of the first failing segment. */
int64_t orc_random_round_batch(uint64_t seed, uint64_t round, int32_t shared, int64_t n,
                               const int64_t *rlh, const int64_t *lpk, int64_t stride,
                               const int32_t *pos_in, int32_t *pos_out, int64_t *R_out) {
  int64_t *kept = (int64_t *)malloc((size_t)stride * sizeof(int64_t));
  if (!kept) return 1;
  for (int64_t s = 0; s < n; ++s) {
    int64_t R = orc_random_round_segment(seed, round, rlh[3 * s], rlh[3 * s + 1], rlh[3 * s + 2],
                                         shared, lpk[3 * s], lpk[3 * s + 1], lpk[3 * s + 2],
                                         pos_in + s * stride, pos_out + s * stride, kept);
    if (R < 0) {
      free(kept);
      return s + 1;
    }
    R_out[s] = R;
    for (int64_t i = R; i < stride; ++i) pos_out[s * stride + i] = -1;
  }
  free(kept);
  return 0;
}

/* Batched orc_random_round_segment_ex; lpk[3*s..] = (L, P, K) with P the
 * protected length actually used (the sink count under sink protection). */
int64_t orc_random_round_batch_ex(uint64_t seed, uint64_t round, int32_t shared, int64_t block,
                                  int32_t hole_fill, int64_t n, const int64_t *rlh,
                                  const int64_t *lpk, int64_t stride, const int32_t *pos_in,
                                  int32_t *pos_out, int64_t *R_out) {
  for (int64_t s = 0; s < n; ++s) {
    int64_t R = orc_random_round_segment_ex(seed, round, rlh[3 * s], rlh[3 * s + 1], rlh[3 * s + 2],
                                            shared, block, hole_fill, lpk[3 * s], lpk[3 * s + 1],
                                            lpk[3 * s + 2], pos_in + s * stride, pos_out + s * stride);
    if (R < 0) return s + 1;
    R_out[s] = R;
    for (int64_t i = R; i < stride; ++i) pos_out[s * stride + i] = -1;
  }
  return 0;
}

/* ------------------------------------------------------------------ */
/* bf16 rounding (round to nearest, ties to even, 8 significant bits). */
/* ------------------------------------------------------------------ */

/* The beacon scoring copy is the beacon rounded once to the cache dtype.
 * bfloat16 keeps 8 significant bits (1 implicit + 7 stored) and the fp32
 * exponent range; values here stay in the normal range. */
double orc_round_bf16(double x) {
  if (x == 0.0 || isnan(x) || isinf(x)) return x;
  int e;
  double m = frexp(x, &e);          /* x = m * 2^e, 0.5 <= |m| < 1 */
  double q = nearbyint(ldexp(m, 8)); /* default mode: nearest, ties to even */
  return ldexp(q, e - 8);
}

/* ------------------------------------------------------------------ */
/* BeaconKV beacon maintenance [BX §3.2; BA].                          */
/* ------------------------------------------------------------------ */

/* One periodic update of the B beacons of one segment from n_pts points
 * (the decode queries since the previous update, already ordered by
 * (step, query head) and with project() = identity).
 *  - init != 0 (first update of the segment): beacon i starts as point
 *    floor(i * n_pts / B) with count 0; n_pts < B is an error.
 *  - assignment: every point goes to the beacon with the smallest squared
 *    Euclidean distance, computed against the beacons as they were before
 *    this update; ties go to the lowest beacon index.  If assign_override
 *    is given, it is used instead (staged parity).
 *  - update: c_i <- (n_i c_i + sum of assigned points) / (n_i + m_i),
 *    n_i <- n_i + m_i; beacons with no assigned point are unchanged.
 * Readings: the explainer's pseudocode names init_beacons, nearest_neighbor
 * and periodically_update_beacons without defining them; the rules above are
 * the plainest ones consistent with "incremental clustering" and with a
 * beacon being a compact representative of its cluster.
 * Returns 0, or -1 (n_pts < B on init, bad override, allocation failure). */
int32_t orc_beacon_update(int64_t n_pts, int64_t B, int64_t d, const double *pts,
                          double *beacons, int64_t *counts, int32_t init,
                          const int32_t *assign_override, int32_t *assign_out) {
  if (B <= 0 || d <= 0 || n_pts < 0) return -1;
  if (init) {
    if (n_pts < B) return -1;
    for (int64_t i = 0; i < B; ++i) {
      int64_t src = (i * n_pts) / B;
      memcpy(beacons + i * d, pts + src * d, (size_t)d * sizeof(double));
      counts[i] = 0;
    }
  }
  for (int64_t p = 0; p < n_pts; ++p) {
    if (assign_override) {
      if (assign_override[p] < 0 || assign_override[p] >= B) return -1;
      assign_out[p] = assign_override[p];
      continue;
    }
    int64_t best = 0;
    double best_d = INFINITY;
    for (int64_t i = 0; i < B; ++i) {
      double dist = 0.0;
      for (int64_t k = 0; k < d; ++k) {
        double diff = pts[p * d + k] - beacons[i * d + k];
        dist += diff * diff;
      }
      if (dist < best_d) {
        best_d = dist;
        best = i;
      }
    }
    assign_out[p] = (int32_t)best;
  }
  double *sum = (double *)calloc((size_t)(B * d), sizeof(double));
  int64_t *m = (int64_t *)calloc((size_t)B, sizeof(int64_t));
  if (!sum || !m) {
    free(sum);
    free(m);
    return -1;
  }
  for (int64_t p = 0; p < n_pts; ++p) {
    int64_t i = assign_out[p];
    m[i] += 1;
    for (int64_t k = 0; k < d; ++k) sum[i * d + k] += pts[p * d + k];
  }
  for (int64_t i = 0; i < B; ++i) {
    if (m[i] == 0) continue;
    double n = (double)counts[i];
    for (int64_t k = 0; k < d; ++k)
      beacons[i * d + k] = (n * beacons[i * d + k] + sum[i * d + k]) / (n + (double)m[i]);
    counts[i] += m[i];
  }
  free(sum);
  free(m);
  return 0;
}

/* ------------------------------------------------------------------ */
/* BeaconKV key score (the build's own definition; the pages leave the  */
/* importance rule open, [BX §3.2 "mark_important"]).                  */
/* ------------------------------------------------------------------ */

/* keys [L][d], beacons [B][d] (the scoring copies).  For every beacon b and
 * every cached key j < L (prompt included):
 *     z_bj  = (c_b . k_j) / sqrt(d)
 *     lse_b = log sum_j exp(z_bj)        (computed as max + log sum exp(z - max))
 * and for every generated position j in [P, L):
 *     score_j = max_b exp(z_bj - lse_b)
 * i.e. the largest share of attention mass any beacon puts on key j.
 * score_out[0..L-P), lse_out[0..B) (nullable).  Returns 0 or -1. */
int32_t orc_beacon_score(int64_t L, int64_t P, int64_t B, int64_t d, const double *keys,
                         const double *beacons, double *score_out, double *lse_out) {
  if (L <= 0 || P < 0 || P > L || B <= 0 || d <= 0) return -1;
  double *z = (double *)malloc((size_t)(B * L) * sizeof(double));
  double *lse = (double *)malloc((size_t)B * sizeof(double));
  if (!z || !lse) {
    free(z);
    free(lse);
    return -1;
  }
  double inv_sqrt_d = 1.0 / sqrt((double)d);
  for (int64_t b = 0; b < B; ++b) {
    for (int64_t j = 0; j < L; ++j) {
      double dot = 0.0;
      for (int64_t k = 0; k < d; ++k) dot += beacons[b * d + k] * keys[j * d + k];
      z[b * L + j] = dot * inv_sqrt_d;
    }
  }
  for (int64_t b = 0; b < B; ++b) {
    double mx = -INFINITY;
    for (int64_t j = 0; j < L; ++j)
      if (z[b * L + j] > mx) mx = z[b * L + j];
    double s = 0.0;
    for (int64_t j = 0; j < L; ++j) s += exp(z[b * L + j] - mx);
    lse[b] = mx + log(s);
  }
  for (int64_t j = P; j < L; ++j) {
    double best = -INFINITY;
    for (int64_t b = 0; b < B; ++b) {
      double p = exp(z[b * L + j] - lse[b]);
      if (p > best) best = p;
    }
    score_out[j - P] = best;
  }
  if (lse_out)
    for (int64_t b = 0; b < B; ++b) lse_out[b] = lse[b];
  free(z);
  free(lse);
  return 0;
}

/* ------------------------------------------------------------------ */
/* BeaconKV cluster-level trigger (the build's reading of [BX] §3.2:   */
/* "query -> cluster -> KV" and mark_important(cluster_id, KV)).       */
/* ------------------------------------------------------------------ */

/* Each query of the latest update window lands in one cluster (its nearest
 * beacon); the trigger raises the importance of the keys that cluster's
 * beacon attends to.  With m_b the number of window queries assigned to
 * beacon b and z_bj, lse_b as in orc_beacon_score:
 *     importance_j = sum_b (m_b / sum_b' m_b') * exp(z_bj - lse_b),  j in [P, L)
 * i.e. the attention mass key j receives when every window query is replaced
 * by its cluster's beacon.  All m_b = 0 gives importance 0 everywhere.
 * keys [L][d], beacons [B][d], trig [B] (counts, >= 0); score_out[0..L-P). */
int32_t orc_beacon_trigger_score(int64_t L, int64_t P, int64_t B, int64_t d, const double *keys,
                                 const double *beacons, const double *trig, double *score_out) {
  if (L <= 0 || P < 0 || P > L || B <= 0 || d <= 0) return -1;
  double total = 0.0;
  for (int64_t b = 0; b < B; ++b) {
    if (trig[b] < 0) return -1;
    total += trig[b];
  }
  double *z = (double *)malloc((size_t)(B * L) * sizeof(double));
  double *lse = (double *)malloc((size_t)B * sizeof(double));
  if (!z || !lse) {
    free(z);
    free(lse);
    return -1;
  }
  const double rsqrt_d = 1.0 / sqrt((double)d);
  for (int64_t b = 0; b < B; ++b)
    for (int64_t j = 0; j < L; ++j) {
      double dot = 0.0;
      for (int64_t k = 0; k < d; ++k) dot += beacons[b * d + k] * keys[j * d + k];
      z[b * L + j] = dot * rsqrt_d;
    }
  for (int64_t b = 0; b < B; ++b) {
    double mx = -INFINITY;
    for (int64_t j = 0; j < L; ++j)
      if (z[b * L + j] > mx) mx = z[b * L + j];
    double sum = 0.0;
    for (int64_t j = 0; j < L; ++j) sum += exp(z[b * L + j] - mx);
    lse[b] = mx + log(sum);
  }
  for (int64_t j = P; j < L; ++j) {
    double acc = 0.0;
    if (total > 0)
      for (int64_t b = 0; b < B; ++b) acc += (trig[b] / total) * exp(z[b * L + j] - lse[b]);
    score_out[j - P] = acc;
  }
  free(z);
  free(lse);
  return 0;
}

/* ------------------------------------------------------------------ */
/* Decode attention over a request's cached rows [RA, "发现四": every     */
/* selector shares the same paged attention kernels; what they attend  */
/* to is the compacted cache].                                         */
/* ------------------------------------------------------------------ */

/* Scaled dot-product attention of one decode query over L cached rows:
 *     s_j = scale * (q . k_j),  j < L
 *     out = sum_j exp(s_j - lse) v_j,  lse = log sum_j exp(s_j)
 * (lse computed as max + log sum exp(s - max)).  q [d], k [L][d],
 * v [L][d]; out [d].  L = 0 gives out = 0 and lse = -inf. */
void orc_decode_attention(int64_t L, int64_t d, const double *q, const double *k, const double *v,
                          double scale, double *out, double *lse_out) {
  for (int64_t c = 0; c < d; ++c) out[c] = 0.0;
  if (L <= 0) {
    *lse_out = -INFINITY;
    return;
  }
  double *s = (double *)malloc((size_t)L * sizeof(double));
  if (!s) {
    *lse_out = NAN;
    return;
  }
  double mx = -INFINITY;
  for (int64_t j = 0; j < L; ++j) {
    double dot = 0.0;
    for (int64_t c = 0; c < d; ++c) dot += q[c] * k[j * d + c];
    s[j] = scale * dot;
    if (s[j] > mx) mx = s[j];
  }
  double sum = 0.0;
  for (int64_t j = 0; j < L; ++j) sum += exp(s[j] - mx);
  double lse = mx + log(sum);
  for (int64_t j = 0; j < L; ++j) {
    double w = exp(s[j] - lse);
    for (int64_t c = 0; c < d; ++c) out[c] += w * v[j * d + c];
  }
  *lse_out = lse;
  free(s);
}

/* Grouped-query form for one (request, layer): Hq query heads over Hkv
 * key/value heads, G = Hq / Hkv consecutive query heads per KV head (query
 * head hq reads KV head hq / G, the grouping the beacon update uses for its
 * points).  q [Hq][d], k and v [Hkv][L][d], out [Hq][d], lse [Hq]. */
void orc_decode_attention_gqa(int64_t Hq, int64_t Hkv, int64_t L, int64_t d, const double *q,
                              const double *k, const double *v, double scale, double *out,
                              double *lse) {
  int64_t G = Hq / Hkv;
  for (int64_t hq = 0; hq < Hq; ++hq) {
    int64_t h = hq / G;
    orc_decode_attention(L, d, q + hq * d, k + h * L * d, v + h * L * d, scale, out + hq * d,
                         lse + hq);
  }
}
