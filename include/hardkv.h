/*
 * hardkv.h — C ABI of the HARD-KV decode-step library (libhardkv.so, sm_100a).
 *
 * HARD-KV ("HARD-KV: Head-Adaptive Regularization for Decoding-time KV
 * Compression", technical summary sec. 2 "Methodology") keeps each attention
 * layer's KV cache in three tiers per (sequence b, KV head h):
 *   Dense     positions [d_lo, len)   most recent tokens, contiguous (Tier 1)
 *   Sparse    positions [s_lo, d_lo)  aged-out tokens; calibrated top-p keeps a
 *                                     head-adaptive subset (Tier 2)
 *   Condensed C slots                 oldest tokens, evicted or merged (Tier 3)
 * and runs every decode step through four stages (sec. 2.A): (1) linear append
 * to Dense; (2) Logits Calibration + top-p -> selection masks; (3) Index
 * Regularization: kept rows rewritten into a contiguous fixed-capacity layout
 * (sec. 2.C Rewrite Cache, Flatten Index to the maximum length) or only indexed
 * (Sparse Loading), per head by a layout policy; the index also in its sum form on
 * demand, the rewritten rows optionally in a shared pool of 16-row blocks (sec. 2.C
 * head-wise block manager); (4) eviction or weighted merge of the oldest block; then
 * decode attention over the tiers.
 *
 * Conventions for every entry point:
 *  - Pointers marked "device" are CUDA device pointers owned by the caller; the
 *    library allocates nothing, never synchronises, keeps no state between calls
 *    and only enqueues work on `stream`. Every entry point can be captured in a
 *    CUDA graph (shapes come from the descriptor, tier boundaries live on the
 *    device).
 *  - Every device pointer must be 16-byte aligned; head_dim * element size is a
 *    multiple of 16 by construction (head_dim 64 or 128).
 *  - Element type of K, V, q, k_new, v_new is `desc->dtype` (IEEE float32 or
 *    bfloat16). Attention output is float32.
 *  - Layouts are row-major, innermost dimension last:
 *      ring K/V  [B, H, R, d]   position p of unit (b,h) lives in row p mod R
 *      compact   [B, H, Cap, d] slots 0..n-1 valid (or pool blocks: hardkv_cache)
 *      condensed [B, H, C, d]   weights [B, H, C] float32 (0 = empty slot)
 *      q [B, Hq, d]; query head qh belongs to KV head qh / (Hq / H)
 *  - Return value: HARDKV_OK (0) or a negative HARDKV_E* code. Arguments are
 *    validated before anything is enqueued; on an error nothing is enqueued.
 *    HARDKV_ECUDA means a launch failed; hardkv_strerror() then names the CUDA
 *    error. Anomalies found on the device (inconsistent boundaries, capacity
 *    clamps, merge near-ties) are recorded in the caller's status words, never
 *    trapped.
 */
#ifndef HARDKV_H
#define HARDKV_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define HARDKV_OK 0
#define HARDKV_EINVAL (-1)   /* bad descriptor field, NULL pointer or p outside (0,1] */
#define HARDKV_EALIGN (-2)   /* a pointer is not 16-byte aligned */
#define HARDKV_EDTYPE (-3)   /* dtype not HARDKV_F32 / HARDKV_BF16 */
#define HARDKV_ECAP   (-4)   /* capacity rule broken (Cap < 1, R too small, R % 64) */
#define HARDKV_ECUDA  (-5)   /* a CUDA launch or copy failed */
#define HARDKV_ESCRATCH (-6) /* too large for the built-in scratch of the allocation-free
                                entry point (hardkv_score_calibrate_topp_static) */

enum { HARDKV_F32 = 0, HARDKV_BF16 = 1 };
enum { HARDKV_EVICT = 0, HARDKV_MERGE = 1 };
/* Which sequences reselect their Sparse subset in a call:
 * ALL   = every sequence;
 * MOVED = only sequences whose last hardkv_append moved a block (moved[b] != 0),
 *         i.e. each sequence reselects once per block of decode steps. */
enum { HARDKV_SELECT_ALL = 0, HARDKV_SELECT_MOVED = 1 };
/* Selection rule of a reselecting unit:
 * TOPP = calibrated top-p (the method: a head-adaptive budget);
 * TOPK = the k highest scores of every head (the fixed-budget selection the method is
 *        compared with; sec. 2.B "Top-k vs. Top-p", sec. 4). */
enum { HARDKV_RULE_TOPP = 0, HARDKV_RULE_TOPK = 1 };
/* Logits Calibration temperature:
 * TAU     = the caller's tau[b,h] (NULL: 1);
 * ENTROPY = per (b,h), the tau in [1/64, 64] for which the entropy of softmax(s / tau)
 *           over the candidates equals the mean entropy of the raw attention
 *           softmax_j(q_g . k_j / sqrt(d)) of the head's queries g over the same
 *           candidates (sec. 2.A Tier 2, a budget "based on the attention entropy";
 *           sec. 2.B; sec. 3, distribution alterations mapped onto the raw attention). */
enum { HARDKV_CAL_TAU = 0, HARDKV_CAL_ENTROPY = 1 };
/* Index Regularization layout of a reselected (b,h) (sec. 2.C):
 * REWRITE     = Rewrite Cache: the kept K/V rows are copied into the compact layout
 *               and later steps read them there (contiguous);
 * SPARSE_LOAD = Sparse Loading: only the flattened index (sp_idx, n_kept) is written;
 *               attention reads the kept rows in place from the ring through it;
 * MTI         = per (b,h), rewrite or load by the Memory-Time Integral rule of
 *               hardkv_layout_policy. */
enum { HARDKV_LAYOUT_REWRITE = 0, HARDKV_LAYOUT_SPARSE_LOAD = 1, HARDKV_LAYOUT_MTI = 2 };

/* Layout policy of the regularization (sec. 2.C "trade-off": the one-off rewrite cost
 * against the per-step decode gain, with budget thresholds L_lower and L_upper).
 * Under HARDKV_LAYOUT_MTI a reselected (b,h) keeping n rows is rewritten iff
 *   n > l_upper, or l_lower <= n <= l_upper and 1 < reuse_steps * gather_surcharge,
 * i.e. when writing the rows once costs less than reading them scattered in each of
 * the reuse_steps later steps that keep this selection (a contiguous read costs 1 per
 * byte, a scattered one 1 + gather_surcharge, a write 1). */
typedef struct {
  int32_t mode;             /* HARDKV_LAYOUT_* */
  int32_t reuse_steps;      /* later steps reading this selection; < 0: derived from the
                               select mode (ALL: 0, the next step reselects; MOVED:
                               block - 1, the selection lives until the next block move) */
  int32_t l_lower, l_upper; /* budget thresholds (rows) */
  float gather_surcharge;   /* > 0: extra cost per byte of a scattered row read */
} hardkv_layout_policy;

/* Device status words (caller-allocated uint32[HARDKV_STATUS_WORDS], zeroed by the
 * caller when it wants to start counting). */
#define HARDKV_STATUS_WORDS 8
enum {
  HARDKV_ST_FLAGS = 0,      /* OR of HARDKV_DEV_* bits */
  HARDKV_ST_CLAMPS = 1,     /* selections whose top-p count exceeded Cap */
  HARDKV_ST_NEAR_TIES = 2,  /* merges whose best two cosines differ by <= 1e-6 */
  HARDKV_ST_MERGED = 3,     /* tokens merged into the Condensed tier */
  HARDKV_ST_MOVES = 4,      /* block moves (one per sequence and move) */
  HARDKV_ST_SELECTIONS = 5  /* (sequence, head) top-p selections performed */
};
#define HARDKV_DEV_RING_OVERFLOW 1u  /* append would overwrite a live ring row: skipped */
#define HARDKV_DEV_BAD_BOUNDS    2u  /* s_lo <= d_lo <= len broken or span > R: unit skipped */
#define HARDKV_DEV_SEGMENTS      4u  /* attention partition had to drop a segment */
#define HARDKV_DEV_WAIT_TIMEOUT  8u  /* a pipeline wait hit its iteration limit */
#define HARDKV_DEV_SELECT       16u  /* top-p found no cut (inconsistent input): unit kept all */
#define HARDKV_DEV_POOL_SHORT   32u  /* paged compact tier: a rewritten selection got fewer
                                        blocks than it needed and kept its first rows only */
#define HARDKV_DEV_CHECK        64u  /* bounds-checked build (libhardkv_checked.so) only: an
                                        index was out of range; that access was skipped */

/* Rows per block of the paged compact tier (hardkv_cache::k_pool). */
#define HARDKV_PAGE_ROWS 16
/* Words of hardkv_cache::pool_ctl. */
enum { HARDKV_POOL_FREE = 0, HARDKV_POOL_RETURNED = 1, HARDKV_POOL_CTL_WORDS = 4 };

/* Static shape of one attention layer's cascade cache. */
typedef struct {
  int32_t batch;            /* B: sequences */
  int32_t n_q_heads;        /* Hq: query heads; Hq % H == 0, G = Hq / H in 1..16 */
  int32_t n_kv_heads;       /* H: KV heads */
  int32_t head_dim;         /* d: 64 or 128 */
  int32_t block;            /* tokens per block moved between tiers, 1..64 */
  int32_t dense_window;     /* W: Dense tier holds W .. W+block-1 tokens */
  int32_t condensed_slots;  /* C: Condensed slots per (b,h), >= 1 (<= 2048 for MERGE) */
  int32_t n_sink;           /* slots [0, n_sink) are pinned (never merged into) */
  int32_t sparse_cap;       /* Cap: compact rows per (b,h), >= 1 */
  int32_t ring_rows;        /* R: raw rows per (b,h); multiple of 64, <= 262144; the
                               live span [s_lo, len) must stay <= R
                               (R >= Sparse + W + block) */
  int32_t dtype;            /* HARDKV_F32 or HARDKV_BF16 */
  int32_t condense_mode;    /* HARDKV_EVICT or HARDKV_MERGE */
} hardkv_desc;

/* The cache state: all device pointers, caller-owned. */
typedef struct {
  void *k_ring, *v_ring;    /* [B,H,R,d] raw rows (Dense + Sparse candidates) */
  int32_t *len;             /* [B] tokens so far (positions 0..len-1) */
  int32_t *d_lo;            /* [B] first Dense position */
  int32_t *s_lo;            /* [B] first Sparse position (positions < s_lo are condensed) */
  int32_t *moved;           /* [B] 1 if the last append moved a block, else 0 */
  void *k_sp, *v_sp;        /* [B,H,Cap,d] compact (regularized) kept rows */
  int32_t *sp_idx;          /* [B,H,Cap] position of each compact slot, -1 = pad */
  int32_t *n_kept;          /* [B,H] compact slots in use */
  int32_t *sp_mode;         /* [B,H] layout of the unit's current selection: 1 = its rows
                               were rewritten into k_sp / v_sp, 0 = they are loaded in
                               place from the ring through sp_idx */
  void *k_cd, *v_cd;        /* [B,H,C,d] Condensed slots */
  float *w_cd;              /* [B,H,C] Condensed weights (tokens merged in), 0 = empty */
  uint32_t *status;         /* [HARDKV_STATUS_WORDS] device counters and flags */
  /* Paged compact tier: the head-wise block manager (sec. 2.C "Metadati": fine-grained,
   * head-adaptive allocation with static shapes and persistent pointers). k_pool NULL:
   * compact rows live in k_sp / v_sp ([B,H,Cap,d], Cap rows reserved per head). Otherwise
   * k_sp / v_sp are unused (may be NULL) and compact slot j of (b,h) is row
   *   blk_tab[(b*H + h) * tab_blocks + j / HARDKV_PAGE_ROWS] * HARDKV_PAGE_ROWS
   *     + j % HARDKV_PAGE_ROWS
   * of k_pool / v_pool, with tab_blocks = ceil(Cap / HARDKV_PAGE_ROWS): each head holds
   * only the blocks its current selection needs, from one pool shared by all heads.
   * A head that reselects with the Rewrite Cache layout and keeps n rows ends with
   * ceil(n / HARDKV_PAGE_ROWS) blocks (a Sparse-Loading head with none): it keeps its
   * first blocks, returns the rest to ret_list and takes what it lacks from the top of
   * free_list. Returned blocks join free_list at the start of the next step (in the
   * append kernel, or before a standalone regularization). If free_list runs short the
   * head keeps the rows its blocks hold, in position order, and HARDKV_DEV_POOL_SHORT
   * is raised. The caller sets up free_list = {0, 1, ..., pool_blocks-1},
   * pool_ctl = {pool_blocks, 0, 0, 0} and blk_cnt = 0 once; everything after that is
   * kept on the device. */
  void *k_pool, *v_pool;    /* [pool_blocks, HARDKV_PAGE_ROWS, d] or NULL */
  int32_t *blk_tab;         /* [B, H, tab_blocks] block ids of each head's compact slots */
  int32_t *blk_cnt;         /* [B, H] blocks each head holds */
  int32_t *free_list;       /* [pool_blocks] free block ids, [0, pool_ctl[FREE]) valid */
  int32_t *ret_list;        /* [pool_blocks] block ids returned since the last merge */
  int32_t *pool_ctl;        /* [HARDKV_POOL_CTL_WORDS] free count, returned count */
  int64_t pool_blocks;      /* blocks in the pool (ignored when k_pool is NULL) */
} hardkv_cache;

/* Arguments of one fused decode step. */
typedef struct {
  const void *q;            /* [B,Hq,d] this step's queries */
  const void *k_new;        /* [B,H,d] this step's key */
  const void *v_new;        /* [B,H,d] this step's value */
  const float *tau;         /* [B,H] calibration temperatures (device), or NULL = 1 */
  float p;                  /* top-p mass, 0 < p <= 1 (p = 1 keeps every candidate) */
  int32_t select_mode;      /* HARDKV_SELECT_ALL or HARDKV_SELECT_MOVED */
  uint32_t *mask;           /* [B,H,mask_words] selection masks out (device), or NULL */
  float *out;               /* [B,Hq,d] attention output */
  cudaEvent_t *stage_events;/* NULL, or HARDKV_STEP_EVENTS events recorded before the
                               first stage and after each stage (capture-safe) */
  int32_t rule;             /* HARDKV_RULE_TOPP (0, default) or HARDKV_RULE_TOPK */
  int32_t top_k;            /* RULE_TOPK: kept count per (b,h), 1..Cap (p is ignored) */
  int32_t calibration;      /* HARDKV_CAL_TAU (0, default) or HARDKV_CAL_ENTROPY (tau is
                               then ignored) */
  float *tau_out;           /* [B,H] (device) or NULL: the temperature each reselecting
                               unit used (1 under RULE_TOPK) */
  const hardkv_layout_policy *layout;  /* host struct, or NULL = HARDKV_LAYOUT_REWRITE */
} hardkv_step_args;
#define HARDKV_STEP_EVENTS 6  /* start, append, condense, score, topp, attend */

/* Bytes of scratch the library needs for this descriptor (caller allocates; the
 * content need not be initialised and is not read across calls except as noted). */
size_t hardkv_workspace_bytes(const hardkv_desc *desc);

/* uint32 words per (b,h) in a selection mask: bit j of unit (b,h) = Sparse
 * candidate j, i.e. position s_lo[b] + j. */
int32_t hardkv_mask_words(const hardkv_desc *desc);

/* Check a descriptor alone. Returns HARDKV_OK or the error code the entry points
 * would return. Pure host code: no CUDA call. */
int hardkv_validate(const hardkv_desc *desc);

/* Stage 1 (sec. 2.A stage (1), "linear append to the Dense cache").
 * For each sequence b: writes k_new[b,h], v_new[b,h] (device, [B,H,d]) to ring row
 * len[b] mod R, then len[b] += 1. If now len - d_lo >= W + block, one block moves
 * Dense->Sparse (d_lo += block) and the oldest Sparse block leaves for the Condensed
 * tier (s_lo += block); moved[b] records whether that happened. If the write would
 * overrun the ring (len - s_lo >= R) the sequence is skipped and
 * HARDKV_DEV_RING_OVERFLOW is raised. */
int hardkv_append(const hardkv_desc *desc, const hardkv_cache *cache,
                  const void *k_new, const void *v_new, void *ws, cudaStream_t stream);

/* Stage 4 (sec. 2.A Tier 3, "eviction or weighted merge"). For each sequence with
 * moved[b] != 0, the block of positions [s_lo - block, s_lo) that just left the
 * Sparse tier is, per KV head: EVICT — dropped (nothing to do); MERGE — folded token
 * by token (position order) into the Condensed slot s >= n_sink with w_s > 0 of
 * highest cosine similarity (ties -> lowest s): k_s <- (w_s k_s + k_x)/(w_s + 1),
 * v_s likewise (float64 arithmetic, rounded to nearest even in the storage dtype),
 * w_s += 1. Must follow the hardkv_append of the same step. */
int hardkv_condense(const hardkv_desc *desc, const hardkv_cache *cache, void *ws,
                    cudaStream_t stream);

/* Stage 2 (sec. 2.B Logits Calibration; sec. 2.A Tier 2 calibrated top-p).
 * For each selected (b,h) (select_mode), over the Sparse candidates j
 * (positions s_lo + j < d_lo):
 *   s_j = max_{g in group(h)} (q_g . k_j) / sqrt(d)       max-pooled logit
 *   p_j = softmax_j(s_j / tau[b,h])                       calibration
 *   keep the shortest prefix of the (s desc, position asc) order whose mass is
 *   >= p (p = 1 keeps all), at most Cap of them.
 * Writes mask[b,h,:] (device uint32 [B,H,mask_words]; bit j set = kept; bits past
 * the Sparse length are 0). tau: device float [B,H] or NULL (all 1). */
int hardkv_score_calibrate_topp(const hardkv_desc *desc, const hardkv_cache *cache,
                                const void *q, const float *tau, float p,
                                int32_t select_mode, uint32_t *mask, void *ws,
                                cudaStream_t stream);

/* Stage 2 with the entropy-matched calibration (HARDKV_CAL_ENTROPY above): as
 * hardkv_score_calibrate_topp, but each selected (b,h) solves its own temperature
 * tau[b,h] in [1/64, 64] so that the calibrated distribution softmax(s / tau) over its
 * candidates has the mean entropy of the raw attention distributions of its queries
 * (Newton steps on 1/tau inside a bisection bracket, on the device). tau_out: device
 * float [B,H] receiving the solved temperatures, or NULL. */
int hardkv_score_calibrate_entropy_topp(const hardkv_desc *desc, const hardkv_cache *cache,
                                        const void *q, float p, int32_t select_mode,
                                        uint32_t *mask, float *tau_out, void *ws,
                                        cudaStream_t stream);

/* Stage 2 with the fixed-budget rule (HARDKV_RULE_TOPK): for each selected (b,h), the
 * same scores s_j, then the k candidates first in the (s desc, position asc) order are
 * kept (all of them when there are at most k); 1 <= k <= Cap. No calibration and no
 * capacity clamp. mask as in hardkv_score_calibrate_topp. */
int hardkv_score_topk(const hardkv_desc *desc, const hardkv_cache *cache, const void *q,
                      int32_t k, int32_t select_mode, uint32_t *mask, void *ws,
                      cudaStream_t stream);

/* Stage 2b/2c on importance scores the caller supplies (any metric in place of the
 * max-pooled logit: sec. 2.B calibrates "scores" into one probability space, whatever
 * produced them). scores: device float [B,H,R], candidate j of (b,h) (position
 * s_lo + j, j < d_lo - s_lo) at scores[(b*H + h)*R + j], 16-byte aligned; other entries
 * do not affect the result (the row is copied in 16-byte units, so up to three entries
 * past a head's candidates are read). rule HARDKV_RULE_TOPP: calibrated top-p with tau (device float [B,H] or
 * NULL = 1) and 0 < p <= 1, at most Cap kept, exactly as hardkv_score_calibrate_topp
 * after its score stage; HARDKV_RULE_TOPK: the top_k best (1 <= top_k <= Cap; p and
 * tau unused). The head's maximum is taken from the scores themselves. mask as in
 * hardkv_score_calibrate_topp; pass it to hardkv_regularize(_policy) to finish stage 3.
 * Scores must be finite: non-finite ones are not checked and select unspecified
 * candidates (every access stays in bounds). */
int hardkv_select_from_scores(const hardkv_desc *desc, const hardkv_cache *cache,
                              const float *scores, const float *tau, float p, int32_t rule,
                              int32_t top_k, int32_t select_mode, uint32_t *mask, void *ws,
                              cudaStream_t stream);

/* Stage 3 (sec. 2.C Index Regularization: Rewrite Cache + Flatten Index to the max
 * length). For each selected (b,h): the kept candidates of `mask` (device, layout as
 * above), in ascending position order, go to compact slots 0..n-1 — K and V rows
 * copied from the ring, sp_idx[slot] = position — with n = min(popcount, Cap) (a
 * larger mask keeps its first Cap, counted as a clamp); sp_idx[n..Cap) = -1;
 * n_kept = n. Payload rows of pad slots are not written. */
int hardkv_regularize(const hardkv_desc *desc, const hardkv_cache *cache,
                      const uint32_t *mask, int32_t select_mode, void *ws,
                      cudaStream_t stream);

/* Stage 3 with a layout policy: as hardkv_regularize, but each selected (b,h) is
 * rewritten or only indexed (Sparse Loading) as `policy` decides (NULL = rewrite);
 * sp_mode[b,h] records the choice for the attention of this and later steps. */
int hardkv_regularize_policy(const hardkv_desc *desc, const hardkv_cache *cache,
                             const uint32_t *mask, int32_t select_mode,
                             const hardkv_layout_policy *policy, void *ws,
                             cudaStream_t stream);

/* Flatten Index to the sum of the lengths (sec. 2.C: the index is regularized to the
 * maximum length -- sp_idx [B,H,Cap], padded with -1 -- or to the sum of the lengths).
 * Reads n_kept and sp_idx of every (b,h) (u = b*H + h) and writes, on the device,
 *   offsets[u] = sum_{v < u} n_kept[v],   offsets[B*H] = sum of all n_kept,
 *   flat[offsets[u] + j] = sp_idx[u, j]   for j < n_kept[u]
 * (n_kept clamped to [0, Cap]). offsets: int32 [B*H + 1]; flat: int32 with room for
 * B*H*Cap entries (the largest total); both 16-byte aligned, owned by the caller.
 * Entries of flat past the total are not written (a valid descriptor keeps B*H*Cap
 * below 2^31, so the offsets fit an int32). */
int hardkv_flatten_sum(const hardkv_desc *desc, const hardkv_cache *cache, int32_t *offsets,
                       int32_t *flat, cudaStream_t stream);

/* Decode attention over the three tiers (implied by sec. 1 / sec. 5: attention runs
 * on the regularized layout). For each query head g of KV head h:
 *   out = sum_t softmax_t(l_t) v_t over
 *         Dense positions [d_lo, len)                    l = q.k / sqrt(d)
 *       U compact slots < n_kept with sp_idx >= s_lo     l = q.k / sqrt(d)
 *         (row read from k_sp / v_sp when sp_mode = 1, from the ring row of
 *          position sp_idx when sp_mode = 0)
 *       U Condensed slots with w > 0                     l = q.k / sqrt(d) + ln w
 * as one joint softmax (split-K partials combined by log-sum-exp).
 * out: device float [B,Hq,d]. */
int hardkv_decode_attn(const hardkv_desc *desc, const hardkv_cache *cache,
                       const void *q, float *out, void *ws, cudaStream_t stream);

/* One fused decode step (sec. 2.A four-stage pipeline): append, condense (MERGE
 * only), score + calibration + selection (args->rule, args->calibration), then
 * regularize fused with attention: the
 * kept rows are gathered once, written to the compact layout and attended in the
 * same pass. Results equal hardkv_append; hardkv_condense;
 * hardkv_score_calibrate_topp; hardkv_regularize; hardkv_decode_attn.
 * All pointers in `args` are device pointers. */
int hardkv_decode_step(const hardkv_desc *desc, const hardkv_cache *cache,
                       const hardkv_step_args *args, void *ws, cudaStream_t stream);

/* hardkv_decode_step with the per-step tensors in HOST memory (pinned memory makes
 * the copies asynchronous): args->q, k_new, v_new and tau (if not NULL) are read from
 * the host, args->out is written to the host; the copies and the step are enqueued
 * on `stream` and the caller synchronises before reading `out`. args->mask and
 * args->tau_out, if not NULL, are device pointers. Every argument is checked before
 * the first copy is enqueued. Staging buffers live in the workspace. Pinned, mapped
 * and 16-byte aligned k_new, v_new and out buffers (cudaHostAlloc memory under
 * unified addressing) are read / written by the kernels in place instead of copied,
 * and such a q is copied to its staging buffer by the first kernel of the step (one
 * copy fewer on the stream); tau is always copied. */
int hardkv_decode_step_host(const hardkv_desc *desc, const hardkv_cache *cache,
                            const hardkv_step_args *host_args, void *ws,
                            cudaStream_t stream);

/* Allocation-free variant of hardkv_score_calibrate_topp (no counterpart in the
 * paper: it only changes where the stage's scratch lives).
 *
 * Some callers cannot call cudaMalloc or hand this library a workspace: a plugin
 * inside a host framework whose caching allocator owns all device memory and offers
 * no scratch to this stage, code that runs while another component holds a stream
 * capture in a mode that forbids allocation, or a latency-critical loop that cannot
 * afford the synchronisation an allocation may cause. For them this entry point
 * takes the same inputs and outputs as hardkv_score_calibrate_topp (q, tau, p,
 * select_mode, mask: device pointers, same layouts and results) but no workspace:
 * the fp32 score array and the per-tile maxima live in a file-scope device array of
 * hardkv_static_scratch_bytes() bytes (32 MiB) that every GPU which loads the library
 * holds until the process exits. It calls no cudaMalloc, cudaFree or allocating
 * library routine.
 *  - Limit: B*H*ring_rows*4 bytes of scores plus the tile maxima must fit in that
 *    array; larger problems return HARDKV_ESCRATCH (nothing is enqueued).
 *  - The first call on a device looks up the array's device address with
 *    cudaGetSymbolAddress while that device is current; make that first call before
 *    any stream capture that includes this entry point. The address is then kept for
 *    the life of the process: a caller that resets the device (cudaDeviceReset) must
 *    not call this entry point on that device afterwards.
 *  - Every call, on every stream, shares the one array and leaves its contents there;
 *    nothing in it needs to start at zero (each call writes what it reads). Calls whose
 *    executions overlap on the GPU race on the array: serialise them (one stream, or
 *    events). */
int hardkv_score_calibrate_topp_static(const hardkv_desc *desc, const hardkv_cache *cache,
                                       const void *q, const float *tau, float p,
                                       int32_t select_mode, uint32_t *mask,
                                       cudaStream_t stream);

/* Size in bytes of the built-in scratch used by hardkv_score_calibrate_topp_static. */
size_t hardkv_static_scratch_bytes(void);

/* Diagnostic (no counterpart in the paper): runs the bounded wait that every pipeline
 * of this library uses on an mbarrier that nothing completes, with at most `limit`
 * polls (1..65536). The wait gives up, ORs HARDKV_DEV_WAIT_TIMEOUT into
 * status[HARDKV_ST_FLAGS], writes `limit` to status[7] and the kernel returns: the
 * path a pipeline takes when a copy never lands, exercised without any copy in flight.
 * status: device uint32[HARDKV_STATUS_WORDS]. */
int hardkv_selftest_wait_timeout(uint32_t *status, uint32_t limit, cudaStream_t stream);

/* Human-readable text of a return code (for HARDKV_ECUDA: the last CUDA error seen
 * by this thread). The string is static or thread-local; do not free it. */
const char *hardkv_strerror(int code);

#ifdef __cplusplus
}
#endif
#endif /* HARDKV_H */
