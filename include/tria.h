/*
 * tria.h -- C ABI of the B200 (sm_100a) TriAttention KV-cache prune step.
 *
 * What the library computes (TriAttention, arXiv 2604.04921, as described by
 * the romaanj.github.io review, section "Method", and the dimensionstp.github.io
 * review, sections 2-2 and 3-2):
 *
 *   calibration   per (layer, query head, RoPE pair f): centre E[q_f] (complex),
 *                 mean norm E|q_f| and concentration R_f = |E[q_f]| / E|q_f|
 *                 over sample pre-RoPE queries;
 *   key score     s_h(t) = mean_{delta in offsets} sum_f |E[q_f]| |k_f|
 *                            cos(w_f (cur + delta - pos_t) + arg E[q_f] - arg k_f)
 *                        + sum_f (1 - R_f) E|q_f| |k_f|
 *                 with k_f the pre-RoPE pair of the cached key, w_f = theta^(-2f/D);
 *   aggregation   z-score of s_h over the sequence's keys (population sigma,
 *                 z = 0 if sigma = 0), then the max over the query heads h that
 *                 share the key's KV head (h / G == kv head);
 *   selection     top-`budget` keys per (layer, KV head, sequence) by
 *                 (score desc, slot asc);
 *   compaction    survivors move in place to slots [0, kept) in ascending slot
 *                 order; seq_len becomes kept.
 *
 * Conventions shared by every call
 * --------------------------------
 * - Pointers marked DEVICE must point to memory of the current CUDA device;
 *   HOST pointers are read during the call only.  The caller owns every
 *   buffer, the workspace included; the library allocates nothing and keeps
 *   no global mutable state.
 * - `stream` is a cudaStream_t passed as void*; NULL is the legacy default
 *   stream.  Every call is asynchronous on it: argument errors are returned
 *   synchronously before anything is launched; launch failures return
 *   TRIA_ERR_CUDA.  Inconsistencies only the device can see (a sequence
 *   length beyond its segment, a malformed selection list, a wait that ran
 *   out) set bits in the workspace's device error word, readable with
 *   tria_get_device_error() after the stream has been synchronised.
 *   Nothing traps.
 * - Cache layout: K and V are bf16 [L][Hkv][cap_total][D] (post-RoPE keys),
 *   pos is int32 [L][Hkv][cap_total].  Sequence b owns slots
 *   [seq_start[b], seq_start[b+1]) of every (layer, KV head) row; its live
 *   keys are the first seq_len[b] of them (or the first unit_len of each
 *   (layer, KV head, sequence) unit, when the cache has per-unit lengths),
 *   with ascending positions.
 * - Slot indices in selection lists are relative to the segment start.
 * - Query head h uses KV head h / G, G = n_q_heads / n_kv_heads.
 * - Supported shapes: head_dim in {64, 128, 256}; G in {1, 2, 4, 8, 16};
 *   batch <= TRIA_MAX_BATCH; 1 <= n_offsets <= TRIA_MAX_OFFSETS; every
 *   segment capacity <= TRIA_MAX_SEGMENT; 1 <= budget <= TRIA_MAX_SEGMENT.
 */
#ifndef TRIA_H
#define TRIA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TRIA_OK = 0,
  TRIA_ERR_INVALID_ARG = 1,   /* a null, negative, inconsistent or misaligned argument */
  TRIA_ERR_UNSUPPORTED = 2,   /* a valid shape this build has no kernel for */
  TRIA_ERR_WORKSPACE = 3,     /* workspace null, misaligned or smaller than tria_workspace_size */
  TRIA_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
  TRIA_ERR_DEVICE_FLAG = 5    /* returned by tria_get_device_error when a device bit is set */
} tria_status;

#define TRIA_ROPE_HALF_SPLIT 0   /* pair f = (v[f], v[f + D/2]) */
#define TRIA_ROPE_INTERLEAVED 1  /* pair f = (v[2f], v[2f + 1]) */

#define TRIA_NO_TRIG 1u          /* ablation: score without the trigonometric term */
#define TRIA_NO_CONC_WEIGHT 2u   /* ablation: norm term weighted by E|q_f| instead of (1-R_f)E|q_f| */
/* tria_prune / tria_prune_noalloc as one persistent cooperative launch (every CTA scores
   a share of each group of units, and grid rounds order the selection and compaction
   steps) instead of the fold, score and unit kernels.  Same results; shapes that launch
   cannot take run the default kernels.  Set the flag before tria_workspace_size: the
   launch needs its own workspace regions. */
#define TRIA_FUSED_PRUNE 4u

#define TRIA_DTYPE_F32 0
#define TRIA_DTYPE_BF16 1

#define TRIA_MAX_BATCH 256
#define TRIA_MAX_OFFSETS 4096
#define TRIA_MAX_SEGMENT (1 << 18)

/* device error word bits */
#define TRIA_DEVERR_SEQ_LEN 1      /* seq_len[b] < 0 or > segment capacity: that sequence skipped */
#define TRIA_DEVERR_SELECTION 2    /* tria_compact: selection not ascending / out of range: unit skipped */
#define TRIA_DEVERR_TIMEOUT 4      /* a bounded wait on an mbarrier ran out: results invalid */
#define TRIA_DEVERR_SEGMENT_BIG 8  /* a live sequence exceeded the kernel's per-unit capacity */
#define TRIA_DEVERR_SEGMENT_FULL 16 /* tria_append: no free slot in a segment: that sequence skipped */
#define TRIA_DEVERR_BUDGET 32      /* a head budget outside [1, budget]: that KV head's units skipped */

/* Host-side description of the prune problem, copied by value. */
typedef struct {
  int32_t num_layers;   /* L >= 1 */
  int32_t batch;        /* B, 1..TRIA_MAX_BATCH */
  int32_t n_q_heads;    /* Hq, a multiple of n_kv_heads */
  int32_t n_kv_heads;   /* Hkv >= 1 */
  int32_t head_dim;     /* D */
  double rope_theta;    /* RoPE base, > 1 */
  int32_t rope_layout;  /* TRIA_ROPE_HALF_SPLIT or TRIA_ROPE_INTERLEAVED */
  int32_t budget;       /* keys kept per (layer, KV head, sequence) */
  const int32_t *offsets; /* HOST [n_offsets] future query offsets, each >= 1 */
  int32_t n_offsets;
  uint32_t flags;       /* 0, or TRIA_NO_TRIG / TRIA_NO_CONC_WEIGHT / TRIA_FUSED_PRUNE */
  int32_t prune_window; /* >= 0.  tria_prune / tria_prune_noalloc prune a sequence only
                           once seq_len >= budget + max(prune_window, 1) (a decode loop
                           that calls tria_prune after every tria_append then prunes each
                           sequence back to budget every prune_window decoded tokens);
                           0 or 1: every sequence with seq_len > budget.  Other calls
                           ignore it. */
  const int32_t *head_budgets; /* DEVICE int32 [L][Hkv], or NULL.  Head-specific budgets
                           (romaanj.github.io review, "Future work": compression refined
                           with budgets per head; the pages give no rule for choosing
                           them, so they are an input): the units of KV head g of layer
                           l keep head_budgets[l*Hkv + g] keys, each in [1, budget]
                           (budget stays the length of every selection list, and an
                           entry outside that range sets TRIA_DEVERR_BUDGET and leaves
                           that head's units as they are).  Needs cache->unit_len: the
                           units of one sequence then hold different numbers of keys.
                           The prune window applies per unit: head budget + window. */
} tria_config;

/* The cache.  Device pointers except seq_start. */
typedef struct {
  void *k;                 /* DEVICE bf16 [L][Hkv][cap_total][D], 16-byte aligned */
  void *v;                 /* DEVICE bf16 [L][Hkv][cap_total][D], 16-byte aligned */
  int32_t *pos;            /* DEVICE int32 [L][Hkv][cap_total], 16-byte aligned */
  int32_t *seq_len;        /* DEVICE int32 [B], live keys per sequence (in/out) */
  int32_t *cur_pos;        /* DEVICE int32 [B], position of each sequence's newest token
                              (read by the scoring calls, advanced by tria_append) */
  const int64_t *seq_start;/* HOST int64 [B+1], nondecreasing, seq_start[B] <= cap_total */
  int64_t cap_total;       /* slots per (layer, KV head) row */
  int32_t *unit_len;       /* DEVICE int32 [L][Hkv][B] (in/out), or NULL.  When set, the
                              live keys of unit (l, g, b) are the first unit_len[(l*Hkv +
                              g)*B + b] slots of its segment (units of one sequence may
                              differ, as after a prune with head budgets); seq_len is then
                              neither read nor written and may be NULL. */
} tria_cache;

/* Calibration statistics, DEVICE float32, 16-byte aligned. */
typedef struct {
  const float *centre;     /* [L][Hq][D/2][2]  E[q_f] as (re, im) */
  const float *mean_norm;  /* [L][Hq][D/2]     E|q_f| */
  const float *mrl;        /* [L][Hq][D/2]     R_f */
} tria_stats;

/* Bytes of workspace the calls below need for this problem (the largest over
 * all calls).  The workspace holds the intermediate results of the steps the
 * problem statement lists (dimensionstp.github.io review, section 2-1, steps
 * 1-6: score every cached key, normalise per head, keep the top budget, evict
 * the rest): folded weights, per-head scores, their sums, selection lists and
 * the error word.  Only the shapes and cache->seq_start/cap_total are read. */
tria_status tria_workspace_size(const tria_config *cfg, const tria_cache *cache, size_t *bytes);

/* Prepares a workspace for the steps of the problem statement (dimensionstp.github.io
 * review, section 2-1, steps 1-6): clears its device error word and its
 * synchronisation words (async on stream).  Call once after allocating a
 * workspace, and again after TRIA_DEVERR_TIMEOUT; the error word is otherwise
 * sticky across calls. */
tria_status tria_workspace_init(void *ws, size_t ws_bytes, void *stream);

/* Offline calibration (romaanj.github.io review, "Method"; dimensionstp.github.io
 * review, section 3-1): q_pre is DEVICE [L][n_samples][Hq][D] pre-RoPE queries,
 * float32 (q_dtype = TRIA_DTYPE_F32) or bf16 (TRIA_DTYPE_BF16).  Writes the
 * three DEVICE float32 outputs laid out as in tria_stats.  Accumulates in
 * float64.  Only L, Hq, head_dim and rope_layout of cfg are read. */
tria_status tria_calibrate(const tria_config *cfg, const void *q_pre, int32_t q_dtype,
                           int64_t n_samples, float *centre, float *mean_norm, float *mrl,
                           void *stream);

/* Key scores (romaanj.github.io review, "Method"; dimensionstp.github.io review,
 * sections 2-2 and 3-2 (2)-(4), (6)).  Writes DEVICE float32 score
 * [L][Hkv][cap_total], the group max of the z-scores, for every live slot of
 * every sequence; if raw is not NULL, also DEVICE float32 raw
 * [L][Hq][cap_total], the per-query-head score s_h.  Other slots are not
 * written.  Sequences of any length are scored. */
tria_status tria_score(const tria_config *cfg, const tria_stats *stats, const tria_cache *cache,
                       float *score, float *raw, void *ws, size_t ws_bytes, void *stream);

/* Top-budget selection (romaanj.github.io review, "Method"; dimensionstp.github.io
 * review, section 3-2 (5)).  score is DEVICE float32 [L][Hkv][cap_total] (as
 * written by tria_score).  Writes DEVICE int32 sel [L][Hkv][B][budget]: the kept
 * slots in ascending order, -1 after the last one.  A sequence with
 * seq_len <= budget keeps all its slots.  Ties go to the lower slot. */
tria_status tria_select(const tria_config *cfg, const tria_cache *cache, const float *score,
                        int32_t *sel, void *ws, size_t ws_bytes, void *stream);

/* In-place compaction: the eviction that follows the selection
 * (dimensionstp.github.io review, section 3-2 (5), window pruning drops every
 * key outside the kept set; romaanj.github.io review, "Method", the cache is cut
 * back to the budget).  sel is DEVICE int32 [L][Hkv][B][budget] as
 * written by tria_select: strictly ascending slots then -1.  Moves K, V and pos
 * rows sel[j] -> j of each segment and sets seq_len[b] to the number of kept
 * slots (every (layer, KV head) list of a sequence must keep the same count).
 * A list that is not strictly ascending or leaves the segment sets
 * TRIA_DEVERR_SELECTION and that unit is left untouched. */
tria_status tria_compact(const tria_config *cfg, const tria_cache *cache, const int32_t *sel,
                         void *ws, size_t ws_bytes, void *stream);

/* The whole prune step in one call (romaanj.github.io review, "Method";
 * dimensionstp.github.io review, section 2-1, steps 1-6, and section 3-2
 * (2)-(6)): score, z-score + group max, select and
 * compact every (layer, KV head, sequence) with seq_len > budget (and
 * seq_len >= budget + cfg->prune_window); other sequences are left untouched.
 * seq_len is read once at the start and rewritten at the end.  If sel_out is
 * not NULL it receives the selection as tria_select would write it for the
 * sequences that were pruned and for those with seq_len <= budget; the rows of
 * sequences held back by prune_window are not written.  By default three
 * kernels (fold, score, unit) chained by programmatic dependent launch;
 * cfg->flags TRIA_FUSED_PRUNE selects one persistent cooperative launch. */
tria_status tria_prune(const tria_config *cfg, const tria_stats *stats, const tria_cache *cache,
                       int32_t *sel_out, void *ws, size_t ws_bytes, void *stream);

/* The decode-loop step before the prune (romaanj.github.io review, "Background":
 * the cache grows by one key and value per decoded token; dimensionstp.github.io
 * review, section 3-2 (5), window-based pruning).  k_new and v_new are DEVICE bf16
 * [L][Hkv][B][D], 16-byte aligned: the new token of every sequence.  For every
 * (layer, KV head, sequence) the token's K and V rows go to slot
 * seq_start[b] + seq_len[b] and its position cur_pos[b] + 1 to pos; then
 * seq_len[b] and cur_pos[b] advance by one.  A sequence whose segment has no
 * free slot (seq_len[b] == segment capacity) is left unchanged and sets
 * TRIA_DEVERR_SEGMENT_FULL; one with seq_len[b] out of range sets
 * TRIA_DEVERR_SEQ_LEN.  Two kernel launches, no host synchronisation: a decode
 * step (tria_append, then tria_prune with cfg->prune_window) can be captured in
 * a CUDA graph and replayed.  ws as for the other calls (only its error word is
 * used). */
tria_status tria_append(const tria_config *cfg, const tria_cache *cache, const void *k_new,
                        const void *v_new, void *ws, size_t ws_bytes, void *stream);

/* Decode attention over the pruned cache: the step after the prune in a decode
 * loop (romaanj.github.io review, "Results": decoding reads the budgeted cache,
 * which is where the throughput gain comes from; dimensionstp.github.io review,
 * section 6, Limitations: in serving the pruned cache meets the attention kernel).
 * The cache stores post-RoPE keys, so positions are not needed.  For layer
 * `layer`, every sequence b and query head h (KV head h / G):
 *   out[b][h] = sum_{t < seq_len[b]} softmax_t(scale * q[b][h] . k_t) v_t
 * over the live slots t of segment b; scale <= 0 selects the usual 1/sqrt(D)
 * (any positive finite scale is used as given).  q is DEVICE bf16 [B][Hq][D], 16-byte
 * aligned; out is DEVICE float32 [B][Hq][D]; a sequence with seq_len 0 gets
 * zeros.  Accumulates in float32 with a running maximum (no overflow for any
 * finite logits).  A seq_len out of range sets TRIA_DEVERR_SEQ_LEN and that
 * sequence's rows are not written.  ws as for the other calls, sized for this
 * cfg and cache: besides its error word, a call over few (sequence, KV head)
 * pairs with long segments uses the workspace's raw-score region for partial
 * results and leaves the words it counts with back at zero.  Like every call,
 * it must not overlap another call on the same workspace. */
tria_status tria_decode_attention(const tria_config *cfg, const tria_cache *cache, int32_t layer,
                                  const void *q, float scale, float *out, void *ws,
                                  size_t ws_bytes, void *stream);

/* tria_prune (same passages: romaanj.github.io review, "Method";
 * dimensionstp.github.io review, sections 2-1 and 3-2) with a cudaEvent_t
 * (as void*) recorded on `stream` before each of its kernels and after the
 * last: events[0..n_stages].  Returns the number of stages in *n_stages
 * (events must hold TRIA_PRUNE_MAX_STAGES + 1) and, if stage_ids is not NULL
 * (HOST, TRIA_PRUNE_MAX_STAGES entries), the kernel of each stage as an index
 * for tria_prune_stage_name.  tria_prune runs three kernels (fold, score,
 * unit); with TRIA_FUSED_PRUNE it runs one persistent launch for the shapes that
 * launch takes (every supported shape except head_dim 256 with G >= 8).  For
 * per-kernel timing only. */
#define TRIA_PRUNE_MAX_STAGES 8
tria_status tria_prune_profiled(const tria_config *cfg, const tria_stats *stats,
                                const tria_cache *cache, int32_t *sel_out, void *ws,
                                size_t ws_bytes, void *stream, void *const *events,
                                int32_t *n_stages, int32_t *stage_ids);

/* Name of the kernel with index i (0 fold, 1 score, 2 unit, 3 the fused prune
 * kernel; the steps of the dimensionstp.github.io review, section 2-1, as this
 * library groups them), "" for any other i. */
const char *tria_prune_stage_name(int32_t i);

/* Reads the workspace's device error word into *code (synchronous: waits for
 * `stream`): the inconsistencies that only the device sees while it runs the
 * steps of the problem statement (dimensionstp.github.io review, section 2-1,
 * steps 1-6), such as a sequence length beyond its segment.  Returns
 * TRIA_ERR_DEVICE_FLAG if any bit is set, TRIA_OK otherwise. */
tria_status tria_get_device_error(const void *ws, int32_t *code, void *stream);

/* tria_prune for callers that cannot allocate device memory.  This entry point
 * has no counterpart in the paper: it exists for callers such as a serving
 * engine that reserves all device memory at start-up and forbids allocation in
 * its decode loop (cudaMalloc may fail once its pool owns the memory, and
 * cudaFree waits for the whole device).  Same inputs, outputs and results as
 * tria_prune, but the workspace is a fixed array of TRIA_NOALLOC_SCRATCH_BYTES
 * inside the library's device image; the call allocates nothing.
 *   - Problems whose tria_workspace_size exceeds TRIA_NOALLOC_SCRATCH_BYTES
 *     return TRIA_ERR_UNSUPPORTED before anything is launched (16 MiB holds,
 *     for example, one layer of 32 query heads over 32768 cached slots).
 *   - CUDA loads the part of the library that holds the array lazily: the
 *     first call on a device (with that device current) looks up the array's
 *     address with cudaGetSymbolAddress, which loads it and so reserves its
 *     TRIA_NOALLOC_SCRATCH_BYTES on that device until the process exits.
 *     Make that first call at start-up, before reserving the device's memory
 *     for a pool and before any stream capture; later calls reserve nothing.
 *     A first call that fails (TRIA_ERR_CUDA) is retried by the next call.
 *   - Every call on a device shares the array.  Each call clears the array's
 *     error word; the other parts that must start at zero start zero and every
 *     call leaves them zero.  Calls whose kernels may overlap on one device
 *     (different streams, no ordering) race.
 *   - device_error, if not NULL, is a DEVICE int32 that receives the call's
 *     device error word (TRIA_DEVERR_* bits, 0 if none) at the end of the call,
 *     in stream order; the scratch cannot be passed to tria_get_device_error.
 */
#define TRIA_NOALLOC_SCRATCH_BYTES (16 << 20)
tria_status tria_prune_noalloc(const tria_config *cfg, const tria_stats *stats,
                               const tria_cache *cache, int32_t *sel_out, int32_t *device_error,
                               void *stream);

/* Human-readable name of a status returned by the calls above (which follow the
 * dimensionstp.github.io review, section 2-1). */
const char *tria_status_string(tria_status s);

/* Version string of this implementation of the prune step (romaanj.github.io
 * review, "Method"). */
const char *tria_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TRIA_H */
