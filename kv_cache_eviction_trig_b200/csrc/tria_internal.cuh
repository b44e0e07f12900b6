// Internal declarations shared by the CUDA translation units of libtria.
// Device primitives are written directly in PTX for sm_100a.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tria.h"

namespace tria {

// ------------------------------------------------------------------ workspace layout
// The workspace starts with a fixed prefix that holds state which must be zero
// when a call starts (tria_workspace_init clears it; the fused prune kernel leaves
// it zero): the error word, the fused kernel's synchronisation words, bucket
// counters and histograms.  After it come the per-call regions of either path
// (fold/score/unit kernels, or the fused kernel); a call uses one path, so the
// two share the same bytes.
constexpr size_t kWsErr = 0;
constexpr size_t kWsSync = 256;
constexpr size_t kWsBcount = 256 + 16 * 128;  // after kSyncWords lines of 128 bytes
constexpr size_t kWsHist = 4096;
constexpr size_t kWsPrefix = kWsHist + 2ull * 32 * 4096 * 4;  // 2 slots x 32 units x 4096 bins

struct WsLayout {
  size_t err;       // int32 device error word (+ padding)
  size_t seqlen;    // int32 [B]   snapshot of seq_len taken at the start of a call
  size_t w;         // float [L*Hkv*B][D/4][G][6]  folded weights (fold kernel)
  size_t raw;       // float [L][Hq][cap]  raw scores when the caller gives none
  size_t sel;       // int32 [L][Hkv][B][budget] selection scratch
  size_t partials;  // double [L*Hkv*B][max_slots][score warps][G][2] sums of s and s^2
  int32_t max_slots;
  // fused prune kernel (same bytes as the regions above)
  int fused;        // the fused kernel runs this problem's prune
  size_t f_ea, f_w, f_raw, f_csum, f_partial, f_zk, f_bucket, f_above, f_thr, f_kcount, f_klist,
      f_khaz, f_stage_k, f_stage_v, f_stage_pos;
  size_t total;
};
WsLayout ws_layout(const tria_config &cfg, const int64_t *seq_start, int64_t cap_total);

// How the score kernel's grid divides the key chunks (a function of the shapes,
// seq_start and the current device's SM count).
struct ScoreGrid {
  int chunk_keys;       // keys per chunk
  int chunks_per_row;   // chunks of one (layer, KV head) row over all sequences
  int64_t total;        // chunks over all rows
  int chunks_per_cta;
  int grid;
  int max_slots;        // most CTAs whose chunk runs meet one unit
};
ScoreGrid score_grid(const tria_config &cfg, const int64_t *seq_start);

// ------------------------------------------------------------------ kernel parameters
#ifndef TRIA_SCORE_WARPS
#define TRIA_SCORE_WARPS 8
#endif
#ifndef TRIA_SCORE_KPT_CAP
#define TRIA_SCORE_KPT_CAP 4
#endif
#ifndef TRIA_SCORE_TC_WARPS
#define TRIA_SCORE_TC_WARPS 11
#endif
constexpr int kScoreConsumerWarps = TRIA_SCORE_WARPS;  // build-time tunables: consumer warps of
constexpr int kScoreTcWarps = TRIA_SCORE_TC_WARPS;     // the FMA form and of the tensor-core form
// the larger of the two: sizes the workspace for the score kernel's partial sums, which
// hold one entry per (unit, CTA slot, consumer warp) of the form that ran
constexpr int kScoreMaxWarps = kScoreConsumerWarps > kScoreTcWarps ? kScoreConsumerWarps : kScoreTcWarps;
constexpr int kScoreKptCap = TRIA_SCORE_KPT_CAP;
#ifndef TRIA_SCORE_JU
#define TRIA_SCORE_JU 4
#endif
constexpr int kScoreJu = TRIA_SCORE_JU;  // pairs of RoPE pairs per inner iteration: 1, 2 or 4
constexpr int kScoreRingBytes = 220 * 1024;  // shared memory for key chunks and weights

#ifndef TRIA_UNIT_THREADS
#define TRIA_UNIT_THREADS 1024
#endif
constexpr int kUnitThreads = TRIA_UNIT_THREADS;  // build-time tunable: 256, 512 or 1024
constexpr int kUnitCluster = 8;
constexpr int kUnitClustersAtOnce = 15;   // 8-CTA clusters of 200 KB resident at once on a B200
constexpr int kUnit4ClustersAtOnce = 33;  // 4-CTA clusters of 200 KB resident at once on a B200
constexpr int kUnitSmemLarge = 200 * 1024;  // one CTA per SM

struct FoldParams {
  const int32_t *cur_pos;   // [B]
  const int32_t *seq_len;   // [B] caller's live lengths
  const int32_t *unit_len;  // [U] per-unit live lengths (instead of seq_len), or null
  int32_t *seqlen_snap;     // [B], or [U] with per-unit lengths, out
  int64_t units;
  int32_t *err;
  const float2 *centre;     // [L][Hq][F]
  const float *mean_norm;   // [L][Hq][F]
  const float *mrl;         // [L][Hq][F]
  float *w;                 // [L*Hkv*B][F/2][G][6] out
  double theta;
  int32_t D, B, L, Hkv, Hq, G;
  uint32_t flags;
  int64_t seg_cap[TRIA_MAX_BATCH];
  double omega[128];        // w_f = theta^(-2f/D), f < D/2
  double2 A[128];           // mean over the offsets of e^{i w_f delta} (0 without the trig term)
};

struct alignas(64) ScoreParams {
  CUtensorMap tmap;         // K as a 2-D bf16 tensor [L*Hkv*cap][D], 128-byte swizzled boxes
  const float *w;           // folded weights (written by the fold kernel)
  const int32_t *seq_len;   // [B] caller's live lengths (not modified during the call)
  const int32_t *unit_len;  // [U] per-unit live lengths instead, or null
  const int32_t *head_budget;  // [L*Hkv] per-head budgets (with skip_short), or null
  int32_t tc;               // 1: the tensor-core form (kScoreTcWarps consumer warps)
  int32_t budget, window;   // with skip_short: units shorter than budget + max(window, 1) are skipped
  float *raw;               // [L][Hq][cap]
  double *partials;         // per (unit, slot, warp): float64 sums of s and s^2 per head
  int32_t max_slots;
  int32_t *err;
  int64_t cap;
  int32_t L, Hkv, Hq, B;
  int32_t prune_from;       // with skip_short: the shortest seq_len that is pruned
  int32_t skip_short;       // 1: sequences with seq_len < prune_from are not scored
  int32_t chunks_per_row;   // chunk_prefix[B]
  int32_t chunks_per_cta;
  int32_t total_chunks;     // < 2^31 (checked on the host)
  int64_t seg_start[TRIA_MAX_BATCH + 1];
  int32_t chunk_prefix[TRIA_MAX_BATCH + 1];
};

enum UnitMode : int32_t { kModeZmax = 0, kModeSelect = 1, kModeCompact = 2, kModePrune = 3 };

struct UnitParams {
  uint8_t *k;               // bf16 rows
  uint8_t *v;
  int32_t *pos;
  const float *raw;         // [L][Hq][cap]      (zmax, prune)
  const double *partials;   // the score kernel's per-(unit, slot, warp) sums (zmax, prune)
  int32_t max_slots, chunks_per_cta, chunks_per_row;
  int32_t score_warps;      // consumer warps the score kernel ran with (entries per slot)
  int32_t chunk_prefix[TRIA_MAX_BATCH + 1];
  float *score;             // [L][Hkv][cap]     (zmax writes, select reads)
  int32_t *sel;             // [L][Hkv][B][budget]
  const int32_t *seqlen;    // [B] snapshot (zmax, select, prune), or [U] with unit_mode
  int32_t *seq_len_out;     // [B] (compact, prune), or [U] with unit_mode
  int32_t unit_mode;        // lengths per (layer, KV head, sequence) unit
  const int32_t *head_budget;  // [L*Hkv] per-head budgets, or null
  int32_t window;           // prune: a unit is pruned once T >= its budget + max(window, 1)
  int32_t *err;
  int64_t cap;
  int32_t L, Hkv, Hq, B, G, D, budget;
  int32_t prune_from;       // prune: the shortest seq_len that is pruned (> budget)
  int32_t mode;
  int32_t write_short_sel;  // prune: also write identity lists for seq_len <= budget
  int32_t smem_bytes;       // dynamic shared memory of the launch
  int32_t cluster;          // CTAs per unit (1, 4 or kUnitCluster)
  int64_t seg_start[TRIA_MAX_BATCH + 1];
};

// ------------------------------------------------------------------ fused prune kernel
// One cooperative, persistent launch (one CTA per SM) scores, z-scores, selects and
// compacts every unit.  Units are taken in groups of consecutive units; every CTA
// scores an equal share of each group's key chunks, and select warps finish a group
// (through four grid-wide rounds on counters in the workspace) while the consumer
// warps already score the next one.
constexpr int kPruneConsumerWarps = 8;
constexpr int kPruneSelectWarps = 4;
constexpr int kPruneThreads = (kPruneConsumerWarps + 1 + kPruneSelectWarps) * 32;
constexpr int kPruneRangeKeys = 8192;  // keys of one CTA's share of a group, at most (fewer for G > 4)
constexpr int kPruneHistBins = 4096;   // bins of a unit's z histogram (1/256 over [-8, 8))
constexpr int kPruneBucketMax = 4096;  // threshold-bin keys gathered by every CTA
constexpr int kPruneMaxGroupUnits = 32;
// sync words (int32) at the start of the persistent prefix of the workspace, each on
// its own 128-byte line (word w at int offset w * kSyncStride): every CTA polls them
enum PruneSync : int { kSyncA = 0, kSyncB = 2, kSyncC = 4, kSyncD = 6, kSyncExit = 8,
                       kSyncAbort = 9, kSyncP1 = 10, kSyncP2 = 11, kSyncE = 12, kSyncWords = 16 };
constexpr int kSyncStride = 32;

struct alignas(64) PruneParams {
  CUtensorMap tmap;           // K as [L*Hkv*cap][D] bf16, 128-byte swizzled boxes
  uint8_t *k, *v;             // bf16 rows
  int32_t *pos;
  int32_t *seq_len;           // [B] in/out (null with per-unit lengths)
  int32_t *unit_len;          // [U] in/out per-unit lengths, or null
  const int32_t *head_budget; // [L*Hkv] per-head budgets, or null
  const int32_t *cur_pos;     // [B]
  const float2 *centre;       // [L][Hq][F]
  const float *mean_norm;     // [L][Hq][F]
  const float *mrl;           // [L][Hq][F]
  int32_t *sel_out;           // [U][budget] or null
  int32_t *err;
  int32_t *sync;              // kSyncWords
  int32_t *bcount;            // [2][kPruneMaxGroupUnits] bucket fill counters (zero at rest)
  uint32_t *hist;             // [2][kPruneMaxGroupUnits][kPruneHistBins] (zero at rest)
  double2 *ea;                // [B][F] e^{i w_f cur_b} * mean_delta e^{i w_f delta} (prologue)
  float *w;                   // [U][F/2][G][6] folded weights of every unit (prologue)
  float *raw;                 // [2][ncta][range_keys][G]
  double *csum;               // [2][ncta][range_chunks][G][2] per-chunk sums of s, s^2 (consumers)
  double *partial;            // [2][ncta][ug][G][2] per CTA and unit of the group
  uint32_t *zk;               // [2][zk_stride] z keys of a group, by chunk position
  unsigned long long *bucket; // [2][ug][kPruneBucketMax] (key << 18 | ~slot) of threshold bins
  int32_t *above;             // [2][ug][ncta] per covering CTA: keys above the threshold bin
  unsigned long long *thr;    // [2][ug] threshold key of an exactly selected unit
  int32_t *kcount;            // [2][ug][ncta] per covering CTA: kept keys (exact path)
  int32_t *klist;             // [ug][budget] kept slots of every unit of a group, by destination
  int32_t *khaz;              // [2][kPruneMaxGroupUnits] kept slots below the unit's budget
  uint8_t *stage_k, *stage_v; // [ug][budget] rows
  int32_t *stage_pos;         // [ug][budget]
  int64_t cap;
  int64_t zk_stride;
  int32_t L, Hkv, Hq, B, budget, window, write_short_sel, flags;
  int32_t units, ug, ngroups, ncta, cpr, range_keys, range_units, range_chunks;
  int64_t seg_start[TRIA_MAX_BATCH + 1];
  int32_t chunk_prefix[TRIA_MAX_BATCH + 1];
  double omega[128];          // w_f = theta^(-2f/D)
  double2 A[128];             // mean over the offsets of e^{i w_f delta} (0 without the trig term)
};

struct PrunePlan {
  int ok;                     // 0: the fused kernel cannot run this problem
  int chunk_keys, ncta, ug, ngroups, cpr, range_keys, range_units;
  int64_t zk_stride;
};
PrunePlan prune_plan(const tria_config &cfg, const int64_t *seq_start);
bool prune_supported(int D, int G, int layout);
size_t prune_smem_bytes(int D, int G);
cudaError_t launch_prune(const PruneParams &p, int D, int G, int layout, cudaStream_t s);

// ------------------------------------------------------------------ launchers (host)
cudaError_t launch_fold(const FoldParams &p, cudaStream_t s);
cudaError_t launch_score(const ScoreParams &p, int D, int G, int layout, int grid,
                         cudaStream_t s, bool pdl);
bool score_supported(int D, int G, int layout);
// Whether the score kernel takes its tensor-core form for this shape and chunk run.
bool score_uses_tc(int D, int G, int chunks_per_cta);
int score_chunk_keys(int D, int G);
// Encodes the tensor map of the key cache viewed as [rows][D] bf16.
cudaError_t make_key_tensor_map(CUtensorMap *map, const void *k, int D, int64_t rows,
                                int box_rows);
cudaError_t launch_unit(const UnitParams &p, int units, cudaStream_t s, bool pdl);
// CTAs per unit: 8 (one cluster) for few units, 1 for many units whose segments fit.
int unit_cluster_size(int64_t units, int64_t max_segment);
int unit_smem_bytes();
// Decode-loop append: the new token's K, V rows and position into each segment's
// next free slot, then seq_len and cur_pos advance (two launches).
struct AppendParams {
  int32_t *unit_len;        // [L][Hkv][B] per-unit lengths (instead of seq_len), or null
  const uint8_t *k_new;     // bf16 [L][Hkv][B][D]
  const uint8_t *v_new;
  uint8_t *k;               // bf16 [L][Hkv][cap][D]
  uint8_t *v;
  int32_t *pos;             // [L][Hkv][cap]
  int32_t *seq_len;         // [B]
  int32_t *cur_pos;         // [B]
  int32_t *err;
  int64_t cap;
  int32_t L, Hkv, B, D;
  int64_t seg_start[TRIA_MAX_BATCH + 1];
};
cudaError_t launch_append(const AppendParams &p, cudaStream_t s);
cudaError_t launch_calibrate(const void *q, int q_dtype, int64_t L, int64_t N, int64_t Hq,
                             int64_t D, int layout, float *centre, float *mean_norm, float *mrl,
                             cudaStream_t s);
int device_sm_count();

}  // namespace tria

// ------------------------------------------------------------------ device primitives
#ifdef __CUDACC__
namespace tria {
namespace dev {

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

#ifndef TRIA_MBAR_HINT_NS
#define TRIA_MBAR_HINT_NS 1000
#endif
constexpr uint32_t kMbarHintNs = TRIA_MBAR_HINT_NS;  // build-time tunable

// One bounded try: returns true once the phase with the given parity has completed.
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity), "r"(kMbarHintNs)  // suspend-time hint
      : "memory");
  return done != 0;
}

// Waits with an iteration limit (about 2 s at the 1 us hint, and never less than
// the try's own time limit per iteration); false if it ran out.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity) {
  for (uint32_t i = 0; i < 2000000u; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

// 1-D bulk copy global -> shared, completion counted on an mbarrier (no multicast).
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// 2-D tiled tensor load global -> shared (box given by the tensor map), completion
// counted on an mbarrier; no multicast.  x is the innermost (element) coordinate.
__device__ __forceinline__ void tma_load_2d(void *dst, const void *map, int32_t x, int32_t y,
                                            uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
      : "memory");
}

// An L2 policy that evicts the lines it tags first (for data read once, so that it
// does not push out scratch that is read again).
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// tma_load_2d with an L2 cache policy.
__device__ __forceinline__ void tma_load_2d_hint(void *dst, const void *map, int32_t x, int32_t y,
                                                 uint64_t *bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar)), "l"(pol)
      : "memory");
}

__device__ __forceinline__ void named_barrier(uint32_t id, uint32_t threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Arrives at a named barrier without waiting for it.
__device__ __forceinline__ void named_barrier_arrive(uint32_t id, uint32_t threads) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// bf16 pair in one 32-bit word -> two floats (exact widening).
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// float -> uint32 whose unsigned order is the float order (+0 and -0 made equal first).
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f == 0.0f ? 0.0f : f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Programmatic dependent launch: let the next kernel of the stream start / wait
// until the previous kernel of the stream has completed and its writes are visible.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void set_error(int32_t *err, int32_t bit) {
  atomicOr(reinterpret_cast<int *>(err), bit);
}

}  // namespace dev
}  // namespace tria
#endif
