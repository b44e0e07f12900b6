// Internal declarations shared by the CUDA translation units of libtria.
// Device primitives are written directly in PTX for sm_100a.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "tria.h"

namespace tria {

// ------------------------------------------------------------------ workspace layout
struct WsLayout {
  size_t err;       // int32 device error word (+ padding)
  size_t seqlen;    // int32 [B]   snapshot of seq_len taken at the start of a call
  size_t ea;        // double2 [B][F]  e^{i w_f cur_b} * mean_delta e^{i w_f delta}
  size_t raw;       // float [L][Hq][cap]  raw scores when the caller gives none
  size_t score;     // float [L][Hkv][cap] group-max z-scores (tria_prune does not need it)
  size_t sel;       // int32 [L][Hkv][B][budget] selection scratch
  size_t partials;  // double [L*Hkv*B][max_slots][G][2] per-CTA sums of s and s^2
  int32_t max_slots;
  size_t total;
};
WsLayout ws_layout(const tria_config &cfg, const int64_t *seq_start, int64_t cap_total);

// ------------------------------------------------------------------ kernel parameters
constexpr int kScoreConsumerWarps = 16;
constexpr int kScoreThreads = (kScoreConsumerWarps + 1) * 32;
constexpr int kScoreStages = 3;
constexpr int kScoreTileBytes = 64 * 1024;   // bytes of K per pipeline stage

constexpr int kUnitThreads = 1024;
constexpr int kUnitCluster = 8;
constexpr int kUnitSmemSmall = 112 * 1024;  // smaller footprint (more clusters resident)
constexpr int kUnitSmemLarge = 200 * 1024;  // one CTA per SM

struct FoldParams {
  const int32_t *cur_pos;   // [B]
  const int32_t *seq_len;   // [B] caller's live lengths
  int32_t *seqlen_snap;     // [B] out
  double2 *ea;              // [B][F] out
  int32_t *err;
  double theta;
  int32_t D, B, n_offsets;
  uint32_t flags;
  int64_t seg_cap[TRIA_MAX_BATCH];
  int32_t offsets[TRIA_MAX_OFFSETS];
};

struct ScoreParams {
  const uint8_t *k;         // bf16 rows [L][Hkv][cap][D]
  const float2 *centre;     // [L][Hq][F]
  const float *mean_norm;   // [L][Hq][F]
  const float *mrl;         // [L][Hq][F]
  const double2 *ea;        // [B][F]  (written by the fold kernel)
  const int32_t *seq_len;   // [B] caller's live lengths (not modified during the call)
  float *raw;               // [L][Hq][cap]
  double *partials;         // [units][max_slots][G][2]
  int32_t *err;
  int64_t cap;
  int32_t max_slots;
  int32_t L, Hkv, Hq, B, budget;
  int32_t skip_short;       // 1: sequences with seq_len <= budget are not scored
  int32_t no_conc_weight;   // ablation flag
  int32_t tiles_per_row;    // tile_prefix[B]
  int32_t tiles_per_cta;
  int64_t total_tiles;
  int64_t seg_start[TRIA_MAX_BATCH + 1];
  int32_t tile_prefix[TRIA_MAX_BATCH + 1];
};

enum UnitMode : int32_t { kModeZmax = 0, kModeSelect = 1, kModeCompact = 2, kModePrune = 3 };

struct UnitParams {
  uint8_t *k;               // bf16 rows
  uint8_t *v;
  int32_t *pos;
  const float *raw;         // [L][Hq][cap]      (zmax, prune)
  const double *partials;   // [units][max_slots][G][2] from the score kernel (zmax, prune)
  int32_t max_slots, tiles_per_cta, tiles_per_row, tile_keys;
  int32_t tile_prefix[TRIA_MAX_BATCH + 1];
  float *score;             // [L][Hkv][cap]     (zmax writes, select reads)
  int32_t *sel;             // [L][Hkv][B][budget]
  const int32_t *seqlen;    // [B] snapshot (zmax, select, prune)
  int32_t *seq_len_out;     // [B] (compact, prune)
  int32_t *err;
  int64_t cap;
  int32_t L, Hkv, Hq, B, G, D, budget;
  int32_t mode;
  int32_t write_short_sel;  // prune: also write identity lists for sequences not pruned
  int32_t smem_bytes;       // dynamic shared memory of the launch
  int64_t seg_start[TRIA_MAX_BATCH + 1];
};

// ------------------------------------------------------------------ launchers (host)
cudaError_t launch_fold(const FoldParams &p, int F, cudaStream_t s);
cudaError_t launch_score(const ScoreParams &p, int D, int G, int layout, int grid,
                         cudaStream_t s, bool pdl);
bool score_supported(int D, int G, int layout);
int score_tile_keys(int D);
cudaError_t launch_unit(const UnitParams &p, int units, cudaStream_t s, bool pdl);
int unit_cluster_size();
int unit_smem_bytes(int units, int64_t max_segment);
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

// One bounded try: returns true once the phase with the given parity has completed.
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity), "r"(1000u)  // suspend hint: 1 us
      : "memory");
  return done != 0;
}

// Waits with an iteration limit (about 2 s at the 1 us hint); false if it ran out.
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

__device__ __forceinline__ void named_barrier(uint32_t id, uint32_t threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
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
