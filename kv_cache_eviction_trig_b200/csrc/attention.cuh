// Decode attention over the pruned cache (the step after the prune).
#pragma once

#include "tria_internal.cuh"

namespace tria {

struct alignas(64) AttnParams {
  CUtensorMap tk, tv;       // K and V as 2-D bf16 tensors [L*Hkv*cap][D], boxes of 64 x 128,
                            // 128-byte swizzled (tensor-core path only)
  int32_t mma;              // 1: the tensor-core path (tk and tv are valid)
  int32_t split;            // clusters per (sequence, KV head) on the tensor-core path (1 or 4)
  float *scratch;           // split 4: [units][4][16 + 8 D] per-cluster partial results
  int32_t *counters;        // split 4: [units] arrivals, zero at rest
  const uint16_t *q;        // bf16 [B][Hq][D]
  const uint16_t *k;        // bf16 [L][Hkv][cap][D]
  const uint16_t *v;
  const int32_t *seq_len;   // [B]
  const int32_t *unit_len;  // [L][Hkv][B] per-unit lengths (instead of seq_len), or null
  float *out;               // [B][Hq][D]
  int32_t *err;
  int64_t cap;
  int32_t layer, B, Hkv, Hq, G, D;
  float scale;
  int64_t seg_start[TRIA_MAX_BATCH + 1];
};

bool attention_supported(int D, int G);
// Whether the tensor-core path takes this shape (D = 64 or 128, G <= 8).
bool attention_mma_supported(int D, int G);
cudaError_t launch_attention(const AttnParams &p, cudaStream_t s);

}  // namespace tria
