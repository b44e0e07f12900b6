// Decode attention over the pruned cache (the step after the prune).
#pragma once

#include "tria_internal.cuh"

namespace tria {

struct AttnParams {
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
cudaError_t launch_attention(const AttnParams &p, cudaStream_t s);

}  // namespace tria
