// Decode-loop append: the step that feeds the prune.  While a model decodes,
// every new token's key and value join the cache (romaanj.github.io review,
// "Background"), and the cache is pruned back to the budget once per window of
// decoded tokens (dimensionstp.github.io review, section 3-2 (5), window-based
// pruning; the prune kernels take the window as a length threshold).
//
// Two launches in stream order, so that every row copy has read seq_len[b]
// before it advances:
//   append_rows_kernel     one warp per (layer, KV head, sequence): copies the
//                          new K and V rows (16-byte vectors) into slot
//                          seq_start[b] + seq_len[b] and writes the position
//                          cur_pos[b] + 1;
//   append_advance_kernel  one thread per sequence: seq_len[b] += 1,
//                          cur_pos[b] += 1.
// Both kernels skip a sequence whose seq_len is out of range or whose segment is
// full, and the row kernel flags it.  With per-unit lengths (unit_len) every
// unit appends at its own length, and a sequence is skipped whole when any of
// its units is full or out of range (every warp of the row kernel and the
// sequence's block of the advance kernel check all of the sequence's units).
#include "tria_internal.cuh"

namespace tria {

static_assert(TRIA_MAX_BATCH <= 256, "one block advances every sequence");

namespace {

// With per-unit lengths: 0 if every unit of sequence b has a free slot, else the
// error bit the worst unit raises (the lanes of one warp share the units).
__device__ __forceinline__ int units_blocked(const AppendParams &p, int b, int64_t cap_b,
                                             int lane, int width) {
  int bad = 0;
  for (int64_t lg = lane; lg < (int64_t)p.L * p.Hkv; lg += width) {
    const int32_t T = p.unit_len[lg * p.B + b];
    if (T < 0 || (int64_t)T > cap_b) bad |= TRIA_DEVERR_SEQ_LEN;
    else if ((int64_t)T == cap_b) bad |= TRIA_DEVERR_SEGMENT_FULL;
  }
  return bad;
}

__global__ void __launch_bounds__(256) append_rows_kernel(const __grid_constant__ AppendParams p) {
  const int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;  // (l*Hkv + g)*B + b
  const int lane = threadIdx.x & 31;
  if (row >= (int64_t)p.L * p.Hkv * p.B) return;
  const int b = (int)(row % p.B);
  const int64_t lg = row / p.B;
  const int64_t cap_b = p.seg_start[b + 1] - p.seg_start[b];
  int32_t T;
  if (p.unit_len) {
    const int bad = __reduce_or_sync(0xffffffffu, units_blocked(p, b, cap_b, lane, 32));
    if (bad) {
      if (lg == 0 && lane == 0) dev::set_error(p.err, bad & TRIA_DEVERR_SEQ_LEN ? TRIA_DEVERR_SEQ_LEN
                                                                              : TRIA_DEVERR_SEGMENT_FULL);
      return;
    }
    T = p.unit_len[row];
  } else {
    T = p.seq_len[b];
    if (T < 0 || (int64_t)T >= cap_b) {
      if (lg == 0 && lane == 0)
        dev::set_error(p.err, (T < 0 || (int64_t)T > cap_b) ? TRIA_DEVERR_SEQ_LEN
                                                            : TRIA_DEVERR_SEGMENT_FULL);
      return;
    }
  }
  const int64_t slot = lg * p.cap + p.seg_start[b] + T;
  const int nv = p.D >> 3;  // 16-byte vectors per row
  const uint4 *ks = reinterpret_cast<const uint4 *>(p.k_new) + row * nv;
  const uint4 *vs = reinterpret_cast<const uint4 *>(p.v_new) + row * nv;
  uint4 *kd = reinterpret_cast<uint4 *>(p.k) + slot * nv;
  uint4 *vd = reinterpret_cast<uint4 *>(p.v) + slot * nv;
  for (int i = lane; i < 2 * nv; i += 32) {
    if (i < nv)
      kd[i] = ks[i];
    else
      vd[i - nv] = vs[i - nv];
  }
  if (lane == 0) p.pos[slot] = p.cur_pos[b] + 1;
}

__global__ void __launch_bounds__(256) append_advance_kernel(const __grid_constant__ AppendParams p) {
  if (p.unit_len) {
    // one block per sequence: every unit's length grows by one, unless one is blocked
    const int b = blockIdx.x;
    const int64_t cap_b = p.seg_start[b + 1] - p.seg_start[b];
    const int bad = __syncthreads_or(units_blocked(p, b, cap_b, threadIdx.x, blockDim.x));
    if (bad) return;  // flagged above
    for (int64_t lg = threadIdx.x; lg < (int64_t)p.L * p.Hkv; lg += blockDim.x)
      p.unit_len[lg * p.B + b] += 1;
    if (threadIdx.x == 0) p.cur_pos[b] = p.cur_pos[b] + 1;
    return;
  }
  const int b = threadIdx.x;
  if (b >= p.B) return;
  const int32_t T = p.seq_len[b];
  if (T < 0 || (int64_t)T >= p.seg_start[b + 1] - p.seg_start[b]) return;  // flagged above
  p.seq_len[b] = T + 1;
  p.cur_pos[b] = p.cur_pos[b] + 1;
}

}  // namespace

cudaError_t launch_append(const AppendParams &p, cudaStream_t s) {
  const int64_t threads = (int64_t)p.L * p.Hkv * p.B * 32;
  const int64_t blocks = (threads + 255) / 256;
  if (blocks > INT32_MAX) return cudaErrorInvalidValue;
  append_rows_kernel<<<(unsigned)blocks, 256, 0, s>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  append_advance_kernel<<<p.unit_len ? p.B : 1, 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace tria
