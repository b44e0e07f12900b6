// Decode attention over the pruned cache: the step after the prune in a decode
// loop (romaanj.github.io review, "Results": decoding reads the budgeted cache;
// dimensionstp.github.io review, section 6, Limitations: in serving the pruned
// cache meets the attention kernel).  One new query token per sequence; for each
// query head h of KV head g = h / G
//   out[b][h] = sum_t softmax_t(scale * q[b][h] . k_t) v_t,  t < seq_len[b]
// (or t < the unit's own length, when the cache has per-unit lengths).
// The cache holds post-RoPE keys, so the (non-contiguous) positions of the
// surviving keys play no part.
//
// Design (sm_100a): one 8-CTA cluster per (sequence, KV head); CTA r takes the
// r-th contiguous slice of the live keys and walks it in tiles of 256 keys with
// a running maximum (online softmax) for all G query heads of the group, so the
// group's keys and values are read from HBM once.  In a tile, thread i scores
// key i against the G queries (16-byte loads of its key row, queries broadcast
// from shared memory), then threads split the head dimension (and, for D < 256,
// the tile's keys) to accumulate p * v with coalesced loads of each value row.
// The eight partial results (running max, sum of exponentials, unnormalised
// output) are combined by rank 0 through distributed shared memory; no
// workspace and no second kernel.  Float32 throughout, expf for the weights.
#include <cooperative_groups.h>

#include <math.h>

#include "attention.cuh"

namespace cg = cooperative_groups;

namespace tria {

namespace {

constexpr int kAttnCluster = 8;
constexpr int kAttnThreads = 256;
constexpr int kAttnTile = 256;  // keys per tile: one per thread when scoring

__device__ __forceinline__ float bf16_to_f(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

template <int D, int G>
__global__ void __cluster_dims__(kAttnCluster, 1, 1) __launch_bounds__(kAttnThreads, 1)
    attention_kernel(const __grid_constant__ AttnParams p) {
  constexpr int KG = kAttnThreads / D;  // key groups in the p*v pass
  static_assert(KG >= 1 && KG * D == kAttnThreads, "D divides the block");
  __shared__ __align__(16) float qo[G][D];          // the queries, later the partial output
  __shared__ __align__(16) float sc[G][kAttnTile];  // tile scores / weights, later p*v partials
  __shared__ float mrun[G], lrun[G], alpha[G];

  cg::cluster_group cl = cg::this_cluster();
  const int r = (int)cl.block_rank();
  const int unit = blockIdx.x / kAttnCluster;  // b * Hkv + g
  const int b = unit / p.Hkv, g = unit - b * p.Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t cap_b = p.seg_start[b + 1] - p.seg_start[b];
  const int32_t T = p.unit_len ? p.unit_len[((int64_t)p.layer * p.Hkv + g) * p.B + b] : p.seq_len[b];
  if (T < 0 || (int64_t)T > cap_b) {  // the same decision in every CTA of the cluster
    if (r == 0 && tid == 0 && (g == 0 || p.unit_len)) dev::set_error(p.err, TRIA_DEVERR_SEQ_LEN);
    return;
  }
  const int t0 = (int)((int64_t)T * r / kAttnCluster), t1 = (int)((int64_t)T * (r + 1) / kAttnCluster);
  const size_t row0 = ((size_t)p.layer * p.Hkv + g) * p.cap + p.seg_start[b];
  const uint16_t *kb = p.k + row0 * D;
  const uint16_t *vb = p.v + row0 * D;
  const uint16_t *qb = p.q + ((size_t)b * p.Hq + (size_t)g * G) * D;

  for (int i = tid; i < G * D; i += kAttnThreads) (&qo[0][0])[i] = bf16_to_f(qb[i]);
  if (tid < G) {
    mrun[tid] = -INFINITY;
    lrun[tid] = 0.0f;
  }
  const int d = tid % D, kg = tid / D;
  float acc[G];
#pragma unroll
  for (int h = 0; h < G; ++h) acc[h] = 0.0f;
  __syncthreads();

  for (int tile = t0; tile < t1; tile += kAttnTile) {
    const int n = min(kAttnTile, t1 - tile);
    // scores of key tile + tid against the G queries
    if (tid < n) {
      const uint4 *kr = reinterpret_cast<const uint4 *>(kb + (size_t)(tile + tid) * D);
      float s[G];
#pragma unroll
      for (int h = 0; h < G; ++h) s[h] = 0.0f;
#pragma unroll 8
      for (int i = 0; i < D / 8; ++i) {
        const uint4 w = __ldg(kr + i);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float x0 = bf16_to_f(ws[j] & 0xffffu), x1 = bf16_to_f(ws[j] >> 16);
#pragma unroll
          for (int h = 0; h < G; ++h) {
            s[h] = fmaf(x0, qo[h][8 * i + 2 * j], s[h]);
            s[h] = fmaf(x1, qo[h][8 * i + 2 * j + 1], s[h]);
          }
        }
      }
#pragma unroll
      for (int h = 0; h < G; ++h) sc[h][tid] = s[h] * p.scale;
    }
    __syncthreads();
    // running maximum per head (a warp per head)
    for (int h = warp; h < G; h += kAttnThreads / 32) {
      float mx = -INFINITY;
      for (int j = lane; j < n; j += 32) mx = fmaxf(mx, sc[h][j]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      if (lane == 0) {
        const float mnew = fmaxf(mrun[h], mx);
        alpha[h] = mrun[h] == -INFINITY ? 0.0f : expf(mrun[h] - mnew);
        mrun[h] = mnew;
      }
    }
    __syncthreads();
    if (tid < n) {
#pragma unroll
      for (int h = 0; h < G; ++h) sc[h][tid] = expf(sc[h][tid] - mrun[h]);
    }
    __syncthreads();
    // sum of the weights (a warp per head) and the weighted values (all threads)
    for (int h = warp; h < G; h += kAttnThreads / 32) {
      float sum = 0.0f;
      for (int j = lane; j < n; j += 32) sum += sc[h][j];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (lane == 0) lrun[h] = lrun[h] * alpha[h] + sum;
    }
#pragma unroll
    for (int h = 0; h < G; ++h) acc[h] *= alpha[h];
    // eight value loads in flight per thread, then their products in key order
    int j = kg;
    for (; j + 7 * KG < n; j += 8 * KG) {
      float vv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) vv[u] = bf16_to_f(__ldg(vb + (size_t)(tile + j + u * KG) * D + d));
#pragma unroll
      for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int h = 0; h < G; ++h) acc[h] = fmaf(sc[h][j + u * KG], vv[u], acc[h]);
    }
    for (; j < n; j += KG) {
      const float vv = bf16_to_f(__ldg(vb + (size_t)(tile + j) * D + d));
#pragma unroll
      for (int h = 0; h < G; ++h) acc[h] = fmaf(sc[h][j], vv, acc[h]);
    }
    __syncthreads();  // sc, alpha and lrun are rewritten by the next tile
  }
  // partial output of this CTA: the key groups' sums, into qo (the queries are done)
  float *part = &sc[0][0];  // [KG][G][D] = kAttnThreads * G floats
#pragma unroll
  for (int h = 0; h < G; ++h) part[((size_t)kg * G + h) * D + d] = acc[h];
  __syncthreads();
  for (int i = tid; i < G * D; i += kAttnThreads) {
    float o = 0.0f;
    for (int k = 0; k < KG; ++k) o += part[(size_t)k * G * D + i];
    (&qo[0][0])[i] = o;
  }
  cl.sync();  // every CTA's running max, sum and partial output are complete
  if (r == 0) {
    float *outb = p.out + ((size_t)b * p.Hq + (size_t)g * G) * D;
    for (int i = tid; i < G * D; i += kAttnThreads) {
      const int h = i / D;
      float M = -INFINITY;
#pragma unroll
      for (int q = 0; q < kAttnCluster; ++q) M = fmaxf(M, cl.map_shared_rank(&mrun[0], q)[h]);
      float L = 0.0f, O = 0.0f;
      if (M != -INFINITY) {
#pragma unroll
        for (int q = 0; q < kAttnCluster; ++q) {
          const float mq = cl.map_shared_rank(&mrun[0], q)[h];
          const float e = mq == -INFINITY ? 0.0f : expf(mq - M);
          L = fmaf(cl.map_shared_rank(&lrun[0], q)[h], e, L);
          O = fmaf(cl.map_shared_rank(&qo[0][0], q)[i], e, O);
        }
      }
      outb[i] = L > 0.0f ? O / L : 0.0f;
    }
  }
  cl.sync();  // the peers' shared memory stays valid until rank 0 has read it
}

template <int D>
cudaError_t launch_d(const AttnParams &p, cudaStream_t s, unsigned grid) {
  switch (p.G) {
    case 1: attention_kernel<D, 1><<<grid, kAttnThreads, 0, s>>>(p); break;
    case 2: attention_kernel<D, 2><<<grid, kAttnThreads, 0, s>>>(p); break;
    case 4: attention_kernel<D, 4><<<grid, kAttnThreads, 0, s>>>(p); break;
    case 8: attention_kernel<D, 8><<<grid, kAttnThreads, 0, s>>>(p); break;
    case 16: attention_kernel<D, 16><<<grid, kAttnThreads, 0, s>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace

bool attention_supported(int D, int G) {
  return (D == 64 || D == 128 || D == 256) && (G == 1 || G == 2 || G == 4 || G == 8 || G == 16);
}

cudaError_t launch_attention(const AttnParams &p, cudaStream_t s) {
  const int64_t grid = (int64_t)p.B * p.Hkv * kAttnCluster;
  if (grid > INT32_MAX) return cudaErrorInvalidValue;
  switch (p.D) {
    case 64: return launch_d<64>(p, s, (unsigned)grid);
    case 128: return launch_d<128>(p, s, (unsigned)grid);
    case 256: return launch_d<256>(p, s, (unsigned)grid);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace tria
