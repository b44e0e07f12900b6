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
// Design (sm_100a): one cluster of CL CTAs per (sequence, KV head), one CTA per
// SM, CL the largest power of two (at most 8) that keeps the launch in one wave.
// (On the tensor-core path, up to 9 pairs with a segment of 8192 slots or more take
// four clusters of 4 each, whose results the pair's last CTA merges.)  CTA r takes the r-th contiguous slice of the live keys
// and walks it in tiles of 16384 / D keys with a running maximum (online
// softmax) for all G query heads of the group, so the group's keys and values are
// read from HBM once.  The tiles stream into three shared-memory stages with bulk
// asynchronous copies (one for the tile's K rows, one for its V rows), the next
// two tiles' copies in flight while the current one is computed.  In a tile, LPK
// lanes score a key, each over D / LPK of its dims with those dims of the query
// heads held in registers, and a butterfly adds their parts; then thread
// (kg, dg) accumulates p * v over columns [dg * VP, dg * VP + VP) of the tile's
// rows kg, kg + KG, ....  Every CTA then combines a slice of the output from the
// CL partial results (running max, sum of exponentials, unnormalised output)
// through distributed shared memory; no workspace and no second kernel.  Float32
// throughout, expf for the weights; every sum is taken in a fixed order.  A
// bounded wait that runs out sets TRIA_DEVERR_TIMEOUT.
#include <cooperative_groups.h>

#include <cuda_bf16.h>
#include <math.h>

#include "attention.cuh"
#include "mma_sync.cuh"

namespace cg = cooperative_groups;

namespace tria {

namespace {

constexpr int kAttnThreads = 256;
constexpr int kAttnNW = kAttnThreads / 32;

__device__ __forceinline__ float bf16_to_f(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

template <int D, int G>
struct AttnShape {
  static constexpr int TILE = 16384 / D;          // keys per tile (32 KB of K, 32 KB of V)
  static constexpr int VROW = 2 * D;              // a K or V row in shared memory (bytes)
  static constexpr int KROW = VROW;
  static constexpr int KST = TILE * KROW, VST = TILE * VROW;
  static constexpr int STAGE = KST + VST;
  static constexpr int VP = G >= 16 ? 4 : 8;      // values of a row per thread in p * v
  // scoring: HQ query heads per pass, LPK lanes per key, DPL dims per lane, so that a
  // lane holds at most 64 query values in registers
  static constexpr int HQ = G * D <= 2048 ? G : 2048 / D;
  static constexpr int LPK0 = HQ * D / 64 < 1 ? 1 : HQ * D / 64;
  static constexpr int LPK = LPK0 > 32 ? 32 : LPK0;
  static constexpr int DPL = D / LPK;
  static_assert(HQ >= 1 && G % HQ == 0 && (LPK & (LPK - 1)) == 0 && DPL * LPK == D, "scoring");
  static_assert(DPL % 8 == 0 || DPL == 4, "16-byte (or 8-byte) key loads");
  static_assert(HQ * DPL <= 64, "query registers");
  static constexpr int DG = D / VP, KG = kAttnThreads / DG;
  static constexpr int NST = 3;                             // stages in flight
  static constexpr int QS = NST * STAGE;                    // float [G][D]
  static constexpr int SC = QS + G * D * 4;                 // float [G][TILE]
  static constexpr int BAR = SC + G * TILE * 4;             // NST mbarriers
  static constexpr int SMEM = BAR + 8 * NST;
  static_assert(DG * VP == D && KG * DG == kAttnThreads && TILE <= kAttnThreads, "shape");
  static_assert(KST % 128 == 0 && STAGE % 128 == 0 && QS % 16 == 0, "aligned regions");
};

template <int D, int G, int CL>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attention_kernel(const __grid_constant__ AttnParams p) {
  using S = AttnShape<D, G>;
  constexpr int TILE = S::TILE, VP = S::VP, DG = S::DG, KG = S::KG;
  extern __shared__ __align__(128) uint8_t sm[];
  float (*qs)[D] = reinterpret_cast<float (*)[D]>(sm + S::QS);  // queries, then partial output
  float (*sc)[TILE] = reinterpret_cast<float (*)[TILE]>(sm + S::SC);
  uint64_t *bar = reinterpret_cast<uint64_t *>(sm + S::BAR);
  __shared__ float mrun[G], lrun[G], alpha[G];
  __shared__ float pm[CL][G], pl[CL][G];
  __shared__ int all_ok;

  cg::cluster_group cl = cg::this_cluster();
  const int r = (int)cl.block_rank();
  const int unit = blockIdx.x / CL;  // b * Hkv + g
  const int b = unit / p.Hkv, g = unit - b * p.Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t cap_b = p.seg_start[b + 1] - p.seg_start[b];
  const int32_t T = p.unit_len ? p.unit_len[((int64_t)p.layer * p.Hkv + g) * p.B + b] : p.seq_len[b];
  if (T < 0 || (int64_t)T > cap_b) {  // the same decision in every CTA of the cluster
    if (r == 0 && tid == 0 && (g == 0 || p.unit_len)) dev::set_error(p.err, TRIA_DEVERR_SEQ_LEN);
    return;
  }
  const int t0 = (int)((int64_t)T * r / CL), t1 = (int)((int64_t)T * (r + 1) / CL);
  const int ntiles = (t1 - t0 + TILE - 1) / TILE;
  const size_t row0 = ((size_t)p.layer * p.Hkv + g) * p.cap + p.seg_start[b];
  const uint8_t *kb = reinterpret_cast<const uint8_t *>(p.k + row0 * D);
  const uint8_t *vb = reinterpret_cast<const uint8_t *>(p.v + row0 * D);
  const uint16_t *qb = p.q + ((size_t)b * p.Hq + (size_t)g * G) * D;

  if (tid == 0) {
#pragma unroll
    for (int q = 0; q < S::NST; ++q) dev::mbar_init(&bar[q], 1);
    dev::fence_mbar_init();
    all_ok = 1;
  }
  for (int i = tid; i < G * D; i += kAttnThreads) (&qs[0][0])[i] = bf16_to_f(qb[i]);
  if (tid < G) {
    mrun[tid] = -INFINITY;
    lrun[tid] = 0.0f;
  }
  __syncthreads();
  // thread 0 streams tile i into stage i % NST: the tile's K rows and its V rows,
  // one bulk copy each (the rows of a segment are contiguous)
  auto issue = [&](int i) {
    const int s = i % S::NST, k0 = t0 + i * TILE, n = min(TILE, t1 - k0);
    uint8_t *st = sm + s * S::STAGE;
    dev::mbar_arrive_expect_tx(&bar[s], (uint32_t)(2 * n * S::VROW));
    dev::bulk_g2s(st, kb + (size_t)k0 * S::VROW, (uint32_t)(n * S::VROW), &bar[s]);
    dev::bulk_g2s(st + S::KST, vb + (size_t)k0 * S::VROW, (uint32_t)(n * S::VROW), &bar[s]);
  };
  if (tid == 0)
    for (int i = 0; i < S::NST && i < ntiles; ++i) issue(i);
  const int dg = tid % DG, kg = tid / DG;
  float acc[G][VP];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < VP; ++e) acc[h][e] = 0.0f;

  for (int i = 0; i < ntiles; ++i) {
    const int s = i % S::NST, n = min(TILE, t1 - (t0 + i * TILE));
    const uint8_t *ks = sm + s * S::STAGE, *vs = ks + S::KST;
    if (!dev::mbar_wait(&bar[s], (uint32_t)(i / S::NST) & 1u)) all_ok = 0;
    __syncthreads();
    if (!all_ok) {  // the copies never arrived: give up on this unit
      if (tid == 0) {
        dev::set_error(p.err, TRIA_DEVERR_TIMEOUT);
        // the other stages' copies (issued for the next tiles) may still land: wait
        // for them, with a limit, before the shared memory is given up
        for (int q = i + 1; q < i + S::NST && q < ntiles; ++q)
          (void)dev::mbar_wait(&bar[q % S::NST], (uint32_t)(q / S::NST) & 1u);
      }
      __syncthreads();
      break;
    }
    // scores: LPK lanes per key, each with DPL of the key's dims (16-byte chunks
    // sub, sub + LPK, ... of the row, so that the lanes of a key read consecutive
    // chunks) and those dims of HQ query heads in registers; the LPK partial dots
    // meet in a butterfly
    {
      constexpr int HQ = S::HQ, LPK = S::LPK, DPL = S::DPL, KPW = 32 / LPK;
      const int sub = lane % LPK, kw = lane / LPK;
#pragma unroll 1
      for (int h0 = 0; h0 < G; h0 += HQ) {
        float qr[HQ][DPL];
#pragma unroll
        for (int h = 0; h < HQ; ++h)
#pragma unroll
          for (int d = 0; d < DPL; ++d)
            qr[h][d] = DPL % 8 == 0 ? qs[h0 + h][((d >> 3) * LPK + sub) * 8 + (d & 7)]
                                    : qs[h0 + h][sub * DPL + d];
        for (int jb = warp * KPW; jb < n; jb += kAttnNW * KPW) {
          const int j = jb + kw;  // (rows at or past n hold stale data: not written out)
          const uint8_t *kr = ks + j * S::KROW;
          float part[HQ];
#pragma unroll
          for (int h = 0; h < HQ; ++h) part[h] = 0.0f;
          if constexpr (DPL % 8 == 0) {
#pragma unroll
            for (int c = 0; c < DPL / 8; ++c) {
              const uint4 w = reinterpret_cast<const uint4 *>(kr)[c * LPK + sub];
              const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const float x0 = bf16_to_f(ws[q] & 0xffffu), x1 = bf16_to_f(ws[q] >> 16);
#pragma unroll
                for (int h = 0; h < HQ; ++h) {
                  part[h] = fmaf(x0, qr[h][8 * c + 2 * q], part[h]);
                  part[h] = fmaf(x1, qr[h][8 * c + 2 * q + 1], part[h]);
                }
              }
            }
          } else {
            const uint2 w = reinterpret_cast<const uint2 *>(kr)[sub];
            const float x[4] = {bf16_to_f(w.x & 0xffffu), bf16_to_f(w.x >> 16),
                                bf16_to_f(w.y & 0xffffu), bf16_to_f(w.y >> 16)};
#pragma unroll
            for (int h = 0; h < HQ; ++h)
#pragma unroll
              for (int d = 0; d < 4; ++d) part[h] = fmaf(x[d], qr[h][d], part[h]);
          }
#pragma unroll
          for (int o = LPK / 2; o > 0; o >>= 1)
#pragma unroll
            for (int h = 0; h < HQ; ++h) part[h] += __shfl_xor_sync(0xffffffffu, part[h], o);
          if (sub == 0 && j < n) {
#pragma unroll
            for (int h = 0; h < HQ; ++h) sc[h0 + h][j] = part[h] * p.scale;
          }
        }
      }
    }
    __syncthreads();
    // running maximum per head (a warp per head)
    for (int h = warp; h < G; h += kAttnNW) {
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
    for (int idx = tid; idx < G * n; idx += kAttnThreads) {
      const int h = idx / n, j = idx - h * n;
      sc[h][j] = expf(sc[h][j] - mrun[h]);
    }
    __syncthreads();
    // sum of the weights (a warp per head) and the weighted values (all threads)
    for (int h = warp; h < G; h += kAttnNW) {
      float sum = 0.0f;
      for (int j = lane; j < n; j += 32) sum += sc[h][j];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (lane == 0) lrun[h] = lrun[h] * alpha[h] + sum;
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float a = alpha[h];
#pragma unroll
      for (int e = 0; e < VP; ++e) acc[h][e] *= a;
    }
    for (int j = kg; j < n; j += KG) {
      const uint8_t *vr = vs + j * S::VROW + dg * VP * 2;
      float x[VP];
      if constexpr (VP == 8) {
        const uint4 w = *reinterpret_cast<const uint4 *>(vr);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          x[2 * q] = bf16_to_f(ws[q] & 0xffffu);
          x[2 * q + 1] = bf16_to_f(ws[q] >> 16);
        }
      } else {
        const uint2 w = *reinterpret_cast<const uint2 *>(vr);
        x[0] = bf16_to_f(w.x & 0xffffu);
        x[1] = bf16_to_f(w.x >> 16);
        x[2] = bf16_to_f(w.y & 0xffffu);
        x[3] = bf16_to_f(w.y >> 16);
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float wt = sc[h][j];
#pragma unroll
        for (int e = 0; e < VP; ++e) acc[h][e] = fmaf(wt, x[e], acc[h][e]);
      }
    }
    __syncthreads();  // stage s, sc, alpha and lrun are free again
    if (tid == 0 && i + S::NST < ntiles) issue(i + S::NST);
  }
  // partial output of this CTA: the key groups' sums, added in key-group order
  for (int i = tid; i < G * D; i += kAttnThreads) (&qs[0][0])[i] = 0.0f;
  __syncthreads();
  for (int k = 0; k < KG; ++k) {
    if (kg == k) {
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < VP; ++e) qs[h][dg * VP + e] += acc[h][e];
    }
    __syncthreads();
  }
  cl.sync();  // every CTA's running max, sum and partial output are complete
  for (int i = tid; i < CL * G; i += kAttnThreads) {
    const int q = i / G, h = i - q * G;
    pm[q][h] = cl.map_shared_rank(&mrun[0], q)[h];
    pl[q][h] = cl.map_shared_rank(&lrun[0], q)[h];
  }
  __syncthreads();
  // CTA r writes its slice of the G * D outputs
  float *outb = p.out + ((size_t)b * p.Hq + (size_t)g * G) * D;
  const int e0 = G * D * r / CL, e1 = G * D * (r + 1) / CL;
  for (int i = e0 + tid; i < e1; i += kAttnThreads) {
    const int h = i / D;
    float M = -INFINITY;
#pragma unroll
    for (int q = 0; q < CL; ++q) M = fmaxf(M, pm[q][h]);
    float L = 0.0f, O = 0.0f;
    if (M != -INFINITY) {
      float part[CL];
#pragma unroll
      for (int q = 0; q < CL; ++q) part[q] = cl.map_shared_rank(&qs[0][0], q)[i];
#pragma unroll
      for (int q = 0; q < CL; ++q) {
        const float e = pm[q][h] == -INFINITY ? 0.0f : expf(pm[q][h] - M);
        L = fmaf(pl[q][h], e, L);
        O = fmaf(part[q], e, O);
      }
    }
    outb[i] = L > 0.0f ? O / L : 0.0f;
  }
  cl.sync();  // the peers' shared memory stays valid until every CTA has read it
}

// ------------------------------------------------------------------ tensor-core path
// For D = 64 or 128 and G <= 8 the two products of a tile run on the tensor cores
// (mma.sync m16n8k16, bf16 inputs, float32 accumulators):
//   S^T = K Q^T     warp w scores keys [16w, 16w + 16) of the tile for the G heads
//                   (padded to 8); K comes straight from the TMA-swizzled stage
//                   and the queries stay in registers.  bf16 x bf16 products are
//                   exact, so the scores equal the float32 dot products up to the
//                   order of the additions.
//   O^T += V^T P^T  warp w owns 16 of the output dims (D = 64: 16 dims and half of
//                   the tile's keys); P (the exponentials, in [0, 1]) is written to
//                   shared memory as a bf16 pair hi + lo (16 significant bits), and
//                   both parts multiply V, so the weights keep float32-level accuracy.
// The tiles stream in by 2-D TMA loads with 128-byte swizzle; rows of the last tile
// past the slice are masked out of the softmax, and their V rows are zeroed.
template <int D>
struct MmaShape {
  static constexpr int TILE = 128;
  static constexpr int NBOX = D / 64;
  static constexpr int BOXB = TILE * 128;             // one box: 128 rows x 64 dims
  static constexpr int TB = NBOX * BOXB;              // a tile's K (or V)
  static constexpr int STAGE = 2 * TB;
  static constexpr int NST = D == 64 ? 4 : 3;
  static constexpr int PROW = TILE * 2 + 16;          // bytes per head row of P^T (padded)
  static constexpr int OFF_Q = NST * STAGE;           // bf16 [8][D] queries
  static constexpr int OFF_P = OFF_Q + 8 * D * 2;     // bf16 [2][8][PROW / 2]: hi, lo
  static constexpr int OFF_O = OFF_P + 2 * 8 * PROW;  // float [8][D] partial output
  static constexpr int OFF_W = OFF_O + 8 * D * 4;     // float [2][8 warps][8]: max, sum
  static constexpr int OFF_BAR = OFF_W + 2 * 64 * 4;
  static constexpr int SMEM = OFF_BAR + 8 * NST + 1024;  // + room to align to 1024
  static_assert(D == 64 || D == 128, "tensor-core path");
};

template <int D, int G, int CL, int SPLIT>
__global__ void __launch_bounds__(256, 1)
    attention_mma_kernel(const __grid_constant__ AttnParams p) {
  using M = MmaShape<D>;
  constexpr int TILE = M::TILE, NBOX = M::NBOX, NST = M::NST, KS = D / 16;
  static_assert(G <= 8, "heads padded to 8");
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = smem_raw + ((1024u - (dev::smem_addr(smem_raw) & 1023u)) & 1023u);
  uint16_t *qsm = reinterpret_cast<uint16_t *>(sm + M::OFF_Q);
  uint8_t *pt = sm + M::OFF_P;
  float *osm = reinterpret_cast<float *>(sm + M::OFF_O);
  float *wmx = reinterpret_cast<float *>(sm + M::OFF_W);
  float *wsm = wmx + 64;
  uint64_t *bar = reinterpret_cast<uint64_t *>(sm + M::OFF_BAR);
  __shared__ float mrun[8], lrun[8];
  __shared__ float pm[CL][8], pl[CL][8];
  __shared__ int all_ok;

  cg::cluster_group cl = cg::this_cluster();
  const int r = (int)cl.block_rank();
  const int ci = blockIdx.x / CL;                // cluster
  const int unit = ci / SPLIT, half = ci % SPLIT;  // unit = b * Hkv + g
  const int b = unit / p.Hkv, g = unit - b * p.Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t cap_b = p.seg_start[b + 1] - p.seg_start[b];
  // the queries (bf16 [8][D], heads past G zero) load alongside the live length
  constexpr int QW = 4 * D / 256;  // 32-bit words of the queries per thread
  const uint16_t *qb = p.q + ((size_t)b * p.Hq + (size_t)g * G) * D;
  uint32_t qv[QW];
#pragma unroll
  for (int k = 0; k < QW; ++k) {
    const int w = tid + 256 * k;
    qv[k] = w < G * D / 2 ? reinterpret_cast<const uint32_t *>(qb)[w] : 0u;
  }
  if (tid == 0) {
    // the tensor maps' descriptors travel to the TMA unit meanwhile
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.tk)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.tv)) : "memory");
  }
  const int32_t T = p.unit_len ? p.unit_len[((int64_t)p.layer * p.Hkv + g) * p.B + b] : p.seq_len[b];
  if (T < 0 || (int64_t)T > cap_b) {  // the same decision in every CTA of the unit
    if (r == 0 && half == 0 && tid == 0 && (g == 0 || p.unit_len))
      dev::set_error(p.err, TRIA_DEVERR_SEQ_LEN);
    return;
  }
  // the unit's keys are split over SPLIT * CL CTAs
  const int part = half * CL + r;
  const int t0 = (int)((int64_t)T * part / (SPLIT * CL));
  const int t1 = (int)((int64_t)T * (part + 1) / (SPLIT * CL));
  const int ntiles = (t1 - t0 + TILE - 1) / TILE;
  // tensor row of the segment's slot 0 (the host checked that every row fits int32)
  const int32_t y0 = (int32_t)(((int64_t)p.layer * p.Hkv + g) * p.cap + p.seg_start[b]);

  auto issue = [&](int i) {  // thread 0: tile i into stage i % NST
    const int s = i % NST;
    uint8_t *st = sm + s * M::STAGE;
    const int32_t y = y0 + t0 + i * TILE;
    // the stage's earlier contents were read (and its V tail zeroed) through the
    // generic proxy: order that before the tensor copies overwrite it
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    dev::mbar_arrive_expect_tx(&bar[s], (uint32_t)M::STAGE);
#pragma unroll
    for (int bx = 0; bx < NBOX; ++bx) {
      dev::tma_load_2d(st + bx * M::BOXB, &p.tk, bx * 64, y, &bar[s]);
      dev::tma_load_2d(st + M::TB + bx * M::BOXB, &p.tv, bx * 64, y, &bar[s]);
    }
  };
  if (tid == 0) {
#pragma unroll
    for (int q = 0; q < NST; ++q) dev::mbar_init(&bar[q], 1);
    dev::fence_mbar_init();
    all_ok = 1;
    for (int i = 0; i < NST && i < ntiles; ++i) issue(i);  // before the queries are stored
  }
#pragma unroll
  for (int k = 0; k < QW; ++k) reinterpret_cast<uint32_t *>(qsm)[tid + 256 * k] = qv[k];
  if (tid < 8) {
    mrun[tid] = -INFINITY;
    lrun[tid] = 0.0f;
  }
  __syncthreads();

  // queries as the B operand of S^T = K Q^T, one fragment pair per 16 dims
  uint32_t qf[KS][2];
  {
    const uint32_t qa = dev::smem_addr(qsm) + (uint32_t)((lane & 7) * D * 2 + ((lane >> 3) & 1) * 16);
#pragma unroll
    for (int t = 0; t < KS; ++t) ldsm_x2(qa + t * 32, qf[t]);
  }
  const int hA = 2 * (lane & 3), hB = hA + 1;  // the heads of this lane's accumulators
  // O^T: dims dm + lane / 4 (+ 8), heads hA, hB; the P hi and lo products apart
  float o[4] = {0.0f, 0.0f, 0.0f, 0.0f}, ol[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  const int dm = D == 128 ? 16 * warp : 16 * (warp & 3);
  const int j0 = D == 128 ? 0 : 4 * (warp >> 2), j1 = D == 128 ? 8 : j0 + 4;
  const uint32_t pth = dev::smem_addr(pt), ptl = pth + 8 * M::PROW;
  uint16_t *pth_g = reinterpret_cast<uint16_t *>(pt), *ptl_g = pth_g + 4 * M::PROW;

  for (int i = 0; i < ntiles; ++i) {
    const int s = i % NST, n = min(TILE, t1 - (t0 + i * TILE));
    uint8_t *ks = sm + s * M::STAGE, *vs = ks + M::TB;
    if (!dev::mbar_wait(&bar[s], (uint32_t)(i / NST) & 1u)) all_ok = 0;
    // the V rows past the slice are zeroed (they may hold anything)
    for (int idx = tid; idx < (TILE - n) * NBOX * 8; idx += 256) {
      const int row = n + idx / (NBOX * 8), rest = idx % (NBOX * 8);
      *reinterpret_cast<uint4 *>(vs + (rest >> 3) * M::BOXB + row * 128 + (rest & 7) * 16) =
          make_uint4(0u, 0u, 0u, 0u);
    }
    // S^T for keys [16 warp, 16 warp + 16)
    float sacc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    {
      // even and odd 16-dim steps in two accumulator chains
      float s2[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      const int mat = lane >> 3, key = 16 * warp + (mat & 1) * 8 + (lane & 7);
      const uint32_t kb = dev::smem_addr(ks);
#pragma unroll
      for (int t = 0; t < KS; t += 2) {
        uint32_t a[4], a2[4];
        ldsm_x4(swz<M::BOXB>(kb, key, 16 * t + (mat >> 1) * 8), a);
        ldsm_x4(swz<M::BOXB>(kb, key, 16 * (t + 1) + (mat >> 1) * 8), a2);
        mma_bf16(sacc, a, qf[t]);
        mma_bf16(s2, a2, qf[t + 1]);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) sacc[e] += s2[e];
    }
    const int keyA = 16 * warp + (lane >> 2), keyB = keyA + 8;
    float sv[4];
    sv[0] = keyA < n ? sacc[0] * p.scale : -INFINITY;
    sv[1] = keyA < n ? sacc[1] * p.scale : -INFINITY;
    sv[2] = keyB < n ? sacc[2] * p.scale : -INFINITY;
    sv[3] = keyB < n ? sacc[3] * p.scale : -INFINITY;
    float mA = fmaxf(sv[0], sv[2]), mB = fmaxf(sv[1], sv[3]);
#pragma unroll
    for (int o2 = 4; o2 < 32; o2 <<= 1) {
      mA = fmaxf(mA, __shfl_xor_sync(0xffffffffu, mA, o2));
      mB = fmaxf(mB, __shfl_xor_sync(0xffffffffu, mB, o2));
    }
    if (lane < 4) {
      wmx[warp * 8 + hA] = mA;
      wmx[warp * 8 + hB] = mB;
    }
    __syncthreads();
    if (!all_ok) {  // the copies never arrived: give up on this unit
      if (tid == 0) {
        dev::set_error(p.err, TRIA_DEVERR_TIMEOUT);
        for (int q = i + 1; q < i + NST && q < ntiles; ++q)
          (void)dev::mbar_wait(&bar[q % NST], (uint32_t)(q / NST) & 1u);
      }
      __syncthreads();
      break;
    }
    // new running maxima of this lane's heads (the tile has at least one key)
    float tmA = -INFINITY, tmB = -INFINITY;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      tmA = fmaxf(tmA, wmx[w * 8 + hA]);
      tmB = fmaxf(tmB, wmx[w * 8 + hB]);
    }
    const float MA = fmaxf(mrun[hA], tmA), MB = fmaxf(mrun[hB], tmB);
    const float alA = mrun[hA] == -INFINITY ? 0.0f : expf(mrun[hA] - MA);
    const float alB = mrun[hB] == -INFINITY ? 0.0f : expf(mrun[hB] - MB);
    float pv[4];
    pv[0] = expf(sv[0] - MA);
    pv[1] = expf(sv[1] - MB);
    pv[2] = expf(sv[2] - MA);
    pv[3] = expf(sv[3] - MB);
    float sA = pv[0] + pv[2], sB = pv[1] + pv[3];
#pragma unroll
    for (int o2 = 4; o2 < 32; o2 <<= 1) {
      sA += __shfl_xor_sync(0xffffffffu, sA, o2);
      sB += __shfl_xor_sync(0xffffffffu, sB, o2);
    }
    if (lane < 4) {
      wsm[warp * 8 + hA] = sA;
      wsm[warp * 8 + hB] = sB;
    }
    // P^T as bf16 hi + lo: row = head, column = key
    {
      const int keys[4] = {keyA, keyA, keyB, keyB}, heads[4] = {hA, hB, hA, hB};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const __nv_bfloat16 hi = __float2bfloat16_rn(pv[e]);
        const __nv_bfloat16 lo = __float2bfloat16_rn(pv[e] - __bfloat162float(hi));
        const int at = heads[e] * (M::PROW / 2) + keys[e];
        pth_g[at] = __bfloat16_as_ushort(hi);
        ptl_g[at] = __bfloat16_as_ushort(lo);
      }
    }
    __syncthreads();
    // O^T = alpha O^T + V^T P^T over this warp's dims (and, for D = 64, half of the keys)
    o[0] *= alA;
    o[1] *= alB;
    o[2] *= alA;
    o[3] *= alB;
    ol[0] *= alA;
    ol[1] *= alB;
    ol[2] *= alA;
    ol[3] *= alB;
    {
      const int mat = lane >> 3;
      const uint32_t vb = dev::smem_addr(vs);
      const uint32_t pa = (uint32_t)((lane & 7) * M::PROW + ((lane >> 3) & 1) * 16);
#pragma unroll
      for (int j = j0; j < j1; ++j) {
        uint32_t a[4], bh[2], bl[2];
        ldsm_x4_t(swz<M::BOXB>(vb, 16 * j + (mat >> 1) * 8 + (lane & 7), dm + (mat & 1) * 8), a);
        ldsm_x2(pth + pa + 32 * j, bh);
        ldsm_x2(ptl + pa + 32 * j, bl);
        mma_bf16(o, a, bh);
        mma_bf16(ol, a, bl);
      }
    }
    if (tid < 8) {  // running max and sum of head tid (every thread has read them)
      float tm = -INFINITY, ts = 0.0f;
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        tm = fmaxf(tm, wmx[w * 8 + tid]);
        ts += wsm[w * 8 + tid];
      }
      const float Mn = fmaxf(mrun[tid], tm);
      const float al = mrun[tid] == -INFINITY ? 0.0f : expf(mrun[tid] - Mn);
      lrun[tid] = lrun[tid] * al + ts;
      mrun[tid] = Mn;
    }
    __syncthreads();  // stage s, P^T and the warp arrays are free again
    if (tid == 0 && i + NST < ntiles) issue(i + NST);
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) o[e] += ol[e];
  // this CTA's unnormalised output O[h][d] (D = 64: the two key halves added in order)
  const int dA = dm + (lane >> 2), dB = dA + 8;
  if (D == 128 || warp < 4) {
    osm[hA * D + dA] = o[0];
    osm[hB * D + dA] = o[1];
    osm[hA * D + dB] = o[2];
    osm[hB * D + dB] = o[3];
  }
  if (D == 64) {
    __syncthreads();
    if (warp >= 4) {
      osm[hA * D + dA] += o[0];
      osm[hB * D + dA] += o[1];
      osm[hA * D + dB] += o[2];
      osm[hB * D + dB] += o[3];
    }
  }
  __syncthreads();
  cl.sync();  // every CTA's running max, sum and partial output are complete
  for (int i = tid; i < CL * 8; i += 256) {
    const int q = i / 8, h = i - q * 8;
    pm[q][h] = cl.map_shared_rank(&mrun[0], q)[h];
    pl[q][h] = cl.map_shared_rank(&lrun[0], q)[h];
  }
  __syncthreads();
  float *outb = p.out + ((size_t)b * p.Hq + (size_t)g * G) * D;
  // SPLIT > 1: this cluster's result (its max, sum and unnormalised output per head)
  float *mine = SPLIT > 1 ? p.scratch + ((size_t)unit * SPLIT + half) * (16 + 8 * D) : nullptr;
  if (SPLIT > 1 && r == 0 && tid < G) {
    float Mx = -INFINITY, L = 0.0f;
    for (int q = 0; q < CL; ++q) Mx = fmaxf(Mx, pm[q][tid]);
    if (Mx != -INFINITY)
      for (int q = 0; q < CL; ++q)
        L = fmaf(pl[q][tid], pm[q][tid] == -INFINITY ? 0.0f : expf(pm[q][tid] - Mx), L);
    mine[tid] = Mx;
    mine[8 + tid] = L;
  }
  const int e0 = G * D * r / CL, e1 = G * D * (r + 1) / CL;
  for (int i = e0 + tid; i < e1; i += 256) {
    const int h = i / D;
    float Mx = -INFINITY;
#pragma unroll
    for (int q = 0; q < CL; ++q) Mx = fmaxf(Mx, pm[q][h]);
    float L = 0.0f, O = 0.0f;
    if (Mx != -INFINITY) {
      float part[CL];
#pragma unroll
      for (int q = 0; q < CL; ++q) part[q] = cl.map_shared_rank(osm, q)[i];
#pragma unroll
      for (int q = 0; q < CL; ++q) {
        const float e = pm[q][h] == -INFINITY ? 0.0f : expf(pm[q][h] - Mx);
        L = fmaf(pl[q][h], e, L);
        O = fmaf(part[q], e, O);
      }
    }
    if (SPLIT > 1) mine[16 + i] = O;
    else outb[i] = L > 0.0f ? O / L : 0.0f;
  }
  cl.sync();  // the peers' shared memory stays valid until every CTA has read it
  if constexpr (SPLIT > 1) {
    // the last of the unit's CTAs to finish merges the SPLIT clusters' results
    __shared__ int last;
    __threadfence();  // this thread's part of the cluster's result is visible device-wide
    __syncthreads();
    if (tid == 0) last = atomicAdd(p.counters + unit, 1) == SPLIT * CL - 1;
    __syncthreads();
    if (last) {
      __threadfence();
      const float *r0 = p.scratch + (size_t)unit * SPLIT * (16 + 8 * D);
      for (int i = tid; i < G * D; i += 256) {
        const int h = i / D;
        float m[SPLIT], l[SPLIT], oq[SPLIT], Mx = -INFINITY;
#pragma unroll
        for (int q = 0; q < SPLIT; ++q) {  // every load issued before any is used
          m[q] = __ldcg(r0 + q * (16 + 8 * D) + h);
          l[q] = __ldcg(r0 + q * (16 + 8 * D) + 8 + h);
          oq[q] = __ldcg(r0 + q * (16 + 8 * D) + 16 + i);
        }
#pragma unroll
        for (int q = 0; q < SPLIT; ++q) Mx = fmaxf(Mx, m[q]);
        float O = 0.0f, L = 0.0f;
        if (Mx != -INFINITY) {
#pragma unroll
          for (int q = 0; q < SPLIT; ++q) {
            const float a = m[q] == -INFINITY ? 0.0f : expf(m[q] - Mx);
            L = fmaf(l[q], a, L);
            O = fmaf(oq[q], a, O);
          }
        }
        outb[i] = L > 0.0f ? O / L : 0.0f;
      }
      if (tid == 0) p.counters[unit] = 0;  // zero at rest for the next call
    }
  }
}

template <int D, int G, int CL, int SPLIT>
cudaError_t launch_mma_dgs(const AttnParams &p, cudaStream_t s, int units) {
  using M = MmaShape<D>;
  auto kern = attention_mma_kernel<D, G, CL, SPLIT>;
  static bool set[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  if (dev < 0 || dev >= 64 || !set[dev]) {
    const cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, M::SMEM);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) set[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)units * CL * SPLIT, 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.dynamicSmemBytes = M::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

template <int D, int G, int CL>
cudaError_t launch_mma_dg(const AttnParams &p, cudaStream_t s, int units) {
  if constexpr (CL == 4) {
    if (p.split == 4) return launch_mma_dgs<D, G, 4, 4>(p, s, units);
  }
  return launch_mma_dgs<D, G, CL, 1>(p, s, units);
}

template <int D, int CL>
cudaError_t launch_mma_d(const AttnParams &p, cudaStream_t s, int units) {
  switch (p.G) {
    case 1: return launch_mma_dg<D, 1, CL>(p, s, units);
    case 2: return launch_mma_dg<D, 2, CL>(p, s, units);
    case 4: return launch_mma_dg<D, 4, CL>(p, s, units);
    case 8: return launch_mma_dg<D, 8, CL>(p, s, units);
    default: return cudaErrorInvalidValue;
  }
}

template <int CL>
cudaError_t launch_mma_cl(const AttnParams &p, cudaStream_t s, int units) {
  return p.D == 64 ? launch_mma_d<64, CL>(p, s, units) : launch_mma_d<128, CL>(p, s, units);
}

template <int D, int G, int CL>
cudaError_t launch_dg(const AttnParams &p, cudaStream_t s, int units) {
  using S = AttnShape<D, G>;
  auto kern = attention_kernel<D, G, CL>;
  static bool set[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  if (dev < 0 || dev >= 64 || !set[dev]) {
    const cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) set[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)units * CL, 1, 1);
  cfg.blockDim = dim3(kAttnThreads, 1, 1);
  cfg.dynamicSmemBytes = S::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

template <int D, int CL>
cudaError_t launch_d(const AttnParams &p, cudaStream_t s, int units) {
  switch (p.G) {
    case 1: return launch_dg<D, 1, CL>(p, s, units);
    case 2: return launch_dg<D, 2, CL>(p, s, units);
    case 4: return launch_dg<D, 4, CL>(p, s, units);
    case 8: return launch_dg<D, 8, CL>(p, s, units);
    case 16: return launch_dg<D, 16, CL>(p, s, units);
    default: return cudaErrorInvalidValue;
  }
}

template <int CL>
cudaError_t launch_cl(const AttnParams &p, cudaStream_t s, int units) {
  switch (p.D) {
    case 64: return launch_d<64, CL>(p, s, units);
    case 128: return launch_d<128, CL>(p, s, units);
    case 256: return launch_d<256, CL>(p, s, units);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

bool attention_supported(int D, int G) {
  return (D == 64 || D == 128 || D == 256) && (G == 1 || G == 2 || G == 4 || G == 8 || G == 16);
}

bool attention_mma_supported(int D, int G) {
  return (D == 64 || D == 128) && (G == 1 || G == 2 || G == 4 || G == 8);
}

cudaError_t launch_attention(const AttnParams &p, cudaStream_t s) {
  const int64_t units = (int64_t)p.B * p.Hkv;
  if (units * 16 > INT32_MAX) return cudaErrorInvalidValue;
  int sms = 148;
  {
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess)
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms < 1) sms = 148;
  }
  // one CTA per SM: the largest cluster (a power of two up to 8) that keeps the
  // launch in one wave (a B200 holds 15 clusters of 8 such CTAs at once, 33 of 4,
  // 74 of 2)
  int cl = 1;
  while (cl < 8 && units * cl * 2 <= sms) cl *= 2;
  if (p.mma) {
    // few (sequence, KV head) pairs: four 4-CTA clusters each (a B200 holds 33 such
    // clusters at once, but only 15 of 8), merged by the unit's last CTA
    if (p.split == 4 && units * 16 <= sms) return launch_mma_cl<4>(p, s, (int)units);
    AttnParams q = p;
    q.split = 1;
    switch (cl) {
      case 1: return launch_mma_cl<1>(q, s, (int)units);
      case 2: return launch_mma_cl<2>(q, s, (int)units);
      case 4: return launch_mma_cl<4>(q, s, (int)units);
      default: return launch_mma_cl<8>(q, s, (int)units);
    }
  }
  switch (cl) {
    case 1: return launch_cl<1>(p, s, (int)units);
    case 2: return launch_cl<2>(p, s, (int)units);
    case 4: return launch_cl<4>(p, s, (int)units);
    default: return launch_cl<8>(p, s, (int)units);
  }
}

}  // namespace tria
