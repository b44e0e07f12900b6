// Raw key scores, one streaming pass over the cached keys.
//
// For every live key t of every (layer l, KV head g, sequence b) and every
// query head h of g's group (romaanj.github.io review, "Method";
// dimensionstp.github.io review, sections 2-2 and 3-2 (2)-(4)):
//   s_h(t) = sum_f [ Re(conj(ktilde_f) * W_hf) + Nw_hf * |ktilde_f| ]
//   W_hf   = c_hf * EA_bf          (trig term with offsets and cur folded in, see fold.cu)
//   Nw_hf  = (1 - R_hf) * E|q_hf|  (norm term; |k_f| = |ktilde_f| since RoPE keeps norms)
// ktilde is the stored post-RoPE bf16 key widened exactly to float; all sums
// are float32.
//
// Design (sm_100a): a persistent grid, one CTA per SM, each taking a
// contiguous run of key chunks (32 to 128 keys, 8 to 16 KB).  One producer
// thread streams the live chunks into a ring of shared-memory slots with 2-D
// TMA tensor loads (128-byte swizzled boxes of 64 head-dim elements, no
// multicast) and tags each slot with a descriptor; eight consumer warps take
// the slots round-robin, each warp a whole chunk.  A consumer lane scores KPT
// whole keys: it reads its rows from the swizzled boxes (conflict-free across
// the warp), widens bf16 pairs to float, forms |k_f| and accumulates all G
// heads with the paired FP32 FMA of sm_100 (__ffma2_rn on two RoPE pairs at a
// time).  The folded weights of a unit (3 KB at D = 128, G = 4) are brought
// into one of two shared-memory weight slots by a bulk copy when the producer
// reaches the unit, and read as broadcasts.  No cross-lane reduction and no
// synchronisation between consumer warps are needed.  For D <= 128 and G <= 8 a
// second consumer form scores each 16-key block on the tensor cores instead (see
// "tensor-core form" below); the launch takes it at G = 8, or when a CTA scores many
// chunks.
#include <cudaTypedefs.h>

#include <mutex>

#include "mma_sync.cuh"
#include "tria_internal.cuh"

namespace tria {

template <int D, int G>
struct ScoreShape {
  static constexpr int F = D / 2;
  static constexpr int FP = F / 2;                                 // RoPE pair pairs
  static constexpr int KPT_D = 256 / D;                            // 16 KB chunks
  // keys per lane: bounded by the FMA form's accumulator registers, except at G = 8 with
  // D <= 128, which always takes the tensor-core form (64-key chunks: 276 against 349 us
  // for 32-key chunks on 4 x 131072 keys)
  static constexpr int KPT_G = G <= 2 ? 4 : (G == 4 ? 2 : (G == 8 && D <= 128 ? 2 : 1));
  static constexpr int KPT0 = KPT_D < KPT_G ? KPT_D : KPT_G;
  static constexpr int KPT = KPT0 < kScoreKptCap ? KPT0 : kScoreKptCap;  // keys per lane
  static constexpr int CH = 32 * KPT;                              // keys per chunk
  static constexpr int NBOX = D / 64;                              // 128-byte boxes per row
  static constexpr int BOXB = CH * 128;                            // bytes per box region
  static constexpr int CB = CH * 2 * D;                            // bytes per chunk
  static constexpr int WB = FP * G * 24;                           // weight bytes per unit
  static constexpr int NSLOT0 = (kScoreRingBytes - 2 * WB) / CB;
  static constexpr int NSLOT = NSLOT0 < 24 ? NSLOT0 : 24;
  static constexpr bool OK = (D == 64 || D == 128 || D == 256) &&
                             (G == 1 || G == 2 || G == 4 || G == 8 || G == 16) && NSLOT > kScoreConsumerWarps;
  static constexpr bool TC_OK = OK && NSLOT > kScoreTcWarps;  // the tensor-core form's consumers
  static constexpr size_t SMEM = 1024 + (size_t)NSLOT * CB + 2ull * WB + (size_t)NSLOT * 16 +
                                 2ull * NSLOT * 8 + 2ull * 8 + 4ull * TRIA_MAX_BATCH + 32 * 20;
};

__device__ __forceinline__ float sqrt_approx(float x) {
  float y;
  asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// A bf16 pair (one 32-bit word) widened exactly into a float pair.
__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t w) {
  return make_float2(dev::bf16lo(w), dev::bf16hi(w));
}

// Row r of a chunk lives in the 128-byte-swizzled box regions the TMA wrote:
// 16-byte unit u of the row's 128 bytes in a box is stored at unit u ^ (r & 7).

// The x and y words of RoPE pairs 2*JU*it .. 2*JU*it + 2*JU-1 of row r: x pairs (f, f+1)
// in xw[j] for f = 2*JU*it + 2j, likewise y (JU = 4, 2 or 1 words per load).
template <int D, int CH, int LAYOUT, int JU>
__device__ __forceinline__ void load_pairs(const uint8_t *chunk, int r, int it, uint32_t (&xw)[JU],
                                           uint32_t (&yw)[JU]) {
  constexpr int F = D / 2;
  constexpr int BOXB = CH * 128;
  if constexpr (LAYOUT == TRIA_ROPE_HALF_SPLIT) {
    const int dx = 2 * JU * it, dy = F + 2 * JU * it;  // first element of the x and y runs
    const uint8_t *ax = chunk + (dx >> 6) * BOXB + r * 128 + ((((dx & 63) >> 3) ^ (r & 7)) << 4) + (dx & 7) * 2;
    const uint8_t *ay = chunk + (dy >> 6) * BOXB + r * 128 + ((((dy & 63) >> 3) ^ (r & 7)) << 4) + (dy & 7) * 2;
    if constexpr (JU == 4) {
      const uint4 a = *reinterpret_cast<const uint4 *>(ax), b = *reinterpret_cast<const uint4 *>(ay);
      xw[0] = a.x; xw[1] = a.y; xw[2] = a.z; xw[3] = a.w;
      yw[0] = b.x; yw[1] = b.y; yw[2] = b.z; yw[3] = b.w;
    } else if constexpr (JU == 2) {
      const uint2 a = *reinterpret_cast<const uint2 *>(ax), b = *reinterpret_cast<const uint2 *>(ay);
      xw[0] = a.x; xw[1] = a.y;
      yw[0] = b.x; yw[1] = b.y;
    } else {
      xw[0] = *reinterpret_cast<const uint32_t *>(ax);
      yw[0] = *reinterpret_cast<const uint32_t *>(ay);
    }
  } else {
    // interleaved: word q holds (x_q, y_q); regroup into x and y pairs
    const int d0 = 4 * JU * it;
    const uint8_t *a0 = chunk + (d0 >> 6) * BOXB + r * 128 + ((((d0 & 63) >> 3) ^ (r & 7)) << 4) + (d0 & 7) * 2;
    uint32_t w[2 * JU];
    if constexpr (JU == 4) {
      const uint8_t *a1 = chunk + (d0 >> 6) * BOXB + r * 128 + (((((d0 & 63) >> 3) + 1) ^ (r & 7)) << 4);
      const uint4 a = *reinterpret_cast<const uint4 *>(a0), b = *reinterpret_cast<const uint4 *>(a1);
      w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w; w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
    } else if constexpr (JU == 2) {
      const uint4 a = *reinterpret_cast<const uint4 *>(a0);
      w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    } else {
      const uint2 a = *reinterpret_cast<const uint2 *>(a0);
      w[0] = a.x; w[1] = a.y;
    }
#pragma unroll
    for (int i = 0; i < JU; ++i) {
      xw[i] = __byte_perm(w[2 * i], w[2 * i + 1], 0x5410);  // (x_2i, x_2i+1)
      yw[i] = __byte_perm(w[2 * i], w[2 * i + 1], 0x7632);  // (y_2i, y_2i+1)
    }
  }
}

// Row, sequence and first key of chunk c (chunks are laid out row by row, and
// within a row sequence by sequence).
__device__ __forceinline__ void chunk_coords(const ScoreParams &p, int c, int &row, int &b,
                                             int &j) {
  row = c / p.chunks_per_row;
  const int rem = c - row * p.chunks_per_row;
  int lo = 0, hi = p.B;  // largest lo with chunk_prefix[lo] <= rem
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (p.chunk_prefix[mid] <= rem) lo = mid; else hi = mid;
  }
  b = lo;
  j = rem - p.chunk_prefix[lo];  // chunk index within the segment
}

// acc += wx * x + wy * y + wn * n, two RoPE pairs at a time.
__device__ __forceinline__ void fma3(float2 &acc, float2 wx, float2 wy, float2 wn, float2 x,
                                     float2 y, float2 n) {
  acc = __ffma2_rn(wx, x, acc);
  acc = __ffma2_rn(wy, y, acc);
  acc = __ffma2_rn(wn, n, acc);
}

// ---------------------------------------------------------------- tensor-core form
// For D = 64 or 128 and G <= 8 a warp scores each 16-key block of its chunk with
// mma.sync m16n8k16 (bf16 operands, float32 accumulators) instead of per-lane FMAs:
//   s = K Wt + Nrm Wn
// K the 16 x D block of stored keys straight from the swizzled chunk (exact bf16),
// Wt (D x 2G) the trigonometric weights on every stored dim (Re W_f on x_f, Im W_f on
// y_f), Nrm (16 x F) the norms |k_f| and Wn (F x 2G) the norm weights.  Each float32
// weight enters as a bf16 pair hi + lo in columns h and G + h (so s_h is column h
// plus column G + h, 16 significant bits of every weight); each norm enters as a
// bf16 pair too (Nrm_hi and Nrm_lo, two MMAs), so the products keep float32-level
// accuracy.  The norms are formed from the A fragments of K themselves: with the
// half-split layout x_f and y_f sit at the same fragment position of the k-steps t
// and t + D/32; with the interleaved layout one register holds (x_f, y_f), and the
// norm matrix takes its frequencies in the order the registers hold them
// (column 2q + e of freq step u is f = 16u + q + 4e, column 2q + 8 + e is
// f = 16u + 8 + q + 4e), which the norm weights follow.
template <int D, int G>
struct TcShape {
  static constexpr int F = D / 2;
  static constexpr int KS = D / 16;                // k-steps over the stored dims
  static constexpr int FS = F / 16;                // k-steps over the frequencies
  static constexpr int NB = 2 * G > 8 ? 2 * G / 8 : 1;  // n-blocks of 8 columns
};

// Frequency of column kk (0..15) of frequency step u of the norm matrix.
template <int LAYOUT>
__device__ __forceinline__ int norm_freq(int u, int kk) {
  if constexpr (LAYOUT == TRIA_ROPE_HALF_SPLIT) return 16 * u + kk;
  else return 16 * u + 8 * (kk >> 3) + ((kk & 7) >> 1) + 4 * (kk & 1);
}

// This lane's B fragments of Wt and Wn from the unit's float weights in shared
// memory ([F/2][G][6]: Re W, Re W, Im W, Im W, Nw, Nw for the pairs 2fp, 2fp+1).
template <int D, int G, int LAYOUT>
__device__ __forceinline__ void tc_weights(const float *wu, int lane,
                                           uint32_t (&bt)[TcShape<D, G>::KS][TcShape<D, G>::NB][2],
                                           uint32_t (&bn)[TcShape<D, G>::FS][TcShape<D, G>::NB][2]) {
  using T = TcShape<D, G>;
  constexpr int F = T::F;
  const int k0 = 2 * (lane & 3);
  auto col = [&](int nb, float w) -> float {  // hi or lo part of weight w for this lane's column
    const int c = 8 * nb + (lane >> 2);
    if (c >= 2 * G) return 0.0f;
    const float hi = dev::bf16lo(pack_bf16x2(w, 0.0f));  // w rounded to bf16
    return c < G ? hi : w - hi;
  };
  auto head = [&](int nb) { const int c = 8 * nb + (lane >> 2); return c < G ? c : (c < 2 * G ? c - G : 0); };
  auto wt = [&](int d, int h) -> float {  // weight on stored dim d for head h
    int f, im;
    if constexpr (LAYOUT == TRIA_ROPE_HALF_SPLIT) { f = d < F ? d : d - F; im = d >= F; }
    else { f = d >> 1; im = d & 1; }
    return wu[(f >> 1) * 6 * G + 6 * h + 2 * im + (f & 1)];
  };
  auto wn = [&](int f, int h) -> float { return wu[(f >> 1) * 6 * G + 6 * h + 4 + (f & 1)]; };
#pragma unroll
  for (int nb = 0; nb < T::NB; ++nb) {
    const int h = head(nb);
#pragma unroll
    for (int t = 0; t < T::KS; ++t) {
      const int d = 16 * t + k0;
      bt[t][nb][0] = pack_bf16x2(col(nb, wt(d, h)), col(nb, wt(d + 1, h)));
      bt[t][nb][1] = pack_bf16x2(col(nb, wt(d + 8, h)), col(nb, wt(d + 9, h)));
    }
#pragma unroll
    for (int u = 0; u < T::FS; ++u) {
      bn[u][nb][0] = pack_bf16x2(col(nb, wn(norm_freq<LAYOUT>(u, k0), h)),
                                 col(nb, wn(norm_freq<LAYOUT>(u, k0 + 1), h)));
      bn[u][nb][1] = pack_bf16x2(col(nb, wn(norm_freq<LAYOUT>(u, k0 + 8), h)),
                                 col(nb, wn(norm_freq<LAYOUT>(u, k0 + 9), h)));
    }
  }
}

// Norms of two (x, y) pairs given as bf16 pairs of x and of y, as the bf16 pairs
// hi and lo of the norm matrix.
__device__ __forceinline__ void tc_norms(uint32_t xw, uint32_t yw, uint32_t &hi, uint32_t &lo) {
  const float2 X = bf16x2_to_f2(xw), Y = bf16x2_to_f2(yw);
  const float2 n2 = __ffma2_rn(Y, Y, __fmul2_rn(X, X));
  const float na = sqrt_approx(n2.x), nb = sqrt_approx(n2.y);
  hi = pack_bf16x2(na, nb);
  const float2 h = bf16x2_to_f2(hi);
  lo = pack_bf16x2(na - h.x, nb - h.y);
}

// Accumulators of 16 keys (rows mb*16 ..) of a chunk at shared address cs for all
// 2G columns: acc[nb] as the C fragment of n-block nb.
template <int D, int G, int LAYOUT, int BOXB>
__device__ __forceinline__ void tc_block(uint32_t cs, int mb, int lane,
                                         const uint32_t (&bt)[TcShape<D, G>::KS][TcShape<D, G>::NB][2],
                                         const uint32_t (&bn)[TcShape<D, G>::FS][TcShape<D, G>::NB][2],
                                         float (&acc)[TcShape<D, G>::NB][4]) {
  using T = TcShape<D, G>;
  uint32_t a[T::KS][4];
  {
    const int mat = lane >> 3, key = 16 * mb + (mat & 1) * 8 + (lane & 7);
#pragma unroll
    for (int t = 0; t < T::KS; ++t) ldsm_x4(swz<BOXB>(cs, key, 16 * t + (mat >> 1) * 8), a[t]);
  }
  float an[T::NB][4];
#pragma unroll
  for (int nb = 0; nb < T::NB; ++nb)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[nb][e] = an[nb][e] = 0.0f;
#pragma unroll
  for (int t = 0; t < T::KS; ++t)
#pragma unroll
    for (int nb = 0; nb < T::NB; ++nb) mma_bf16(acc[nb], a[t], bt[t][nb]);
#pragma unroll
  for (int u = 0; u < T::FS; ++u) {
    uint32_t nh[4], nl[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      if constexpr (LAYOUT == TRIA_ROPE_HALF_SPLIT) {
        tc_norms(a[u][r], a[u + T::KS / 2][r], nh[r], nl[r]);
      } else {
        // registers r (rows r0 or r0 + 8) of k-steps 2u (r < 2) and 2u + 1 (r >= 2): a
        // register holds (x_f, y_f); two of them give the pair of norms of columns
        // (2q, 2q + 1) resp. (2q + 8, 2q + 9)
        const uint32_t *ka = a[2 * u + (r >> 1)];
        const uint32_t wa = ka[r & 1], wb = ka[(r & 1) + 2];
        tc_norms(__byte_perm(wa, wb, 0x5410), __byte_perm(wa, wb, 0x7632), nh[r], nl[r]);
      }
    }
#pragma unroll
    for (int nb = 0; nb < T::NB; ++nb) {
      mma_bf16(an[nb], nh, bn[u][nb]);
      mma_bf16(an[nb], nl, bn[u][nb]);
    }
  }
#pragma unroll
  for (int nb = 0; nb < T::NB; ++nb)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[nb][e] += an[nb][e];
}

template <int D, int G, int LAYOUT, bool TCF>
__global__ void __launch_bounds__(((TCF ? kScoreTcWarps : kScoreConsumerWarps) + 1) * 32, 1)
    score_kernel(const __grid_constant__ ScoreParams p) {
  using S = ScoreShape<D, G>;
  constexpr int F = S::F, FP = S::FP, KPT = S::KPT, CH = S::CH, CB = S::CB;
  constexpr int NW = TCF ? kScoreTcWarps : kScoreConsumerWarps;  // consumer warps
  constexpr int NSLOT = S::NSLOT;

  constexpr int WB = S::WB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *ring = smem_raw + ((1024u - (dev::smem_addr(smem_raw) & 1023u)) & 1023u);
  uint8_t *wring = ring + (size_t)NSLOT * CB;                        // [2][WB] weight slots
  int4 *desc = reinterpret_cast<int4 *>(wring + 2 * WB);  // per slot: row, b | wslot, key0, n
  uint64_t *full = reinterpret_cast<uint64_t *>(desc + NSLOT);
  uint64_t *empty = full + NSLOT;
  uint64_t *wfull = empty + NSLOT;                         // [2] weight slot loaded
  int32_t *live = reinterpret_cast<int32_t *>(wfull + 2);  // [B] keys to score per sequence
  int4 *tab = reinterpret_cast<int4 *>(live + TRIA_MAX_BATCH);  // [32] chunk descriptors
  int32_t *taby = reinterpret_cast<int32_t *>(tab + 32);          // [32] their tensor rows

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NSLOT; ++s) {
      dev::mbar_init(&full[s], 1);
      dev::mbar_init(&empty[s], 1);
    }
    dev::mbar_init(&wfull[0], 1);
    dev::mbar_init(&wfull[1], 1);
    dev::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) dev::pdl_launch_dependents();
  const int c0 = blockIdx.x * p.chunks_per_cta;
  const int c1 = min(c0 + p.chunks_per_cta, p.total_chunks);
  // Keys to score of unit (row, b): the live length, 0 if out of range or (with
  // skip_short) too short to prune; per sequence from `live`, or per unit.
  auto live_of = [&](int row, int b) -> int {
    if (!p.unit_len) return live[b];
    int32_t T = p.unit_len[(int64_t)row * p.B + b];
    if (T < 0 || (int64_t)T > p.seg_start[b + 1] - p.seg_start[b]) return 0;  // flagged by the fold
    if (p.skip_short) {
      const int bud = p.head_budget ? p.head_budget[row] : p.budget;
      if (bud < 1 || bud > p.budget) return 0;
      if ((int64_t)T < (int64_t)bud + (p.window > 1 ? p.window : 1)) return 0;
    }
    return T;
  };
  // The first unit with live chunks: its weights are copied by the consumers
  // themselves straight from L2 (not queued behind the key stream) into slot 0.
  auto find_first_unit = [&]() {
    for (int c = c0; c < c1; ++c) {
      int row, b, jc;
      chunk_coords(p, c, row, b, jc);
      if (live_of(row, b) > jc * CH) return row * p.B + b;
      c += max(0, (p.chunk_prefix[b + 1] - p.chunk_prefix[b]) - jc - 1);  // skip the dead rest
    }
    return -1;
  };
  // Named barriers: 1 the consumers among themselves; 2 the consumers' warm-up is
  // done (the producer may start the key stream); 3 the producer's live lengths are
  // written (the consumers may read them).

  if (warp == NW) {
    // ---------------------------------------------------------------- producer
    for (int b = lane; b < p.B && !p.unit_len; b += 32) {
      int32_t T = p.seq_len[b];
      if (T < 0 || (int64_t)T > p.seg_start[b + 1] - p.seg_start[b]) T = 0;  // flagged by the fold
      if (p.skip_short && T < p.prune_from) T = 0;
      live[b] = T;
    }
    __syncwarp();
    __threadfence_block();
    dev::named_barrier_arrive(3, (NW + 1) * 32);
    const int first_unit = find_first_unit();
    // lane 0's state: slot positions, weight slots
    uint32_t q = 0;
    bool failed = false;
    int64_t cur_unit = first_unit;  // its weights were put in slot 0 by the consumers
    int wslot = 0;
    bool prefilled = first_unit >= 0;  // the current unit's weights came from the consumers
    uint32_t wuse[2] = {0, 0};    // bulk fills of each weight slot so far (barrier phases)
    int64_t wlast[2] = {-1, -1};  // last chunk position that read each weight slot
    // Weight fills wait for the fold kernel; the first ones are held back until the
    // ring is full, so the first key chunks stream in while the fold runs.
    bool folded = false;
    int npend = 0;
    int pend_slot[2] = {0, 0};
    int64_t pend_unit[2] = {0, 0};
    auto flush = [&]() {
      if (npend == 0) return;
      if (!folded) {
        dev::pdl_wait();  // the weights come from the fold kernel
        folded = true;
      }
      for (int i = 0; i < npend; ++i) {
        dev::mbar_arrive_expect_tx(&wfull[pend_slot[i]], WB);
        dev::bulk_g2s(wring + pend_slot[i] * WB,
                      reinterpret_cast<const uint8_t *>(p.w) + pend_unit[i] * WB, WB,
                      &wfull[pend_slot[i]]);
      }
      npend = 0;
    };
    // The consumers first run their chunk code once (see below); the key stream
    // starts after that, so their instruction fetches do not queue behind it.
    dev::named_barrier(2, (NW + 1) * 32);
    // The 32 lanes describe 32 chunks at a time in parallel; lane 0 then issues them.
    for (int cg0 = c0; cg0 < c1; cg0 += 32) {
      {
        const int c = cg0 + lane;
        int row = 0, lo = 0, key0 = 0, n = 0;
        if (c < c1) {
          int jc;
          chunk_coords(p, c, row, lo, jc);
          key0 = jc * CH;
          n = min(max(live_of(row, lo) - key0, 0), CH);
        }
        tab[lane] = make_int4(row, lo, key0, n);
        taby[lane] = (int32_t)((int64_t)row * p.cap + p.seg_start[lo] + key0);
      }
      __syncwarp();
      if (lane == 0 && !failed) {
        const int cnt = min(32, c1 - cg0);
        for (int i = 0; i < cnt; ++i) {
          const int4 e = tab[i];
          const int row = e.x, lo = e.y, key0 = e.z, n = e.w;
          if (n == 0) continue;
          const uint32_t s = q % NSLOT, use = q / NSLOT;
          if (use > 0 && !dev::mbar_wait(&empty[s], (use - 1) & 1)) {
            failed = true;
            break;
          }
          const int64_t unit = (int64_t)row * p.B + lo;
          if (unit != cur_unit) {
            // the unit's weights go to the other weight slot, once every chunk that read
            // that slot's previous weights has been released (all positions up to
            // q - NSLOT are: the waits above covered them)
            const int j = wslot ^ 1;
            if (wlast[j] >= 0) {
              flush();  // the chunks awaited below need their weights
              for (int64_t pp = (int64_t)q - NSLOT + 1; pp <= wlast[j] && !failed; ++pp) {
                // pp > q - NSLOT: position pp's slot was not reused yet, so the parity is its own
                if (pp >= 0) failed = !dev::mbar_wait(&empty[pp % NSLOT], (uint32_t)(pp / NSLOT) & 1);
              }
              if (failed) break;
            }
            pend_slot[npend] = j;
            pend_unit[npend] = unit;
            ++npend;
            if (folded) flush();
            ++wuse[j];
            wslot = j;
            cur_unit = unit;
            prefilled = false;
          }
          wlast[wslot] = q;
          // weight tag: 4 for the consumers' own fill, else slot | phase parity << 1
          const int wtag = prefilled ? 4 : (wslot | (int)(((wuse[wslot] - 1) & 1) << 1));
          desc[s] = make_int4(row, lo | (wtag << 16), key0, n);
          dev::mbar_arrive_expect_tx(&full[s], CB);
          const int32_t y = taby[i];
#pragma unroll
          for (int bx = 0; bx < S::NBOX; ++bx)
            dev::tma_load_2d(ring + (size_t)s * CB + bx * S::BOXB, &p.tmap, bx * 64, y, &full[s]);
          ++q;
          if (q >= (uint32_t)NSLOT) flush();  // the ring is full: wait for the fold now
        }
      }
      failed = __shfl_sync(0xffffffffu, failed, 0);
      if (failed) break;
      __syncwarp();  // lane 0 has read the table
    }
    if (lane == 0) {
      if (!failed) flush();
      // one end marker per consumer warp
      for (int t = 0; t < NW && !failed; ++t) {
        const uint32_t s = q % NSLOT, use = q / NSLOT;
        if (use > 0 && !dev::mbar_wait(&empty[s], (use - 1) & 1)) {
          failed = true;
          break;
        }
        desc[s] = make_int4(0, 0, 0, -1);
        dev::mbar_arrive(&full[s]);
        ++q;
      }
      if (failed) {
        dev::set_error(p.err, TRIA_DEVERR_TIMEOUT);
        // let the copies already issued land before the CTA can retire
        const uint32_t first = q > (uint32_t)NSLOT ? q - NSLOT : 0;
        for (uint32_t u = first; u < q; ++u) dev::mbar_wait(&full[u % NSLOT], (u / NSLOT) & 1);
      }
    }
    dev::pdl_wait();  // this grid never completes before the fold it depends on
    return;
  }

  // ------------------------------------------------------------------ consumers
  int wseen = -1;  // weight slot and fill parity last waited for
  // the tensor-core form's B fragments of the current weights, and their tag
  constexpr bool TC = TCF && (D == 64 || D == 128) && G <= 8 && CH % 16 == 0;
  using TS = TcShape<D, G>;
  uint32_t bt[TC ? TS::KS : 1][TC ? TS::NB : 1][2], bn[TC ? TS::FS : 1][TC ? TS::NB : 1][2];
  int ftag = -1;
  // float64 sums of s and s^2 of this lane's keys for the current unit; each warp
  // writes one entry per unit its CTA's chunk run meets (zeros where it had none)
  int u_first = 0, u_last = -1, first_unit = -1;  // set after the warm-up
  double s1[G], s2[G];
#pragma unroll
  for (int h = 0; h < G; ++h) { s1[h] = 0.0; s2[h] = 0.0; }
  auto write_unit = [&](int u, bool zero) {
    double v[2 * G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      double a = zero ? 0.0 : s1[h], b2 = zero ? 0.0 : s2[h];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        a += __shfl_xor_sync(0xffffffffu, a, o);
        b2 += __shfl_xor_sync(0xffffffffu, b2, o);
      }
      v[2 * h] = a;
      v[2 * h + 1] = b2;
    }
    const int row = u / p.B, b = u - row * p.B;
    if (p.chunk_prefix[b + 1] == p.chunk_prefix[b]) return;  // an empty segment: never read
    const int slot = (int)blockIdx.x - (row * p.chunks_per_row + p.chunk_prefix[b]) / p.chunks_per_cta;
    if (slot < 0 || slot >= p.max_slots) return;
    double *dst = p.partials + (((int64_t)u * p.max_slots + slot) * NW + warp) * (2 * G);
    if (lane < 2 * G) {
#pragma unroll
      for (int i = 0; i < 2 * G; ++i)
        if (lane == i) dst[i] = v[i];
    }
  };
  int cur = -1, next_unwritten = 0;
  // The first pass is a warm-up: one inner iteration and the epilogue of the chunk
  // code on whatever the ring holds, storing nothing (n = 0), so that the code is
  // fetched before the key stream saturates the memory system.
  bool warm = true;
#pragma unroll 1
  for (uint32_t q = warp;;) {
    uint32_t s = 0;
    int row = 0, b = 0, key0 = 0, n = 0, wtag = 0;
    if (!warm) {
      s = q % NSLOT;
      const uint32_t use = q / NSLOT;
      // the slot's previous chunk was released, so the parity below is this use's
      if ((use > 0 && !dev::mbar_wait(&empty[s], (use - 1) & 1)) ||
          !dev::mbar_wait(&full[s], use & 1)) {
        if (lane == 0) dev::set_error(p.err, TRIA_DEVERR_TIMEOUT);
        break;
      }
      const int4 d = desc[s];
      if (d.w < 0) break;
      row = d.x;
      b = d.y & 0xffff;
      key0 = d.z;
      n = d.w;
      const int unit = row * p.B + b;
      if (unit != cur) {
        if (cur >= 0) {
          write_unit(cur, false);
          next_unwritten = cur + 1;
        }
        for (int u = next_unwritten; u < unit; ++u) write_unit(u, true);
        next_unwritten = unit;
        cur = unit;
#pragma unroll
        for (int h = 0; h < G; ++h) { s1[h] = 0.0; s2[h] = 0.0; }
      }
      wtag = d.y >> 16;  // weight slot | fill parity << 1, or 4: slot 0 by the consumers
      if (wtag != wseen) {
        if (!dev::mbar_wait(&wfull[wtag & 1], (uint32_t)(wtag >> 1))) {
          if (lane == 0) dev::set_error(p.err, TRIA_DEVERR_TIMEOUT);
          break;
        }
        wseen = wtag;
      }
    }
    const float *wu = reinterpret_cast<const float *>(wring + (wtag & 1) * WB);
    const uint8_t *chunk = ring + (size_t)s * CB;
    const int l = row / p.Hkv, g = row - l * p.Hkv;
    float *rawp = p.raw + ((size_t)l * p.Hq + (size_t)g * G) * p.cap + p.seg_start[b] + key0;

    if constexpr (TC) {
      if (wtag != ftag) {  // the unit's weights as this lane's B fragments
        tc_weights<D, G, LAYOUT>(wu, lane, bt, bn);
        ftag = wtag;
      }
      const uint32_t cs = dev::smem_addr(chunk);
      const int q4 = lane & 3, r0 = lane >> 2;
      const int nmb = warm ? 1 : CH / 16;
#pragma unroll 1
      for (int mb = 0; mb < nmb; ++mb) {
        float acc[TcShape<D, G>::NB][4];
        tc_block<D, G, LAYOUT, S::BOXB>(cs, mb, lane, bt, bn, acc);
        // s_h = column h + column G + h: this lane ends with heads 2 q4, 2 q4 + 1 of keys
        // r0 and r0 + 8 (G >= 2), or head 0 (G = 1)
        float v[4];
        if constexpr (G == 8) {
#pragma unroll
          for (int e = 0; e < 4; ++e) v[e] = acc[0][e] + acc[1][e];
        } else if constexpr (G == 4 || G == 2) {
#pragma unroll
          for (int e = 0; e < 4; ++e) v[e] = acc[0][e] + __shfl_xor_sync(0xffffffffu, acc[0][e], G / 2);
        } else {
          v[0] = acc[0][0] + acc[0][1];
          v[2] = acc[0][2] + acc[0][3];
          v[1] = v[3] = 0.0f;
        }
        if (G == 1 ? q4 == 0 : 2 * q4 < G) {
          const int hA = G == 1 ? 0 : 2 * q4;
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const int r = 16 * mb + r0 + 8 * half;
            if (r < n) {
#pragma unroll
              for (int e = 0; e < (G == 1 ? 1 : 2); ++e) {
                const float x = v[2 * half + e];
                rawp[(size_t)(hA + e) * p.cap + r] = x;
#pragma unroll
                for (int h = 0; h < G; ++h)
                  if (h == hA + e) {
                    s1[h] += (double)x;
                    s2[h] = fma((double)x, (double)x, s2[h]);
                  }
              }
            }
          }
        }
      }
    } else {
    float2 acc[KPT][G];
#pragma unroll
    for (int k = 0; k < KPT; ++k)
#pragma unroll
      for (int h = 0; h < G; ++h) acc[k][h] = make_float2(0.0f, 0.0f);

    constexpr int JU = kScoreJu;
    const int iters = warm ? 1 : FP / JU;
#pragma unroll 1
    for (int it = 0; it < iters; ++it) {
      uint32_t xw[KPT][JU], yw[KPT][JU];
#pragma unroll
      for (int k = 0; k < KPT; ++k) load_pairs<D, CH, LAYOUT, JU>(chunk, lane + 32 * k, it, xw[k], yw[k]);
#pragma unroll
      for (int j = 0; j < JU; ++j) {
        const float *wf = wu + (size_t)(JU * it + j) * 6 * G;
        float2 X[KPT], Y[KPT], N[KPT];
#pragma unroll
        for (int k = 0; k < KPT; ++k) {
          X[k] = bf16x2_to_f2(xw[k][j]);
          Y[k] = bf16x2_to_f2(yw[k][j]);
          const float2 n2 = __ffma2_rn(Y[k], Y[k], __fmul2_rn(X[k], X[k]));
          N[k] = make_float2(sqrt_approx(n2.x), sqrt_approx(n2.y));
        }
        if constexpr (G % 2 == 0) {
#pragma unroll
          for (int hp = 0; hp < G / 2; ++hp) {
            const float4 *w4 = reinterpret_cast<const float4 *>(wf + 12 * hp);
            const float4 A = w4[0], B4 = w4[1], C = w4[2];
            const float2 wx0 = make_float2(A.x, A.y), wy0 = make_float2(A.z, A.w);
            const float2 wn0 = make_float2(B4.x, B4.y), wx1 = make_float2(B4.z, B4.w);
            const float2 wy1 = make_float2(C.x, C.y), wn1 = make_float2(C.z, C.w);
#pragma unroll
            for (int k = 0; k < KPT; ++k) {
              fma3(acc[k][2 * hp], wx0, wy0, wn0, X[k], Y[k], N[k]);
              fma3(acc[k][2 * hp + 1], wx1, wy1, wn1, X[k], Y[k], N[k]);
            }
          }
        } else {
          const float2 *w2 = reinterpret_cast<const float2 *>(wf);
          const float2 wx = w2[0], wy = w2[1], wn = w2[2];
#pragma unroll
          for (int k = 0; k < KPT; ++k) fma3(acc[k][0], wx, wy, wn, X[k], Y[k], N[k]);
        }
      }
    }
#pragma unroll
    for (int k = 0; k < KPT; ++k) {
      const int r = lane + 32 * k;
      if (r < n) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float v = acc[k][h].x + acc[k][h].y;
          rawp[(size_t)h * p.cap + r] = v;
          s1[h] += (double)v;
          s2[h] = fma((double)v, (double)v, s2[h]);
        }
      }
    }
    }  // the FMA form
    if (warm) {
      warm = false;
      ftag = -1;  // the warm-up built fragments from whatever the weight slot held
      dev::named_barrier_arrive(2, (NW + 1) * 32);  // the producer may start the stream
      {
        int row, b, j;
        chunk_coords(p, c0, row, b, j);
        u_first = row * p.B + b;
        chunk_coords(p, max(c1 - 1, c0), row, b, j);
        u_last = row * p.B + b;
        next_unwritten = u_first;
      }
      dev::named_barrier(3, (NW + 1) * 32);  // the live lengths are written
      first_unit = find_first_unit();
      if (first_unit >= 0) {
        dev::pdl_wait();  // the weights come from the fold kernel
        const uint4 *src = reinterpret_cast<const uint4 *>(reinterpret_cast<const uint8_t *>(p.w) +
                                                           (int64_t)first_unit * WB);
        for (int i = threadIdx.x; i < WB / 16; i += NW * 32)
          reinterpret_cast<uint4 *>(wring)[i] = src[i];
        dev::named_barrier(1, NW * 32);
        wseen = 4;  // the tag of these weights
      }
      continue;
    }
    __syncwarp();
    if (lane == 0) dev::mbar_arrive(&empty[s]);
    q += NW;
  }
  if (c0 < c1) {
    if (cur >= 0) {
      write_unit(cur, false);
      next_unwritten = cur + 1;
    }
    for (int u = next_unwritten; u <= u_last; ++u) write_unit(u, true);
  }
}

template <int D, int G, int LAYOUT, bool TCF>
static cudaError_t launch_one(const ScoreParams &p, int grid, cudaStream_t s, bool pdl) {
  using S = ScoreShape<D, G>;
  if constexpr (!S::OK || (TCF && !S::TC_OK)) {
    return cudaErrorInvalidValue;
  } else {
    auto kern = score_kernel<D, G, LAYOUT, TCF>;
    static bool configured[64] = {};  // per device: the attribute is set once per process
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
    if (dev < 0 || dev >= 64 || !configured[dev]) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)S::SMEM);
      if (e != cudaSuccess) return e;
      if (dev >= 0 && dev < 64) configured[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3(((TCF ? kScoreTcWarps : kScoreConsumerWarps) + 1) * 32, 1, 1);
    cfg.dynamicSmemBytes = S::SMEM;
    cfg.stream = s;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, p);
  }
}

// The tensor-core form costs more per CTA (a larger warm-up, fragment builds per unit)
// and less per key: on a B200 it is ahead for G = 8, and for smaller groups once a CTA
// scores kScoreTcChunks chunks or more (one 8B-shaped layer, 28 chunks per CTA: 27.2
// against 28.8 us; 36 layers, about 1000 per CTA: 488 against 457 us).
constexpr int kScoreTcChunks = 64;

bool score_uses_tc(int D, int G, int chunks_per_cta) {
  return (D == 64 || D == 128) && (G == 1 || G == 2 || G == 4 || G == 8) &&
         (G == 8 || chunks_per_cta >= kScoreTcChunks);
}

template <int D, int G, int LAYOUT>
static cudaError_t launch_g(const ScoreParams &p, int grid, cudaStream_t s, bool pdl) {
  if constexpr ((D == 64 || D == 128) && G <= 8) {
    if (p.tc) return launch_one<D, G, LAYOUT, true>(p, grid, s, pdl);
  }
  if (p.tc) return cudaErrorInvalidValue;  // the tensor-core form does not take this shape
  return launch_one<D, G, LAYOUT, false>(p, grid, s, pdl);
}

template <int D, int LAYOUT>
static cudaError_t dispatch_g(const ScoreParams &p, int G, int grid, cudaStream_t s, bool pdl) {
  switch (G) {
    case 1: return launch_g<D, 1, LAYOUT>(p, grid, s, pdl);
    case 2: return launch_g<D, 2, LAYOUT>(p, grid, s, pdl);
    case 4: return launch_g<D, 4, LAYOUT>(p, grid, s, pdl);
    case 8: return launch_g<D, 8, LAYOUT>(p, grid, s, pdl);
    case 16: return launch_g<D, 16, LAYOUT>(p, grid, s, pdl);
    default: return cudaErrorInvalidValue;
  }
}

template <int D>
static int chunk_keys_g(int G) {
  switch (G) {
    case 1: return ScoreShape<D, 1>::OK ? ScoreShape<D, 1>::CH : 0;
    case 2: return ScoreShape<D, 2>::OK ? ScoreShape<D, 2>::CH : 0;
    case 4: return ScoreShape<D, 4>::OK ? ScoreShape<D, 4>::CH : 0;
    case 8: return ScoreShape<D, 8>::OK ? ScoreShape<D, 8>::CH : 0;
    case 16: return ScoreShape<D, 16>::OK ? ScoreShape<D, 16>::CH : 0;
    default: return 0;
  }
}

int score_chunk_keys(int D, int G) {
  switch (D) {
    case 64: return chunk_keys_g<64>(G);
    case 128: return chunk_keys_g<128>(G);
    case 256: return chunk_keys_g<256>(G);
    default: return 0;
  }
}

bool score_supported(int D, int G, int layout) {
  if (layout != TRIA_ROPE_HALF_SPLIT && layout != TRIA_ROPE_INTERLEAVED) return false;
  return score_chunk_keys(D, G) > 0;
}

cudaError_t make_key_tensor_map(CUtensorMap *map, const void *k, int D, int64_t rows,
                                int box_rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  static std::once_flag once;
  std::call_once(once, []() {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!encode) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(k), dims,
                            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t launch_score(const ScoreParams &p, int D, int G, int layout, int grid,
                         cudaStream_t s, bool pdl) {
  if (layout == TRIA_ROPE_HALF_SPLIT) {
    switch (D) {
      case 64: return dispatch_g<64, TRIA_ROPE_HALF_SPLIT>(p, G, grid, s, pdl);
      case 128: return dispatch_g<128, TRIA_ROPE_HALF_SPLIT>(p, G, grid, s, pdl);
      case 256: return dispatch_g<256, TRIA_ROPE_HALF_SPLIT>(p, G, grid, s, pdl);
    }
  } else {
    switch (D) {
      case 64: return dispatch_g<64, TRIA_ROPE_INTERLEAVED>(p, G, grid, s, pdl);
      case 128: return dispatch_g<128, TRIA_ROPE_INTERLEAVED>(p, G, grid, s, pdl);
      case 256: return dispatch_g<256, TRIA_ROPE_INTERLEAVED>(p, G, grid, s, pdl);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace tria
