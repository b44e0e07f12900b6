// Raw key scores, one streaming pass over the cached keys.
//
// For every live key t of every (layer l, KV head g, sequence b) and every
// query head h of g's group (romaanj.github.io review, "Method";
// dimensionstp.github.io review, sections 2-2 and 3-2 (2)-(4)):
//   s_h(t) = sum_f [ Re(conj(ktilde_f) * W_hf) + Nw_hf * |ktilde_f| ]
//   W_hf   = c_hf * EA_bf          (trig term with offsets and cur folded in, see fold.cu)
//   Nw_hf  = (1 - R_hf) * E|q_hf|  (norm term; |k_f| = |ktilde_f| since RoPE keeps norms)
// ktilde is the stored post-RoPE bf16 key widened exactly to float; all sums
// are float32.  The kernel also leaves, per (unit, CTA, head), the float64
// sums of s and s^2 over the keys it scored, which the z-score needs.
//
// Design (sm_100a): a persistent grid, one CTA per SM, each taking a
// contiguous run of 64 KB key tiles.  One producer warp streams tiles into a
// 3-stage shared-memory ring with 1-D bulk copies (cp.async.bulk, completion
// on mbarriers, no multicast); sixteen consumer warps compute.  A consumer
// lane owns PPL RoPE pairs of a key and works on two keys at once; the unit's
// weights sit in shared memory in lane order (one broadcast read serves the
// lanes of all keys in a warp) and pair up two RoPE pairs per 64-bit register
// for the sm_100 paired FP32 FMA (__ffma2_rn).  The LPK lanes of a key
// combine their partial sums by a reduce-scatter (each shuffle level halves
// the values a lane holds); the heads are assigned to register slots in a
// lane-dependent order when the weights are laid out, so no selects are
// needed and each lane ends with its heads' totals, which it stores.
#include "tria_internal.cuh"

namespace tria {

template <int D, int G>
struct ScoreShape {
  static constexpr int F = D / 2;
  static constexpr int PPL = 8;                                   // pairs per lane
  static constexpr int P2 = PPL / 2;                              // paired registers per lane
  static constexpr int LPK = F / PPL;                             // lanes per key
  static constexpr int KPW = 32 / LPK;                            // key groups per warp
  static constexpr int VL = G > LPK ? G / LPK : 1;                // head totals a lane ends with
  static constexpr int ROW = 2 * D;                               // bytes per key row
  static constexpr int TILE = kScoreTileBytes / ROW;              // keys per tile
  static constexpr int NW = kScoreConsumerWarps;
  static constexpr int KEYS_PER_WARP = TILE / NW;
  static constexpr int STEPS = KEYS_PER_WARP / (2 * KPW);         // two keys per lane per step
  static constexpr int WENT = P2 * G * LPK;                       // weight entries per unit
  static constexpr bool OK = (LPK >= 1) && (LPK <= 32) && (STEPS * 2 * KPW == KEYS_PER_WARP) &&
                             (STEPS >= 1) && (G <= 16);
  static constexpr size_t SMEM_STAGES = (size_t)kScoreStages * TILE * ROW;
  static constexpr size_t SMEM_W = (size_t)WENT * 24;             // float4 (wx, wy) + float2 nw
  static constexpr size_t SMEM_PART = (size_t)NW * G * 2 * 8;     // per-warp float64 partials
  static constexpr size_t SMEM = SMEM_STAGES + SMEM_W + SMEM_PART + 2ull * kScoreStages * 8;
};

struct TileRef {
  int32_t row;   // l * Hkv + g
  int32_t b;
  int64_t key0;  // first key of the tile within the segment
  int32_t n;     // live keys in the tile (0: nothing to do)
};

__device__ __forceinline__ TileRef tile_of(const ScoreParams &p, int64_t t, int tile_keys) {
  TileRef r;
  r.row = (int32_t)(t / p.tiles_per_row);
  const int32_t rem = (int32_t)(t - (int64_t)r.row * p.tiles_per_row);
  int lo = 0, hi = p.B;  // largest b with tile_prefix[b] <= rem
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (p.tile_prefix[mid] <= rem) lo = mid; else hi = mid;
  }
  r.b = lo;
  r.key0 = (int64_t)(rem - p.tile_prefix[lo]) * tile_keys;
  int32_t T = p.seq_len[lo];
  if (T < 0 || (int64_t)T > p.seg_start[lo + 1] - p.seg_start[lo]) T = 0;  // flagged by the fold
  int64_t n = (int64_t)T - r.key0;
  n = n < 0 ? 0 : (n > tile_keys ? tile_keys : n);
  if (p.skip_short && T <= p.budget) n = 0;
  r.n = (int32_t)n;
  return r;
}

__device__ __forceinline__ float sqrt_approx(float x) {
  float y;
  asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// A bf16 pair (one 32-bit word) widened exactly into a float pair.
__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t w) {
  return make_float2(dev::bf16lo(w), dev::bf16hi(w));
}

// Reduce-scatter over the lanes of a key: at offset O, a lane holding V values
// keeps the first V/2 and adds its partner's second half; once one value is
// left the remaining levels are a plain butterfly sum.
template <int O, int V, int G>
__device__ __forceinline__ void reduce_scatter(float (&a)[G], float (&b)[G]) {
  if constexpr (O >= 1) {
    if constexpr (V > 1) {
      constexpr int H = V / 2;
#pragma unroll
      for (int k = 0; k < H; ++k) {
        a[k] += __shfl_xor_sync(0xffffffffu, a[k + H], O);
        b[k] += __shfl_xor_sync(0xffffffffu, b[k + H], O);
      }
      reduce_scatter<O / 2, H, G>(a, b);
    } else {
      a[0] += __shfl_xor_sync(0xffffffffu, a[0], O);
      b[0] += __shfl_xor_sync(0xffffffffu, b[0], O);
      reduce_scatter<O / 2, 1, G>(a, b);
    }
  }
}

// The PPL pairs a lane owns in a key row held in shared memory, as two words
// of x (and of y) per paired register: x pairs (f0+2i, f0+2i+1) in xw[i].
template <int D, int PPL, int LAYOUT>
__device__ __forceinline__ void load_row(const uint8_t *rowp, int f0, uint32_t (&xw)[PPL / 2],
                                         uint32_t (&yw)[PPL / 2]) {
  static_assert(PPL == 8, "lanes own eight pairs");
  if constexpr (LAYOUT == TRIA_ROPE_HALF_SPLIT) {
    const uint4 a = *reinterpret_cast<const uint4 *>(rowp + 2 * f0);
    const uint4 b = *reinterpret_cast<const uint4 *>(rowp + D + 2 * f0);
    xw[0] = a.x; xw[1] = a.y; xw[2] = a.z; xw[3] = a.w;
    yw[0] = b.x; yw[1] = b.y; yw[2] = b.z; yw[3] = b.w;
  } else {
    // interleaved: word q holds (x_q, y_q); regroup into x and y pairs
    const uint4 a = *reinterpret_cast<const uint4 *>(rowp + 4 * f0);
    const uint4 b = *reinterpret_cast<const uint4 *>(rowp + 4 * f0 + 16);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      xw[i] = __byte_perm(w[2 * i], w[2 * i + 1], 0x5410);  // (x_2i, x_2i+1)
      yw[i] = __byte_perm(w[2 * i], w[2 * i + 1], 0x7632);  // (y_2i, y_2i+1)
    }
  }
}

template <int D, int G, int LAYOUT>
__global__ void __launch_bounds__(kScoreThreads, 1)
    score_kernel(const __grid_constant__ ScoreParams p) {
  using S = ScoreShape<D, G>;
  constexpr int F = S::F, PPL = S::PPL, P2 = S::P2, LPK = S::LPK, KPW = S::KPW, VL = S::VL;
  constexpr int ROW = S::ROW, TILE = S::TILE, NW = S::NW, NST = kScoreStages;

  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t *stage = smem;
  float4 *wxy = reinterpret_cast<float4 *>(smem + S::SMEM_STAGES);           // [P2][G][LPK]
  float2 *wn = reinterpret_cast<float2 *>(wxy + S::WENT);                     // [P2][G][LPK]
  double *wpart = reinterpret_cast<double *>(wn + S::WENT);                   // [NW][G][2]
  uint64_t *full = reinterpret_cast<uint64_t *>(wpart + NW * G * 2);
  uint64_t *empty = full + NST;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      dev::mbar_init(&full[s], 1);
      dev::mbar_init(&empty[s], NW);
    }
    dev::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) dev::pdl_launch_dependents();

  const int64_t t0 = (int64_t)blockIdx.x * p.tiles_per_cta;
  int64_t t1 = t0 + p.tiles_per_cta;
  if (t1 > p.total_tiles) t1 = p.total_tiles;

  if (warp == NW) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      uint32_t it = 0;
      bool failed = false;
      for (int64_t t = t0; t < t1 && !failed; ++t) {
        const TileRef tl = tile_of(p, t, TILE);
        if (tl.n <= 0) continue;
        const uint32_t s = it % NST, use = it / NST;
        if (use > 0 && !dev::mbar_wait(&empty[s], (use - 1) & 1)) {
          dev::set_error(p.err, TRIA_DEVERR_TIMEOUT);
          failed = true;
          break;
        }
        const uint32_t bytes = (uint32_t)tl.n * ROW;
        const uint8_t *src =
            p.k + ((size_t)tl.row * p.cap + p.seg_start[tl.b] + tl.key0) * (size_t)ROW;
        dev::mbar_arrive_expect_tx(&full[s], bytes);
        dev::bulk_g2s(stage + (size_t)s * TILE * ROW, src, bytes, &full[s]);
        ++it;
      }
      if (failed) {
        // let the copies already issued land before the CTA can retire
        const uint32_t first = it > (uint32_t)NST ? it - NST : 0;
        for (uint32_t u = first; u < it; ++u) dev::mbar_wait(&full[u % NST], (u / NST) & 1);
      }
    }
    dev::pdl_wait();  // this grid never completes before the fold it depends on
    return;
  }

  // ------------------------------------------------------------------ consumers
  const int ct = threadIdx.x;  // consumer thread index, 0 .. NW*32-1
  const int kg = lane / LPK, li = lane % LPK, f0 = li * PPL;
  // register slot k of this lane holds head (k ^ hmask) of the group, so that the
  // reduce-scatter leaves heads (v ^ hmask), v < VL, in slots 0 .. VL-1
  int hmask = 0;
#pragma unroll
  for (int lv = 0; (G >> (lv + 1)) > 0 && (LPK >> (lv + 1)) > 0; ++lv)
    if (li & (LPK >> (lv + 1))) hmask |= (G >> (lv + 1));
  const bool writer = LPK <= G || (li & (LPK / G - 1)) == 0;  // duplicates stay quiet
  dev::pdl_wait();  // the folded offset factors come from the fold kernel

  double st1[VL], st2[VL];  // this lane's float64 sums of s and s^2 for its heads
  int64_t cached = -1, cur_l = 0, cur_g = 0, cur_b = 0;
  uint32_t it = 0;
  bool failed = false;

  // Publishes this CTA's partial sums for a unit: a fixed-order reduction over
  // the lanes and warps holding each head, then one slot per (unit, CTA).
  auto flush = [&](int64_t unit) {
#pragma unroll
    for (int v = 0; v < VL; ++v) {
      double a = st1[v], b2 = st2[v];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        bool halving = false;  // lanes across a halving level hold different heads
#pragma unroll
        for (int lv = 0; (G >> (lv + 1)) > 0 && (LPK >> (lv + 1)) > 0; ++lv)
          if (o == (LPK >> (lv + 1))) halving = true;
        if (!halving) {
          a += __shfl_xor_sync(0xffffffffu, a, o);
          b2 += __shfl_xor_sync(0xffffffffu, b2, o);
        }
      }
      if (kg == 0 && writer) {
        const int h = v ^ hmask;
        wpart[(warp * G + h) * 2 + 0] = a;
        wpart[(warp * G + h) * 2 + 1] = b2;
      }
    }
    dev::named_barrier(1, NW * 32);
    if (ct < 2 * G) {
      double a = 0.0;
      for (int w = 0; w < NW; ++w) a += wpart[w * G * 2 + ct];
      const int64_t first_tile = (unit / p.B) * p.tiles_per_row + p.tile_prefix[unit % p.B];
      const int64_t slot = blockIdx.x - first_tile / p.tiles_per_cta;
      p.partials[(unit * p.max_slots + slot) * (2 * G) + ct] = a;
    }
    dev::named_barrier(1, NW * 32);
  };

  for (int64_t t = t0; t < t1; ++t) {
    const TileRef tl = tile_of(p, t, TILE);
    if (tl.n <= 0) continue;
    const int64_t unit = (int64_t)tl.row * p.B + tl.b;
    if (unit != cached) {
      if (cached >= 0) flush(cached);
      cached = unit;
      cur_l = tl.row / p.Hkv;
      cur_g = tl.row - cur_l * p.Hkv;
      cur_b = tl.b;
#pragma unroll
      for (int v = 0; v < VL; ++v) { st1[v] = 0.0; st2[v] = 0.0; }
      // lay out the unit's weights in lane order (the previous unit's readers are
      // past the barrier in flush, or this is the first unit)
      for (int e = ct; e < S::WENT; e += NW * 32) {
        const int el = e % LPK, ek = (e / LPK) % G, ei = e / (LPK * G);
        int em = 0;
#pragma unroll
        for (int lv = 0; (G >> (lv + 1)) > 0 && (LPK >> (lv + 1)) > 0; ++lv)
          if (el & (LPK >> (lv + 1))) em |= (G >> (lv + 1));
        const int h = ek ^ em;
        const size_t base = ((size_t)cur_l * p.Hq + (size_t)cur_g * G + h) * F + el * PPL + 2 * ei;
        float wxv[2], wyv[2], nv[2];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const float2 c = p.centre[base + q];
          const double2 ea = p.ea[(size_t)cur_b * F + el * PPL + 2 * ei + q];
          wxv[q] = (float)((double)c.x * ea.x - (double)c.y * ea.y);
          wyv[q] = (float)((double)c.x * ea.y + (double)c.y * ea.x);
          const float r = p.no_conc_weight ? 0.0f : p.mrl[base + q];
          nv[q] = (1.0f - r) * p.mean_norm[base + q];
        }
        wxy[e] = make_float4(wxv[0], wxv[1], wyv[0], wyv[1]);
        wn[e] = make_float2(nv[0], nv[1]);
      }
      dev::named_barrier(1, NW * 32);
    }
    const uint32_t s = it % NST, use = it / NST;
    if (!failed && !dev::mbar_wait(&full[s], use & 1)) {
      dev::set_error(p.err, TRIA_DEVERR_TIMEOUT);
      failed = true;
    }
    if (!failed) {
      const uint8_t *sb = stage + (size_t)s * TILE * ROW;
      float *rawrow = p.raw + ((size_t)cur_l * p.Hq + (size_t)cur_g * G) * p.cap +
                      (size_t)p.seg_start[cur_b] + tl.key0;
#pragma unroll 1
      for (int step = 0; step < S::STEPS; ++step) {
        const int ka = warp * S::KEYS_PER_WARP + step * 2 * KPW + kg, kb = ka + KPW;
        uint32_t xa[P2], ya[P2], xb[P2], yb[P2];
        load_row<D, PPL, LAYOUT>(sb + (size_t)ka * ROW, f0, xa, ya);
        load_row<D, PPL, LAYOUT>(sb + (size_t)kb * ROW, f0, xb, yb);
        // paired float32 arithmetic of sm_100: __ffma2_rn does two FMAs per instruction
        float2 acca[G], accb[G];
#pragma unroll
        for (int k = 0; k < G; ++k) acca[k] = accb[k] = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int i = 0; i < P2; ++i) {
          const float2 XA = bf16x2_to_f2(xa[i]), YA = bf16x2_to_f2(ya[i]);
          const float2 XB = bf16x2_to_f2(xb[i]), YB = bf16x2_to_f2(yb[i]);
          const float2 na2 = __ffma2_rn(YA, YA, __fmul2_rn(XA, XA));
          const float2 nb2 = __ffma2_rn(YB, YB, __fmul2_rn(XB, XB));
          const float2 NA = make_float2(sqrt_approx(na2.x), sqrt_approx(na2.y));
          const float2 NB = make_float2(sqrt_approx(nb2.x), sqrt_approx(nb2.y));
#pragma unroll
          for (int k = 0; k < G; ++k) {
            const int e = (i * G + k) * LPK + li;
            const float4 w4 = wxy[e];
            const float2 WX = make_float2(w4.x, w4.y), WY = make_float2(w4.z, w4.w);
            const float2 WN = wn[e];
            acca[k] = __ffma2_rn(WX, XA, acca[k]);
            accb[k] = __ffma2_rn(WX, XB, accb[k]);
            acca[k] = __ffma2_rn(WY, YA, acca[k]);
            accb[k] = __ffma2_rn(WY, YB, accb[k]);
            acca[k] = __ffma2_rn(WN, NA, acca[k]);
            accb[k] = __ffma2_rn(WN, NB, accb[k]);
          }
        }
        float sa[G], sbv[G];
#pragma unroll
        for (int k = 0; k < G; ++k) {
          sa[k] = acca[k].x + acca[k].y;
          sbv[k] = accb[k].x + accb[k].y;
        }
        reduce_scatter<LPK / 2, G, G>(sa, sbv);
        if (writer) {
#pragma unroll
          for (int v = 0; v < VL; ++v) {
            float *rh = rawrow + (size_t)(v ^ hmask) * p.cap;
            if (ka < tl.n) {
              rh[ka] = sa[v];
              st1[v] += (double)sa[v];
              st2[v] = fma((double)sa[v], (double)sa[v], st2[v]);
            }
            if (kb < tl.n) {
              rh[kb] = sbv[v];
              st1[v] += (double)sbv[v];
              st2[v] = fma((double)sbv[v], (double)sbv[v], st2[v]);
            }
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) dev::mbar_arrive(&empty[s]);
    ++it;
  }
  if (cached >= 0) flush(cached);
}

template <int D, int G, int LAYOUT>
static cudaError_t launch_one(const ScoreParams &p, int grid, cudaStream_t s, bool pdl) {
  using S = ScoreShape<D, G>;
  if constexpr (!S::OK) {
    return cudaErrorInvalidValue;
  } else {
    auto kern = score_kernel<D, G, LAYOUT>;
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
    cfg.blockDim = dim3(kScoreThreads, 1, 1);
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

template <int D, int LAYOUT>
static cudaError_t dispatch_g(const ScoreParams &p, int G, int grid, cudaStream_t s, bool pdl) {
  switch (G) {
    case 1: return launch_one<D, 1, LAYOUT>(p, grid, s, pdl);
    case 2: return launch_one<D, 2, LAYOUT>(p, grid, s, pdl);
    case 4: return launch_one<D, 4, LAYOUT>(p, grid, s, pdl);
    case 8: return launch_one<D, 8, LAYOUT>(p, grid, s, pdl);
    case 16: return launch_one<D, 16, LAYOUT>(p, grid, s, pdl);
    default: return cudaErrorInvalidValue;
  }
}

template <int D>
static bool supported_g(int G) {
  switch (G) {
    case 1: return ScoreShape<D, 1>::OK;
    case 2: return ScoreShape<D, 2>::OK;
    case 4: return ScoreShape<D, 4>::OK;
    case 8: return ScoreShape<D, 8>::OK;
    case 16: return ScoreShape<D, 16>::OK;
    default: return false;
  }
}

bool score_supported(int D, int G, int layout) {
  if (layout != TRIA_ROPE_HALF_SPLIT && layout != TRIA_ROPE_INTERLEAVED) return false;
  switch (D) {
    case 64: return supported_g<64>(G);
    case 128: return supported_g<128>(G);
    case 256: return supported_g<256>(G);
    default: return false;
  }
}

int score_tile_keys(int D) { return kScoreTileBytes / (2 * D); }

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
