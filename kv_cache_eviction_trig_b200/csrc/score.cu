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
// time).  The folded weights are the same for every lane, so they are read as
// broadcast loads that stay in L1.  No cross-lane reduction and no
// synchronisation between consumer warps are needed.
#include <cudaTypedefs.h>

#include <mutex>

#include "tria_internal.cuh"

namespace tria {

template <int D, int G>
struct ScoreShape {
  static constexpr int F = D / 2;
  static constexpr int FP = F / 2;                                 // RoPE pair pairs
  static constexpr int KPT_D = 256 / D;                            // 16 KB chunks
  static constexpr int KPT_G = G <= 2 ? 4 : (G == 4 ? 2 : 1);      // accumulator registers
  static constexpr int KPT0 = KPT_D < KPT_G ? KPT_D : KPT_G;
  static constexpr int KPT = KPT0 < kScoreKptCap ? KPT0 : kScoreKptCap;  // keys per lane
  static constexpr int CH = 32 * KPT;                              // keys per chunk
  static constexpr int NBOX = D / 64;                              // 128-byte boxes per row
  static constexpr int BOXB = CH * 128;                            // bytes per box region
  static constexpr int CB = CH * 2 * D;                            // bytes per chunk
  static constexpr int NW = kScoreConsumerWarps;
  static constexpr int NSLOT = kScoreRingBytes / CB < 24 ? kScoreRingBytes / CB : 24;
  static constexpr bool OK = (D == 64 || D == 128 || D == 256) &&
                             (G == 1 || G == 2 || G == 4 || G == 8 || G == 16) && NSLOT > NW;
  static constexpr size_t SMEM =
      1024 + (size_t)NSLOT * CB + (size_t)NSLOT * 16 + 2ull * NSLOT * 8 + 4ull * TRIA_MAX_BATCH;
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

// 16-byte chunk `c` (0..7) of row `r` of a 128-byte-swizzled box region.
__device__ __forceinline__ uint4 lds_swizzled(const uint8_t *box, int r, int c) {
  return *reinterpret_cast<const uint4 *>(box + r * 128 + ((c ^ (r & 7)) << 4));
}

// The x and y words of RoPE pairs 8*c8 .. 8*c8+7 of row r: x pairs (f, f+1) in xw[j]
// for f = 8*c8 + 2j, likewise y.
template <int D, int CH, int LAYOUT>
__device__ __forceinline__ void load_pairs(const uint8_t *chunk, int r, int c8, uint32_t (&xw)[4],
                                           uint32_t (&yw)[4]) {
  constexpr int F = D / 2;
  constexpr int BOXB = CH * 128;
  if constexpr (LAYOUT == TRIA_ROPE_HALF_SPLIT) {
    const int dx = 8 * c8, dy = F + 8 * c8;  // first element of the x and y runs
    const uint4 a = lds_swizzled(chunk + (dx >> 6) * BOXB, r, (dx & 63) >> 3);
    const uint4 b = lds_swizzled(chunk + (dy >> 6) * BOXB, r, (dy & 63) >> 3);
    xw[0] = a.x; xw[1] = a.y; xw[2] = a.z; xw[3] = a.w;
    yw[0] = b.x; yw[1] = b.y; yw[2] = b.z; yw[3] = b.w;
  } else {
    // interleaved: word q holds (x_q, y_q); regroup into x and y pairs
    const int d0 = 16 * c8;
    const uint8_t *box = chunk + (d0 >> 6) * BOXB;
    const uint4 a = lds_swizzled(box, r, (d0 & 63) >> 3);
    const uint4 b = lds_swizzled(box, r, ((d0 & 63) >> 3) + 1);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      xw[i] = __byte_perm(w[2 * i], w[2 * i + 1], 0x5410);  // (x_2i, x_2i+1)
      yw[i] = __byte_perm(w[2 * i], w[2 * i + 1], 0x7632);  // (y_2i, y_2i+1)
    }
  }
}

// acc += wx * x + wy * y + wn * n, two RoPE pairs at a time.
__device__ __forceinline__ void fma3(float2 &acc, float2 wx, float2 wy, float2 wn, float2 x,
                                     float2 y, float2 n) {
  acc = __ffma2_rn(wx, x, acc);
  acc = __ffma2_rn(wy, y, acc);
  acc = __ffma2_rn(wn, n, acc);
}

template <int D, int G, int LAYOUT>
__global__ void __launch_bounds__(kScoreThreads, 1)
    score_kernel(const __grid_constant__ ScoreParams p) {
  using S = ScoreShape<D, G>;
  constexpr int F = S::F, FP = S::FP, KPT = S::KPT, CH = S::CH, CB = S::CB, NW = S::NW;
  constexpr int NSLOT = S::NSLOT;

  extern __shared__ uint8_t smem_raw[];
  uint8_t *ring = smem_raw + ((1024u - (dev::smem_addr(smem_raw) & 1023u)) & 1023u);
  int4 *desc = reinterpret_cast<int4 *>(ring + (size_t)NSLOT * CB);  // per slot: row, b, key0, n
  uint64_t *full = reinterpret_cast<uint64_t *>(desc + NSLOT);
  uint64_t *empty = full + NSLOT;
  int32_t *live = reinterpret_cast<int32_t *>(empty + NSLOT);  // [B] keys to score per sequence

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NSLOT; ++s) {
      dev::mbar_init(&full[s], 1);
      dev::mbar_init(&empty[s], 1);
    }
    dev::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) dev::pdl_launch_dependents();

  if (warp == NW) {
    // ---------------------------------------------------------------- producer
    for (int b = lane; b < p.B; b += 32) {
      int32_t T = p.seq_len[b];
      if (T < 0 || (int64_t)T > p.seg_start[b + 1] - p.seg_start[b]) T = 0;  // flagged by the fold
      if (p.skip_short && T <= p.budget) T = 0;
      live[b] = T;
    }
    __syncwarp();
    if (lane == 0) {
      const int c0 = blockIdx.x * p.chunks_per_cta;
      const int c1 = min(c0 + p.chunks_per_cta, p.total_chunks);
      uint32_t q = 0;
      bool failed = false;
      for (int c = c0; c < c1 && !failed; ++c) {
        const int row = c / p.chunks_per_row;
        const int rem = c - row * p.chunks_per_row;
        int lo = 0, hi = p.B;  // largest b with chunk_prefix[b] <= rem
        while (hi - lo > 1) {
          const int mid = (lo + hi) >> 1;
          if (p.chunk_prefix[mid] <= rem) lo = mid; else hi = mid;
        }
        const int key0 = (rem - p.chunk_prefix[lo]) * CH;
        const int n = min(max(live[lo] - key0, 0), CH);
        if (n == 0) continue;
        const uint32_t s = q % NSLOT, use = q / NSLOT;
        if (use > 0 && !dev::mbar_wait(&empty[s], (use - 1) & 1)) {
          failed = true;
          break;
        }
        desc[s] = make_int4(row, lo, key0, n);
        dev::mbar_arrive_expect_tx(&full[s], CB);
        const int32_t y = (int32_t)((int64_t)row * p.cap + p.seg_start[lo] + key0);
#pragma unroll
        for (int bx = 0; bx < S::NBOX; ++bx)
          dev::tma_load_2d(ring + (size_t)s * CB + bx * S::BOXB, &p.tmap, bx * 64, y, &full[s]);
        ++q;
      }
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
  dev::pdl_wait();  // the folded weights come from the fold kernel
  for (uint32_t q = warp;; q += NW) {
    const uint32_t s = q % NSLOT, use = q / NSLOT;
    // the slot's previous chunk was released, so the parity below is this use's
    if ((use > 0 && !dev::mbar_wait(&empty[s], (use - 1) & 1)) ||
        !dev::mbar_wait(&full[s], use & 1)) {
      if (lane == 0) dev::set_error(p.err, TRIA_DEVERR_TIMEOUT);
      break;
    }
    const int4 d = desc[s];
    if (d.w < 0) break;
    const int row = d.x, b = d.y, key0 = d.z, n = d.w;
    const int64_t unit = (int64_t)row * p.B + b;
    const float *wu = p.w + (size_t)unit * FP * 6 * G;
    const uint8_t *chunk = ring + (size_t)s * CB;

    float2 acc[KPT][G];
#pragma unroll
    for (int k = 0; k < KPT; ++k)
#pragma unroll
      for (int h = 0; h < G; ++h) acc[k][h] = make_float2(0.0f, 0.0f);

#pragma unroll 1
    for (int c8 = 0; c8 < F / 8; ++c8) {
      uint32_t xw[KPT][4], yw[KPT][4];
#pragma unroll
      for (int k = 0; k < KPT; ++k) load_pairs<D, CH, LAYOUT>(chunk, lane + 32 * k, c8, xw[k], yw[k]);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float *wf = wu + (size_t)(4 * c8 + j) * 6 * G;
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
    const int l = row / p.Hkv, g = row - l * p.Hkv;
    float *rawp = p.raw + ((size_t)l * p.Hq + (size_t)g * G) * p.cap + p.seg_start[b] + key0;
#pragma unroll
    for (int k = 0; k < KPT; ++k) {
      const int r = lane + 32 * k;
      if (r < n) {
#pragma unroll
        for (int h = 0; h < G; ++h) rawp[(size_t)h * p.cap + r] = acc[k][h].x + acc[k][h].y;
      }
    }
    __syncwarp();
    if (lane == 0) dev::mbar_arrive(&empty[s]);
  }
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
