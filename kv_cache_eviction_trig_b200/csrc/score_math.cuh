// Per-key arithmetic of the key score, shared by the kernels that score keys
// out of 128-byte-swizzled shared-memory chunks written by 2-D TMA loads.
//
// For a key t of KV head g and a query head h of g's group (romaanj.github.io
// review, "Method"; dimensionstp.github.io review, sections 2-2 and 3-2 (2)-(4)):
//   s_h(t) = sum_f [ Re(conj(ktilde_f) * W_hf) + Nw_hf * |ktilde_f| ]
// with ktilde the stored post-RoPE key, W_hf = c_hf * e^{i w_f cur} * mean_delta
// e^{i w_f delta} (the trigonometric term with the offsets and the current
// position folded in; the key position cancels) and Nw_hf = (1 - R_hf) E|q_hf|.
// Sums are float32 over exact bf16 inputs.
//
// Weights of one unit sit in shared memory as [F/2][G][6] floats: for the RoPE
// pairs 2fp and 2fp+1 and head h, (Re W, Re W, Im W, Im W, Nw, Nw).
#pragma once

#include "tria_internal.cuh"

namespace tria {

template <int D, int G>
struct KeyShape {
  static constexpr int F = D / 2;
  static constexpr int FP = F / 2;                                 // pairs of RoPE pairs
  static constexpr int KPT_D = 256 / D;                            // 16 KB chunks
  static constexpr int KPT_G = G <= 2 ? 4 : (G == 4 ? 2 : 1);      // accumulator registers
  static constexpr int KPT0 = KPT_D < KPT_G ? KPT_D : KPT_G;
  static constexpr int KPT = KPT0 < kScoreKptCap ? KPT0 : kScoreKptCap;  // keys per lane
  static constexpr int CH = 32 * KPT;                              // keys per chunk
  static constexpr int NBOX = D / 64;                              // 128-byte boxes per row
  static constexpr int BOXB = CH * 128;                            // bytes per box region
  static constexpr int CB = CH * 2 * D;                            // bytes per chunk
  static constexpr int WB = FP * G * 24;                           // weight bytes per unit
  static constexpr int JU = 4;                                     // pair-pairs per iteration
  static_assert(FP % JU == 0, "head_dim must be a multiple of 16");
  static_assert(CB % 1024 == 0, "chunks keep the 1024-byte swizzle alignment");
};

namespace km {

__device__ __forceinline__ float sqrt_approx(float x) {
  float y;
  asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// A bf16 pair (one 32-bit word) widened exactly into a float pair.
__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t w) {
  return make_float2(dev::bf16lo(w), dev::bf16hi(w));
}

// acc += wx * x + wy * y + wn * n, two RoPE pairs at a time.
__device__ __forceinline__ void fma3(float2 &acc, float2 wx, float2 wy, float2 wn, float2 x,
                                     float2 y, float2 n) {
  acc = __ffma2_rn(wx, x, acc);
  acc = __ffma2_rn(wy, y, acc);
  acc = __ffma2_rn(wn, n, acc);
}

// Shared-memory address of the 16-byte unit holding elements e .. e+7 (e a
// multiple of 8) of row r inside a chunk of 128-byte-swizzled boxes: box e / 64
// holds elements [64 box, 64 box + 64) of every row, 128 bytes per row, and unit u
// of a row is stored at unit u ^ (r & 7).  With a = chunk + 128 r + 16 (r & 7)
// (the row's base with its swizzle folded in), the unit sits at
// (a ^ 16 ((e / 8) & 7)) + (e / 64) * BOXB: the XOR touches bits 4-6 only, the box
// offset bits >= 10.
template <int BOXB>
__device__ __forceinline__ uint32_t unit_addr(uint32_t a, int e) {
  return (a ^ (uint32_t)(((e >> 3) & 7) << 4)) + (uint32_t)(e >> 6) * BOXB;
}

// 16-byte shared-memory load.  Volatile: it stays after the mbarrier wait that
// made the TMA-written bytes visible.
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

// The x and y words of RoPE pairs 8 it .. 8 it + 7 of the row whose swizzled base
// (shared-memory address) is a: xw[j] holds the x components of pairs
// (8 it + 2j, 8 it + 2j + 1), likewise yw.
template <int D, int BOXB, int LAYOUT>
__device__ __forceinline__ void load_pairs8(uint32_t a, int it, uint32_t (&xw)[4],
                                            uint32_t (&yw)[4]) {
  constexpr int F = D / 2;
  if constexpr (LAYOUT == TRIA_ROPE_HALF_SPLIT) {
    const uint4 xa = lds128(unit_addr<BOXB>(a, 8 * it));
    const uint4 ya = lds128(unit_addr<BOXB>(a, F + 8 * it));
    xw[0] = xa.x; xw[1] = xa.y; xw[2] = xa.z; xw[3] = xa.w;
    yw[0] = ya.x; yw[1] = ya.y; yw[2] = ya.z; yw[3] = ya.w;
  } else {
    // interleaved: word q holds (x_q, y_q); regroup into x and y pairs
    const uint4 w0 = lds128(unit_addr<BOXB>(a, 16 * it));
    const uint4 w1 = lds128(unit_addr<BOXB>(a, 16 * it + 8));
    const uint32_t w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      xw[i] = __byte_perm(w[2 * i], w[2 * i + 1], 0x5410);  // (x_2i, x_2i+1)
      yw[i] = __byte_perm(w[2 * i], w[2 * i + 1], 0x7632);  // (y_2i, y_2i+1)
    }
  }
}

// Raw scores of the KPT keys r = lane + 32 k of a chunk for the G heads:
// out[k][h] = s_h(key r).  chunk_s is the chunk's shared-memory address, wu the
// unit's weights in shared memory.  `iters` < FP / 4 runs a shortened pass (used
// to fetch the code before the real work starts).
template <int D, int G, int LAYOUT>
__device__ __forceinline__ void score_chunk(uint32_t chunk_s, const float *wu, int lane,
                                            int iters, float (&out)[KeyShape<D, G>::KPT][G]) {
  using S = KeyShape<D, G>;
  constexpr int KPT = S::KPT;
  uint32_t a[KPT];
#pragma unroll
  for (int k = 0; k < KPT; ++k) {
    const uint32_t r = (uint32_t)(lane + 32 * k);
    a[k] = chunk_s + 128u * r + ((r & 7u) << 4);
  }
  float2 acc[KPT][G];
#pragma unroll
  for (int k = 0; k < KPT; ++k)
#pragma unroll
    for (int h = 0; h < G; ++h) acc[k][h] = make_float2(0.0f, 0.0f);

#pragma unroll 1
  for (int it = 0; it < iters; ++it) {
    uint32_t xw[KPT][4], yw[KPT][4];
#pragma unroll
    for (int k = 0; k < KPT; ++k) load_pairs8<D, S::BOXB, LAYOUT>(a[k], it, xw[k], yw[k]);
    const float *wi = wu + (size_t)it * (4 * 6 * G);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float *wf = wi + j * 6 * G;
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
  for (int k = 0; k < KPT; ++k)
#pragma unroll
    for (int h = 0; h < G; ++h) out[k][h] = acc[k][h].x + acc[k][h].y;
}

}  // namespace km
}  // namespace tria
