// Offline calibration (romaanj.github.io review, "Method"; dimensionstp.github.io
// review, section 3-1): for every (layer, query head, RoPE pair f) over the N
// sample pre-RoPE queries,
//   centre_f = mean_n q_f (complex),  mean_f = mean_n |q_f|,  R_f = |centre_f| / mean_f
// (R_f = 0 when mean_f = 0).  One block per (layer, head); float64 accumulation.
#include <cuda_bf16.h>

#include "tria_internal.cuh"

namespace tria {

template <typename Tq>
__device__ __forceinline__ double widen(Tq v);
template <>
__device__ __forceinline__ double widen<float>(float v) { return (double)v; }
template <>
__device__ __forceinline__ double widen<__nv_bfloat16>(__nv_bfloat16 v) {
  return (double)__bfloat162float(v);
}

template <typename Tq>
__global__ void __launch_bounds__(256) calibrate_kernel(const Tq *q, int64_t N, int64_t Hq,
                                                        int D, int layout, float *centre,
                                                        float *mean_norm, float *mrl) {
  const int F = D / 2;
  const int64_t lh = blockIdx.x;
  const int64_t l = lh / Hq, h = lh % Hq;
  const int lanes = blockDim.x / F;  // samples handled in parallel per pair
  const int f = threadIdx.x % F, s0 = threadIdx.x / F;
  const int xi = layout == TRIA_ROPE_HALF_SPLIT ? f : 2 * f;
  const int yi = layout == TRIA_ROPE_HALF_SPLIT ? f + F : 2 * f + 1;
  double sx = 0.0, sy = 0.0, sn = 0.0;
  if (s0 < lanes) {
    for (int64_t n = s0; n < N; n += lanes) {
      const Tq *v = q + ((l * N + n) * Hq + h) * (int64_t)D;
      const double x = widen<Tq>(v[xi]), y = widen<Tq>(v[yi]);
      sx += x;
      sy += y;
      sn += sqrt(x * x + y * y);
    }
  }
  __shared__ double red[3][256];
  red[0][threadIdx.x] = sx;
  red[1][threadIdx.x] = sy;
  red[2][threadIdx.x] = sn;
  __syncthreads();
  if (threadIdx.x < F) {
    double a = 0.0, b = 0.0, m = 0.0;
    for (int k = 0; k < lanes; ++k) {  // fixed order
      a += red[0][k * F + f];
      b += red[1][k * F + f];
      m += red[2][k * F + f];
    }
    a /= (double)N;
    b /= (double)N;
    m /= (double)N;
    const int64_t o = lh * F + f;
    centre[2 * o] = (float)a;
    centre[2 * o + 1] = (float)b;
    mean_norm[o] = (float)m;
    mrl[o] = m > 0.0 ? (float)(sqrt(a * a + b * b) / m) : 0.0f;
  }
}

cudaError_t launch_calibrate(const void *q, int q_dtype, int64_t L, int64_t N, int64_t Hq,
                             int64_t D, int layout, float *centre, float *mean_norm, float *mrl,
                             cudaStream_t s) {
  const unsigned blocks = (unsigned)(L * Hq);
  if (q_dtype == TRIA_DTYPE_F32)
    calibrate_kernel<float><<<blocks, 256, 0, s>>>(static_cast<const float *>(q), N, Hq, (int)D,
                                                   layout, centre, mean_norm, mrl);
  else
    calibrate_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(
        static_cast<const __nv_bfloat16 *>(q), N, Hq, (int)D, layout, centre, mean_norm, mrl);
  return cudaGetLastError();
}

}  // namespace tria
