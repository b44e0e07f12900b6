// Fold of the future-offset average, the current position and the calibrated
// query statistics into one weight triple per (unit, query head, RoPE pair).
//
// The trigonometric term of the key score (romaanj.github.io review, "Method";
// dimensionstp.github.io review, section 2-2) is
//   S_trig = mean_delta sum_f |c_f||k_f| cos(w_f (cur + delta - p) + arg c_f - arg k_f).
// With the pre-RoPE key k_f = ktilde_f e^{-i w_f p} the key's position p cancels
// and the sum becomes Re sum_f conj(ktilde_f) * W_f with
//   W_f  = c_f * EA_f,   EA_f = e^{i w_f cur} * (1/|O|) sum_{delta in O} e^{i w_f delta},
// so the per-key work needs no position and no trigonometry.  The norm term's
// weight is Nw_f = (1 - R_f) E|q_f| (section 3-2 (3)-(4)).
//
// Block (fp, y) handles the RoPE pairs f = 2fp, 2fp+1 (w_f and the offset average
// A_f come from the host, in double precision): it forms EA = e^{i w_f cur} A_f in
// float64 (angles reach ~1e5 rad) for every sequence, then writes, for a share y of
// the (unit, head) pairs, the float32 weights
//   w[unit][fp][h] = (Re W_2fp, Re W_2fp+1, Im W_2fp, Im W_2fp+1, Nw_2fp, Nw_2fp+1).
// Block (0, 0) also snapshots and checks seq_len (blocks (0, y) the per-unit
// lengths, when the cache has them), so that every later kernel of the call sees
// the lengths as they were at its start.
#include "tria_internal.cuh"

namespace tria {

static_assert(TRIA_MAX_BATCH <= 256, "the fold handles one sequence per thread of a block");

__global__ void __launch_bounds__(256) fold_kernel(const __grid_constant__ FoldParams p) {
  dev::pdl_launch_dependents();  // the score kernel may start streaming keys now
  const int fp = blockIdx.x;
  const int F = p.D / 2;
  __shared__ double2 ea[TRIA_MAX_BATCH][2];
  // Loads that do not depend on the trigonometry are issued first.
  const int64_t units = (int64_t)p.L * p.Hkv * p.B;
  const int64_t entries = units * p.G;
  const int64_t e0 = (int64_t)blockIdx.y * blockDim.x + threadIdx.x;
  float2 c0[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
  float r0[2] = {0.f, 0.f}, m0[2] = {0.f, 0.f};
  if (e0 < entries) {
    const int64_t unit = e0 / p.G;
    const int h = (int)(e0 - unit * p.G);
    const int64_t lg = unit / p.B;
    const int l = (int)(lg / p.Hkv), g = (int)(lg % p.Hkv);
    const size_t base0 = ((size_t)l * p.Hq + (size_t)g * p.G + h) * F + 2 * fp;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      c0[q] = p.centre[base0 + q];
      r0[q] = p.mrl[base0 + q];
      m0[q] = p.mean_norm[base0 + q];
    }
  }
  const int32_t cur = threadIdx.x < p.B ? p.cur_pos[threadIdx.x] : 0;
  const bool snap = !p.unit_len && blockIdx.x == 0 && blockIdx.y == 0 && (int)threadIdx.x < p.B;
  const int32_t t_in = snap ? p.seq_len[threadIdx.x] : 0;
  // w_f = theta^(-2f/D), evaluated on the host in double precision
  const double w[2] = {p.omega[2 * fp], p.omega[2 * fp + 1]};
  // the offset average A_f = mean_delta e^{i w_f delta}, from the host (float64)
  const double A[4] = {p.A[2 * fp].x, p.A[2 * fp].y, p.A[2 * fp + 1].x, p.A[2 * fp + 1].y};
  for (int b = threadIdx.x; b < p.B; b += blockDim.x) {
    const int32_t cb = b == (int)threadIdx.x ? cur : p.cur_pos[b];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      double s, c;
      sincos(w[q] * (double)cb, &s, &c);
      const double ax = A[2 * q], ay = A[2 * q + 1];
      ea[b][q] = make_double2(c * ax - s * ay, c * ay + s * ax);
    }
  }
  __syncthreads();

  const int FP = F / 2;
  for (int64_t e = e0; e < entries; e += (int64_t)gridDim.y * blockDim.x) {
    const int64_t unit = e / p.G;
    const int h = (int)(e - unit * p.G);
    const int b = (int)(unit % p.B);
    const int64_t lg = unit / p.B;
    const int l = (int)(lg / p.Hkv), g = (int)(lg % p.Hkv);
    const size_t base = ((size_t)l * p.Hq + (size_t)g * p.G + h) * F + 2 * fp;
    float wx[2], wy[2], nw[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const bool pre = e == e0;  // the first entry's inputs were loaded up front
      const float2 c = pre ? c0[q] : p.centre[base + q];
      const double2 e2 = ea[b][q];
      wx[q] = (float)((double)c.x * e2.x - (double)c.y * e2.y);
      wy[q] = (float)((double)c.x * e2.y + (double)c.y * e2.x);
      const float r = (p.flags & TRIA_NO_CONC_WEIGHT) ? 0.0f : (pre ? r0[q] : p.mrl[base + q]);
      nw[q] = (1.0f - r) * (pre ? m0[q] : p.mean_norm[base + q]);
    }
    float2 *out = reinterpret_cast<float2 *>(p.w + ((size_t)unit * FP + fp) * (6 * p.G) + 6 * h);
    out[0] = make_float2(wx[0], wx[1]);
    out[1] = make_float2(wy[0], wy[1]);
    out[2] = make_float2(nw[0], nw[1]);
  }

  if (snap) {  // B <= TRIA_MAX_BATCH = blockDim.x: one sequence per thread
    int32_t T = t_in;
    if (T < 0 || (int64_t)T > p.seg_cap[threadIdx.x]) {
      dev::set_error(p.err, TRIA_DEVERR_SEQ_LEN);
      T = 0;
    }
    p.seqlen_snap[threadIdx.x] = T;
  }
  if (p.unit_len && blockIdx.x == 0) {  // per-unit lengths: blocks (0, y) share the units
    for (int64_t u = (int64_t)blockIdx.y * blockDim.x + threadIdx.x; u < p.units;
         u += (int64_t)gridDim.y * blockDim.x) {
      int32_t T = p.unit_len[u];
      if (T < 0 || (int64_t)T > p.seg_cap[u % p.B]) {
        dev::set_error(p.err, TRIA_DEVERR_SEQ_LEN);
        T = 0;
      }
      p.seqlen_snap[u] = T;
    }
  }
}

cudaError_t launch_fold(const FoldParams &p, cudaStream_t s) {
  const int FP = p.D / 4;
  const int64_t entries = (int64_t)p.L * p.Hkv * p.B * p.G;
  // about 8 entries per thread, at most 64 blocks per pair
  int64_t y = (entries + 2047) / 2048;
  if (y < 1) y = 1;
  if (y > 64) y = 64;
  fold_kernel<<<dim3((unsigned)FP, (unsigned)y), 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace tria
