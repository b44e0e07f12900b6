// Fold of the future-offset average and the current position into one complex
// factor per (sequence, RoPE pair).
//
// The trigonometric term of the key score (romaanj.github.io review, "Method";
// dimensionstp.github.io review, section 2-2) is
//   S_trig = mean_delta sum_f |c_f||k_f| cos(w_f (cur + delta - p) + arg c_f - arg k_f).
// With the pre-RoPE key k_f = ktilde_f e^{-i w_f p} the key's position p cancels
// and the sum becomes Re sum_f conj(ktilde_f) * c_f * EA_f with
//   EA_f = e^{i w_f cur} * (1/|O|) sum_{delta in O} e^{i w_f delta},
// so the per-key work needs no position and no trigonometry.  EA is formed
// here in float64 (angles reach ~1e5 rad); block f handles pair f.
// Block 0 also snapshots and checks seq_len, so that every later kernel of
// the call sees the lengths as they were at its start.
#include "tria_internal.cuh"

namespace tria {

__global__ void __launch_bounds__(256) fold_kernel(const __grid_constant__ FoldParams p) {
  dev::pdl_launch_dependents();  // the score kernel may start streaming keys now
  const int f = blockIdx.x;
  const double w = pow(p.theta, -2.0 * (double)f / (double)p.D);
  double sc = 0.0, ss = 0.0;
  for (int j = threadIdx.x; j < p.n_offsets; j += blockDim.x) {
    double s, c;
    sincos(w * (double)p.offsets[j], &s, &c);
    sc += c;
    ss += s;
  }
  // fixed-order block reduction (deterministic)
  for (int o = 16; o > 0; o >>= 1) {
    sc += __shfl_xor_sync(0xffffffffu, sc, o);
    ss += __shfl_xor_sync(0xffffffffu, ss, o);
  }
  __shared__ double red[2][8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) { red[0][warp] = sc; red[1][warp] = ss; }
  __syncthreads();
  if (threadIdx.x == 0) {
    double a = 0.0, b = 0.0;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) { a += red[0][i]; b += red[1][i]; }
    red[0][0] = a / (double)p.n_offsets;
    red[1][0] = b / (double)p.n_offsets;
  }
  __syncthreads();
  double ax = red[0][0], ay = red[1][0];
  if (p.flags & TRIA_NO_TRIG) { ax = 0.0; ay = 0.0; }
  const int F = p.D / 2;
  for (int b = threadIdx.x; b < p.B; b += blockDim.x) {
    double s, c;
    sincos(w * (double)p.cur_pos[b], &s, &c);
    p.ea[(size_t)b * F + f] = make_double2(c * ax - s * ay, c * ay + s * ax);
  }
  if (f == 0) {
    for (int b = threadIdx.x; b < p.B; b += blockDim.x) {
      int32_t T = p.seq_len[b];
      if (T < 0 || (int64_t)T > p.seg_cap[b]) {
        dev::set_error(p.err, TRIA_DEVERR_SEQ_LEN);
        T = 0;
      }
      p.seqlen_snap[b] = T;
    }
  }
}

cudaError_t launch_fold(const FoldParams &p, int F, cudaStream_t s) {
  fold_kernel<<<F, 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace tria
