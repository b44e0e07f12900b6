// Per-unit stages of the prune step: one thread-block cluster per
// (layer l, KV head g, sequence b).
//
//   z-score + group max (romaanj.github.io review, "Method"; dimensionstp.github.io
//     review, section 3-2 (6)): mu_h and the population sigma_h of the raw
//     scores over the sequence's T live keys (two passes, float64 sums reduced
//     across the cluster in rank order, so the result is deterministic);
//     z_h = (s_h - mu_h) / sigma_h (0 when sigma_h = 0); score = max_h z_h.
//   selection (same sources, "prune back to budget"; section 3-2 (5)): the
//     `budget` largest scores, ties to the lower slot, by a 4-pass 8-bit radix
//     select on order-preserving 32-bit keys.  Each CTA histograms its slice;
//     every CTA then sums the cluster's histograms through distributed shared
//     memory, so all agree on the threshold without a global round trip.
//     The kept slots are emitted in ascending order.
//   compaction (eviction): kept rows of K, V and pos move in place to slots
//     [0, kept).  A kept slot s_j always satisfies s_j >= j, so reading every
//     source of a batch of destinations before any of them is written (one
//     cluster barrier per batch) makes the in-place gather race-free: a
//     destination row j can only be the source of a kept key with index <= j,
//     which belongs to this batch or an earlier one.
//
// Cluster barriers are hardware barriers (barrier.cluster); there are no
// spin-waits in this kernel.
#include <cooperative_groups.h>

#include "tria_internal.cuh"

namespace cg = cooperative_groups;

namespace tria {

namespace {

constexpr int kCtl = 8 * 1024;  // control region at the start of shared memory
constexpr int kMaxG = 16;
constexpr int kWarps = kUnitThreads / 32;

struct Ctl {
  uint32_t hist[2][256];
  uint32_t tot[256];
  double part[2][kMaxG];   // this CTA's partial sums (pass 0: s, pass 1: (s - mu)^2)
  double mu[kMaxG];
  double inv_sigma[kMaxG];
  double wred[kWarps][kMaxG];
  int32_t cnt[4];          // gt, eq (selection) / first_neg, bad (compaction check)
  int32_t bc[8];           // broadcast scalars
  int32_t scan[2][kWarps + 1];
};
static_assert(sizeof(Ctl) <= kCtl, "control region too small");

__device__ __forceinline__ double block_sum_d(double v, double *wred_col, int stride) {
  // returns the block sum in thread 0 only; wred_col[w * stride]
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) wred_col[warp * stride] = v;
  return v;
}

// exclusive block scan of one int per thread; returns the exclusive prefix and the total
__device__ __forceinline__ int block_excl_scan(int v, int32_t *wtot, int *total) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int incl = v;
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) wtot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kWarps ? wtot[lane] : 0;
    int wi = w;
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += t;
    }
    if (lane < kWarps) wtot[lane] = wi - w;  // exclusive warp offsets
    if (lane == kWarps - 1) wtot[kWarps] = wi;
  }
  __syncthreads();
  const int out = wtot[warp] + incl - v;
  *total = wtot[kWarps];
  __syncthreads();
  return out;
}

}  // namespace

__global__ void __launch_bounds__(kUnitThreads, 1) unit_kernel(const __grid_constant__ UnitParams p) {
  cg::cluster_group cl = cg::this_cluster();
  const int CL = (int)cl.num_blocks();
  const int r = (int)cl.block_rank();
  const int64_t unit = blockIdx.x / CL;
  const int b = (int)(unit % p.B);
  const int g = (int)((unit / p.B) % p.Hkv);
  const int l = (int)(unit / ((int64_t)p.B * p.Hkv));
  const int64_t row = (int64_t)l * p.Hkv + g;
  const int64_t seg = p.seg_start[b];
  const int64_t seg_cap = p.seg_start[b + 1] - seg;
  const int G = p.G;
  const int tid = threadIdx.x, nthr = blockDim.x;

  extern __shared__ __align__(128) uint8_t smem[];
  Ctl &c = *reinterpret_cast<Ctl *>(smem);
  uint8_t *data = smem + kCtl;
  const size_t data_bytes = (size_t)kUnitSmemBytes - kCtl;
  int32_t *sel = p.sel + (row * p.B + b) * (int64_t)p.budget;

  int kept = 0;
  // ------------------------------------------------------------ compaction only
  if (p.mode == kModeCompact) {
    const int64_t j0 = (int64_t)p.budget * r / CL, j1 = (int64_t)p.budget * (r + 1) / CL;
    int first_neg = (int)j1, bad = 0;
    for (int64_t j = j0 + tid; j < j1; j += nthr) {
      const int32_t s = __ldcg(sel + j);
      const int32_t prev = j > 0 ? __ldcg(sel + j - 1) : -1;
      if (s < -1 || s >= seg_cap) bad = 1;
      if (s >= 0 && j > 0 && (prev < 0 || s <= prev)) bad = 1;  // ascending, no slot after a -1
      if (s < 0) first_neg = min(first_neg, (int)j);
    }
    if (tid == 0) { c.cnt[2] = (int)j1; c.cnt[3] = 0; }
    __syncthreads();
    atomicMin(&c.cnt[2], first_neg);
    if (bad) atomicOr(&c.cnt[3], 1);
    cl.sync();
    int any_bad = 0;
    kept = p.budget;
    for (int q = 0; q < CL; ++q) {
      const Ctl *peer = cl.map_shared_rank(&c, q);
      kept = min(kept, peer->cnt[2]);
      any_bad |= peer->cnt[3];
    }
    cl.sync();  // peers' control regions are no longer read after this point
    if (any_bad) {
      if (r == 0 && tid == 0) dev::set_error(p.err, TRIA_DEVERR_SELECTION);
      return;
    }
  } else {
    const int32_t T = p.seqlen[b];
    if (T < 0 || (int64_t)T > seg_cap) {
      if (r == 0 && tid == 0) dev::set_error(p.err, TRIA_DEVERR_SEQ_LEN);
      return;  // same decision in every CTA of the cluster
    }
    const bool selects = (p.mode == kModeSelect || p.mode == kModePrune);
    if (selects && T <= p.budget) {
      // sequence at or under budget: every slot is kept, nothing moves
      if (p.mode == kModeSelect || p.write_short_sel) {
        const int64_t j0 = (int64_t)p.budget * r / CL, j1 = (int64_t)p.budget * (r + 1) / CL;
        for (int64_t j = j0 + tid; j < j1; j += nthr) sel[j] = j < T ? (int32_t)j : -1;
      }
      return;
    }
    if (T == 0) return;
    const int64_t lo = (int64_t)T * r / CL, hi = (int64_t)T * (r + 1) / CL;
    const int n = (int)(hi - lo);
    const int nmax = (int)((T + CL - 1) / CL);
    if ((size_t)nmax * 4 > data_bytes) {
      if (r == 0 && tid == 0) dev::set_error(p.err, TRIA_DEVERR_SEGMENT_BIG);
      return;  // every CTA of the cluster takes this branch (same T)
    }
    uint32_t *zkey = reinterpret_cast<uint32_t *>(data);

    if (p.mode == kModeZmax || p.mode == kModePrune) {
      // ---------------------------------------------------- z-score statistics
      const bool cache = (size_t)(G + 1) * nmax * 4 <= data_bytes;
      float *rawc = reinterpret_cast<float *>(data) + nmax;  // [G][nmax]
      const float *rawu = p.raw + ((int64_t)l * p.Hq + (int64_t)g * G) * p.cap + seg;
      for (int j = 0; j < G; ++j) {
        const float *s = rawu + (int64_t)j * p.cap;
        double acc = 0.0;
        for (int i = tid; i < n; i += nthr) {
          const float v = s[lo + i];
          if (cache) rawc[(size_t)j * nmax + i] = v;
          acc += (double)v;
        }
        block_sum_d(acc, &c.wred[0][j], kMaxG);
      }
      __syncthreads();
      if (tid < G) {
        double a = 0.0;
        for (int w = 0; w < kWarps; ++w) a += c.wred[w][tid];
        c.part[0][tid] = a;
      }
      cl.sync();
      if (tid < G) {
        double a = 0.0;
        for (int q = 0; q < CL; ++q) a += cl.map_shared_rank(&c, q)->part[0][tid];
        c.mu[tid] = a / (double)T;
      }
      __syncthreads();
      for (int j = 0; j < G; ++j) {
        const float *s = rawu + (int64_t)j * p.cap;
        const double mu = c.mu[j];
        double acc = 0.0;
        for (int i = tid; i < n; i += nthr) {
          const double d = (double)(cache ? rawc[(size_t)j * nmax + i] : s[lo + i]) - mu;
          acc += d * d;
        }
        block_sum_d(acc, &c.wred[0][j], kMaxG);
      }
      __syncthreads();
      if (tid < G) {
        double a = 0.0;
        for (int w = 0; w < kWarps; ++w) a += c.wred[w][tid];
        c.part[1][tid] = a;
      }
      cl.sync();
      if (tid < G) {
        double a = 0.0;
        for (int q = 0; q < CL; ++q) a += cl.map_shared_rank(&c, q)->part[1][tid];
        const double sigma = sqrt(a / (double)T);
        c.inv_sigma[tid] = sigma > 0.0 ? 1.0 / sigma : 0.0;
      }
      __syncthreads();
      // ---------------------------------------------------- z and group max
      float *score = p.score + row * p.cap + seg;
      for (int i = tid; i < n; i += nthr) {
        double zmax = -1.0e300;
        for (int j = 0; j < G; ++j) {
          const float v = cache ? rawc[(size_t)j * nmax + i] : rawu[(int64_t)j * p.cap + lo + i];
          const double z = ((double)v - c.mu[j]) * c.inv_sigma[j];
          zmax = z > zmax ? z : zmax;
        }
        const float zf = (float)zmax;
        if (p.mode == kModeZmax) score[lo + i] = zf == 0.0f ? 0.0f : zf;
        else zkey[i] = dev::order_key(zf);
      }
      if (p.mode == kModeZmax) {
        cl.sync();  // peers may still read this CTA's partial sums
        return;
      }
    } else {
      const float *score = p.score + row * p.cap + seg;
      for (int i = tid; i < n; i += nthr) zkey[i] = dev::order_key(score[lo + i]);
    }
    __syncthreads();

    // ------------------------------------------------------------ radix select
    uint32_t prefix = 0, mask = 0;
    int krem = p.budget;
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      uint32_t *H = c.hist[pass & 1];
      for (int i = tid; i < 256; i += nthr) H[i] = 0;
      __syncthreads();
      for (int i = tid; i < n; i += nthr) {
        const uint32_t key = zkey[i];
        if ((key & mask) == prefix) atomicAdd(&H[(key >> shift) & 255u], 1u);
      }
      cl.sync();
      for (int i = tid; i < 256; i += nthr) {
        uint32_t a = 0;
        for (int q = 0; q < CL; ++q) a += cl.map_shared_rank(H, q)[i];
        c.tot[i] = a;
      }
      __syncthreads();
      if (tid < 32) {
        uint32_t cnt8[8], s = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) { cnt8[i] = c.tot[tid * 8 + i]; s += cnt8[i]; }
        uint32_t incl = s;  // inclusive suffix over lanes (this lane and above)
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t t = __shfl_down_sync(0xffffffffu, incl, o);
          if (tid + o < 32) incl += t;
        }
        const uint32_t above = incl - s;  // candidates in higher lanes
        if (above < (uint32_t)krem && (uint32_t)krem <= incl) {
          uint32_t cum = above;
          for (int i = 7; i >= 0; --i) {
            if (cum + cnt8[i] >= (uint32_t)krem) {
              c.bc[0] = tid * 8 + i;
              c.bc[1] = krem - (int)cum;
              break;
            }
            cum += cnt8[i];
          }
        }
      }
      __syncthreads();
      const uint32_t d = (uint32_t)c.bc[0];
      krem = c.bc[1];
      prefix |= d << shift;
      mask |= 255u << shift;
      __syncthreads();
    }
    const uint32_t thr = prefix;
    const int k_eq = krem;  // keys equal to thr that are kept (the lowest slots)

    // ------------------------------------------------------------ emit kept slots
    const int RL = (n + nthr - 1) / nthr;
    const int a0 = min(n, tid * RL), a1 = min(n, a0 + RL);
    int gt = 0, eq = 0;
    for (int i = a0; i < a1; ++i) {
      const uint32_t key = zkey[i];
      gt += key > thr;
      eq += key == thr;
    }
    int tot_gt, tot_eq;
    const int gt_x = block_excl_scan(gt, c.scan[0], &tot_gt);
    const int eq_x = block_excl_scan(eq, c.scan[1], &tot_eq);
    (void)gt_x;
    if (tid == 0) { c.cnt[0] = tot_gt; c.cnt[1] = tot_eq; }
    cl.sync();
    if (tid == 0) {
      int eqb = 0, base = 0;
      for (int q = 0; q < CL; ++q) {
        const Ctl *peer = cl.map_shared_rank(&c, q);
        const int qg = peer->cnt[0], qe = peer->cnt[1];
        const int take = max(0, min(qe, k_eq - eqb));
        if (q == r) { c.bc[2] = eqb; c.bc[3] = base; }
        eqb += qe;
        base += qg + take;
      }
    }
    __syncthreads();
    const int eq_before = c.bc[2] + eq_x;
    const int take = max(0, min(eq, k_eq - eq_before));
    int dummy;
    const int out0 = c.bc[3] + block_excl_scan(gt + take, c.scan[0], &dummy);
    {
      int o = out0, er = eq_before;
      for (int i = a0; i < a1; ++i) {
        const uint32_t key = zkey[i];
        bool keep = key > thr;
        if (key == thr) { keep = er < k_eq; ++er; }
        if (keep) {
          if (o < p.budget) sel[o] = (int32_t)(lo + i);
          ++o;
        }
      }
    }
    __threadfence();
    cl.sync();  // selection list complete and visible; peers' control regions no longer read
    if (p.mode == kModeSelect) return;
    kept = p.budget;
  }

  // -------------------------------------------------------------- in-place compaction
  const int ROW = 2 * p.D;                 // bytes per K or V row
  const int VPR = ROW / 16;                // 16-byte vectors per row
  const int row_bytes = 2 * ROW + 4;       // staged K + V + pos
  const int cap_rows = (int)(data_bytes / row_bytes);
  const int64_t j0 = (int64_t)p.budget * r / CL, j1 = (int64_t)p.budget * (r + 1) / CL;
  const int range_max = (p.budget + CL - 1) / CL;
  const int batches = (range_max + cap_rows - 1) / cap_rows;
  uint4 *sk = reinterpret_cast<uint4 *>(data);                    // [cap_rows][VPR]
  uint4 *sv = sk + (size_t)cap_rows * VPR;                         // [cap_rows][VPR]
  int32_t *sp = reinterpret_cast<int32_t *>(sv + (size_t)cap_rows * VPR);  // [cap_rows]
  const int64_t rbase = row * p.cap + seg;
  uint4 *kg4 = reinterpret_cast<uint4 *>(p.k + (size_t)rbase * ROW);
  uint4 *vg4 = reinterpret_cast<uint4 *>(p.v + (size_t)rbase * ROW);
  int32_t *pg = p.pos + rbase;
  for (int bt = 0; bt < batches; ++bt) {
    const int64_t a = j0 + (int64_t)bt * cap_rows;
    int64_t e = a + cap_rows;
    if (e > j1) e = j1;
    if (e > kept) e = kept;
    const int nb = e > a ? (int)(e - a) : 0;
    for (int idx = tid; idx < nb * VPR; idx += nthr) {
      const int jj = idx / VPR, v = idx - jj * VPR;
      const int32_t s = __ldcg(sel + a + jj);
      if (s < 0 || s >= seg_cap) {  // cannot happen for a well-formed list; never read outside
        if (v == 0) dev::set_error(p.err, TRIA_DEVERR_SELECTION);
        continue;
      }
      if (s != a + jj) {
        sk[(size_t)jj * VPR + v] = kg4[(size_t)s * VPR + v];
        sv[(size_t)jj * VPR + v] = vg4[(size_t)s * VPR + v];
        if (v == 0) sp[jj] = pg[s];
      }
    }
    cl.sync();  // every source row of this batch has been read, cluster-wide
    for (int idx = tid; idx < nb * VPR; idx += nthr) {
      const int jj = idx / VPR, v = idx - jj * VPR;
      const int32_t s = __ldcg(sel + a + jj);
      if (s >= 0 && s < seg_cap && s != a + jj) {
        kg4[(size_t)(a + jj) * VPR + v] = sk[(size_t)jj * VPR + v];
        vg4[(size_t)(a + jj) * VPR + v] = sv[(size_t)jj * VPR + v];
        if (v == 0) pg[a + jj] = sp[jj];
      }
    }
    __syncthreads();  // staging buffer reused by the next batch
  }
  if (r == 0 && tid == 0 && l == 0 && g == 0) p.seq_len_out[b] = kept;
}

static int g_cluster[64];  // per device: chosen cluster size (0 = not yet chosen)

int unit_cluster_size() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 8;
  if (g_cluster[dev]) return g_cluster[dev];
  cudaFuncSetAttribute(unit_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kUnitSmemBytes);
  cudaFuncSetAttribute(unit_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  int chosen = 8;
  for (int cs : {16, 8}) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cs, 1, 1);
    cfg.blockDim = dim3(kUnitThreads, 1, 1);
    cfg.dynamicSmemBytes = kUnitSmemBytes;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = cs;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, unit_kernel, &cfg) == cudaSuccess && n > 0) {
      chosen = cs;
      break;
    }
    cudaGetLastError();
  }
  g_cluster[dev] = chosen;
  return chosen;
}

cudaError_t launch_unit(const UnitParams &p, int units, cudaStream_t s) {
  const int cs = unit_cluster_size();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)units * cs, 1, 1);
  cfg.blockDim = dim3(kUnitThreads, 1, 1);
  cfg.dynamicSmemBytes = kUnitSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = cs;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, unit_kernel, p);
}

}  // namespace tria
