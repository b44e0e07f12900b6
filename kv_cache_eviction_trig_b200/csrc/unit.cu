// Per-unit stages of the prune step: one thread-block cluster per
// (layer l, KV head g, sequence b).
//
//   z-score + group max (romaanj.github.io review, "Method"; dimensionstp.github.io
//     review, section 3-2 (6)): mu_h and the population sigma_h of the raw
//     scores over the sequence's T live keys; z_h = (s_h - mu_h) / sigma_h
//     (0 when sigma_h = 0); score = max_h z_h.  mu and sigma come from the
//     float64 sums of s and s^2 the score kernel leaves per (CTA, head), added
//     here in a fixed order, so the result is deterministic.
//   selection (same sources, "prune back to budget"; section 3-2 (5)): the
//     `budget` largest scores, ties to the lower slot, by a 4-pass 8-bit radix
//     select on order-preserving 32-bit keys.  Each CTA histograms its slice in
//     shared memory; every CTA then sums the cluster's histograms through
//     distributed shared memory (all peers read in parallel), so all agree on
//     the threshold without a global round trip.  Kept slots are emitted in
//     ascending order.
//   compaction (eviction): kept rows of K, V and pos move in place to slots
//     [0, kept).  A kept slot s_j always satisfies s_j >= j, so reading every
//     source of a batch of destinations before any of them is written (one
//     cluster barrier per batch) makes the in-place gather race-free: a
//     destination row j can only be the source of a kept key with index <= j,
//     which belongs to this batch or an earlier one.  Rows move through shared
//     memory with 1-D bulk copies (cp.async.bulk) in both directions.
//
// Cluster barriers are hardware barriers; the only other waits are on this
// CTA's own bulk copies and are bounded.  The kernel is launched as a
// programmatic dependent of the score kernel and waits for it
// (griddepcontrol.wait) before reading anything that kernel or the fold wrote.
#include <cooperative_groups.h>

#include "tria_internal.cuh"

namespace cg = cooperative_groups;

namespace tria {

namespace {

constexpr int kCtl = 20 * 1024;  // control region at the start of shared memory
constexpr int kMaxG = 16;
constexpr int kMaxCluster = 16;
constexpr int kWarps = kUnitThreads / 32;

struct Ctl {
  uint64_t cbar;                    // compaction bulk-load barrier
  uint32_t hist[2][256];
  uint32_t tot[256];
  double gath[1][kMaxG][2];         // the unit's sums of s and s^2 per head
  float mu_hi[kMaxG], mu_lo[kMaxG];  // mean split into two floats (hi + lo)
  float inv_sigma[kMaxG];
  int32_t cnt[4];                   // gt, eq of this CTA / first_neg, bad (compaction check)
  int32_t peer_cnt[kMaxCluster][2];
  int32_t bc[8];                    // broadcast scalars
  int32_t scan[kWarps + 1];
};
static_assert(sizeof(Ctl) <= kCtl, "control region too small");

// Exclusive block scan of one int per thread; also returns the block total.
__device__ __forceinline__ int block_excl_scan(int v, int32_t *wtot, int *total) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) wtot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int w = lane < kWarps ? wtot[lane] : 0;
    int wi = w;
#pragma unroll
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
  return out;
}

// 1-D bulk copy shared -> global (bulk-group completion).
__device__ __forceinline__ void bulk_s2g(void *dst, const void *src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
               "r"(dev::smem_addr(src)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

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
  const int lane = tid & 31;

  extern __shared__ __align__(128) uint8_t smem[];
  Ctl &c = *reinterpret_cast<Ctl *>(smem);
  uint8_t *data = smem + kCtl;
  const size_t data_bytes = (size_t)p.smem_bytes - kCtl;
  int32_t *sel = p.sel + (row * p.B + b) * (int64_t)p.budget;

  if (tid == 0) {
    dev::mbar_init(&c.cbar, (uint32_t)nthr);
    dev::fence_mbar_init();
  }
  for (int i = tid; i < 256; i += nthr) c.hist[0][i] = 0;
  __syncthreads();
  dev::pdl_wait();

  int kept = 0;
  if (p.mode == kModeCompact) {
    // ------------------------------------------------------------ check the list
    const int64_t j0 = (int64_t)p.budget * r / CL, j1 = (int64_t)p.budget * (r + 1) / CL;
    int first_neg = p.budget, bad = 0;  // index of the first -1 (budget if none)
    for (int64_t j = j0 + tid; j < j1; j += nthr) {
      const int32_t s = __ldcg(sel + j);
      const int32_t prev = j > 0 ? __ldcg(sel + j - 1) : -1;
      if (s < -1 || s >= seg_cap) bad = 1;
      if (s >= 0 && j > 0 && (prev < 0 || s <= prev)) bad = 1;  // ascending, no slot after a -1
      if (s < 0) first_neg = min(first_neg, (int)j);
    }
    if (tid == 0) { c.cnt[2] = p.budget; c.cnt[3] = 0; }
    __syncthreads();
    atomicMin(&c.cnt[2], first_neg);
    if (bad) atomicOr(&c.cnt[3], 1);
    cl.sync();
    if (tid < CL) {
      const Ctl *peer = cl.map_shared_rank(&c, tid);
      c.peer_cnt[tid][0] = peer->cnt[2];
      c.peer_cnt[tid][1] = peer->cnt[3];
    }
    cl.sync();  // peers' control regions are not read after this point
    int any_bad = 0;
    kept = p.budget;
    for (int q = 0; q < CL; ++q) {
      kept = min(kept, c.peer_cnt[q][0]);
      any_bad |= c.peer_cnt[q][1];
    }
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
    const int nmax4 = (nmax + 3) & ~3;
    if ((size_t)nmax4 * 4 > data_bytes) {
      if (r == 0 && tid == 0) dev::set_error(p.err, TRIA_DEVERR_SEGMENT_BIG);
      return;  // every CTA of the cluster takes this branch (same T)
    }
    uint32_t *zkey = reinterpret_cast<uint32_t *>(data);

    if (p.mode == kModeZmax || p.mode == kModePrune) {
      // ---------------------------------------------------- z-score statistics
      // The score kernel left float64 sums of s and s^2 per (CTA, head) for this
      // unit; the CTAs that scored it are those whose tile runs meet its live tiles.
      const float *rawu = p.raw + ((int64_t)l * p.Hq + (int64_t)g * G) * p.cap + seg;
      if (tid < 2 * G) {
        const int64_t first_tile = row * p.tiles_per_row + p.tile_prefix[b];
        const int64_t live_tiles = ((int64_t)T + p.tile_keys - 1) / p.tile_keys;
        const int64_t c0 = first_tile / p.tiles_per_cta;
        const int64_t c1 = (first_tile + live_tiles - 1) / p.tiles_per_cta;
        const double *pu = p.partials + unit * (int64_t)p.max_slots * (2 * G);
        double a = 0.0;
        for (int64_t q = 0; q <= c1 - c0; ++q) a += pu[q * (2 * G) + tid];  // fixed order
        c.gath[0][tid >> 1][tid & 1] = a;
      }
      __syncthreads();
      if (tid < G) {
        const double m = c.gath[0][tid][0] / (double)T;
        const double var = c.gath[0][tid][1] / (double)T - m * m;
        c.mu_hi[tid] = (float)m;
        c.mu_lo[tid] = (float)(m - (double)c.mu_hi[tid]);
        c.inv_sigma[tid] = var > 0.0 ? (float)(1.0 / sqrt(var)) : 0.0f;
      }
      __syncthreads();
      // ---------------------------------------------------- z and group max
      float *score = p.score + row * p.cap + seg;
      for (int i = tid; i < n; i += nthr) {
        float zf = -3.0e38f;
        for (int j = 0; j < G; ++j) {
          const float v = rawu[(int64_t)j * p.cap + lo + i];
          const float z = ((v - c.mu_hi[j]) - c.mu_lo[j]) * c.inv_sigma[j];
          zf = fmaxf(zf, z);
        }
        if (p.mode == kModeZmax) score[lo + i] = zf == 0.0f ? 0.0f : zf;
        else zkey[i] = dev::order_key(zf);
      }
      if (p.mode == kModeZmax) return;
    } else {
      const float *score = p.score + row * p.cap + seg;
      for (int i = tid; i < n; i += nthr) zkey[i] = dev::order_key(score[lo + i]);
    }
    for (int i = n + tid; i < nmax4; i += nthr) zkey[i] = 0u;  // padding never matches a prefix
    __syncthreads();

    // ------------------------------------------------------------ radix select
    // hist[0] was zeroed at kernel start; each pass zeroes the other buffer for
    // the next pass after the cluster barrier (peers finished reading it then).
    uint32_t prefix = 0, mask = 0;
    int krem = p.budget;
    const uint4 *zkey4 = reinterpret_cast<const uint4 *>(zkey);
    const int n4 = nmax4 >> 2;
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      uint32_t *H = c.hist[pass & 1];
      for (int i = tid; i < n4; i += nthr) {
        const uint4 kv = zkey4[i];
        const uint32_t ks[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          // padding keys are 0: they match only while prefix == 0 and mask == 0
          if ((ks[e] & mask) == prefix && 4 * i + e < n) {
            const uint32_t d = (ks[e] >> shift) & 255u;
            const uint32_t peers = __match_any_sync(__activemask(), d);
            if ((uint32_t)lane == (uint32_t)(__ffs(peers) - 1)) atomicAdd(&H[d], (uint32_t)__popc(peers));
          }
        }
      }
      cl.sync();
      for (int i = tid; i < 256; i += nthr) {
        uint32_t v[kMaxCluster];
#pragma unroll
        for (int q = 0; q < kMaxCluster; ++q) v[q] = q < CL ? cl.map_shared_rank(H, q)[i] : 0u;
        uint32_t a = 0;
#pragma unroll
        for (int q = 0; q < kMaxCluster; ++q) a += v[q];
        c.tot[i] = a;
        c.hist[(pass + 1) & 1][i] = 0;
      }
      __syncthreads();
      if (tid < 32) {
        uint32_t cnt8[8], s = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) { cnt8[i] = c.tot[tid * 8 + i]; s += cnt8[i]; }
        uint32_t incl = s;  // inclusive suffix over lanes (this lane and above)
#pragma unroll
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
      prefix |= (uint32_t)c.bc[0] << shift;
      mask |= 255u << shift;
      krem = c.bc[1];
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
    int tot_pk;
    const int x_pk = block_excl_scan((gt << 16) | eq, c.scan, &tot_pk);  // n < 65536
    const int gt_x = x_pk >> 16, eq_x = x_pk & 0xffff;
    if (tid == 0) { c.cnt[0] = tot_pk >> 16; c.cnt[1] = tot_pk & 0xffff; }
    cl.sync();
    if (tid < CL) {
      const Ctl *peer = cl.map_shared_rank(&c, tid);
      c.peer_cnt[tid][0] = peer->cnt[0];
      c.peer_cnt[tid][1] = peer->cnt[1];
    }
    __syncthreads();
    if (tid == 0) {
      int eqb = 0, base = 0;
      for (int q = 0; q < CL; ++q) {
        const int qg = c.peer_cnt[q][0], qe = c.peer_cnt[q][1];
        const int take = max(0, min(qe, k_eq - eqb));
        if (q == r) { c.bc[2] = base; c.bc[3] = take; }
        eqb += qe;
        base += qg + take;
      }
    }
    __syncthreads();
    {
      const int take_cta = c.bc[3];  // equal keys this CTA keeps: its first take_cta ones
      int o = c.bc[2] + gt_x + min(eq_x, take_cta), er = eq_x;
      for (int i = a0; i < a1; ++i) {
        const uint32_t key = zkey[i];
        bool keep = key > thr;
        if (key == thr) { keep = er < take_cta; ++er; }
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
  const int ROW = 2 * p.D;                          // bytes per K or V row
  constexpr int kItemsPerThread = 2;                 // row copies a thread issues per batch
  const int cap_rows = min((int)(data_bytes / (2 * (size_t)ROW)), kItemsPerThread * nthr / 2);
  // Batch bt covers the destinations [bt * CL * cap_rows, (bt + 1) * CL * cap_rows) of the
  // whole cluster (CTA r takes the r-th chunk), so every destination written in a batch
  // precedes every destination, and hence every source, of the batches after it.
  const int64_t per_batch = (int64_t)CL * cap_rows;
  const int batches = (int)((kept + per_batch - 1) / per_batch);
  const int64_t rbase = row * p.cap + seg;
  uint8_t *kg = p.k + (size_t)rbase * ROW;
  uint8_t *vg = p.v + (size_t)rbase * ROW;
  int32_t *pg = p.pos + rbase;
  uint8_t *sk = data;                                // [cap_rows][ROW]
  uint8_t *sv = data + (size_t)cap_rows * ROW;       // [cap_rows][ROW]
  bool failed = false;
  for (int bt = 0; bt < batches; ++bt) {
    const int64_t a = (int64_t)bt * per_batch + (int64_t)r * cap_rows;
    int64_t e = a + cap_rows;
    if (e > kept) e = kept;
    const int nb = e > a ? (int)(e - a) : 0;
    // item it = 2 * row + {0: K row (and pos), 1: V row}
    int32_t src[kItemsPerThread], rp[kItemsPerThread];
    uint32_t bytes = 0;
#pragma unroll
    for (int u = 0; u < kItemsPerThread; ++u) {
      const int item = tid + u * nthr, jj = item >> 1;
      src[u] = -1;
      if (jj < nb) {
        const int32_t s = __ldcg(sel + a + jj);
        if (s >= 0 && s < seg_cap) {
          if (s != a + jj) { src[u] = s; bytes += (uint32_t)ROW; }
        } else if ((item & 1) == 0) {
          dev::set_error(p.err, TRIA_DEVERR_SELECTION);
        }
      }
    }
    if (!failed) {
      dev::mbar_arrive_expect_tx(&c.cbar, bytes);
#pragma unroll
      for (int u = 0; u < kItemsPerThread; ++u) {
        if (src[u] >= 0) {
          const int item = tid + u * nthr, jj = item >> 1;
          if ((item & 1) == 0) {
            dev::bulk_g2s(sk + (size_t)jj * ROW, kg + (size_t)src[u] * ROW, ROW, &c.cbar);
            rp[u] = pg[src[u]];
          } else {
            dev::bulk_g2s(sv + (size_t)jj * ROW, vg + (size_t)src[u] * ROW, ROW, &c.cbar);
          }
        }
      }
      if (!dev::mbar_wait(&c.cbar, bt & 1)) {
        dev::set_error(p.err, TRIA_DEVERR_TIMEOUT);
        failed = true;
      }
    }
    cl.sync();  // every source row of this batch has been read, cluster-wide
    if (!failed) {
#pragma unroll
      for (int u = 0; u < kItemsPerThread; ++u) {
        if (src[u] >= 0) {
          const int item = tid + u * nthr, jj = item >> 1;
          if ((item & 1) == 0) {
            bulk_s2g(kg + (size_t)(a + jj) * ROW, sk + (size_t)jj * ROW, ROW);
            pg[a + jj] = rp[u];
          } else {
            bulk_s2g(vg + (size_t)(a + jj) * ROW, sv + (size_t)jj * ROW, ROW);
          }
        }
      }
      bulk_commit();
      bulk_wait_read0();  // this thread's staged rows may be overwritten by the next batch
    }
    __syncthreads();
  }
  bulk_wait0();
  if (r == 0 && tid == 0 && l == 0 && g == 0) p.seq_len_out[b] = kept;
}

// Launch configuration: 8-CTA clusters of 1024 threads, one CTA per SM
// (portable cluster size; 15 clusters are resident at once on a B200).
int unit_cluster_size() { return kUnitCluster; }

int unit_smem_bytes(int units, int64_t max_segment) {
  (void)units;
  (void)max_segment;  // the large size holds the keys of a TRIA_MAX_SEGMENT segment per CTA
  static bool configured[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 64 && !configured[dev]) {
    cudaFuncSetAttribute(unit_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kUnitSmemLarge);
    configured[dev] = true;
  }
  return kUnitSmemLarge;
}

cudaError_t launch_unit(const UnitParams &p, int units, cudaStream_t s, bool pdl) {
  const int cs = kUnitCluster;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)units * cs, 1, 1);
  cfg.blockDim = dim3(kUnitThreads, 1, 1);
  cfg.dynamicSmemBytes = p.smem_bytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, unit_kernel, p);
}

}  // namespace tria
