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
//     `budget` largest scores, ties to the lower slot, on order-preserving
//     32-bit keys.  While the keys are computed, each is counted into a
//     cluster-wide 12-bit histogram with remote shared-memory atomics (CTA q
//     owns one eighth of the bins); after one barrier every CTA reads the whole
//     histogram and names the bucket holding the budget-th key.  Usually that
//     bucket is small: every CTA then gathers the bucket's keys from all peers
//     (in slot order) and finishes the selection alone, exactly, so it also
//     knows how many keys every peer keeps without another exchange.  A bucket
//     too large to gather is refined by further cluster-wide rounds (12 then 8
//     bits); if it is still large, its keys are all equal and the ties go to
//     the lowest slots.
//   compaction (eviction): kept rows of K, V and pos move in place to slots
//     [0, kept).  A kept slot s_j always satisfies s_j >= j, so reading every
//     source of a batch of destinations before any of them is written (one
//     cluster barrier per batch) makes the in-place gather race-free: a
//     destination row j can only be the source of a kept key with index <= j,
//     which belongs to this batch or an earlier one.  Sources are staged in
//     shared memory with 16-byte asynchronous copies; each CTA's destination
//     rows are contiguous and go back with one bulk copy per tensor.
//
// Cluster barriers are hardware barriers; there are no spin-waits.  The kernel
// is launched as a programmatic dependent of the score kernel and waits for it
// (griddepcontrol.wait) before reading anything that kernel or the fold wrote.
#include <cooperative_groups.h>

#include "tria_internal.cuh"

namespace cg = cooperative_groups;

namespace tria {

namespace {

constexpr int kCtl = 24 * 1024;  // control region at the start of shared memory
constexpr int kMaxG = 16;
constexpr int kMaxCluster = 16;
constexpr int kWarps = kUnitThreads / 32;
constexpr int kBins = 4096;                   // cluster-wide histogram bins (12-bit digits)
constexpr int kSlice = kBins / kUnitCluster;  // bins each CTA of the cluster owns
constexpr int kCandMax = 4096;                // bucket keys a CTA may gather
constexpr int kLocalBins = 1024;              // bins of the rounds inside a gathered bucket

struct Ctl {
  double sums[kMaxG][2];            // the unit's sums of s and s^2 per head
  float mu_hi[kMaxG], mu_lo[kMaxG];  // mean split into two floats (hi + lo)
  float inv_sigma[kMaxG];
  int32_t cnt[8];                   // this CTA's published counts
  int32_t peer[kMaxCluster][4];     // peers' counts, gathered
  int32_t off[kMaxCluster + 1];     // offsets of the peers' bucket lists in the gathered copy
  int32_t bc[8];                    // broadcast scalars
  int32_t gcnt[kMaxCluster][2];     // per peer: bucket keys above the threshold, equal to it
  int32_t scan[kWarps + 1];
  uint32_t lh[kLocalBins];          // histogram of the rounds inside a gathered bucket
  uint32_t slice[3][kSlice];        // this CTA's slice of the cluster histogram, per round
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
  __syncthreads();
  return out;
}

// Counts bin d of a cluster-wide histogram whose bins are spread over the CTAs'
// slices (owner = d / per_owner), one remote atomic per distinct d in the warp.
__device__ __forceinline__ void cluster_hist_add(cg::cluster_group &cl, uint32_t *slice,
                                                 uint32_t d, int per_owner_log2) {
  const uint32_t peers = __match_any_sync(__activemask(), d);
  if ((threadIdx.x & 31) == (uint32_t)(__ffs(peers) - 1)) {
    uint32_t *dst = cl.map_shared_rank(slice, (int)(d >> per_owner_log2));
    atomicAdd(dst + (d & ((1u << per_owner_log2) - 1)), (uint32_t)__popc(peers));
  }
}

// Finds, in a histogram of `nbins` counts ordered by increasing key, the bin
// holding the krem-th largest counted key.  Every thread returns the bin, the
// number of counted keys above it and the bin's own count (block-wide).
__device__ __forceinline__ void find_bin(const uint32_t *tot, int nbins, int krem, int32_t *bc,
                                         int32_t *wtot, int *bin, int *above, int *count) {
  const int per = (nbins + (int)blockDim.x - 1) / (int)blockDim.x;
  const int b0 = threadIdx.x * per;
  const int b1 = min(nbins, b0 + per);
  int s = 0;
  for (int i = b0; i < b1; ++i) s += (int)tot[i];
  if (threadIdx.x == 0) { bc[0] = 0; bc[1] = 0; bc[2] = 0; }
  int total;
  const int excl = block_excl_scan(s, wtot, &total);  // ends with a barrier
  const int higher = total - excl - s;  // counted keys in bins above this thread's range
  if (higher < krem && krem <= higher + s) {
    int cum = higher;
    for (int i = b1 - 1; i >= b0; --i) {
      const int c = (int)tot[i];
      if (cum + c >= krem) {
        bc[0] = i;
        bc[1] = cum;
        bc[2] = c;
        break;
      }
      cum += c;
    }
  }
  __syncthreads();
  *bin = bc[0];
  *above = bc[1];
  *count = bc[2];
  __syncthreads();
}

// Peer whose range [off[q], off[q+1]) holds index i (off has CL+1 entries).
__device__ __forceinline__ int owner_of(const int32_t *off, int CL, int i) {
  int q = 0;
  while (q + 1 < CL && off[q + 1] <= i) ++q;
  return q;
}

__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dev::smem_addr(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dev::smem_addr(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
// Shared-memory writes of this thread (generic proxy) become visible to bulk copies.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
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

template <int G>
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
  const int tid = threadIdx.x, nthr = blockDim.x;

  extern __shared__ __align__(128) uint8_t smem[];
  Ctl &c = *reinterpret_cast<Ctl *>(smem);
  uint8_t *data = smem + kCtl;
  const size_t data_bytes = (size_t)p.smem_bytes - kCtl;
  int32_t *sel = p.sel + (row * p.B + b) * (int64_t)p.budget;

  // prologue (overlaps the score kernel's tail): clear the histogram slices of all
  // rounds, and make sure every peer has before anyone counts into them
  for (int i = tid; i < 3 * kSlice; i += nthr) (&c.slice[0][0])[i] = 0u;
  cl.sync();
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
    if (tid == 0) { c.cnt[0] = p.budget; c.cnt[1] = 0; }
    __syncthreads();
    atomicMin(&c.cnt[0], first_neg);
    if (bad) atomicOr(&c.cnt[1], 1);
    cl.sync();
    if (tid < CL) {
      const Ctl *peer = cl.map_shared_rank(&c, tid);
      c.peer[tid][0] = peer->cnt[0];
      c.peer[tid][1] = peer->cnt[1];
    }
    cl.sync();  // peers' control regions are not read after this point
    int any_bad = 0;
    kept = p.budget;
    for (int q = 0; q < CL; ++q) {
      kept = min(kept, c.peer[q][0]);
      any_bad |= c.peer[q][1];
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
    // data region: zkey[nmax4] | tot[kBins] | cand_key[cap] | cand_slot[cap]
    const size_t fixed = (size_t)nmax4 * 4 + (size_t)kBins * 4;
    const int cand_cap = fixed + 8ull * 256 <= data_bytes
                             ? (int)min((size_t)kCandMax, (data_bytes - fixed) / 8) : 0;
    if (cand_cap == 0) {
      if (r == 0 && tid == 0) dev::set_error(p.err, TRIA_DEVERR_SEGMENT_BIG);
      return;  // every CTA of the cluster takes this branch (same T)
    }
    uint32_t *zkey = reinterpret_cast<uint32_t *>(data);
    uint32_t *tot = zkey + nmax4;  // [kBins] the cluster histogram, read back
    uint32_t *cand_key = tot + kBins;
    int32_t *cand_slot = reinterpret_cast<int32_t *>(cand_key + cand_cap);

    if (p.mode == kModeZmax || p.mode == kModePrune) {
      // ---------------------------------------------------- z-score statistics
      // The score kernel left float64 sums of s and s^2 per (CTA, head) for this
      // unit; the CTAs that scored it are those whose tile runs meet its live tiles.
      {
        const int64_t first_tile = row * p.tiles_per_row + p.tile_prefix[b];
        const int64_t live_tiles = ((int64_t)T + p.tile_keys - 1) / p.tile_keys;
        const int64_t c0 = first_tile / p.tiles_per_cta;
        const int64_t c1 = (first_tile + live_tiles - 1) / p.tiles_per_cta;
        const int nv = (int)(c1 - c0 + 1) * 2 * G;
        const double *pu = p.partials + unit * (int64_t)p.max_slots * (2 * G);
        double *tmp = reinterpret_cast<double *>(data);  // scratch before the keys exist
        for (int i = tid; i < nv; i += nthr) tmp[i] = pu[i];
        __syncthreads();
        if (tid < 2 * G) {
          double a = 0.0;
          for (int i = tid; i < nv; i += 2 * G) a += tmp[i];  // fixed order
          c.sums[tid >> 1][tid & 1] = a;
        }
        __syncthreads();
        if (tid < G) {
          const double m = c.sums[tid][0] / (double)T;
          const double var = c.sums[tid][1] / (double)T - m * m;
          c.mu_hi[tid] = (float)m;
          c.mu_lo[tid] = (float)(m - (double)c.mu_hi[tid]);
          c.inv_sigma[tid] = var > 0.0 ? (float)(1.0 / sqrt(var)) : 0.0f;
        }
        __syncthreads();
      }
      // ---------------------------------------------------- z and group max
      const float *rawu = p.raw + ((int64_t)l * p.Hq + (int64_t)g * G) * p.cap + seg + lo;
      float *score = p.score + row * p.cap + seg + lo;
      float mh[G], ml[G], is[G];
#pragma unroll
      for (int j = 0; j < G; ++j) { mh[j] = c.mu_hi[j]; ml[j] = c.mu_lo[j]; is[j] = c.inv_sigma[j]; }
      constexpr int U = G <= 4 ? 4 : (G <= 8 ? 2 : 1);  // keys per thread per round of loads
      for (int i0 = tid; i0 < n; i0 += U * nthr) {
        float v[U][G];
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
          for (int j = 0; j < G; ++j)
            v[u][j] = i0 + u * nthr < n ? rawu[(int64_t)j * p.cap + i0 + u * nthr] : 0.0f;
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int i = i0 + u * nthr;
          if (i < n) {
            float zf = -3.0e38f;
#pragma unroll
            for (int j = 0; j < G; ++j) zf = fmaxf(zf, ((v[u][j] - mh[j]) - ml[j]) * is[j]);
            if (p.mode == kModeZmax) {
              score[i] = zf == 0.0f ? 0.0f : zf;
            } else {
              const uint32_t key = dev::order_key(zf);
              zkey[i] = key;
              cluster_hist_add(cl, &c.slice[0][0], key >> 20, 9);
            }
          }
        }
      }
      if (p.mode == kModeZmax) return;
    } else {
      const float *score = p.score + row * p.cap + seg + lo;
      for (int i = tid; i < n; i += nthr) {
        const uint32_t key = dev::order_key(score[i]);
        zkey[i] = key;
        cluster_hist_add(cl, &c.slice[0][0], key >> 20, 9);
      }
    }

    // ------------------------------------------------------------ threshold
    // Cluster-wide histogram rounds on digits [31:20], [19:8], [7:0] of the keys,
    // until the bucket of the krem-th largest key is small enough to gather (or
    // the key is fully known).  Round r counts into slice[r] of the owners.
    uint32_t prefix = 0, mask = 0;
    int krem = p.budget, bucket = 0;
    int shift = 20, dbits = 12;
    for (int round = 0;; ++round) {
      const int nb = 1 << dbits;
      const int per_log2 = dbits - 3;  // bins per owner: nb / 8
      cl.sync();  // every count of this round has landed
      for (int i = tid; i < nb; i += nthr)
        tot[i] = cl.map_shared_rank(&c.slice[round][0], i >> per_log2)[i & ((1 << per_log2) - 1)];
      __syncthreads();
      int bin, above;
      find_bin(tot, nb, krem, c.bc, c.scan, &bin, &above, &bucket);
      prefix |= (uint32_t)bin << shift;
      mask |= (uint32_t)(nb - 1) << shift;
      krem -= above;
      if (bucket <= cand_cap || shift == 0) break;
      // refine: the next digit of the bucket's keys, into the next round's slices
      const int nshift = shift >= 12 ? shift - 12 : 0;
      const int nbits = shift - nshift;
      for (int i = tid; i < n; i += nthr) {
        const uint32_t key = zkey[i];
        if ((key & mask) == prefix)
          cluster_hist_add(cl, &c.slice[round + 1][0], (key >> nshift) & ((1u << nbits) - 1),
                           nbits - 3);
      }
      shift = nshift;
      dbits = nbits;
    }
    // Keys above the bucket are kept, keys below dropped; of the bucket's keys the
    // krem largest are kept (ties: lowest slots).  Each thread owns a contiguous
    // run of this CTA's keys, so runs in thread order are in slot order.
    const int RL = (n + nthr - 1) / nthr;
    const int a0 = min(n, tid * RL), a1 = min(n, a0 + RL);
    int above_local = 0, in_local = 0;
    for (int i = a0; i < a1; ++i) {
      const uint32_t mk = zkey[i] & mask;
      above_local += mk > prefix;
      in_local += mk == prefix;
    }
    const bool gather = bucket <= cand_cap;
    int tot_pk;
    const int x_pk = block_excl_scan((above_local << 16) | in_local, c.scan, &tot_pk);  // n < 65536
    if (gather) {
      int o = x_pk & 0xffff;
      for (int i = a0; i < a1; ++i) {
        const uint32_t key = zkey[i];
        if ((key & mask) == prefix) {
          cand_key[o] = key;
          cand_slot[o] = (int32_t)(lo + i);
          ++o;
        }
      }
    }
    if (tid == 0) { c.cnt[0] = tot_pk >> 16; c.cnt[1] = tot_pk & 0xffff; }
    cl.sync();  // counts and bucket lists complete
    if (tid < CL) {
      const Ctl *peer = cl.map_shared_rank(&c, tid);
      c.peer[tid][0] = peer->cnt[0];  // keys above the bucket
      c.peer[tid][1] = peer->cnt[1];  // keys in the bucket
    }
    if (tid < 2 * kMaxCluster) c.gcnt[tid >> 1][tid & 1] = 0;
    __syncthreads();
    if (tid == 0) {
      c.off[0] = 0;
      for (int q = 0; q < CL; ++q) c.off[q + 1] = c.off[q] + c.peer[q][1];
    }
    __syncthreads();
    uint32_t thr;
    int k_eq;
    if (gather) {
      // every CTA copies the whole bucket (peers in rank order = slot order) into
      // its own `tot` area (free now), then finishes the selection alone
      const int C = c.off[CL];
      uint32_t *gkey = tot;  // [C], C <= cand_cap <= kBins
      for (int i = tid; i < C; i += nthr) {
        const int q = owner_of(c.off, CL, i);
        gkey[i] = cl.map_shared_rank(cand_key, q)[i - c.off[q]];
      }
      __syncthreads();
      // the low bits below the bucket prefix, by 10-bit local rounds
      int rshift = shift, rkrem = krem;
      uint32_t rprefix = prefix, rmask = mask;
      while (rshift > 0) {
        const int nshift = rshift >= 10 ? rshift - 10 : 0;
        const int nbits = rshift - nshift;
        for (int i = tid; i < (1 << nbits); i += nthr) c.lh[i] = 0;
        __syncthreads();
        for (int i = tid; i < C; i += nthr) {
          const uint32_t key = gkey[i];
          if ((key & rmask) == rprefix) atomicAdd(&c.lh[(key >> nshift) & ((1u << nbits) - 1)], 1u);
        }
        __syncthreads();
        int bin, above, cnt;
        find_bin(c.lh, 1 << nbits, rkrem, c.bc, c.scan, &bin, &above, &cnt);
        rprefix |= (uint32_t)bin << nshift;
        rmask |= (uint32_t)((1 << nbits) - 1) << nshift;
        rkrem -= above;
        rshift = nshift;
      }
      thr = rprefix;
      k_eq = rkrem;
      // per peer: bucket keys above thr and equal to thr
      for (int i = tid; i < C; i += nthr) {
        const uint32_t key = gkey[i];
        if (key >= thr) atomicAdd(&c.gcnt[owner_of(c.off, CL, i)][key == thr ? 1 : 0], 1);
      }
      __syncthreads();
    } else {
      // all 32 bits are resolved: every key of the bucket equals prefix
      thr = prefix;
      k_eq = krem;
      if (tid < CL) c.gcnt[tid][1] = c.peer[tid][1];
      __syncthreads();
    }
    // ------------------------------------------------------------ emit kept slots
    // CTA q keeps its keys above the bucket, its bucket keys above thr, and those
    // of its keys equal to thr whose cluster-wide rank in slot order is < k_eq.
    if (tid == 0) {
      int eqb = 0, base = 0;
      for (int q = 0; q < CL; ++q) {
        const int qe = c.gcnt[q][1];
        const int take = max(0, min(qe, k_eq - eqb));
        if (q == r) { c.bc[4] = base; c.bc[5] = eqb; }
        eqb += qe;
        base += c.peer[q][0] + c.gcnt[q][0] + take;
      }
    }
    __syncthreads();
    {
      int gt = 0, eq = 0;
      for (int i = a0; i < a1; ++i) {
        const uint32_t key = zkey[i];
        gt += key > thr;
        eq += key == thr;
      }
      int tot2;
      const int x2 = block_excl_scan((gt << 16) | eq, c.scan, &tot2);
      const int eq_x = x2 & 0xffff;
      int er = c.bc[5] + eq_x;  // cluster-wide rank of this run's first key equal to thr
      int o = c.bc[4] + (x2 >> 16) + max(0, min(eq_x, k_eq - c.bc[5]));
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
    cl.sync();  // selection list complete and visible; peers' shared memory no longer read
    if (p.mode == kModeSelect) return;
    kept = p.budget;
  }

  // -------------------------------------------------------------- in-place compaction
  const int ROW = 2 * p.D;   // bytes per K or V row
  const int VPR = ROW / 16;  // 16-byte vectors per row
  const int cap_rows = (int)(data_bytes / (2 * (size_t)ROW + 8));
  // Batch bt covers the destinations [bt * CL * cap_rows, (bt + 1) * CL * cap_rows) of the
  // whole cluster (CTA r takes the r-th chunk), so every destination written in a batch
  // precedes every destination, and hence every source, of the batches after it.
  const int64_t per_batch = (int64_t)CL * cap_rows;
  const int batches = (int)((kept + per_batch - 1) / per_batch);
  const int64_t rbase = row * p.cap + seg;
  uint8_t *kg = p.k + (size_t)rbase * ROW;
  uint8_t *vg = p.v + (size_t)rbase * ROW;
  int32_t *pg = p.pos + rbase;
  uint8_t *sk = data;                                                     // [cap_rows][ROW]
  uint8_t *sv = data + (size_t)cap_rows * ROW;                            // [cap_rows][ROW]
  int32_t *sp = reinterpret_cast<int32_t *>(data + 2 * (size_t)cap_rows * ROW);  // [cap_rows]
  int32_t *ss = sp + cap_rows;                                            // [cap_rows] sources
  for (int bt = 0; bt < batches; ++bt) {
    const int64_t a = (int64_t)bt * per_batch + (int64_t)r * cap_rows;
    int64_t e = a + cap_rows;
    if (e > kept) e = kept;
    const int nb = e > a ? (int)(e - a) : 0;
    int bad = 0;
    for (int jj = tid; jj < nb; jj += nthr) {
      int32_t s = __ldcg(sel + a + jj);
      if (s < 0 || s >= seg_cap) { bad = 1; s = (int32_t)(a + jj); }  // never read outside
      ss[jj] = s;
    }
    if (bad) dev::set_error(p.err, TRIA_DEVERR_SELECTION);
    __syncthreads();
    for (int it = tid; it < nb * 2 * VPR; it += nthr) {
      const int jj = it / (2 * VPR), w = it - jj * 2 * VPR;
      const size_t s = (size_t)ss[jj];
      if (w < VPR) cp_async16(sk + (size_t)jj * ROW + 16 * w, kg + s * ROW + 16 * w);
      else cp_async16(sv + (size_t)jj * ROW + 16 * (w - VPR), vg + s * ROW + 16 * (w - VPR));
    }
    for (int jj = tid; jj < nb; jj += nthr) cp_async4(sp + jj, pg + ss[jj]);
    cp_async_wait_all();
    fence_proxy_async_smem();  // the staged rows are read back by bulk copies
    __syncthreads();
    cl.sync();  // every source row of this batch has been read, cluster-wide
    if (tid == 0 && nb > 0) {
      bulk_s2g(kg + (size_t)a * ROW, sk, (uint32_t)nb * ROW);
      bulk_s2g(vg + (size_t)a * ROW, sv, (uint32_t)nb * ROW);
      bulk_commit();
    }
    for (int jj = tid; jj < nb; jj += nthr) pg[a + jj] = sp[jj];
    if (tid == 0) bulk_wait_read0();  // the staging buffers may be reused by the next batch
    __syncthreads();
  }
  if (tid == 0) bulk_wait0();
  if (r == 0 && tid == 0 && l == 0 && g == 0) p.seq_len_out[b] = kept;
}

// Launch configuration: 8-CTA clusters of 1024 threads, one CTA per SM
// (portable cluster size; 15 clusters are resident at once on a B200).
int unit_cluster_size() { return kUnitCluster; }

template <int G>
static void configure_unit() {
  cudaFuncSetAttribute(unit_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, kUnitSmemLarge);
}

int unit_smem_bytes(int units, int64_t max_segment) {
  (void)units;
  (void)max_segment;  // the large size holds the keys of a TRIA_MAX_SEGMENT segment per CTA
  static bool configured[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 64 && !configured[dev]) {
    configure_unit<1>();
    configure_unit<2>();
    configure_unit<4>();
    configure_unit<8>();
    configure_unit<16>();
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
  // the group size only shapes the z-score stage
  const int G = (p.mode == kModeZmax || p.mode == kModePrune) ? p.G : 1;
  switch (G) {
    case 1: return cudaLaunchKernelEx(&cfg, unit_kernel<1>, p);
    case 2: return cudaLaunchKernelEx(&cfg, unit_kernel<2>, p);
    case 4: return cudaLaunchKernelEx(&cfg, unit_kernel<4>, p);
    case 8: return cudaLaunchKernelEx(&cfg, unit_kernel<8>, p);
    case 16: return cudaLaunchKernelEx(&cfg, unit_kernel<16>, p);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace tria
