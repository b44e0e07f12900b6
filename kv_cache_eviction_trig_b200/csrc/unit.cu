// Per-unit stages of the prune step: one thread-block cluster per
// (layer l, KV head g, sequence b); CTA r of the cluster owns the r-th slice of
// the sequence's keys.
//
//   z-score + group max (romaanj.github.io review, "Method"; dimensionstp.github.io
//     review, section 3-2 (6)): mu_h and the population sigma_h of the raw
//     scores over the sequence's T live keys; z_h = (s_h - mu_h) / sigma_h
//     (0 when sigma_h = 0); score = max_h z_h.  mu and sigma come from float64
//     sums of s and s^2 that the score kernel leaves per (CTA, warp); every CTA
//     adds them in the same fixed order, so all CTAs hold the same, deterministic
//     statistics without exchanging anything.
//   selection (same sources, "prune back to budget"; section 3-2 (5)): the
//     `budget` largest scores, ties to the lower slot, on order-preserving
//     32-bit keys.  While the keys are computed each CTA counts them into a
//     local 4096-bin histogram (shared-memory atomics).  For z-scores the bins
//     are a fixed grid of width 1/256 over [-8, 8) (a monotone function of the
//     key), so the bin holding the budget-th key usually holds a few dozen keys;
//     for arbitrary scores (tria_select) the bins are the top 12 key bits.  After
//     one barrier every CTA reads the peers' 64 coarse counts, then the 64 fine
//     counts of the coarse bin that holds the budget-th key, and so names its
//     bin.  If that bucket is small, every CTA gathers its keys from all peers
//     (in slot order) and resolves it alone (pairwise ranks, or local radix
//     rounds for larger buckets), so it also knows how many keys every peer keeps
//     without another exchange.  A bucket too large to gather is refined by
//     cluster-wide rounds on the key bits (12, 12, 8; counts land in the owning
//     CTA's slice through remote atomics); if it is still large its keys are all
//     equal and the ties go to the lowest slots.
//   compaction (eviction): kept rows of K, V and pos move in place to slots
//     [0, kept).  A kept slot s_j always satisfies s_j >= j, so reading every
//     source before any destination of the same batch is written (one cluster
//     barrier in between) makes the in-place gather race-free.  Normally CTA q
//     compacts the q-th eighth of the destinations in one batch: whoever emits a
//     kept key stores its slot straight into q's shared-memory list, q stages the
//     rows with 16-byte asynchronous copies and writes them back with one bulk
//     copy per tensor after the barrier.  Larger budgets are compacted in batches
//     in global destination order read from the selection list: every
//     destination written in a batch precedes every source of the later batches.
//
// Cluster barriers are hardware barriers; there are no spin-waits.  The kernel
// is launched as a programmatic dependent of the score kernel and waits for it
// (griddepcontrol.wait) before reading anything that kernel or the fold wrote.
#include <cooperative_groups.h>

#include "tria_internal.cuh"

namespace cg = cooperative_groups;

namespace tria {

namespace {

constexpr int kCtl = 32 * 1024;  // control region at the start of shared memory
constexpr int kMaxG = 16;
constexpr int kMaxCluster = 16;
constexpr int kWarps = kUnitThreads / 32;
static_assert(kWarps >= 1 && kWarps <= 32, "one lane per warp in the emit prefix");
constexpr int kBins = 4096;                   // cluster-wide histogram bins
// A CTA's slices of the cluster histograms of the refinement rounds (12, 12 and 8 key bits),
// stored back to back: kBins / CL, kBins / CL and 256 / CL bins; 2112 words at CL = 4.
constexpr int kSliceWords = 2 * (kBins / 4) + 256 / 4;
constexpr int kRounds = 3;                    // refinement rounds (12, 12, 8 key bits)
constexpr int kCoarse = 64;                   // coarse bins of the first round (64 bins each)
constexpr int kCandMax = 4096;                // bucket keys a CTA may gather
constexpr int kDirectRank = kUnitThreads < 256 ? kUnitThreads : 256;  // buckets ranked pairwise
constexpr int kLocalBins = 1024;              // bins of the rounds inside a gathered bucket
constexpr int kOwnRows = 640;                 // destinations a CTA compacts in one batch
constexpr int kKeptMax = 3072;                // kept keys of one CTA listed for the compactors

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
  int32_t wgt[kWarps], weq[kWarps];  // per warp: its run's keys above and equal to thr
  int32_t src[kOwnRows];            // source slots of this CTA's share of the destinations
  int32_t base[kMaxCluster];        // per peer: first output index of its kept keys
  int32_t keptq[kMaxCluster];       // per peer: its kept keys
  int32_t kept_src[kKeptMax];       // slots of this CTA's kept keys, in output order
  uint32_t coarse[kCoarse];         // this CTA's first-round counts per coarse bin
  uint32_t gc[kUnitCluster][kCoarse];  // the cluster's coarse counts, then fine counts
  uint32_t lh[kLocalBins];          // histogram of the rounds inside a gathered bucket
  uint32_t slice[kSliceWords];      // this CTA's slices of the cluster histograms, per round
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

// First-round bin of a z-score key: the float z it encodes on a grid of width
// 1/256 over [-8, 8), clamped; non-decreasing in the key (NaN keys, which sit
// at the ends of the key order, go to the end bins).
__device__ __forceinline__ uint32_t fine_bin(uint32_t key) {
  const uint32_t u = (key & 0x80000000u) ? (key & 0x7fffffffu) : ~key;
  const float z = __uint_as_float(u);
  if (z != z) return (key & 0x80000000u) ? (uint32_t)(kBins - 1) : 0u;
  const float t = fmaf(z, 256.0f, 2048.0f);
  if (!(t >= 0.0f)) return 0u;
  if (t >= (float)(kBins - 1)) return (uint32_t)(kBins - 1);
  return (uint32_t)t;
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

// One warp: in the counts cnt[q][i] of CL peers over 64 bins ordered by
// increasing key, the bin holding the krem-th largest counted key, the number
// of counted keys above it and its own count (returned to every lane).
template <int CL>
__device__ __forceinline__ void warp_find_bin64(const uint32_t *cnt, int krem, int *bin, int *above,
                                                int *count) {
  const int lane = threadIdx.x & 31;
  const int bh = 63 - 2 * lane, bl = 62 - 2 * lane;  // this lane's bins, higher first
  int ch = 0, cl_ = 0;
#pragma unroll
  for (int q = 0; q < CL; ++q) {
    ch += (int)cnt[q * 64 + bh];
    cl_ += (int)cnt[q * 64 + bl];
  }
  const int s = ch + cl_;
  int incl = s;  // keys in this lane's bins and in all higher bins
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  const int higher = incl - s;
  const bool mine = higher < krem && krem <= incl;
  const uint32_t who = __ballot_sync(0xffffffffu, mine);
  const int src = who ? __ffs(who) - 1 : 0;
  int b = bh, a = higher, c = ch;
  if (higher + ch < krem) { b = bl; a = higher + ch; c = cl_; }
  *bin = __shfl_sync(0xffffffffu, b, src);
  *above = __shfl_sync(0xffffffffu, a, src);
  *count = __shfl_sync(0xffffffffu, c, src);
}

// Peer whose range [off[q], off[q+1]) holds index i (off has CL+1 entries).
template <int CL>
__device__ __forceinline__ int owner_of(const int32_t *off, int i) {
  int q = 0;
#pragma unroll
  for (int k = 1; k < CL; ++k) q += off[k] <= i;
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

// Stages rows src[0..m) of K and V (ROW bytes each) and of pos into shared memory
// with 16-byte (4-byte for pos) asynchronous copies, and waits for them.
__device__ __forceinline__ void stage_rows(const int32_t *src, int m, const uint8_t *kg,
                                           const uint8_t *vg, const int32_t *pg, uint8_t *sk,
                                           uint8_t *sv, int32_t *sp, int ROW, int vlog2) {
  const int VPR = ROW >> 4;
  for (int it = threadIdx.x; it < (m << (vlog2 + 1)); it += blockDim.x) {
    const int jj = it >> (vlog2 + 1), w = it & ((2 << vlog2) - 1);
    const size_t s = (size_t)src[jj];
    if (w < VPR) cp_async16(sk + (size_t)jj * ROW + 16 * w, kg + s * ROW + 16 * w);
    else cp_async16(sv + (size_t)jj * ROW + 16 * (w - VPR), vg + s * ROW + 16 * (w - VPR));
  }
  for (int jj = threadIdx.x; jj < m; jj += blockDim.x) cp_async4(sp + jj, pg + src[jj]);
  cp_async_wait_all();
  fence_proxy_async_smem();  // the staged rows are read back by bulk copies
}

}  // namespace

// MODE: the mode fixed at compile time (the prune step's own instantiation, so that its
// code holds no other mode's branches), or -1 to read it from the parameters.
template <int G, int CL, int MODE>
__global__ void __launch_bounds__(kUnitThreads, 1) unit_kernel(const __grid_constant__ UnitParams p) {
  static_assert(CL == 1 || CL == 4 || CL == kUnitCluster, "a unit is one CTA or a cluster of 4 or 8");
  const int mode = MODE >= 0 ? MODE : p.mode;
  cg::cluster_group cl = cg::this_cluster();
  const int r = (int)cl.block_rank();
  const int64_t unit = blockIdx.x / CL;
  const int b = (int)(unit % p.B);
  const int g = (int)((unit / p.B) % p.Hkv);
  const int l = (int)(unit / ((int64_t)p.B * p.Hkv));
  const int64_t row = (int64_t)l * p.Hkv + g;
  const int64_t seg = p.seg_start[b];
  const int64_t seg_cap = p.seg_start[b + 1] - seg;
  const int tid = threadIdx.x, nthr = blockDim.x;
  // keys this unit keeps (a head budget, or the single budget; p.budget is also the
  // length of every selection list), and whether the unit's budget is valid
  const int32_t bud = p.head_budget ? p.head_budget[row] : p.budget;
  const bool bud_ok = bud >= 1 && bud <= p.budget;

  extern __shared__ __align__(128) uint8_t smem[];
  Ctl &c = *reinterpret_cast<Ctl *>(smem);
  uint8_t *data = smem + kCtl;
  const size_t data_bytes = (size_t)p.smem_bytes - kCtl;
  int32_t *sel = p.sel + (row * p.B + b) * (int64_t)p.budget;

  const int ROW = 2 * p.D;                    // bytes per K or V row
  const int vlog2 = 31 - __clz(ROW >> 4);     // log2 of 16-byte vectors per row
  const int64_t rbase = row * p.cap + seg;
  uint8_t *kg = p.k + (size_t)rbase * ROW;
  uint8_t *vg = p.v + (size_t)rbase * ROW;
  int32_t *pg = p.pos + rbase;

  // prologue (overlaps the score kernel's tail): clear the histogram slices of all
  // rounds; the first cluster barrier below makes every peer's clearing visible
  // before anyone counts into them
  for (int i = tid; i < kSliceWords; i += nthr) c.slice[i] = 0u;
  const bool zmodes = mode == kModeZmax || mode == kModePrune;
  if (!zmodes) cl.sync();
  dev::pdl_wait();

  int kept = 0;
  if (mode == kModeCompact) {
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
    if (any_bad || !bud_ok || kept > bud) {
      if (r == 0 && tid == 0)
        dev::set_error(p.err, any_bad || bud_ok ? TRIA_DEVERR_SELECTION : TRIA_DEVERR_BUDGET);
      return;
    }
  } else {
    const int32_t T = p.seqlen[p.unit_mode ? unit : b];  // issued first: the loads below do not need it
    if (zmodes) {
      // The score kernel left, per (CTA slot, warp), float64 sums of s and s^2 of the
      // unit's keys; every CTA of the cluster adds them in the same fixed order
      // (strided lanes, then a shuffle tree), so all hold identical statistics.  They
      // do not depend on the live length, so their loads overlap its load.
      const int64_t first = (int64_t)row * p.chunks_per_row + p.chunk_prefix[b];
      const int nch = p.chunk_prefix[b + 1] - p.chunk_prefix[b];
      const int slots = nch > 0 ? (int)((first + nch - 1) / p.chunks_per_cta - first / p.chunks_per_cta) + 1 : 0;
      const int entries = slots * p.score_warps;
      const double *pu = p.partials + unit * (int64_t)p.max_slots * p.score_warps * (2 * G);
      const int warp = tid >> 5, lane = tid & 31;
      for (int col = warp; col < 2 * G; col += kWarps) {
        double a = 0.0;
        for (int e = lane; e < entries; e += 32) a += pu[(int64_t)e * (2 * G) + col];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        if (lane == 0) c.sums[col >> 1][col & 1] = a;
      }
    }
    if (T < 0 || (int64_t)T > seg_cap) {
      if (r == 0 && tid == 0) dev::set_error(p.err, TRIA_DEVERR_SEQ_LEN);
      return;  // same decision in every CTA of the cluster
    }
    const bool selects = (mode == kModeSelect || mode == kModePrune);
    if (selects && !bud_ok) {
      if (r == 0 && tid == 0) dev::set_error(p.err, TRIA_DEVERR_BUDGET);
      return;
    }
    if (selects && T <= bud) {
      // sequence at or under budget: every slot is kept, nothing moves
      if (mode == kModeSelect || p.write_short_sel) {
        const int64_t j0 = (int64_t)p.budget * r / CL, j1 = (int64_t)p.budget * (r + 1) / CL;
        for (int64_t j = j0 + tid; j < j1; j += nthr) sel[j] = j < T ? (int32_t)j : -1;
      }
      return;
    }
    // held back by the prune window: the unit is left as it is
    if (mode == kModePrune && (int64_t)T < (int64_t)bud + (p.window > 1 ? p.window : 1)) return;
    if (T == 0) return;
    const int64_t lo = (int64_t)T * r / CL, hi = (int64_t)T * (r + 1) / CL;
    const int n = (int)(hi - lo);
    const int nmax = (int)((T + CL - 1) / CL);
    const int nmax4 = (nmax + 3) & ~3;
    // data region: zkey[nmax4] | tot[kBins] | gslot[kCandMax] | ... |
    //              cand_key[cand_cap] cand_slot[cand_cap] (at the end)
    const size_t fixed = (size_t)nmax4 * 4 + (size_t)kBins * 4 + (size_t)kCandMax * 4;
    const int cand_cap = fixed + 8ull * 256 <= data_bytes
                             ? (int)min((size_t)kCandMax, (data_bytes - fixed) / 8) : 0;
    if (cand_cap == 0) {
      if (r == 0 && tid == 0) dev::set_error(p.err, TRIA_DEVERR_SEGMENT_BIG);
      return;  // every CTA of the cluster takes this branch (same T)
    }
    uint32_t *zkey = reinterpret_cast<uint32_t *>(data);
    uint32_t *tot = zkey + nmax4;  // [kBins] this CTA's first-round histogram, later scratch
    int32_t *gslot = reinterpret_cast<int32_t *>(tot + kBins);  // [kCandMax] gathered slots
    uint32_t *cand_key = reinterpret_cast<uint32_t *>(data + data_bytes) - 2 * cand_cap;
    int32_t *cand_slot = reinterpret_cast<int32_t *>(cand_key + cand_cap);
    for (int i = tid; i < kBins; i += nthr) tot[i] = 0u;
    if (tid < 2) c.cnt[tid] = 0;
    __syncthreads();
    // the first round bins z-scores on a fixed grid, arbitrary scores by their top bits
    const bool fine = zmodes;

    if (zmodes) {
      // ---------------------------------------------------- z-score statistics
      // The score kernel left, per (CTA slot, warp), float64 sums of s and s^2 of the
      // unit's keys; every CTA of the cluster adds them in the same fixed order
      // (strided lanes, then a shuffle tree), so all hold identical statistics.
      const float *rawu = p.raw + ((int64_t)l * p.Hq + (int64_t)g * G) * p.cap + seg + lo;
      // keys per thread per round of loads (U * G raw values in registers)
      constexpr int U = (16384 / kUnitThreads) / (G > 4 ? G : 4) > 0 ? (16384 / kUnitThreads) / (G > 4 ? G : 4) : 1;
      const bool one_round = n <= U * nthr;            // values stay in registers
      float v[U][G];
      auto load = [&](int i0) {
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
          for (int j = 0; j < G; ++j)
            v[u][j] = i0 + u * nthr < n ? rawu[(int64_t)j * p.cap + i0 + u * nthr] : 0.0f;
      };
      if (one_round) load(tid);  // in flight while mu and sigma are formed
      {
        // c.sums were written before the live length was read (a barrier since)
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
      float *score = p.score + row * p.cap + seg + lo;
      float mh[G], ml[G], is[G];
#pragma unroll
      for (int j = 0; j < G; ++j) { mh[j] = c.mu_hi[j]; ml[j] = c.mu_lo[j]; is[j] = c.inv_sigma[j]; }
      auto zround = [&](int i0) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int i = i0 + u * nthr;
          if (i < n) {
            float zf = -3.0e38f;
#pragma unroll
            for (int j = 0; j < G; ++j) zf = fmaxf(zf, ((v[u][j] - mh[j]) - ml[j]) * is[j]);
            if (mode == kModeZmax) {
              score[i] = zf == 0.0f ? 0.0f : zf;
            } else {
              const uint32_t key = dev::order_key(zf);
              zkey[i] = key;
              atomicAdd(&tot[fine_bin(key)], 1u);
            }
          }
        }
      };
      if (one_round) {
        zround(tid);
      } else {
        for (int i0 = tid; i0 < n; i0 += U * nthr) {
          load(i0);
          zround(i0);
        }
      }
      if (mode == kModeZmax) return;
    } else {
      const float *score = p.score + row * p.cap + seg + lo;
      for (int i = tid; i < n; i += nthr) {
        const uint32_t key = dev::order_key(score[i]);
        zkey[i] = key;
        atomicAdd(&tot[key >> 20], 1u);
      }
    }

    // ------------------------------------------------------------ threshold
    // Round 0: the cluster's counts of the first-round bins, coarse then fine.
    __syncthreads();  // local histogram complete
    {
      const int warp = tid >> 5, lane = tid & 31;
      for (int w2 = warp; w2 < kCoarse / 2; w2 += kWarps) {  // coarse bins 2*w2, 2*w2+1
        const int cb = 2 * w2 + (lane >> 4);
        const int f0 = cb * 64 + (lane & 15) * 4;
        uint32_t sum = tot[f0] + tot[f0 + 1] + tot[f0 + 2] + tot[f0 + 3];
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if ((lane & 15) == 0) c.coarse[cb] = sum;
      }
    }
    cl.sync();  // every CTA's first-round histogram is complete
    uint32_t prefix = 0, mask = 0, bin0 = 0;
    int krem = bud, bucket = 0;
    int top = fine ? 32 : 20;  // bits below `top` are not fixed by prefix/mask
    {
      // coarse bin holding the krem-th largest key, then its fine bin
      for (int i = tid; i < CL * kCoarse; i += nthr)
        c.gc[i / kCoarse][i % kCoarse] = cl.map_shared_rank(&c.coarse[0], i / kCoarse)[i % kCoarse];
      __syncthreads();
      if (tid < 32) {
        int bin, above, cnt;
        warp_find_bin64<CL>(&c.gc[0][0], krem, &bin, &above, &cnt);
        if (tid == 0) { c.bc[0] = bin; c.bc[1] = above; }
      }
      __syncthreads();
      const int cbin = c.bc[0];
      krem -= c.bc[1];
      __syncthreads();
      for (int i = tid; i < CL * kCoarse; i += nthr)
        c.gc[i / kCoarse][i % kCoarse] = cl.map_shared_rank(tot, i / kCoarse)[cbin * 64 + i % kCoarse];
      __syncthreads();
      if (tid < 32) {
        int bin, above, cnt;
        warp_find_bin64<CL>(&c.gc[0][0], krem, &bin, &above, &cnt);
        if (tid == 0) { c.bc[0] = cbin * 64 + bin; c.bc[1] = above; c.bc[2] = cnt; }
      }
      __syncthreads();
      const int bin = c.bc[0];
      krem -= c.bc[1];
      bucket = c.bc[2];
      __syncthreads();
      if (fine) {
        bin0 = (uint32_t)bin;
      } else {
        prefix = (uint32_t)bin << 20;
        mask = 0xfff00000u;
      }
    }
    auto in_bucket = [&](uint32_t key) -> bool {
      return (!fine || fine_bin(key) == bin0) && ((key & mask) == prefix);
    };
    // Refinement rounds: the next key-bit digit of the bucket's keys, counted into
    // slice[round] of the owning CTAs, until the bucket is small enough to gather
    // or the key is fully known.  (`tot` is rewritten only after the first barrier
    // below, when every peer has finished reading this CTA's histogram.)
    for (int round = 0; bucket > cand_cap && top > 0; ++round) {
      const int dshift = top >= 12 ? top - 12 : 0;
      const int dbits = top - dshift;
      const int nb = 1 << dbits;
      if constexpr (CL == 1) {
        // one CTA holds the whole unit: count straight into `tot` (its first-round
        // counts are no longer needed)
        for (int i = tid; i < nb; i += nthr) tot[i] = 0u;
        __syncthreads();
        for (int i = tid; i < n; i += nthr) {
          const uint32_t key = zkey[i];
          if (in_bucket(key)) atomicAdd(&tot[(key >> dshift) & (nb - 1)], 1u);
        }
        __syncthreads();
      } else {
        const int per_log2 = dbits - (CL == 8 ? 3 : 2);  // bins per owner: nb / CL
        for (int i = tid; i < n; i += nthr) {
          const uint32_t key = zkey[i];
          if (in_bucket(key))
            cluster_hist_add(cl, &c.slice[round * (kBins / CL)], (key >> dshift) & (nb - 1), per_log2);
        }
        cl.sync();  // every count of this round has landed
        for (int i = tid; i < nb; i += nthr)
          tot[i] = cl.map_shared_rank(&c.slice[round * (kBins / CL)], i >> per_log2)[i & ((1 << per_log2) - 1)];
        __syncthreads();
      }
      int bin, above;
      find_bin(tot, nb, krem, c.bc, c.scan, &bin, &above, &bucket);
      krem -= above;
      prefix |= (uint32_t)bin << dshift;
      mask |= (uint32_t)(nb - 1) << dshift;
      top = dshift;
    }
    // Keys above the bucket are kept, keys below dropped; of the bucket's keys the
    // krem largest are kept (ties: lowest slots).  Each CTA counts its keys above the
    // bucket and lists its bucket keys with their slots (in any order).
    const bool gather = bucket <= cand_cap;
    {
      int above_local = 0;
      for (int i = tid; i < n; i += nthr) {
        const uint32_t key = zkey[i];
        const uint32_t fb = fine ? fine_bin(key) : 0u;
        const bool same_bin = !fine || fb == bin0;
        if (same_bin && (key & mask) == prefix) {
          const int pos = atomicAdd(&c.cnt[1], 1);
          if (gather && pos < cand_cap) {
            cand_key[pos] = key;
            cand_slot[pos] = (int32_t)(lo + i);
          }
        } else {
          above_local += (fine && fb > bin0) || (same_bin && (key & mask) > prefix);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) above_local += __shfl_xor_sync(0xffffffffu, above_local, o);
      if ((tid & 31) == 0 && above_local) atomicAdd(&c.cnt[0], above_local);
    }
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
        const int q = owner_of<CL>(c.off, i);
        gkey[i] = cl.map_shared_rank(cand_key, q)[i - c.off[q]];
        gslot[i] = cl.map_shared_rank(cand_slot, q)[i - c.off[q]];
      }
      __syncthreads();
      if (C <= kDirectRank) {
        // pairwise ranks (larger keys first, then lower slots): the key of rank
        // krem-1 is the threshold
        if (tid < C) {
          const uint32_t key = gkey[tid];
          const int32_t slot = gslot[tid];
          int rank = 0;
          for (int j = 0; j < C; ++j) {
            const uint32_t kj = gkey[j];
            rank += (kj > key) | ((kj == key) & (gslot[j] < slot));
          }
          if (rank == krem - 1) c.bc[6] = (int32_t)key;
        }
        __syncthreads();
        thr = (uint32_t)c.bc[6];
        k_eq = -1;  // from the counts below
      } else {
        // the low bits below the bucket's fixed bits, by 10-bit local rounds
        int rshift = top, rkrem = krem;
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
      }
      // per peer: bucket keys above thr and equal to thr
      for (int i = tid; i < C; i += nthr) {
        const uint32_t key = gkey[i];
        if (key >= thr) atomicAdd(&c.gcnt[owner_of<CL>(c.off, i)][key == thr ? 1 : 0], 1);
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
    // Destination share of each CTA when the unit is compacted in one batch.
    const int per = (bud + CL - 1) / CL;
    const bool balanced_fit = mode == kModePrune &&
                              per <= (int)min((size_t)kOwnRows, data_bytes / (2 * (size_t)ROW + 4));
    if (tid < 32) {
      // lane q < CL: peer q's keys equal to thr before it (eqb), the ones it keeps
      // (take), and the first output index of its kept keys (base)
      const int q = tid;
      const int gt = q < CL ? c.gcnt[q][0] : 0, qe = q < CL ? c.gcnt[q][1] : 0;
      const int ab = q < CL ? c.peer[q][0] : 0;
      int keq = k_eq;
      if (keq < 0) {
        int tgt = gt;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) tgt += __shfl_xor_sync(0xffffffffu, tgt, o);
        keq = krem - tgt;
      }
      int eqi = qe;  // inclusive prefix of equal keys
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, eqi, o);
        if (q >= o) eqi += t;
      }
      const int eqb = eqi - qe;
      const int kq = ab + gt + max(0, min(qe, keq - eqb));
      int ki = kq;  // inclusive prefix of kept keys
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, ki, o);
        if (q >= o) ki += t;
      }
      if (q == r) { c.bc[4] = ki - kq; c.bc[5] = eqb; }
      if (q < CL) { c.base[q] = ki - kq; c.keptq[q] = kq; }
      const int most = __reduce_max_sync(0xffffffffu, q < CL ? kq : 0);
      if (q == 0) { c.bc[3] = keq; c.bc[7] = most; }
    }
    __syncthreads();
    k_eq = c.bc[3];
    const bool balanced = balanced_fit && c.bc[7] <= kKeptMax;
    {
      // Warp w owns a contiguous run of this CTA's keys (runs in warp order are in
      // slot order); its lanes read consecutive keys, so the shared-memory reads are
      // free of bank conflicts, and ballots order the kept keys inside each step.
      const int warp = tid >> 5, lane = tid & 31;
      const int WL = ((n + kWarps - 1) / kWarps + 31) & ~31;
      const int w0 = min(n, warp * WL), w1 = min(n, w0 + WL);
      int gt = 0, eq = 0;
      for (int i = w0 + lane; i < w1; i += 32) {
        const uint32_t key = zkey[i];
        gt += key > thr;
        eq += key == thr;
      }
      gt = __reduce_add_sync(0xffffffffu, gt);
      eq = __reduce_add_sync(0xffffffffu, eq);
      if (lane == 0) { c.wgt[warp] = gt; c.weq[warp] = eq; }
      __syncthreads();
      // keys above thr and keys equal to thr in the runs of the warps before this one
      const int gt_x = __reduce_add_sync(0xffffffffu, lane < warp ? c.wgt[lane] : 0);
      const int eq_x = __reduce_add_sync(0xffffffffu, lane < warp ? c.weq[lane] : 0);
      int er = c.bc[5] + eq_x;  // cluster-wide rank of this run's first key equal to thr
      int o = c.bc[4] + gt_x + max(0, min(eq_x, k_eq - c.bc[5]));
      const uint32_t below = (1u << lane) - 1u;
      for (int i0 = w0; i0 < w1; i0 += 32) {
        const int i = i0 + lane;
        const bool in = i < w1;
        const uint32_t key = in ? zkey[i] : 0u;
        const bool is_eq = in && key == thr;
        const uint32_t eqm = __ballot_sync(0xffffffffu, is_eq);
        const bool keep = in && (key > thr || (is_eq && er + __popc(eqm & below) < k_eq));
        const uint32_t km = __ballot_sync(0xffffffffu, keep);
        const int oi = o + __popc(km & below);
        if (keep && oi < bud) {
          const int32_t slot = (int32_t)(lo + i);
          sel[oi] = slot;
          if (balanced) c.kept_src[oi - c.bc[4]] = slot;  // read by the compacting CTAs
        }
        o += __popc(km);
        er += __popc(eqm);
      }
    }
    // a head budget below the list length leaves the rest of the list empty
    for (int64_t j = bud + (int64_t)(p.budget - bud) * r / CL + tid;
         j < bud + (int64_t)(p.budget - bud) * (r + 1) / CL; j += nthr)
      sel[j] = -1;
    cl.sync();  // selection lists complete and visible; peers' keys are no longer read
    if (mode == kModeSelect) return;
    if (balanced) {
      // ------------------------------------- one batch: this CTA's share of destinations
      const int j0 = r * per;
      const int m = max(0, min(per, bud - j0));
      for (int jj = tid; jj < m; jj += nthr) {
        const int j = j0 + jj;
        int q = 0;  // the peer whose kept keys include output index j
#pragma unroll
        for (int k = 1; k < CL; ++k) q += c.base[k] <= j;
        c.src[jj] = cl.map_shared_rank(&c.kept_src[0], q)[j - c.base[q]];
      }
      __syncthreads();
      uint8_t *sk = data;
      uint8_t *sv = data + (size_t)per * ROW;
      int32_t *sp = reinterpret_cast<int32_t *>(data + 2 * (size_t)per * ROW);
      stage_rows(c.src, m, kg, vg, pg, sk, sv, sp, ROW, vlog2);
      __syncthreads();
      cl.sync();  // every source row of the unit has been read
      if (tid == 0 && m > 0) {
        bulk_s2g(kg + (size_t)j0 * ROW, sk, (uint32_t)m * ROW);
        bulk_s2g(vg + (size_t)j0 * ROW, sv, (uint32_t)m * ROW);
        bulk_commit();
      }
      for (int jj = tid; jj < m; jj += nthr) pg[j0 + jj] = sp[jj];
      if (tid == 0) bulk_wait_read0();  // shared memory stays valid until the copies read it
      if (r == 0 && tid == 0) {
        if (p.unit_mode) p.seq_len_out[unit] = bud;
        else if (l == 0 && g == 0) p.seq_len_out[b] = bud;
      }
      return;
    }
    kept = bud;
  }

  // -------------------------------------------------------------- batched compaction
  const int cap_rows = (int)(data_bytes / (2 * (size_t)ROW + 8));
  // Batch bt covers the destinations [bt * CL * cap_rows, (bt + 1) * CL * cap_rows) of the
  // whole cluster (CTA r takes the r-th chunk), so every destination written in a batch
  // precedes every destination, and hence every source, of the batches after it.
  const int64_t per_batch = (int64_t)CL * cap_rows;
  const int batches = (int)((kept + per_batch - 1) / per_batch);
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
    stage_rows(ss, nb, kg, vg, pg, sk, sv, sp, ROW, vlog2);
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
  if (r == 0 && tid == 0) {
    if (p.unit_mode) p.seq_len_out[unit] = kept;
    else if (l == 0 && g == 0) p.seq_len_out[b] = kept;
  }
}

// Launch configuration: 8-CTA clusters of 1024 threads, one CTA per SM
// (portable cluster size; 15 clusters are resident at once on a B200).
template <int G, int CL>
static void configure_unit() {
  cudaFuncSetAttribute(unit_kernel<G, CL, -1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       kUnitSmemLarge);
  cudaFuncSetAttribute(unit_kernel<G, CL, kModePrune>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       kUnitSmemLarge);
}

int unit_smem_bytes() {
  // the large size holds the keys of a TRIA_MAX_SEGMENT segment per CTA of a cluster
  static bool configured[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 64 && !configured[dev]) {
    configure_unit<1, 1>();
    configure_unit<2, 1>();
    configure_unit<4, 1>();
    configure_unit<8, 1>();
    configure_unit<16, 1>();
    configure_unit<1, 4>();
    configure_unit<2, 4>();
    configure_unit<4, 4>();
    configure_unit<8, 4>();
    configure_unit<16, 4>();
    configure_unit<1, kUnitCluster>();
    configure_unit<2, kUnitCluster>();
    configure_unit<4, kUnitCluster>();
    configure_unit<8, kUnitCluster>();
    configure_unit<16, kUnitCluster>();
    configured[dev] = true;
  }
  return kUnitSmemLarge;
}

int unit_cluster_size(int64_t units, int64_t max_segment) {
  // Few units: a cluster of CTAs per unit (latency).  Many units: one CTA per unit
  // (more units at once), when a CTA's shared memory holds a whole segment's keys:
  // zkey + first-round histogram + gathered slots + a minimal bucket list.  Between
  // the two (up to 33 units whose segments need more than one CTA): clusters of 4,
  // which a B200 holds all at once where clusters of 8 would take several waves.
  const int64_t data = kUnitSmemLarge - kCtl;
  auto fits = [&](int64_t keys) {
    return 4 * ((keys + 3) & ~3ll) + 4ll * kBins + 4ll * kCandMax + 8ll * 256 <= data;
  };
  if (units <= kUnitClustersAtOnce) return kUnitCluster;
  if (fits(max_segment)) return 1;
  if (units <= kUnit4ClustersAtOnce && fits((max_segment + 3) / 4)) return 4;
  return kUnitCluster;
}

template <int CL>
static cudaError_t launch_unit_cl(const UnitParams &p, int units, cudaStream_t s, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)units * CL, 1, 1);
  cfg.blockDim = dim3(kUnitThreads, 1, 1);
  cfg.dynamicSmemBytes = p.smem_bytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  // the group size only shapes the z-score stage
  const int G = (p.mode == kModeZmax || p.mode == kModePrune) ? p.G : 1;
  if (p.mode == kModePrune) {
    switch (G) {
      case 1: return cudaLaunchKernelEx(&cfg, unit_kernel<1, CL, kModePrune>, p);
      case 2: return cudaLaunchKernelEx(&cfg, unit_kernel<2, CL, kModePrune>, p);
      case 4: return cudaLaunchKernelEx(&cfg, unit_kernel<4, CL, kModePrune>, p);
      case 8: return cudaLaunchKernelEx(&cfg, unit_kernel<8, CL, kModePrune>, p);
      case 16: return cudaLaunchKernelEx(&cfg, unit_kernel<16, CL, kModePrune>, p);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (G) {
    case 1: return cudaLaunchKernelEx(&cfg, unit_kernel<1, CL, -1>, p);
    case 2: return cudaLaunchKernelEx(&cfg, unit_kernel<2, CL, -1>, p);
    case 4: return cudaLaunchKernelEx(&cfg, unit_kernel<4, CL, -1>, p);
    case 8: return cudaLaunchKernelEx(&cfg, unit_kernel<8, CL, -1>, p);
    case 16: return cudaLaunchKernelEx(&cfg, unit_kernel<16, CL, -1>, p);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_unit(const UnitParams &p, int units, cudaStream_t s, bool pdl) {
  if (p.cluster == 1) return launch_unit_cl<1>(p, units, s, pdl);
  if (p.cluster == 4) return launch_unit_cl<4>(p, units, s, pdl);
  return launch_unit_cl<kUnitCluster>(p, units, s, pdl);
}

}  // namespace tria
