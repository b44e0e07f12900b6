// The whole prune step in one persistent, cooperative launch: every cached key
// scored, z-scored per query head and maxed over its GQA group, the top `budget`
// keys of each (layer, KV head, sequence) unit kept and compacted in place
// (romaanj.github.io review, "Method"; dimensionstp.github.io review, section 2-1
// steps 1-6 and section 3-2 (2)-(6)).
//
// Work layout.  Key chunks (32-128 keys) are numbered row by row ((layer, KV
// head) rows, sequences within a row), so a unit's chunks are consecutive.
// Units are taken in groups of ug consecutive units, and every CTA (one per SM)
// owns an equal, contiguous share ("range") of each group's chunks.  Within a
// CTA:
//   * one producer warp streams the live chunks of its ranges, group after
//     group, into a ring of shared-memory slots with 2-D TMA loads (128-byte
//     swizzle, no multicast); when the unit changes it computes the unit's
//     folded weights W = c * e^{i w cur} * mean_delta e^{i w delta} and
//     Nw = (1 - R) E|q| into one of two weight slots;
//   * eight consumer warps score the chunks (score_math.cuh) and write the raw
//     per-head scores of the CTA's range to a scratch slot of the group;
//   * four select warps finish each group while the consumers score the next:
//       A  float64 sums of s and s^2 of the range, per unit and head, are
//          published; after the round every covering CTA adds all of them in
//          the same order, so they share bit-identical mu and sigma;
//       B  z = max_h (s_h - mu_h) / sigma_h as an order-preserving 32-bit key
//          per key, counted into the unit's histogram of 4096 bins (a 1/256
//          grid over [-8, 8)); after the round every CTA finds the bin that
//          holds the budget-th key;
//       C  the keys of that bin are published as (key << 18 | ~slot), whose
//          order is the selection order (score desc, slot asc), with the count
//          of keys above the bin; after the round every covering CTA ranks the
//          bin's keys and knows the exact threshold, how many keys each CTA
//          keeps and where its kept keys go.  A bin too large to gather (many
//          equal scores) is resolved exactly by the unit's first CTA alone,
//          with a radix select over all the unit's keys;
//       D  every CTA copies its kept K, V and pos rows to a staging area (out
//          of place); after the round (every source row of the group read) it
//          copies its share of the destinations back into the cache, in place.
//     A round is an atomic arrive on a counter plus a bounded wait for all
//     CTAs; a CTA's select warps take groups in order, so by the time a CTA
//     reaches a round of group g every CTA has finished group g - 1, which
//     makes two alternating slots of every per-group buffer enough.
//
// Every wait is bounded (about 2 s): on expiry the kernel sets
// TRIA_DEVERR_TIMEOUT and an abort word that makes every other wait give up.
// The last CTA to leave resets the synchronisation words, so a workspace is
// ready for the next call without a host-side reset.
#include <cudaTypedefs.h>

#include <algorithm>

#include "score_math.cuh"
#include "tria_internal.cuh"

namespace tria {

namespace {

constexpr int NW = kPruneConsumerWarps;
constexpr int NSW = kPruneSelectWarps;
constexpr int SWT = NSW * 32;               // select threads
constexpr int kSwBarrier = 4;               // named barrier of the select warps
constexpr int kMaxRangeChunks = 128;        // kPruneRangeKeys / 16 (smallest chunk is 32 keys)
constexpr int kRadixBins = 2048;
constexpr int kSlotBits = 18;               // slots < TRIA_MAX_SEGMENT = 2^18
constexpr uint64_t kSlotMask = (1ull << kSlotBits) - 1;
static_assert(TRIA_MAX_SEGMENT <= (1 << kSlotBits), "slots must fit the composite key");

enum UnitModeP : int32_t { kSkip = 0, kShort = 1, kHold = 2, kPruneU = 3 };

struct UEnt {              // one unit met by this CTA's range of the current group
  int32_t u, lc0, nlc;     // unit, first local chunk, local chunks
  int32_t T, bud, mode;    // live length, budget, UnitModeP
  int32_t key0, key1;      // live keys of the range within the unit: [key0, key1)
  int32_t clo, chi;        // first and last CTA covering the unit in this group
  int32_t bstar, above;    // threshold bin; keys of the unit above it
  int32_t bcnt, oc, kc;    // keys in the threshold bin; this CTA's first output index and kept keys
  int32_t pad;
  unsigned long long thr;  // composite threshold
};

struct SwMisc {
  int32_t nu, ok;
  int32_t bc[8];
  int32_t scan[NSW + 1];
  double red[NSW][32];
  double stat[32];
  float mu_hi[16], mu_lo[16], inv_sig[16];
  unsigned long long rv;
};

constexpr int rnd128(int x) { return (x + 127) & ~127; }

// Shared-memory regions after the key ring and the two weight slots, each starting
// on a 128-byte boundary (offsets relative to the end of the weight slots).
struct SmemMap {
  static constexpr int ZKS = 0;                                          // u32 [kPruneRangeKeys]
  static constexpr int R1 = ZKS + rnd128(kPruneRangeKeys * 4);           // 32 KB union
  static constexpr int RH = R1 + 32768;                                  // u32 [kRadixBins]
  static constexpr int CTAB = RH + rnd128(kRadixBins * 4);               // int2 [kMaxRangeChunks]
  static constexpr int UTAB = CTAB + rnd128(kMaxRangeChunks * 8);        // UEnt [kMaxRangeChunks + 1]
  static constexpr int MISC = UTAB + rnd128((kMaxRangeChunks + 1) * (int)sizeof(UEnt));
  static constexpr int SEQ = MISC + rnd128((int)sizeof(SwMisc));         // i32 [TRIA_MAX_BATCH]
  static constexpr int TAB = SEQ + rnd128(TRIA_MAX_BATCH * 4);           // int4 [32]
  static constexpr int TABY = TAB + rnd128(32 * 16);                     // i32 [32]
  static constexpr int EA = TABY + rnd128(32 * 4);                       // double2 [128]
  static constexpr int DESC = EA + rnd128(128 * 16);                     // int4 [NSLOT], barriers
  static constexpr int END = DESC + 1024;
};

template <int D, int G>
struct PruneShape : KeyShape<D, G> {
  using K = KeyShape<D, G>;
  static constexpr int FIXED = 1024 + 2 * K::WB + SmemMap::END;
  static constexpr int LIMIT = 227 * 1024;
  static constexpr int NSLOT0 = (LIMIT - FIXED) / K::CB;
  static constexpr int NSLOT = NSLOT0 < 24 ? NSLOT0 : 24;
  static constexpr bool OK = (D == 64 || D == 128 || D == 256) &&
                             (G == 1 || G == 2 || G == 4 || G == 8 || G == 16) && NSLOT > NW;
  static constexpr size_t SMEM = (size_t)FIXED + (size_t)NSLOT * K::CB;
  static_assert(K::WB % 128 == 0 && K::CB % 128 == 0, "regions after the ring stay aligned");
  static_assert(NSLOT * 16 + (2 * NSLOT + 6) * 8 <= 1024, "descriptors and barriers fit");
};

// ------------------------------------------------------------------ small device helpers
__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ int32_t ld_acquire(const int32_t *p) {
  int32_t v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ int32_t ld_volatile(const int32_t *p) {
  return *reinterpret_cast<const volatile int32_t *>(p);
}
__device__ __forceinline__ void sw_sync() { dev::named_barrier(kSwBarrier, SWT); }

__device__ __forceinline__ void raise_abort(const PruneParams &p) {
  dev::set_error(p.err, TRIA_DEVERR_TIMEOUT);
  atomicExch(p.sync + kSyncAbort, 1);
}

// Bounded mbarrier wait that also gives up once another CTA has aborted.
__device__ __forceinline__ bool wait_bar(const PruneParams &p, uint64_t *bar, uint32_t parity) {
  for (uint32_t i = 0; i < 2000000u; ++i) {
    if (dev::mbar_try_wait(bar, parity)) return true;
    if ((i & 15u) == 15u && ld_volatile(p.sync + kSyncAbort)) return false;
  }
  return false;
}

// Grid round: every CTA adds one to counter `w` (slot g % 2) and waits until all
// CTAs of this and the earlier uses of the slot have arrived.  Called by all select
// threads; returns false (everywhere) when it gave up.
__device__ bool grid_round(const PruneParams &p, SwMisc &ms, int w, int g, int t) {
  sw_sync();  // every select thread's writes precede the arrival
  if (t == 0) {
    int32_t *ctr = p.sync + w + (g & 1);
    const int32_t target = p.ncta * ((g >> 1) + 1);
    __threadfence();
    atomicAdd(ctr, 1);
    bool ok = false;
    const uint64_t t0 = globaltimer();
    for (uint32_t i = 0;; ++i) {
      if (ld_acquire(ctr) >= target) { ok = true; break; }
      if (ld_volatile(p.sync + kSyncAbort)) break;
      if ((i & 31u) == 31u && globaltimer() - t0 > 2000000000ull) {
        raise_abort(p);
        break;
      }
    }
    __threadfence();
    ms.ok = ok;
  }
  sw_sync();
  return ms.ok != 0;
}

// Chunk numbering helpers (all from the parameters).
__device__ __forceinline__ int64_t unit_first_chunk(const PruneParams &p, int64_t u) {
  if (u >= p.units) return (int64_t)p.L * p.Hkv * p.cpr;
  const int64_t row = u / p.B;
  return row * p.cpr + p.chunk_prefix[u - row * p.B];
}
__device__ __forceinline__ void group_chunks(const PruneParams &p, int g, int64_t &cs, int64_t &ce) {
  cs = unit_first_chunk(p, (int64_t)g * p.ug);
  ce = unit_first_chunk(p, min((int64_t)(g + 1) * p.ug, (int64_t)p.units));
}
__device__ __forceinline__ int64_t range_start(const PruneParams &p, int64_t cs, int64_t ce, int c) {
  return cs + (ce - cs) * c / p.ncta;
}
// The CTA whose range holds chunk q of the group [cs, ce).
__device__ __forceinline__ int chunk_owner(const PruneParams &p, int64_t cs, int64_t ce, int64_t q) {
  const int64_t n = ce - cs, x = q - cs;
  return (int)(((x + 1) * p.ncta + n - 1) / n) - 1;
}
// Unit and chunk-within-segment of chunk q.
__device__ __forceinline__ void chunk_unit(const PruneParams &p, int64_t q, int &u, int &jc) {
  const int row = (int)(q / p.cpr);
  const int rem = (int)(q - (int64_t)row * p.cpr);
  int lo = 0, hi = p.B;  // largest lo with chunk_prefix[lo] <= rem
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (p.chunk_prefix[mid] <= rem) lo = mid; else hi = mid;
  }
  u = row * p.B + lo;
  jc = rem - p.chunk_prefix[lo];
}

// Live length, budget and what the call does with unit u (kSkip: a length out of
// range or a head budget outside [1, budget]).
__device__ __forceinline__ void unit_state(const PruneParams &p, const int32_t *seqlen_s, int u,
                                           int &T, int &bud, int &mode) {
  const int b = u % p.B;
  T = p.unit_len ? p.unit_len[u] : seqlen_s[b];
  bud = p.head_budget ? p.head_budget[u / p.B] : p.budget;
  const int64_t capb = p.seg_start[b + 1] - p.seg_start[b];
  if (T < 0 || (int64_t)T > capb || bud < 1 || bud > p.budget) { mode = kSkip; return; }
  const int w = p.window > 1 ? p.window : 1;
  if (T <= bud) mode = kShort;
  else if ((int64_t)T < (int64_t)bud + w) mode = kHold;
  else mode = kPruneU;
}

__device__ __forceinline__ unsigned long long composite(uint32_t key, int slot) {
  return ((unsigned long long)key << kSlotBits) | (kSlotMask - (unsigned long long)slot);
}

// First-round bin of a z-score key on a grid of width 1/256 over [-8, 8), clamped;
// non-decreasing in the key (NaN keys sit at the ends of the key order and go to the
// end bins).
__device__ __forceinline__ uint32_t z_bin(uint32_t key) {
  const uint32_t u = (key & 0x80000000u) ? (key & 0x7fffffffu) : ~key;
  const float z = __uint_as_float(u);
  if (z != z) return (key & 0x80000000u) ? (uint32_t)(kPruneHistBins - 1) : 0u;
  const float t = fmaf(z, 256.0f, 2048.0f);
  if (!(t >= 0.0f)) return 0u;
  if (t >= (float)(kPruneHistBins - 1)) return (uint32_t)(kPruneHistBins - 1);
  return (uint32_t)t;
}

// Exclusive prefix over the select threads of one int each; returns the total too.
__device__ __forceinline__ int sw_excl_scan(SwMisc &ms, int v, int t, int *total) {
  const int w = t >> 5, lane = t & 31;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int x = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += x;
  }
  if (lane == 31) ms.scan[w] = incl;
  sw_sync();
  int before = 0, all = 0;
#pragma unroll
  for (int i = 0; i < NSW; ++i) {
    const int x = ms.scan[i];
    if (i < w) before += x;
    all += x;
  }
  sw_sync();
  *total = all;
  return before + incl - v;
}

// Radix select over n composites (given by get(i)): the krem-th largest
// (1 <= krem <= n).  Composites are below 2^50; digits of 11 bits, high first.
template <class Get>
__device__ unsigned long long radix_select(SwMisc &ms, uint32_t *rh, int n, int krem, Get get,
                                           int t) {
  unsigned long long prefix = 0, mask = 0;
  for (int shift = 44; shift >= 0; shift -= 11) {
    const int bits = shift == 44 ? 6 : 11;  // bits 44..49, then 11-bit digits down to bit 0
    const int nb = 1 << bits;
    for (int i = t; i < nb; i += SWT) rh[i] = 0u;
    sw_sync();
    for (int i = t; i < n; i += SWT) {
      const unsigned long long v = get(i);
      if ((v & mask) == prefix) atomicAdd(&rh[(v >> shift) & (nb - 1)], 1u);
    }
    sw_sync();
    // bin holding the krem-th largest: suffix sums over per-thread runs of bins
    const int per = (nb + SWT - 1) / SWT;
    const int b0 = min(nb, t * per), b1 = min(nb, b0 + per);
    int s = 0;
    for (int i = b0; i < b1; ++i) s += (int)rh[i];
    int total;
    const int excl = sw_excl_scan(ms, s, t, &total);
    const int higher = total - excl - s;  // counted keys in bins above this thread's run
    if (higher < krem && krem <= higher + s) {
      int cum = higher;
      for (int i = b1 - 1; i >= b0; --i) {
        const int c = (int)rh[i];
        if (cum + c >= krem) {
          ms.bc[0] = i;
          ms.bc[1] = cum;
          break;
        }
        cum += c;
      }
    }
    sw_sync();
    const int bin = ms.bc[0];
    krem -= ms.bc[1];
    prefix |= (unsigned long long)bin << shift;
    mask |= (unsigned long long)(nb - 1) << shift;
    sw_sync();
  }
  return prefix;
}

// Folded weights of unit u into a weight slot (one warp; see score_math.cuh for the layout).
template <int D, int G>
__device__ void compute_weights(const PruneParams &p, int u, float *dst, double2 *ea, int lane) {
  constexpr int F = D / 2, FP = F / 2;
  const int b = u % p.B, row = u / p.B;
  const int l = row / p.Hkv, g = row - l * p.Hkv;
  const double cur = (double)p.cur_pos[b];
  for (int f = lane; f < F; f += 32) {
    double s, c;
    sincos(p.omega[f] * cur, &s, &c);
    const double2 a = p.A[f];
    ea[f] = make_double2(c * a.x - s * a.y, c * a.y + s * a.x);
  }
  __syncwarp();
  const bool no_conc = (p.flags & TRIA_NO_CONC_WEIGHT) != 0;
  for (int e = lane; e < FP * G; e += 32) {
    const int fp = e / G, h = e - fp * G;
    const size_t base = ((size_t)l * p.Hq + (size_t)g * G + h) * F + 2 * fp;
    float wx[2], wy[2], nw[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const float2 c = p.centre[base + q];
      const double2 e2 = ea[2 * fp + q];
      wx[q] = (float)((double)c.x * e2.x - (double)c.y * e2.y);
      wy[q] = (float)((double)c.x * e2.y + (double)c.y * e2.x);
      const float r = no_conc ? 0.0f : p.mrl[base + q];
      nw[q] = (1.0f - r) * p.mean_norm[base + q];
    }
    float2 *o = reinterpret_cast<float2 *>(dst + (size_t)(fp * G + h) * 6);
    o[0] = make_float2(wx[0], wx[1]);
    o[1] = make_float2(wy[0], wy[1]);
    o[2] = make_float2(nw[0], nw[1]);
  }
  __syncwarp();
}

// 16-byte copies of nrow rows of rowb bytes (plus one int32 each) from src rows to
// dst rows, all select threads.
__device__ __forceinline__ void copy_rows16(uint8_t *dst, const uint8_t *src, int64_t nbytes, int t) {
  const int64_t nv = nbytes >> 4;
  const uint4 *s = reinterpret_cast<const uint4 *>(src);
  uint4 *d = reinterpret_cast<uint4 *>(dst);
  int64_t i = t;
  for (; i + 3 * SWT < nv; i += 4 * SWT) {
    const uint4 a = s[i], b = s[i + SWT], c = s[i + 2 * SWT], e = s[i + 3 * SWT];
    d[i] = a; d[i + SWT] = b; d[i + 2 * SWT] = c; d[i + 3 * SWT] = e;
  }
  for (; i < nv; i += SWT) d[i] = s[i];
}

}  // namespace

template <int D, int G, int LAYOUT>
__global__ void __launch_bounds__(kPruneThreads, 1)
    prune_kernel(const __grid_constant__ PruneParams p) {
  using S = PruneShape<D, G>;
  constexpr int F = S::F, KPT = S::KPT, CH = S::CH, CB = S::CB, WB = S::WB, NSLOT = S::NSLOT;
  constexpr int ROWB = 2 * D;  // bytes of a K or V row
  extern __shared__ uint8_t smem_raw[];
  uint8_t *ring = smem_raw + ((1024u - (dev::smem_addr(smem_raw) & 1023u)) & 1023u);
  uint8_t *wring = ring + (size_t)NSLOT * CB;
  uint8_t *swb = wring + 2 * WB;  // 128-byte aligned: CB and WB are multiples of 128
  uint32_t *zks = reinterpret_cast<uint32_t *>(swb + SmemMap::ZKS);        // [kPruneRangeKeys]
  uint8_t *r1 = swb + SmemMap::R1;                                         // 32 KB
  uint32_t *lh = reinterpret_cast<uint32_t *>(r1);                         // [4096] local hist
  unsigned long long *bk = reinterpret_cast<unsigned long long *>(r1);     // [4096] bucket
  int32_t *kl = reinterpret_cast<int32_t *>(r1);                           // [2048] kept slots
  uint32_t *rh = reinterpret_cast<uint32_t *>(swb + SmemMap::RH);          // [2048]
  int2 *ctab = reinterpret_cast<int2 *>(swb + SmemMap::CTAB);              // [128]
  UEnt *utab = reinterpret_cast<UEnt *>(swb + SmemMap::UTAB);              // [129]
  SwMisc &ms = *reinterpret_cast<SwMisc *>(swb + SmemMap::MISC);
  int32_t *seqlen_s = reinterpret_cast<int32_t *>(swb + SmemMap::SEQ);     // [B]
  int4 *tab = reinterpret_cast<int4 *>(swb + SmemMap::TAB);                // [32]
  int32_t *taby = reinterpret_cast<int32_t *>(swb + SmemMap::TABY);        // [32]
  double2 *ea = reinterpret_cast<double2 *>(swb + SmemMap::EA);            // [128]
  int4 *desc = reinterpret_cast<int4 *>(swb + SmemMap::DESC);              // [NSLOT]
  uint64_t *full = reinterpret_cast<uint64_t *>(desc + NSLOT);
  uint64_t *empty = full + NSLOT;
  uint64_t *wfull = empty + NSLOT;     // [2]
  uint64_t *gdone = wfull + 2;         // [2] consumer warps finished a group
  uint64_t *rawfree = gdone + 2;       // [2] select warps done with a group's raw scores

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NSLOT; ++s) {
      dev::mbar_init(&full[s], 1);
      dev::mbar_init(&empty[s], 1);
    }
    for (int j = 0; j < 2; ++j) {
      dev::mbar_init(&wfull[j], 1);
      dev::mbar_init(&gdone[j], NW);
      dev::mbar_init(&rawfree[j], 1);
    }
    dev::fence_mbar_init();
  }
  // seq_len as it was at the start of the call (the kernel rewrites it unit by unit)
  if (p.seq_len)
    for (int i = threadIdx.x; i < p.B; i += blockDim.x) seqlen_s[i] = p.seq_len[i];
  __syncthreads();

  if (warp == NW) {
    // ================================================================ producer
    uint32_t q = 0;
    bool failed = false;
    int cur_unit = -1, wslot = 1;
    uint32_t wuse[2] = {0, 0};
    int64_t wlast[2] = {-1, -1};
    // the consumers fetch their code once before the key stream starts
    dev::named_barrier(2, (NW + 1) * 32);
    for (int g = 0; g < p.ngroups && !failed; ++g) {
      int64_t cs, ce;
      group_chunks(p, g, cs, ce);
      const int64_t r0 = range_start(p, cs, ce, c), r1e = range_start(p, cs, ce, c + 1);
      for (int64_t cg0 = r0; cg0 < r1e && !failed; cg0 += 32) {
        {
          const int64_t qq = cg0 + lane;
          int4 e = make_int4(0, 0, 0, 0);
          int32_t y = 0;
          if (qq < r1e) {
            int u, jc, T, bud, mode;
            chunk_unit(p, qq, u, jc);
            unit_state(p, seqlen_s, u, T, bud, mode);
            const int key0 = jc * CH;
            const int n = mode == kPruneU ? min(max(T - key0, 0), CH) : 0;
            e = make_int4(u, key0, (int)(qq - r0), n);
            const int row = u / p.B;
            y = (int32_t)((int64_t)row * p.cap + p.seg_start[u - row * p.B] + key0);
          }
          tab[lane] = e;
          taby[lane] = y;
        }
        __syncwarp();
        const int cnt = (int)(r1e - cg0 < 32 ? r1e - cg0 : 32);
        for (int i = 0; i < cnt; ++i) {
          const int4 e = tab[i];
          if (e.w == 0) continue;
          const uint32_t s = q % NSLOT, use = q / NSLOT;
          int ok = 1;
          if (lane == 0 && use > 0) ok = wait_bar(p, &empty[s], (use - 1) & 1);
          if (!__shfl_sync(0xffffffffu, ok, 0)) { failed = true; break; }
          if (e.x != cur_unit) {
            // the unit's weights go to the other weight slot, once every chunk that read
            // that slot's previous weights has been released (positions up to q - NSLOT
            // were covered by the waits above)
            const int j = wslot ^ 1;
            if (wlast[j] >= 0) {
              if (lane == 0)
                for (int64_t pp = (int64_t)q - NSLOT + 1; pp <= wlast[j] && ok; ++pp)
                  if (pp >= 0) ok = wait_bar(p, &empty[pp % NSLOT], (uint32_t)(pp / NSLOT) & 1);
              if (!__shfl_sync(0xffffffffu, ok, 0)) { failed = true; break; }
            }
            compute_weights<D, G>(p, e.x, reinterpret_cast<float *>(wring + j * WB), ea, lane);
            __threadfence_block();
            __syncwarp();
            if (lane == 0) dev::mbar_arrive(&wfull[j]);
            ++wuse[j];
            wslot = j;
            cur_unit = e.x;
          }
          wlast[wslot] = q;
          if (lane == 0) {
            const int wtag = wslot | (int)(((wuse[wslot] - 1) & 1) << 1);
            desc[s] = make_int4(e.x, e.y, (g << 8) | e.z, e.w | (wtag << 16));
            dev::mbar_arrive_expect_tx(&full[s], CB);
#pragma unroll
            for (int bx = 0; bx < S::NBOX; ++bx)
              dev::tma_load_2d(ring + (size_t)s * CB + bx * S::BOXB, &p.tmap, bx * 64, taby[i],
                               &full[s]);
          }
          ++q;
        }
        __syncwarp();  // the table is read before it is rewritten
      }
    }
    if (lane == 0) {
      // one end marker per consumer warp
      for (int t = 0; t < NW && !failed; ++t) {
        const uint32_t s = q % NSLOT, use = q / NSLOT;
        if (use > 0 && !wait_bar(p, &empty[s], (use - 1) & 1)) { failed = true; break; }
        desc[s] = make_int4(0, 0, 0, -1);
        dev::mbar_arrive(&full[s]);
        ++q;
      }
      if (failed) {
        raise_abort(p);
        // let the copies already issued land before the CTA can retire
        const uint32_t first = q > (uint32_t)NSLOT ? q - NSLOT : 0;
        for (uint32_t u = first; u < q; ++u) dev::mbar_wait(&full[u % NSLOT], (u / NSLOT) & 1);
      }
    }
    return;
  }

  if (warp < NW) {
    // ================================================================ consumers
    int wseen = -1, open_g = 0;
    bool failed = false;
    auto close_group = [&](int h) {
      __threadfence_block();
      __syncwarp();
      if (lane == 0) dev::mbar_arrive(&gdone[h & 1]);
    };
    auto enter_group = [&](int h) -> bool {
      int ok = 1;
      if (h >= 2 && lane == 0) ok = wait_bar(p, &rawfree[h & 1], (uint32_t)((h - 2) >> 1) & 1);
      return __shfl_sync(0xffffffffu, ok, 0) != 0;
    };
    // The first pass is a warm-up: one inner iteration of the chunk code on whatever
    // slot 0 holds, storing nothing, so that the code is fetched before the key stream
    // saturates the memory system; then the producer may start.
    bool warm = true;
#pragma unroll 1
    for (uint32_t q = warp;;) {
      uint32_t s = 0;
      int g = 0, lchunk = 0, n = 0, wtag = 0;
      if (!warm) {
        s = q % NSLOT;
        const uint32_t use = q / NSLOT;
        int ok = 1;
        if (lane == 0)
          ok = (use == 0 || wait_bar(p, &empty[s], (use - 1) & 1)) && wait_bar(p, &full[s], use & 1);
        if (!__shfl_sync(0xffffffffu, ok, 0)) { failed = true; break; }
        const int4 d = desc[s];
        if (d.w < 0) break;
        g = d.z >> 8;
        lchunk = d.z & 255;
        n = d.w & 0xffff;
        wtag = d.w >> 16;
        while (open_g < g && !failed) {
          close_group(open_g);
          ++open_g;
          failed = !enter_group(open_g);
        }
        if (failed) break;
        if (wtag != wseen) {
          int okw = 1;
          if (lane == 0) okw = wait_bar(p, &wfull[wtag & 1], (uint32_t)(wtag >> 1));
          if (!__shfl_sync(0xffffffffu, okw, 0)) { failed = true; break; }
          wseen = wtag;
        }
      }
      float out[KPT][G];
      km::score_chunk<D, G, LAYOUT>(dev::smem_addr(ring + (size_t)s * CB),
                                    reinterpret_cast<const float *>(wring + (wtag & 1) * WB),
                                    lane, warm ? 1 : S::FP / 4, out);
      float *rb = p.raw + (((size_t)(g & 1) * p.ncta + c) * p.range_keys + (size_t)lchunk * CH) * G;
#pragma unroll
      for (int k = 0; k < KPT; ++k) {
        const int r = lane + 32 * k;
        if (r < n) {
          float *o = rb + (size_t)r * G;
          if constexpr (G % 4 == 0) {
#pragma unroll
            for (int h = 0; h < G; h += 4)
              *reinterpret_cast<float4 *>(o + h) =
                  make_float4(out[k][h], out[k][h + 1], out[k][h + 2], out[k][h + 3]);
          } else if constexpr (G == 2) {
            *reinterpret_cast<float2 *>(o) = make_float2(out[k][0], out[k][1]);
          } else {
            o[0] = out[k][0];
          }
        }
      }
      if (warm) {
        warm = false;
        dev::named_barrier_arrive(2, (NW + 1) * 32);  // the producer may start the stream
        continue;
      }
      __syncwarp();
      if (lane == 0) dev::mbar_arrive(&empty[s]);
      q += NW;
    }
    if (failed) {
      if (lane == 0) raise_abort(p);
      return;
    }
    while (open_g < p.ngroups) {
      close_group(open_g);
      ++open_g;
      if (open_g < p.ngroups && !enter_group(open_g)) {
        if (lane == 0) raise_abort(p);
        return;
      }
    }
    return;
  }

  // ================================================================== select warps
  const int t = threadIdx.x - (NW + 1) * 32;
  const int sw_warp = t >> 5;
  bool alive = true;
  // Units whose segments have no chunk never meet a range: CTA u % ncta writes their
  // selection rows (all -1: a valid length there is 0) and reports bad lengths.
  for (int u = c; u < p.units; u += p.ncta) {
    const int row = u / p.B, b = u - row * p.B;
    if (p.chunk_prefix[b + 1] != p.chunk_prefix[b]) continue;
    if ((p.unit_len ? p.unit_len[u] : seqlen_s[b]) != 0) {
      if (t == 0 && (row == 0 || p.unit_len)) dev::set_error(p.err, TRIA_DEVERR_SEQ_LEN);
      continue;
    }
    if (p.sel_out && p.write_short_sel)
      for (int j = t; j < p.budget; j += SWT) p.sel_out[(int64_t)u * p.budget + j] = -1;
  }
  for (int g = 0; g < p.ngroups && alive; ++g) {
    const int slot = g & 1;
    int okg = 1;
    if (t == 0) okg = wait_bar(p, &gdone[slot], (uint32_t)(g >> 1) & 1);
    if (t == 0) ms.ok = okg;
    sw_sync();
    if (!ms.ok) { if (t == 0) raise_abort(p); alive = false; break; }
    int64_t cs, ce;
    group_chunks(p, g, cs, ce);
    const int64_t r0 = range_start(p, cs, ce, c), r1e = range_start(p, cs, ce, c + 1);
    const int m = (int)(r1e - r0);
    const int u0g = g * p.ug;
    // ------------------------------------------------------------ step 0: tables
    if (t < m) {
      int u, jc;
      chunk_unit(p, r0 + t, u, jc);
      ctab[t] = make_int2(u, jc);
    }
    sw_sync();
    if (t == 0) {
      int nu = 0;
      for (int i = 0; i < m; ++i) {
        const int u = ctab[i].x;
        if (nu == 0 || utab[nu - 1].u != u) {
          utab[nu].u = u;
          utab[nu].lc0 = i;
          utab[nu].nlc = 0;
          ++nu;
        }
        ++utab[nu - 1].nlc;
      }
      ms.nu = nu;
    }
    sw_sync();
    const int nu = ms.nu;
    if (t < nu) {
      UEnt &e = utab[t];
      unit_state(p, seqlen_s, e.u, e.T, e.bud, e.mode);
      const int jc0 = ctab[e.lc0].y, jc1 = ctab[e.lc0 + e.nlc - 1].y;
      e.key0 = jc0 * CH;
      e.key1 = e.mode == kPruneU ? max(e.key0, min(e.T, (jc1 + 1) * CH)) : e.key0;
      const int64_t f0 = unit_first_chunk(p, e.u), f1 = unit_first_chunk(p, e.u + 1);
      e.clo = chunk_owner(p, cs, ce, f0);
      e.chi = chunk_owner(p, cs, ce, f1 - 1);
      if (e.mode == kSkip && c == e.clo)
        dev::set_error(p.err, (e.bud < 1 || e.bud > p.budget) ? TRIA_DEVERR_BUDGET
                                                              : TRIA_DEVERR_SEQ_LEN);
    }
    sw_sync();
    // ------------------------------------------------------------ step 1: sums of s, s^2
    for (int i = 0; i < nu; ++i) {
      const UEnt e = utab[i];
      if (e.mode != kPruneU) continue;
      const int nk = e.key1 - e.key0, li0 = e.lc0 * CH;
      const float *rb = p.raw + (((size_t)slot * p.ncta + c) * p.range_keys + li0) * G;
      double s1[G], s2[G];
#pragma unroll
      for (int h = 0; h < G; ++h) { s1[h] = 0.0; s2[h] = 0.0; }
      for (int k = t; k < nk; k += SWT) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const double v = (double)rb[(size_t)k * G + h];
          s1[h] += v;
          s2[h] = fma(v, v, s2[h]);
        }
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          s1[h] += __shfl_xor_sync(0xffffffffu, s1[h], o);
          s2[h] += __shfl_xor_sync(0xffffffffu, s2[h], o);
        }
      }
      if ((t & 31) == 0) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
          ms.red[sw_warp][2 * h] = s1[h];
          ms.red[sw_warp][2 * h + 1] = s2[h];
        }
      }
      sw_sync();
      if (t < 2 * G) {
        double a = 0.0;
#pragma unroll
        for (int w = 0; w < NSW; ++w) a += ms.red[w][t];
        p.partial[(((size_t)slot * p.ncta + c) * p.range_units + i) * (2 * G) + t] = a;
      }
      sw_sync();
    }
    if (!grid_round(p, ms, kSyncA, g, t)) { alive = false; break; }
    // ------------------------------------------------------------ step 2: z keys, histograms
    for (int i = 0; i < nu; ++i) {
      const UEnt e = utab[i];
      if (e.mode != kPruneU) continue;
      // mu and sigma from every covering CTA's sums, added in CTA order
      {
        constexpr int COLS = 2 * G, TPC = SWT / COLS;
        const int col = t / TPC, j = t - col * TPC;
        double a = 0.0;
        for (int cc = e.clo + j; cc <= e.chi; cc += TPC) {
          const int64_t ra = range_start(p, cs, ce, cc);
          if (ra == range_start(p, cs, ce, cc + 1)) continue;  // an empty range publishes nothing
          int uf, jcf;
          chunk_unit(p, ra, uf, jcf);
          const int ul = e.u - uf;
          a += __ldcg(p.partial + (((size_t)slot * p.ncta + cc) * p.range_units + ul) * (2 * G) + col);
        }
        sw_sync();
        reinterpret_cast<double *>(rh)[t] = a;  // the radix histogram area is free here
        sw_sync();
        if (t < COLS) {
          double sum = 0.0;
          for (int k = 0; k < TPC; ++k) sum += reinterpret_cast<double *>(rh)[t * TPC + k];
          ms.stat[t] = sum;
        }
        sw_sync();
        if (t < G) {
          const double mu = ms.stat[2 * t] / (double)e.T;
          const double var = ms.stat[2 * t + 1] / (double)e.T - mu * mu;
          ms.mu_hi[t] = (float)mu;
          ms.mu_lo[t] = (float)(mu - (double)ms.mu_hi[t]);
          ms.inv_sig[t] = var > 0.0 ? (float)(1.0 / sqrt(var)) : 0.0f;
        }
        for (int i2 = t; i2 < kPruneHistBins; i2 += SWT) lh[i2] = 0u;
        sw_sync();
      }
      float mh[G], ml[G], is[G];
#pragma unroll
      for (int h = 0; h < G; ++h) { mh[h] = ms.mu_hi[h]; ml[h] = ms.mu_lo[h]; is[h] = ms.inv_sig[h]; }
      const int nk = e.key1 - e.key0, li0 = e.lc0 * CH;
      const float *rb = p.raw + (((size_t)slot * p.ncta + c) * p.range_keys + li0) * G;
      uint32_t *zg = p.zk + (size_t)slot * p.zk_stride + (size_t)(r0 - cs) * CH + li0;
      for (int k = t; k < nk; k += SWT) {
        float zf = -3.0e38f;
#pragma unroll
        for (int h = 0; h < G; ++h) zf = fmaxf(zf, ((rb[(size_t)k * G + h] - mh[h]) - ml[h]) * is[h]);
        const uint32_t key = dev::order_key(zf);
        zks[li0 + k] = key;
        zg[k] = key;
        atomicAdd(&lh[z_bin(key)], 1u);
      }
      sw_sync();
      uint32_t *hg = p.hist + ((size_t)slot * kPruneMaxGroupUnits + (e.u - u0g)) * kPruneHistBins;
      for (int bn = t; bn < kPruneHistBins; bn += SWT) {
        const uint32_t v = lh[bn];
        if (v) atomicAdd(&hg[bn], v);
      }
      sw_sync();
    }
    if (t == 0) dev::mbar_arrive(&rawfree[slot]);  // the consumers may reuse this raw slot
    if (!grid_round(p, ms, kSyncB, g, t)) { alive = false; break; }
    // ------------------------------------------------------------ step 3: threshold bins
    for (int i = 0; i < nu; ++i) {
      UEnt &eref = utab[i];
      const UEnt e = eref;
      if (e.mode != kPruneU) continue;
      const int ug_i = e.u - u0g;
      const uint32_t *hg = p.hist + ((size_t)slot * kPruneMaxGroupUnits + ug_i) * kPruneHistBins;
      // 32 bins per thread, thread 127 holding the highest
      uint32_t cnt[32];
#pragma unroll
      for (int v4 = 0; v4 < 8; ++v4) {
        const uint4 x = __ldcg(reinterpret_cast<const uint4 *>(hg + t * 32) + v4);
        cnt[4 * v4] = x.x; cnt[4 * v4 + 1] = x.y; cnt[4 * v4 + 2] = x.z; cnt[4 * v4 + 3] = x.w;
      }
      int sum = 0;
#pragma unroll
      for (int k = 0; k < 32; ++k) sum += (int)cnt[k];
      int total;
      const int excl = sw_excl_scan(ms, sum, t, &total);
      const int higher = total - excl - sum;
      const int krem = e.bud;
      if (higher < krem && krem <= higher + sum) {
        int cum = higher;
        bool found = false;
#pragma unroll
        for (int k = 31; k >= 0; --k) {
          const int cc = (int)cnt[k];
          if (!found && cum + cc >= krem) {
            found = true;
            ms.bc[0] = t * 32 + k;
            ms.bc[1] = cum;
            ms.bc[2] = cc;
          }
          if (!found) cum += cc;
        }
      }
      sw_sync();
      const int bstar = ms.bc[0], above = ms.bc[1], bcnt = ms.bc[2];
      sw_sync();
      if (t == 0) { eref.bstar = bstar; eref.above = above; eref.bcnt = bcnt; }
      const int nk = e.key1 - e.key0, li0 = e.lc0 * CH;
      if (bcnt <= kPruneBucketMax) {
        // this range's keys in the bin and above it
        int nc = 0, na = 0;
        for (int k = t; k < nk; k += SWT) {
          const uint32_t bn = z_bin(zks[li0 + k]);
          nc += bn == (uint32_t)bstar;
          na += bn > (uint32_t)bstar;
        }
        int tot_c, tot_a;
        const int off = sw_excl_scan(ms, nc, t, &tot_c);
        sw_excl_scan(ms, na, t, &tot_a);
        if (t == 0) {
          ms.bc[3] = tot_c > 0 ? atomicAdd(p.bcount + slot * kPruneMaxGroupUnits + ug_i, tot_c) : 0;
          p.above[((size_t)slot * p.ug + ug_i) * p.ncta + (c - e.clo)] = tot_a;
        }
        sw_sync();
        unsigned long long *bl = p.bucket + ((size_t)slot * p.ug + ug_i) * kPruneBucketMax;
        int w = ms.bc[3] + off;
        for (int k = t; k < nk; k += SWT) {
          const uint32_t key = zks[li0 + k];
          if (z_bin(key) == (uint32_t)bstar) {
            if (w < kPruneBucketMax) bl[w] = composite(key, e.key0 + k);
            ++w;
          }
        }
        sw_sync();
      } else if (c == e.clo) {
        // a bin too large to gather: this CTA selects the unit exactly over all its keys
        const uint32_t *zu = p.zk + (size_t)slot * p.zk_stride +
                             (size_t)(unit_first_chunk(p, e.u) - cs) * CH;
        const unsigned long long thr = radix_select(
            ms, rh, e.T, e.bud, [&](int k) { return composite(__ldcg(zu + k), k); }, t);
        // kept keys per covering CTA (their slot ranges within the unit)
        const int64_t f0 = unit_first_chunk(p, e.u), f1 = unit_first_chunk(p, e.u + 1);
        for (int cc = e.clo; cc <= e.chi; ++cc) {
          // the CTA's chunks [ra, rb) meet the unit's [f0, f1) in keys [a0, b1)
          const int64_t ra = max(range_start(p, cs, ce, cc), f0);
          const int64_t rb2 = min(range_start(p, cs, ce, cc + 1), f1);
          const int a0 = (int)((ra - f0) * CH);
          const int b1 = rb2 > ra ? (int)(e.T < (rb2 - f0) * CH ? (int64_t)e.T : (rb2 - f0) * CH) : a0;
          int kept = 0;
          for (int k = a0 + t; k < b1; k += SWT) kept += composite(__ldcg(zu + k), k) >= thr;
          int tot;
          sw_excl_scan(ms, kept, t, &tot);
          if (t == 0) p.kcount[((size_t)slot * p.ug + ug_i) * p.ncta + (cc - e.clo)] = tot;
        }
        if (t == 0) p.thr[(size_t)slot * p.ug + ug_i] = thr;
        sw_sync();
      }
    }
    if (!grid_round(p, ms, kSyncC, g, t)) { alive = false; break; }
    // this group's histograms are read by every CTA by now: clear this CTA's share
    {
      const int64_t words = (int64_t)min(p.ug, p.units - u0g) * kPruneHistBins;
      const int64_t w0 = words * c / p.ncta, w1 = words * (c + 1) / p.ncta;
      uint32_t *hb = p.hist + (size_t)slot * kPruneMaxGroupUnits * kPruneHistBins;
      for (int64_t k = w0 + t; k < w1; k += SWT) hb[k] = 0u;
    }
    // ------------------------------------------------------------ step 4: emit and stage
    for (int i = 0; i < nu; ++i) {
      UEnt &eref = utab[i];
      const UEnt e = eref;
      if (e.mode != kPruneU) continue;
      const int ug_i = e.u - u0g;
      const int nk = e.key1 - e.key0, li0 = e.lc0 * CH;
      unsigned long long thr;
      int oc = 0, kc = 0;
      if (e.bcnt <= kPruneBucketMax) {
        const int nb = e.bcnt;
        const unsigned long long *bl = p.bucket + ((size_t)slot * p.ug + ug_i) * kPruneBucketMax;
        for (int k = t; k < nb; k += SWT) bk[k] = __ldcg(bl + k);
        sw_sync();
        const int krem = e.bud - e.above;  // 1 <= krem <= nb
        if (nb <= 4 * SWT) {
          // pairwise ranks: the entry with krem - 1 larger entries is the threshold
          for (int k = t; k < nb; k += SWT) {
            const unsigned long long v = bk[k];
            int rank = 0;
            for (int j = 0; j < nb; ++j) rank += bk[j] > v;
            if (rank == krem - 1) ms.rv = v;
          }
          sw_sync();
          thr = ms.rv;
        } else {
          thr = radix_select(ms, rh, nb, krem, [&](int k) { return bk[k]; }, t);
        }
        // kept keys before this range and in it
        int before = 0, mine = 0;
        for (int k = t; k < nb; k += SWT) {
          const unsigned long long v = bk[k];
          if (v >= thr) {
            const int sl = (int)(kSlotMask - (v & kSlotMask));
            before += sl < e.key0;
            mine += sl >= e.key0 && sl < e.key1;
          }
        }
        const int32_t *ab = p.above + ((size_t)slot * p.ug + ug_i) * p.ncta;
        for (int cc = e.clo + t; cc < c; cc += SWT)
          if (range_start(p, cs, ce, cc) != range_start(p, cs, ce, cc + 1))
            before += __ldcg(ab + (cc - e.clo));
        if (t == 0) mine += __ldcg(ab + (c - e.clo));
        int tb, tm;
        sw_excl_scan(ms, before, t, &tb);
        sw_excl_scan(ms, mine, t, &tm);
        oc = tb;
        kc = tm;
      } else {
        thr = __ldcg(p.thr + (size_t)slot * p.ug + ug_i);
        const int32_t *kb = p.kcount + ((size_t)slot * p.ug + ug_i) * p.ncta;
        int before = 0;
        for (int cc = e.clo + t; cc < c; cc += SWT) before += __ldcg(kb + (cc - e.clo));
        int tb;
        sw_excl_scan(ms, before, t, &tb);
        oc = tb;
        kc = __ldcg(kb + (c - e.clo));
      }
      // the kept keys of a unit fill [0, budget) exactly once; anything else is a bug
      // that must not write outside the unit's rows
      if (oc < 0 || kc < 0 || oc + kc > e.bud) {
        if (t == 0) dev::set_error(p.err, TRIA_DEVERR_SELECTION);
        oc = 0;
        kc = 0;
      }
      // kept slots in slot order: warp w owns a contiguous run, ballots order its keys
      {
        const int WL = ((nk + NSW - 1) / NSW + 31) & ~31;
        const int w0 = min(nk, sw_warp * WL), w1 = min(nk, w0 + WL);
        const int lane_s = t & 31;
        int cnt = 0;
        for (int k = w0 + lane_s; k < w1; k += 32)
          cnt += composite(zks[li0 + k], e.key0 + k) >= thr;
        cnt = __reduce_add_sync(0xffffffffu, cnt);
        if (lane_s == 0) ms.scan[sw_warp] = cnt;
        sw_sync();  // (the bucket in r1 is no longer read: the kept list may overwrite it)
        int o = 0;
        for (int w = 0; w < sw_warp; ++w) o += ms.scan[w];
        const uint32_t below = (1u << lane_s) - 1u;
        int32_t *so = p.sel_out ? p.sel_out + (int64_t)e.u * p.budget : nullptr;
        for (int k0 = w0; k0 < w1; k0 += 32) {
          const int k = k0 + lane_s;
          const bool keep = k < w1 && composite(zks[li0 + k], e.key0 + k) >= thr;
          const uint32_t km = __ballot_sync(0xffffffffu, keep);
          const int oi = o + __popc(km & below);
          if (keep && oi < kc) {
            kl[oi] = e.key0 + k;
            if (so) so[oc + oi] = e.key0 + k;
          }
          o += __popc(km);
        }
        sw_sync();
        if (t == 0) { eref.thr = thr; eref.oc = oc; eref.kc = kc; }
      }
      // stage the kept rows (K, V, pos) at their final index, out of place
      {
        const int row = e.u / p.B, b = e.u - row * p.B;
        const int64_t base = (int64_t)row * p.cap + p.seg_start[b];
        const uint8_t *ks = p.k + (size_t)base * ROWB;
        const uint8_t *vs = p.v + (size_t)base * ROWB;
        uint8_t *kd = p.stage_k + ((size_t)ug_i * p.budget + oc) * ROWB;
        uint8_t *vd = p.stage_v + ((size_t)ug_i * p.budget + oc) * ROWB;
        constexpr int VPR = ROWB / 16;
        const int nv = kc * VPR;
        for (int w = t; w < nv; w += SWT) {
          const int j = w / VPR, x = w - j * VPR;
          const int64_t src = kl[j];
          const uint4 a = __ldcg(reinterpret_cast<const uint4 *>(ks + (size_t)src * ROWB) + x);
          const uint4 bb = __ldcg(reinterpret_cast<const uint4 *>(vs + (size_t)src * ROWB) + x);
          reinterpret_cast<uint4 *>(kd + (size_t)j * ROWB)[x] = a;
          reinterpret_cast<uint4 *>(vd + (size_t)j * ROWB)[x] = bb;
        }
        int32_t *pd = p.stage_pos + (size_t)ug_i * p.budget + oc;
        for (int j = t; j < kc; j += SWT) pd[j] = __ldcg(p.pos + base + kl[j]);
      }
      sw_sync();
    }
    if (!grid_round(p, ms, kSyncD, g, t)) { alive = false; break; }
    // ------------------------------------------------------------ step 5: write back
    for (int i = 0; i < nu; ++i) {
      const UEnt e = utab[i];
      const int row = e.u / p.B, b = e.u - row * p.B;
      const int ug_i = e.u - u0g;
      if (e.mode == kPruneU) {
        const int64_t base = (int64_t)row * p.cap + p.seg_start[b];
        if (e.kc > 0) {
          const uint8_t *ks = p.stage_k + ((size_t)ug_i * p.budget + e.oc) * ROWB;
          const uint8_t *vs = p.stage_v + ((size_t)ug_i * p.budget + e.oc) * ROWB;
          copy_rows16(p.k + (size_t)(base + e.oc) * ROWB, ks, (int64_t)e.kc * ROWB, t);
          copy_rows16(p.v + (size_t)(base + e.oc) * ROWB, vs, (int64_t)e.kc * ROWB, t);
          const int32_t *ps = p.stage_pos + (size_t)ug_i * p.budget + e.oc;
          for (int j = t; j < e.kc; j += SWT) p.pos[base + e.oc + j] = ps[j];
        }
        if (c == e.clo) {
          if (t == 0) {
            if (p.unit_len) p.unit_len[e.u] = e.bud;
            else if (row == 0) p.seq_len[b] = e.bud;
            p.bcount[slot * kPruneMaxGroupUnits + ug_i] = 0;
          }
          // a head budget below the list length leaves the rest of the list empty
          if (p.sel_out)
            for (int j = e.bud + t; j < p.budget; j += SWT) p.sel_out[(int64_t)e.u * p.budget + j] = -1;
        }
      } else if (e.mode == kShort && c == e.clo && p.sel_out && p.write_short_sel) {
        int32_t *so = p.sel_out + (int64_t)e.u * p.budget;
        for (int j = t; j < p.budget; j += SWT) so[j] = j < e.T ? j : -1;
      }
    }
    sw_sync();
  }
  // ------------------------------------------------------------------ leave
  sw_sync();
  if (t == 0) {
    __threadfence();
    const int32_t was = atomicAdd(p.sync + kSyncExit, 1);
    if (was == p.ncta - 1) {
      // the last CTA out: every other CTA is past its last synchronisation
      __threadfence();
      const bool aborted = ld_volatile(p.sync + kSyncAbort) != 0;
      if (aborted) {
        // a group may have stopped half-way: clear what must be zero at rest
        for (int k = 0; k < 2 * kPruneMaxGroupUnits * kPruneHistBins; ++k) p.hist[k] = 0u;
        for (int k = 0; k < 2 * kPruneMaxGroupUnits; ++k) p.bcount[k] = 0;
      }
      for (int k = 0; k < kSyncWords; ++k) p.sync[k] = 0;
      __threadfence();
    }
  }
}

// ------------------------------------------------------------------ host side
template <int D, int G>
static size_t smem_of() {
  if constexpr (PruneShape<D, G>::OK) return PruneShape<D, G>::SMEM;
  return 0;
}

size_t prune_smem_bytes(int D, int G) {
#define TRIA_SMEM_G(DD)                             \
  switch (G) {                                     \
    case 1: return smem_of<DD, 1>();               \
    case 2: return smem_of<DD, 2>();               \
    case 4: return smem_of<DD, 4>();               \
    case 8: return smem_of<DD, 8>();               \
    case 16: return smem_of<DD, 16>();             \
    default: return 0;                             \
  }
  switch (D) {
    case 64: TRIA_SMEM_G(64)
    case 128: TRIA_SMEM_G(128)
    case 256: TRIA_SMEM_G(256)
    default: return 0;
  }
#undef TRIA_SMEM_G
}

static int chunk_keys_of(int D, int G) {
#define TRIA_CH_G(DD)                                         \
  switch (G) {                                               \
    case 1: return KeyShape<DD, 1>::CH;                      \
    case 2: return KeyShape<DD, 2>::CH;                      \
    case 4: return KeyShape<DD, 4>::CH;                      \
    case 8: return KeyShape<DD, 8>::CH;                      \
    case 16: return KeyShape<DD, 16>::CH;                    \
    default: return 0;                                       \
  }
  switch (D) {
    case 64: TRIA_CH_G(64)
    case 128: TRIA_CH_G(128)
    case 256: TRIA_CH_G(256)
    default: return 0;
  }
#undef TRIA_CH_G
}

bool prune_supported(int D, int G, int layout) {
  if (layout != TRIA_ROPE_HALF_SPLIT && layout != TRIA_ROPE_INTERLEAVED) return false;
  return prune_smem_bytes(D, G) > 0;
}

PrunePlan prune_plan(const tria_config &cfg, const int64_t *seq_start) {
  PrunePlan pl{};
  const int G = cfg.n_kv_heads > 0 ? cfg.n_q_heads / cfg.n_kv_heads : 0;
  if (!prune_supported(cfg.head_dim, G, cfg.rope_layout)) return pl;
  const int CH = chunk_keys_of(cfg.head_dim, G);
  pl.chunk_keys = CH;
  pl.ncta = device_sm_count();
  int64_t cpr = 0;
  for (int b = 0; b < cfg.batch; ++b) cpr += (seq_start[b + 1] - seq_start[b] + CH - 1) / CH;
  if (cpr > INT32_MAX / 2) return pl;
  pl.cpr = (int)cpr;
  const int64_t units = (int64_t)cfg.num_layers * cfg.n_kv_heads * cfg.batch;
  if (units > INT32_MAX / 2) return pl;
  const int64_t total = (int64_t)cfg.num_layers * cfg.n_kv_heads * cpr;
  const int64_t cap_chunks = (int64_t)pl.ncta * (kPruneRangeKeys / CH);
  auto unit_chunks = [&](int64_t u) {
    const int b = (int)(u % cfg.batch);
    return (seq_start[b + 1] - seq_start[b] + CH - 1) / CH;
  };
  auto max_group = [&](int64_t ug) {
    int64_t most = 0;
    for (int64_t g0 = 0; g0 < units; g0 += ug) {
      int64_t n = 0;
      for (int64_t u = g0; u < std::min(units, g0 + ug); ++u) n += unit_chunks(u);
      most = std::max(most, n);
    }
    return most;
  };
  // at least two groups when there is enough work (the second one's scoring hides
  // the first one's selection), at most kPruneMaxGroupUnits units, and no CTA share
  // above kPruneRangeKeys keys
  int64_t ug = total >= 8ll * pl.ncta ? (units + 1) / 2 : units;
  ug = std::max<int64_t>(1, std::min<int64_t>(ug, kPruneMaxGroupUnits));
  int64_t most = max_group(ug);
  while (most > cap_chunks && ug > 1) {
    ug = std::max<int64_t>(1, std::min(ug - 1, ug * cap_chunks / most));
    most = max_group(ug);
  }
  if (most > cap_chunks) return pl;  // one unit alone is too large for the ranges
  pl.ug = (int)ug;
  pl.ngroups = (int)((units + ug - 1) / ug);
  const int64_t per_cta = (most + pl.ncta - 1) / pl.ncta;
  pl.range_keys = (int)std::max<int64_t>(CH, per_cta * CH);
  pl.range_units = (int)per_cta + 1;
  pl.zk_stride = most * CH;
  pl.ok = 1;
  return pl;
}

template <int D, int G, int LAYOUT>
static cudaError_t launch_prune_one(const PruneParams &p, cudaStream_t s) {
  using S = PruneShape<D, G>;
  if constexpr (!S::OK) {
    return cudaErrorInvalidValue;
  } else {
    auto kern = prune_kernel<D, G, LAYOUT>;
    static bool configured[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
    if (dev < 0 || dev >= 64 || !configured[dev]) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)S::SMEM);
      if (e != cudaSuccess) return e;
      if (dev >= 0 && dev < 64) configured[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.ncta, 1, 1);
    cfg.blockDim = dim3(kPruneThreads, 1, 1);
    cfg.dynamicSmemBytes = S::SMEM;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;  // all CTAs resident: they wait on one another
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, p);
  }
}

template <int D, int LAYOUT>
static cudaError_t prune_dispatch_g(const PruneParams &p, int G, cudaStream_t s) {
  switch (G) {
    case 1: return launch_prune_one<D, 1, LAYOUT>(p, s);
    case 2: return launch_prune_one<D, 2, LAYOUT>(p, s);
    case 4: return launch_prune_one<D, 4, LAYOUT>(p, s);
    case 8: return launch_prune_one<D, 8, LAYOUT>(p, s);
    case 16: return launch_prune_one<D, 16, LAYOUT>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_prune(const PruneParams &p, int D, int G, int layout, cudaStream_t s) {
  if (layout == TRIA_ROPE_HALF_SPLIT) {
    switch (D) {
      case 64: return prune_dispatch_g<64, TRIA_ROPE_HALF_SPLIT>(p, G, s);
      case 128: return prune_dispatch_g<128, TRIA_ROPE_HALF_SPLIT>(p, G, s);
      case 256: return prune_dispatch_g<256, TRIA_ROPE_HALF_SPLIT>(p, G, s);
    }
  } else {
    switch (D) {
      case 64: return prune_dispatch_g<64, TRIA_ROPE_INTERLEAVED>(p, G, s);
      case 128: return prune_dispatch_g<128, TRIA_ROPE_INTERLEAVED>(p, G, s);
      case 256: return prune_dispatch_g<256, TRIA_ROPE_INTERLEAVED>(p, G, s);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace tria
