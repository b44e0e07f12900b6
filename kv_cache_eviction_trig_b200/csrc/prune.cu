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
//       D  every CTA writes the slots it keeps into the unit's kept list, at
//          their destination index; after the round the covering CTAs split the
//          unit's destinations evenly;
//       E  each CTA copies out of place the kept rows of its share whose slot
//          lies below the unit's budget (a row another destination overwrites);
//          after the round it writes its destinations in place, from that copy
//          or straight from the source slot (slots >= budget are never written).
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
constexpr int kMaxRangeChunks = kPruneRangeKeys / 32;  // the smallest chunk is 32 keys
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
  int32_t bcnt, pad;       // keys in the threshold bin
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
  static constexpr int ZKS = 0;                                          // u16 [kPruneRangeKeys]
  static constexpr int R1 = ZKS + rnd128(kPruneRangeKeys * 2);           // 32 KB union
  static constexpr int RH = R1 + 32768;                                  // u32 [kRadixBins]
  static constexpr int CTAB = RH + rnd128(kRadixBins * 4);               // int2 [kMaxRangeChunks]
  static constexpr int UTAB = CTAB + rnd128(kMaxRangeChunks * 8);        // UEnt [kPruneMaxGroupUnits]
  static constexpr int MISC = UTAB + rnd128(kPruneMaxGroupUnits * (int)sizeof(UEnt));
  static constexpr int SEQ = MISC + rnd128((int)sizeof(SwMisc));         // i32 [TRIA_MAX_BATCH]
  static constexpr int TAB = SEQ + rnd128(TRIA_MAX_BATCH * 4);           // int4 [32]
  static constexpr int TABY = TAB + rnd128(32 * 16);                     // i32 [32]
  static constexpr int DESC = TABY + rnd128(32 * 4);                     // int4 [NSLOT], barriers
  static constexpr int END = DESC + 1024;
};

template <int D, int G>
struct PruneShape : KeyShape<D, G> {
  using K = KeyShape<D, G>;
  static constexpr int FIXED = 1024 + 2 * K::WB + SmemMap::END;
  static constexpr int LIMIT = 227 * 1024 - 256;  // room for the few static shared words
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

__device__ __forceinline__ int32_t *sync_word(const PruneParams &p, int w) {
  return p.sync + w * kSyncStride;
}

__device__ __forceinline__ void raise_abort(const PruneParams &p) {
  dev::set_error(p.err, TRIA_DEVERR_TIMEOUT);
  atomicExch(sync_word(p, kSyncAbort), 1);
}

// Bounded mbarrier wait that also gives up once another CTA has aborted (the abort
// word is looked at rarely: every waiting warp of every CTA would otherwise poll it).
__device__ __forceinline__ bool wait_bar(const PruneParams &p, uint64_t *bar, uint32_t parity) {
  for (uint32_t i = 0; i < 2000000u; ++i) {
    if (dev::mbar_try_wait(bar, parity)) return true;
    if ((i & 1023u) == 1023u && ld_volatile(sync_word(p, kSyncAbort))) return false;
  }
  return false;
}

// Grid round: every CTA adds one to counter `w` (slot g % 2) and waits until all
// CTAs of this and the earlier uses of the slot have arrived.  Called by all select
// threads; returns false (everywhere) when it gave up.
__device__ bool grid_round(const PruneParams &p, SwMisc &ms, int w, int g, int t) {
  sw_sync();  // every select thread's writes precede the arrival
  if (t == 0) {
    int32_t *ctr = sync_word(p, w + (g & 1));
    const int32_t target = p.ncta * ((g >> 1) + 1);
    // a release add: the select threads' writes (ordered before it by the barrier
    // above) are visible to every CTA whose acquiring poll sees the count
    asm volatile("red.release.gpu.global.add.s32 [%0], 1;" ::"l"(ctr) : "memory");
    bool ok = false;
    const uint64_t t0 = globaltimer();
    for (uint32_t i = 0;; ++i) {
      if (ld_acquire(ctr) >= target) { ok = true; break; }
      __nanosleep(64);  // back off: 148 CTAs poll the same line
      if ((i & 63u) == 63u) {
        if (ld_volatile(sync_word(p, kSyncAbort))) break;
        if (globaltimer() - t0 > 2000000000ull) {
          raise_abort(p);
          break;
        }
      }
    }
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

// Polls a grid counter until it reaches `target` (one thread; bounded, with back-off).
__device__ bool poll_counter(const PruneParams &p, int w, int32_t target) {
  int32_t *ctr = sync_word(p, w);
  const uint64_t t0 = globaltimer();
  for (uint32_t i = 0;; ++i) {
    if (ld_acquire(ctr) >= target) return true;
    __nanosleep(64);
    if ((i & 63u) == 63u) {
      if (ld_volatile(sync_word(p, kSyncAbort))) return false;
      if (globaltimer() - t0 > 2000000000ull) {
        raise_abort(p);
        return false;
      }
    }
  }
}

// Prologue, run by every warp but the producer (nt threads, thread wt): the
// folded weights of every unit into p.w.  First EA[b][f] = e^{i w_f cur_b} * A_f
// for every sequence and RoPE pair (float64 sincos, one per entry): when the
// table fits (B * F <= kEaLocal) every CTA computes all of it into shared memory
// (ea_s), else the CTAs share it out through p.ea and one grid round.  Then for
// every (unit, pair pair, head) the weights W = c * EA (trigonometric term) and
// Nw = (1 - R) E|q| (norm term) in the layout of score_math.cuh.  The producer
// copies a unit's weights into shared memory with one bulk copy when it reaches
// the unit.
constexpr int kEaLocal = 2048;
template <int D, int G>
__device__ bool prologue_weights(const PruneParams &p, int c, int wt, int nt, int *ok_s,
                                 double2 *ea_s) {
  constexpr int F = D / 2, FP = F / 2;
  const int64_t stride = (int64_t)p.ncta * nt;
  const bool local = (int64_t)p.B * F <= kEaLocal;
  if (local) {
    for (int e = wt; e < p.B * F; e += nt) {
      const int b = e / F, f = e - b * F;
      double sn, cs;
      sincos(p.omega[f] * (double)p.cur_pos[b], &sn, &cs);
      const double2 a = p.A[f];
      ea_s[e] = make_double2(cs * a.x - sn * a.y, cs * a.y + sn * a.x);
    }
    dev::named_barrier(5, nt);
  } else {
    for (int64_t e = (int64_t)c * nt + wt; e < (int64_t)p.B * F; e += stride) {
      const int b = (int)(e / F), f = (int)(e - (int64_t)b * F);
      double sn, cs;
      sincos(p.omega[f] * (double)p.cur_pos[b], &sn, &cs);
      const double2 a = p.A[f];
      p.ea[e] = make_double2(cs * a.x - sn * a.y, cs * a.y + sn * a.x);
    }
    dev::named_barrier(5, nt);
    if (wt == 0) {
      __threadfence();
      atomicAdd(sync_word(p, kSyncP1), 1);
      *ok_s = poll_counter(p, kSyncP1, p.ncta);
      __threadfence();
    }
    dev::named_barrier(5, nt);
    if (!*ok_s) return false;
  }
  const bool no_conc = (p.flags & TRIA_NO_CONC_WEIGHT) != 0;
  const int64_t per_unit = (int64_t)FP * G;
  for (int64_t e = (int64_t)c * nt + wt; e < (int64_t)p.units * per_unit; e += stride) {
    const int u = (int)(e / per_unit);
    const int r = (int)(e - (int64_t)u * per_unit);
    const int fp = r / G, h = r - fp * G;
    const int b = u % p.B, row = u / p.B;
    const int l = row / p.Hkv, g = row - l * p.Hkv;
    const size_t base = ((size_t)l * p.Hq + (size_t)g * G + h) * F + 2 * fp;
    float wx[2], wy[2], nw[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const float2 cc = p.centre[base + q];
      const size_t ei = (size_t)b * F + 2 * fp + q;
      const double2 e2 = local ? ea_s[ei] : __ldcg(p.ea + ei);
      wx[q] = (float)((double)cc.x * e2.x - (double)cc.y * e2.y);
      wy[q] = (float)((double)cc.x * e2.y + (double)cc.y * e2.x);
      const float rr = no_conc ? 0.0f : p.mrl[base + q];
      nw[q] = (1.0f - rr) * p.mean_norm[base + q];
    }
    float2 *o = reinterpret_cast<float2 *>(p.w + (size_t)e * 6);
    o[0] = make_float2(wx[0], wx[1]);
    o[1] = make_float2(wy[0], wy[1]);
    o[2] = make_float2(nw[0], nw[1]);
  }
  // the weights are read by bulk copies (the async proxy) of every CTA
  asm volatile("fence.proxy.async.global;" ::: "memory");
  dev::named_barrier(5, nt);  // (also: the shared table is no longer read)
  if (wt == 0) {
    __threadfence();
    atomicAdd(sync_word(p, kSyncP2), 1);
  }
  return true;
}

// The G raw scores of local key k of a range, through L2.
template <int G>
__device__ __forceinline__ void load_raw(const float *rb, int k, float (&v)[G]) {
  if constexpr (G % 4 == 0) {
#pragma unroll
    for (int h = 0; h < G; h += 4) {
      const float4 x = __ldcg(reinterpret_cast<const float4 *>(rb + (size_t)k * G + h));
      v[h] = x.x; v[h + 1] = x.y; v[h + 2] = x.z; v[h + 3] = x.w;
    }
  } else if constexpr (G == 2) {
    const float2 x = __ldcg(reinterpret_cast<const float2 *>(rb + (size_t)k * 2));
    v[0] = x.x; v[1] = x.y;
  } else {
    v[0] = __ldcg(rb + k);
  }
}

// Keys each select thread loads at once (all loads in flight before any use).
// (13 warps: one SM sub-partition holds four of them, so its 16K registers cap a
// thread at 128; the batches stay small enough not to spill.)
template <int G>
struct SwBatch { static constexpr int KB = G <= 2 ? 8 : (G == 4 ? 4 : (G == 8 ? 2 : 1)); };


// Sums NV per-lane doubles over the warp, leaving each total in the lanes of one
// index: at the first log2(NV) butterfly levels a lane keeps half of its values and
// sends the other half, so NV sums cost NV - 1 + (5 - log2 NV) shuffles instead of
// 5 NV.  Returns the index of the total that v[0] holds; the lanes whose low
// 5 - log2(NV) bits are 0 hold each total once.  The order of the additions is fixed.
template <int NV>
__device__ __forceinline__ int warp_sum_scatter(double (&v)[NV], int lane) {
  static_assert(NV >= 1 && NV <= 32 && (NV & (NV - 1)) == 0, "a power of two up to 32");
  int idx = 0;
#pragma unroll
  for (int lev = 0; lev < 5; ++lev) {
    const int o = 16 >> lev;
    const int n = NV >> lev;  // values this lane still holds
    if (n > 1) {
      const bool up = (lane & o) != 0;
#pragma unroll
      for (int i = 0; i < n / 2; ++i) {
        const double send = up ? v[i] : v[i + n / 2];
        const double keep = up ? v[i + n / 2] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
      }
      if (up) idx += n / 2;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
    }
  }
  return idx;
}

// ------------------------------------------------------------------ compaction helpers
constexpr int kCopyPiece = 4096;  // destinations per pass (two int lists in the 32 KB area)
constexpr int kCopyRows = 8;      // row steps per warp in flight

// Loads kept-list entries [q0, q0 + n) into ksh and lists in mv (any order) the
// destinations that move: src != j, and with hazards_only also src < lim (a kept row
// that another destination overwrites); otherwise src < lim guards against a broken
// list (lim = T).  Returns the number of moves (all select threads).
__device__ int gather_moves(SwMisc &ms, const int32_t *klg, int q0, int n, int lim,
                            bool hazards_only, int32_t *ksh, int32_t *mv, int t) {
  if (t == 0) ms.bc[4] = 0;
  for (int j = t; j < n; j += SWT) ksh[j] = __ldcg(klg + q0 + j);
  sw_sync();
  for (int j0 = 0; j0 < n; j0 += SWT) {
    const int j = j0 + t;
    bool m = false;
    if (j < n) {
      const int src = ksh[j];
      m = src != q0 + j && (unsigned)src < (unsigned)lim;
    }
    const uint32_t bal = __ballot_sync(0xffffffffu, m);
    int w0 = 0;
    if ((t & 31) == 0 && bal) w0 = atomicAdd(&ms.bc[4], __popc(bal));
    w0 = __shfl_sync(0xffffffffu, w0, 0);
    if (m) mv[w0 + __popc(bal & ((1u << (t & 31)) - 1u))] = j;
  }
  sw_sync();
  const int nm = ms.bc[4];
  sw_sync();
  return nm;
}

// Copies the nm listed rows: destination q0 + j takes row ksh[j] of the unit (or its
// staged copy).  A row's K and V are 2 * ROWB / 16 vectors of 16 bytes; a warp moves
// RPW rows per step (VPL vectors per lane), kCopyRows steps with every load in flight
// before the first store; the row's first lane moves its position.
template <int ROWB>
__device__ __noinline__ void copy_rows(const PruneParams &p, const int32_t *ksh, const int32_t *mv,
                                       int nm, int q0, int64_t base, int bud, int ug_i,
                                       bool from_stage, bool to_stage, int t) {
  constexpr int VPR = ROWB / 16;                 // vectors per K (or V) row
  constexpr int VT = 2 * VPR;                    // K and V
  constexpr int RPW = VT >= 32 ? 1 : 32 / VT;    // rows per warp step
  constexpr int VPL = VT >= 32 ? VT / 32 : 1;    // vectors per lane per row
  constexpr int LPR = 32 / RPW;                  // lanes per row
  const int lane = t & 31, wid = t >> 5;
  const int rsub = lane / LPR, lr = lane - rsub * LPR;
  const size_t st0 = (size_t)ug_i * p.budget;
  for (int r0 = wid * RPW * kCopyRows; r0 < nm; r0 += NSW * RPW * kCopyRows) {
    uint4 a[kCopyRows][VPL];
    int32_t ps[kCopyRows];
#pragma unroll
    for (int u = 0; u < kCopyRows; ++u) {
      const int r = r0 + u * RPW + rsub;
      if (r < nm) {
        const int j = mv[r], src = ksh[j], d = q0 + j;
        const bool stg = from_stage && src < bud;
        const uint8_t *kr = stg ? p.stage_k + (st0 + d) * ROWB : p.k + (size_t)(base + src) * ROWB;
        const uint8_t *vr = stg ? p.stage_v + (st0 + d) * ROWB : p.v + (size_t)(base + src) * ROWB;
#pragma unroll
        for (int e = 0; e < VPL; ++e) {
          const int x = lr + e * LPR;  // vector of the row's K | V
          a[u][e] = __ldcg(reinterpret_cast<const uint4 *>(x < VPR ? kr : vr) + (x < VPR ? x : x - VPR));
        }
        if (lr == 0) ps[u] = __ldcg(stg ? p.stage_pos + st0 + d : p.pos + base + src);
      }
    }
#pragma unroll
    for (int u = 0; u < kCopyRows; ++u) {
      const int r = r0 + u * RPW + rsub;
      if (r < nm) {
        const int d = q0 + mv[r];
        uint8_t *kr = to_stage ? p.stage_k + (st0 + d) * ROWB : p.k + (size_t)(base + d) * ROWB;
        uint8_t *vr = to_stage ? p.stage_v + (st0 + d) * ROWB : p.v + (size_t)(base + d) * ROWB;
#pragma unroll
        for (int e = 0; e < VPL; ++e) {
          const int x = lr + e * LPR;
          reinterpret_cast<uint4 *>(x < VPR ? kr : vr)[x < VPR ? x : x - VPR] = a[u][e];
        }
        if (lr == 0) {
          if (to_stage) p.stage_pos[st0 + d] = ps[u];
          else p.pos[base + d] = ps[u];
        }
      }
    }
  }
  sw_sync();  // the lists are reused by the next piece
}

}  // namespace

// The select warps: the weight prologue, then, group after group, steps 0-5 and the
// rounds between them (kept out of line so that its registers do not crowd the
// scoring loop's).
// The current group as one CTA's select warps see it (the select steps below are
// kept out of line, so that each gets the registers to itself).
struct GrpCtx {
  int g, slot, u0g, nu, m;
  int64_t cs, ce, r0;
};

// Step 0: the range's chunks and the units they belong to; returns the units met.
template <int D, int G>
__device__ __noinline__ int sel_tables(const PruneParams &p, uint8_t *swb, const GrpCtx x) {
  using S = PruneShape<D, G>;
  constexpr int CH = S::CH;
  constexpr int ROWB = 2 * D;  // bytes of a K or V row
  uint16_t *zks = reinterpret_cast<uint16_t *>(swb + SmemMap::ZKS);
  uint8_t *r1 = swb + SmemMap::R1;
  uint32_t *lh = reinterpret_cast<uint32_t *>(r1);
  unsigned long long *bk = reinterpret_cast<unsigned long long *>(r1);
  int32_t *ksh = reinterpret_cast<int32_t *>(r1);
  int32_t *mv = reinterpret_cast<int32_t *>(r1) + kCopyPiece;
  uint32_t *rh = reinterpret_cast<uint32_t *>(swb + SmemMap::RH);
  int2 *ctab = reinterpret_cast<int2 *>(swb + SmemMap::CTAB);
  UEnt *utab = reinterpret_cast<UEnt *>(swb + SmemMap::UTAB);
  SwMisc &ms = *reinterpret_cast<SwMisc *>(swb + SmemMap::MISC);
  int32_t *seqlen_s = reinterpret_cast<int32_t *>(swb + SmemMap::SEQ);
  const int c = blockIdx.x;
  const int t = threadIdx.x - (NW + 1) * 32;
  const int sw_warp = t >> 5;
  const int g = x.g, slot = x.slot, u0g = x.u0g, m = x.m;
  const int64_t cs = x.cs, ce = x.ce, r0 = x.r0;
  const uint32_t *zr = p.zk + (size_t)slot * p.zk_stride + (size_t)(r0 - cs) * CH;  // range keys
  (void)ROWB; (void)zks; (void)lh; (void)bk; (void)ksh; (void)mv; (void)rh; (void)ctab;
  (void)utab; (void)seqlen_s; (void)sw_warp; (void)g; (void)u0g; (void)m; (void)ce; (void)zr;
    // ------------------------------------------------------------ step 0: tables
    for (int i = t; i < m; i += SWT) {
      int u, jc;
      chunk_unit(p, r0 + i, u, jc);
      ctab[i] = make_int2(u, jc);
    }
    sw_sync();
    // one entry per unit met: chunk i opens one when its unit differs from chunk i - 1's
    int nu = 0;
    for (int i0 = 0; i0 < m; i0 += SWT) {
      const int i = i0 + t;
      const int st = (i < m && (i == 0 || ctab[i].x != ctab[i - 1].x)) ? 1 : 0;
      int tot;
      const int ex = sw_excl_scan(ms, st, t, &tot);
      if (st) {
        utab[nu + ex].u = ctab[i].x;
        utab[nu + ex].lc0 = i;
      }
      nu += tot;
    }
    sw_sync();
    if (t < nu) {
      UEnt &e = utab[t];
      e.nlc = (t + 1 < nu ? utab[t + 1].lc0 : m) - e.lc0;
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
  return nu;
}

// Step 1: the range's sums of s and s^2 per unit and head.
template <int D, int G>
__device__ __noinline__ void sel_sums(const PruneParams &p, uint8_t *swb, const GrpCtx x) {
  using S = PruneShape<D, G>;
  constexpr int CH = S::CH;
  constexpr int ROWB = 2 * D;  // bytes of a K or V row
  uint16_t *zks = reinterpret_cast<uint16_t *>(swb + SmemMap::ZKS);
  uint8_t *r1 = swb + SmemMap::R1;
  uint32_t *lh = reinterpret_cast<uint32_t *>(r1);
  unsigned long long *bk = reinterpret_cast<unsigned long long *>(r1);
  int32_t *ksh = reinterpret_cast<int32_t *>(r1);
  int32_t *mv = reinterpret_cast<int32_t *>(r1) + kCopyPiece;
  uint32_t *rh = reinterpret_cast<uint32_t *>(swb + SmemMap::RH);
  int2 *ctab = reinterpret_cast<int2 *>(swb + SmemMap::CTAB);
  UEnt *utab = reinterpret_cast<UEnt *>(swb + SmemMap::UTAB);
  SwMisc &ms = *reinterpret_cast<SwMisc *>(swb + SmemMap::MISC);
  int32_t *seqlen_s = reinterpret_cast<int32_t *>(swb + SmemMap::SEQ);
  const int c = blockIdx.x;
  const int t = threadIdx.x - (NW + 1) * 32;
  const int sw_warp = t >> 5;
  const int g = x.g, slot = x.slot, u0g = x.u0g, m = x.m;
  const int64_t cs = x.cs, ce = x.ce, r0 = x.r0;
  const uint32_t *zr = p.zk + (size_t)slot * p.zk_stride + (size_t)(r0 - cs) * CH;  // range keys
  (void)ROWB; (void)zks; (void)lh; (void)bk; (void)ksh; (void)mv; (void)rh; (void)ctab;
  (void)utab; (void)seqlen_s; (void)sw_warp; (void)g; (void)u0g; (void)m; (void)ce; (void)zr;
  const int nu = x.nu;
    // ------------------------------------------------------------ step 1: sums of s, s^2
    // the consumers' per-chunk sums over the range's live chunks of each unit, added
    // in a fixed order
    for (int i = 0; i < nu; ++i) {
      const UEnt e = utab[i];
      if (e.mode != kPruneU) continue;
      constexpr int COLS = 2 * G, TPC = SWT / COLS;
      const int col = t / TPC, j = t - col * TPC;
      const int nlive = (e.key1 - e.key0 + CH - 1) / CH;
      const double *cb = p.csum + (((size_t)slot * p.ncta + c) * p.range_chunks + e.lc0) * COLS + col;
      double a = 0.0;
#pragma unroll 4
      for (int lc = j; lc < nlive; lc += TPC) a += __ldcg(cb + (size_t)lc * COLS);
      reinterpret_cast<double *>(rh)[t] = a;  // the radix histogram area is free here
      sw_sync();
      if (t < COLS) {
        double sum = 0.0;
        for (int k = 0; k < TPC; ++k) sum += reinterpret_cast<double *>(rh)[t * TPC + k];
        p.partial[(((size_t)slot * p.ncta + c) * p.ug + (e.u - u0g)) * COLS + t] = sum;
      }
      sw_sync();
    }
}

// Step 2: z keys and the units' histograms.
template <int D, int G>
__device__ __noinline__ void sel_zkeys(const PruneParams &p, uint8_t *swb, const GrpCtx x) {
  using S = PruneShape<D, G>;
  constexpr int CH = S::CH;
  constexpr int ROWB = 2 * D;  // bytes of a K or V row
  uint16_t *zks = reinterpret_cast<uint16_t *>(swb + SmemMap::ZKS);
  uint8_t *r1 = swb + SmemMap::R1;
  uint32_t *lh = reinterpret_cast<uint32_t *>(r1);
  unsigned long long *bk = reinterpret_cast<unsigned long long *>(r1);
  int32_t *ksh = reinterpret_cast<int32_t *>(r1);
  int32_t *mv = reinterpret_cast<int32_t *>(r1) + kCopyPiece;
  uint32_t *rh = reinterpret_cast<uint32_t *>(swb + SmemMap::RH);
  int2 *ctab = reinterpret_cast<int2 *>(swb + SmemMap::CTAB);
  UEnt *utab = reinterpret_cast<UEnt *>(swb + SmemMap::UTAB);
  SwMisc &ms = *reinterpret_cast<SwMisc *>(swb + SmemMap::MISC);
  int32_t *seqlen_s = reinterpret_cast<int32_t *>(swb + SmemMap::SEQ);
  const int c = blockIdx.x;
  const int t = threadIdx.x - (NW + 1) * 32;
  const int sw_warp = t >> 5;
  const int g = x.g, slot = x.slot, u0g = x.u0g, m = x.m;
  const int64_t cs = x.cs, ce = x.ce, r0 = x.r0;
  const uint32_t *zr = p.zk + (size_t)slot * p.zk_stride + (size_t)(r0 - cs) * CH;  // range keys
  (void)ROWB; (void)zks; (void)lh; (void)bk; (void)ksh; (void)mv; (void)rh; (void)ctab;
  (void)utab; (void)seqlen_s; (void)sw_warp; (void)g; (void)u0g; (void)m; (void)ce; (void)zr;
  const int nu = x.nu;
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
          // (every non-empty range between the first and the last covering CTA's meets the unit)
          if (range_start(p, cs, ce, cc) == range_start(p, cs, ce, cc + 1)) continue;
          a += __ldcg(p.partial + (((size_t)slot * p.ncta + cc) * p.ug + (e.u - u0g)) * (2 * G) + col);
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
      constexpr int KB = SwBatch<G>::KB;
      for (int k0 = t; k0 < nk; k0 += SWT * KB) {
        float v[KB][G];
#pragma unroll
        for (int j = 0; j < KB; ++j)
          if (k0 + j * SWT < nk) load_raw<G>(rb, k0 + j * SWT, v[j]);
#pragma unroll
        for (int j = 0; j < KB; ++j) {
          const int k = k0 + j * SWT;
          if (k < nk) {
            float zf = -3.0e38f;
#pragma unroll
            for (int h = 0; h < G; ++h) zf = fmaxf(zf, ((v[j][h] - mh[h]) - ml[h]) * is[h]);
            const uint32_t key = dev::order_key(zf);
            const uint32_t bn = z_bin(key);
            zks[li0 + k] = (uint16_t)bn;
            zg[k] = key;
            atomicAdd(&lh[bn], 1u);
          }
        }
      }
      sw_sync();
      uint32_t *hg = p.hist + ((size_t)slot * kPruneMaxGroupUnits + (e.u - u0g)) * kPruneHistBins;
      for (int bn = t; bn < kPruneHistBins; bn += SWT) {
        const uint32_t v = lh[bn];
        if (v) atomicAdd(&hg[bn], v);
      }
      sw_sync();
    }
}

// Step 3: threshold bins, and the keys in them published.
template <int D, int G>
__device__ __noinline__ void sel_bins(const PruneParams &p, uint8_t *swb, const GrpCtx x) {
  using S = PruneShape<D, G>;
  constexpr int CH = S::CH;
  constexpr int ROWB = 2 * D;  // bytes of a K or V row
  uint16_t *zks = reinterpret_cast<uint16_t *>(swb + SmemMap::ZKS);
  uint8_t *r1 = swb + SmemMap::R1;
  uint32_t *lh = reinterpret_cast<uint32_t *>(r1);
  unsigned long long *bk = reinterpret_cast<unsigned long long *>(r1);
  int32_t *ksh = reinterpret_cast<int32_t *>(r1);
  int32_t *mv = reinterpret_cast<int32_t *>(r1) + kCopyPiece;
  uint32_t *rh = reinterpret_cast<uint32_t *>(swb + SmemMap::RH);
  int2 *ctab = reinterpret_cast<int2 *>(swb + SmemMap::CTAB);
  UEnt *utab = reinterpret_cast<UEnt *>(swb + SmemMap::UTAB);
  SwMisc &ms = *reinterpret_cast<SwMisc *>(swb + SmemMap::MISC);
  int32_t *seqlen_s = reinterpret_cast<int32_t *>(swb + SmemMap::SEQ);
  const int c = blockIdx.x;
  const int t = threadIdx.x - (NW + 1) * 32;
  const int sw_warp = t >> 5;
  const int g = x.g, slot = x.slot, u0g = x.u0g, m = x.m;
  const int64_t cs = x.cs, ce = x.ce, r0 = x.r0;
  const uint32_t *zr = p.zk + (size_t)slot * p.zk_stride + (size_t)(r0 - cs) * CH;  // range keys
  (void)ROWB; (void)zks; (void)lh; (void)bk; (void)ksh; (void)mv; (void)rh; (void)ctab;
  (void)utab; (void)seqlen_s; (void)sw_warp; (void)g; (void)u0g; (void)m; (void)ce; (void)zr;
  const int nu = x.nu;
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
          const uint32_t bn = zks[li0 + k];
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
          if (zks[li0 + k] == (uint32_t)bstar) {
            if (w < kPruneBucketMax) bl[w] = composite(__ldcg(zr + li0 + k), e.key0 + k);
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
}

// Step 4: exact thresholds and the kept lists.
template <int D, int G>
__device__ __noinline__ void sel_emit(const PruneParams &p, uint8_t *swb, const GrpCtx x) {
  using S = PruneShape<D, G>;
  constexpr int CH = S::CH;
  constexpr int ROWB = 2 * D;  // bytes of a K or V row
  uint16_t *zks = reinterpret_cast<uint16_t *>(swb + SmemMap::ZKS);
  uint8_t *r1 = swb + SmemMap::R1;
  uint32_t *lh = reinterpret_cast<uint32_t *>(r1);
  unsigned long long *bk = reinterpret_cast<unsigned long long *>(r1);
  int32_t *ksh = reinterpret_cast<int32_t *>(r1);
  int32_t *mv = reinterpret_cast<int32_t *>(r1) + kCopyPiece;
  uint32_t *rh = reinterpret_cast<uint32_t *>(swb + SmemMap::RH);
  int2 *ctab = reinterpret_cast<int2 *>(swb + SmemMap::CTAB);
  UEnt *utab = reinterpret_cast<UEnt *>(swb + SmemMap::UTAB);
  SwMisc &ms = *reinterpret_cast<SwMisc *>(swb + SmemMap::MISC);
  int32_t *seqlen_s = reinterpret_cast<int32_t *>(swb + SmemMap::SEQ);
  const int c = blockIdx.x;
  const int t = threadIdx.x - (NW + 1) * 32;
  const int sw_warp = t >> 5;
  const int g = x.g, slot = x.slot, u0g = x.u0g, m = x.m;
  const int64_t cs = x.cs, ce = x.ce, r0 = x.r0;
  const uint32_t *zr = p.zk + (size_t)slot * p.zk_stride + (size_t)(r0 - cs) * CH;  // range keys
  (void)ROWB; (void)zks; (void)lh; (void)bk; (void)ksh; (void)mv; (void)rh; (void)ctab;
  (void)utab; (void)seqlen_s; (void)sw_warp; (void)g; (void)u0g; (void)m; (void)ce; (void)zr;
  const int nu = x.nu;
    // this group's histograms are read by every CTA by now: clear this CTA's share
    {
      const int64_t words = (int64_t)min(p.ug, p.units - u0g) * kPruneHistBins;
      const int64_t w0 = words * c / p.ncta, w1 = words * (c + 1) / p.ncta;
      uint32_t *hb = p.hist + (size_t)slot * kPruneMaxGroupUnits * kPruneHistBins;
      for (int64_t k = w0 + t; k < w1; k += SWT) hb[k] = 0u;
    }
    // ------------------------------------------------------------ step 4: emit
    for (int i = 0; i < nu; ++i) {
      const UEnt e = utab[i];
      if (e.mode != kPruneU) continue;
      const int ug_i = e.u - u0g;
      const int nk = e.key1 - e.key0, li0 = e.lc0 * CH;
      const int bstar = e.bstar;
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
      // kept slots in slot order into the unit's kept list (by destination index):
      // thread t owns a contiguous run of the range's keys, read as 16-byte groups of
      // bins; the unit's range that holds slot bud - 1 also publishes how many kept
      // slots lie below bud (the rows the compaction must move out of place first)
      {
        const int RUN = ((nk + SWT - 1) / SWT + 7) & ~7;
        const int k0 = min(nk, t * RUN), k1 = min(nk, k0 + RUN);
        const int lim = e.bud - e.key0;
        const uint4 *zv = reinterpret_cast<const uint4 *>(zks + li0);
        // a key is kept if its bin is above the threshold bin, or in it and not below thr
        auto kept = [&](int k, uint32_t bn) {
          return bn > (uint32_t)bstar ||
                 (bn == (uint32_t)bstar && composite(__ldcg(zr + li0 + k), e.key0 + k) >= thr);
        };
        int cnt = 0, cbel = 0;
        for (int k = k0; k < k1; k += 8) {
          const uint4 q = zv[k >> 3];
          const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int kk = k + i;
            const uint32_t bn = (w4[i >> 1] >> (16 * (i & 1))) & 0xffffu;
            if (kk < k1 && kept(kk, bn)) {
              ++cnt;
              cbel += kk < lim;
            }
          }
        }
        int tot, totb;
        const int off = sw_excl_scan(ms, cnt, t, &tot);
        sw_excl_scan(ms, cbel, t, &totb);
        if (t == 0) {
          if (tot != kc) dev::set_error(p.err, TRIA_DEVERR_SELECTION);
          if (e.key0 <= e.bud - 1 && e.bud - 1 < e.key1)
            p.khaz[slot * kPruneMaxGroupUnits + ug_i] = oc + totb;
        }
        int32_t *so = p.sel_out ? p.sel_out + (int64_t)e.u * p.budget : nullptr;
        int32_t *klg = p.klist + (size_t)ug_i * p.budget;
        int o = oc + off;
        for (int k = k0; k < k1; k += 8) {
          const uint4 q = zv[k >> 3];
          const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int kk = k + i;
            const uint32_t bn = (w4[i >> 1] >> (16 * (i & 1))) & 0xffffu;
            if (kk < k1 && kept(kk, bn)) {
              if (o < oc + kc) {
                klg[o] = e.key0 + kk;
                if (so) so[o] = e.key0 + kk;
              }
              ++o;
            }
          }
        }
      }
      sw_sync();
    }
}

// Step 5a: the kept rows that another destination overwrites, copied out of place.
template <int D, int G>
__device__ __noinline__ void sel_stage(const PruneParams &p, uint8_t *swb, const GrpCtx x) {
  using S = PruneShape<D, G>;
  constexpr int CH = S::CH;
  constexpr int ROWB = 2 * D;  // bytes of a K or V row
  uint16_t *zks = reinterpret_cast<uint16_t *>(swb + SmemMap::ZKS);
  uint8_t *r1 = swb + SmemMap::R1;
  uint32_t *lh = reinterpret_cast<uint32_t *>(r1);
  unsigned long long *bk = reinterpret_cast<unsigned long long *>(r1);
  int32_t *ksh = reinterpret_cast<int32_t *>(r1);
  int32_t *mv = reinterpret_cast<int32_t *>(r1) + kCopyPiece;
  uint32_t *rh = reinterpret_cast<uint32_t *>(swb + SmemMap::RH);
  int2 *ctab = reinterpret_cast<int2 *>(swb + SmemMap::CTAB);
  UEnt *utab = reinterpret_cast<UEnt *>(swb + SmemMap::UTAB);
  SwMisc &ms = *reinterpret_cast<SwMisc *>(swb + SmemMap::MISC);
  int32_t *seqlen_s = reinterpret_cast<int32_t *>(swb + SmemMap::SEQ);
  const int c = blockIdx.x;
  const int t = threadIdx.x - (NW + 1) * 32;
  const int sw_warp = t >> 5;
  const int g = x.g, slot = x.slot, u0g = x.u0g, m = x.m;
  const int64_t cs = x.cs, ce = x.ce, r0 = x.r0;
  const uint32_t *zr = p.zk + (size_t)slot * p.zk_stride + (size_t)(r0 - cs) * CH;  // range keys
  (void)ROWB; (void)zks; (void)lh; (void)bk; (void)ksh; (void)mv; (void)rh; (void)ctab;
  (void)utab; (void)seqlen_s; (void)sw_warp; (void)g; (void)u0g; (void)m; (void)ce; (void)zr;
  const int nu = x.nu;
    // ------------------------------------------------------------ step 5: compaction
    // Every unit's kept list (by destination) is complete.  The CTAs that meet the
    // unit split its destinations [0, bud) in proportion to their key ranges, which
    // partition [0, T) (kept keys cluster in slot ranges, so a split by source would
    // leave some CTAs far more rows than others).  A kept row whose slot lies inside
    // [0, bud) may be overwritten by another destination: those rows are first copied
    // out of place (5a), and after one more round every destination is written (5b),
    // from the staged copy or straight from its slot (slots >= bud are never written).
    // The kept slots below bud are the first Kh destinations (Kh from the range that
    // holds slot bud - 1), which 5a splits evenly too.
    // Both passes put the share's list in shared memory, gather the rows to move, and
    // copy them with kCopyRows rows per warp in flight before the stores.
    for (int i = 0; i < nu; ++i) {  // 5a
      const UEnt e = utab[i];
      if (e.mode != kPruneU) continue;
      const int ug_i = e.u - u0g;
      // the kept slots below bud are the first Kh destinations: split those evenly
      const int Kh = __ldcg(p.khaz + slot * kPruneMaxGroupUnits + ug_i);
      if (Kh < 0 || Kh > e.bud) {
        if (t == 0) dev::set_error(p.err, TRIA_DEVERR_SELECTION);
        continue;
      }
      const int d0 = (int)((int64_t)Kh * e.key0 / e.T), d1 = (int)((int64_t)Kh * e.key1 / e.T);
      const int row = e.u / p.B, b = e.u - row * p.B;
      const int64_t base = (int64_t)row * p.cap + p.seg_start[b];
      const int32_t *klg = p.klist + (size_t)ug_i * p.budget;
      for (int q0 = d0; q0 < d1; q0 += kCopyPiece) {
        const int n = min(kCopyPiece, d1 - q0);
        int nm = gather_moves(ms, klg, q0, n, e.bud, /*hazards_only=*/true, ksh, mv, t);
        copy_rows<ROWB>(p, ksh, mv, nm, q0, base, e.bud, ug_i, /*from_stage=*/false,
                        /*to_stage=*/true, t);
      }
    }
}

// Step 5b: every destination written, and the units' lengths.
template <int D, int G>
__device__ __noinline__ void sel_write(const PruneParams &p, uint8_t *swb, const GrpCtx x) {
  using S = PruneShape<D, G>;
  constexpr int CH = S::CH;
  constexpr int ROWB = 2 * D;  // bytes of a K or V row
  uint16_t *zks = reinterpret_cast<uint16_t *>(swb + SmemMap::ZKS);
  uint8_t *r1 = swb + SmemMap::R1;
  uint32_t *lh = reinterpret_cast<uint32_t *>(r1);
  unsigned long long *bk = reinterpret_cast<unsigned long long *>(r1);
  int32_t *ksh = reinterpret_cast<int32_t *>(r1);
  int32_t *mv = reinterpret_cast<int32_t *>(r1) + kCopyPiece;
  uint32_t *rh = reinterpret_cast<uint32_t *>(swb + SmemMap::RH);
  int2 *ctab = reinterpret_cast<int2 *>(swb + SmemMap::CTAB);
  UEnt *utab = reinterpret_cast<UEnt *>(swb + SmemMap::UTAB);
  SwMisc &ms = *reinterpret_cast<SwMisc *>(swb + SmemMap::MISC);
  int32_t *seqlen_s = reinterpret_cast<int32_t *>(swb + SmemMap::SEQ);
  const int c = blockIdx.x;
  const int t = threadIdx.x - (NW + 1) * 32;
  const int sw_warp = t >> 5;
  const int g = x.g, slot = x.slot, u0g = x.u0g, m = x.m;
  const int64_t cs = x.cs, ce = x.ce, r0 = x.r0;
  const uint32_t *zr = p.zk + (size_t)slot * p.zk_stride + (size_t)(r0 - cs) * CH;  // range keys
  (void)ROWB; (void)zks; (void)lh; (void)bk; (void)ksh; (void)mv; (void)rh; (void)ctab;
  (void)utab; (void)seqlen_s; (void)sw_warp; (void)g; (void)u0g; (void)m; (void)ce; (void)zr;
  const int nu = x.nu;
    auto share = [&](const UEnt &e, int &d0, int &d1) {
      d0 = (int)((int64_t)e.bud * e.key0 / e.T);
      d1 = (int)((int64_t)e.bud * e.key1 / e.T);
    };
    for (int i = 0; i < nu; ++i) {  // 5b
      const UEnt e = utab[i];
      const int row = e.u / p.B, b = e.u - row * p.B;
      const int ug_i = e.u - u0g;
      if (e.mode == kPruneU) {
        int d0, d1;
        share(e, d0, d1);
        const int64_t base = (int64_t)row * p.cap + p.seg_start[b];
        const int32_t *klg = p.klist + (size_t)ug_i * p.budget;
        for (int q0 = d0; q0 < d1; q0 += kCopyPiece) {
          const int n = min(kCopyPiece, d1 - q0);
          int nm = gather_moves(ms, klg, q0, n, e.T, /*hazards_only=*/false, ksh, mv, t);
          copy_rows<ROWB>(p, ksh, mv, nm, q0, base, e.bud, ug_i, /*from_stage=*/true,
                          /*to_stage=*/false, t);
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
}

// The select warps: the weight prologue, then, group after group, steps 0-5 and the
// grid rounds between them.
template <int D, int G>
__device__ __noinline__ void select_role(const PruneParams &p, uint8_t *swb, uint64_t *gdone,
                                         uint64_t *rawfree, int *pro_ok_s) {
  uint8_t *r1 = swb + SmemMap::R1;
  SwMisc &ms = *reinterpret_cast<SwMisc *>(swb + SmemMap::MISC);
  int32_t *seqlen_s = reinterpret_cast<int32_t *>(swb + SmemMap::SEQ);     // [B]
  const int c = blockIdx.x;
  const int t = threadIdx.x - (NW + 1) * 32;
  bool alive = prologue_weights<D, G>(p, c, NW * 32 + t, (NW + NSW) * 32, pro_ok_s,
                                     reinterpret_cast<double2 *>(r1));
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
  if (!alive && t == 0) raise_abort(p);
  for (int g = 0; g < p.ngroups && alive; ++g) {
    const int slot = g & 1;
    int okg = 1;
    if (t == 0) okg = wait_bar(p, &gdone[slot], (uint32_t)(g >> 1) & 1);
    if (t == 0) ms.ok = okg;
    sw_sync();
    if (!ms.ok) { if (t == 0) raise_abort(p); alive = false; break; }
    GrpCtx x;
    x.g = g;
    x.slot = slot;
    x.u0g = g * p.ug;
    group_chunks(p, g, x.cs, x.ce);
    x.r0 = range_start(p, x.cs, x.ce, c);
    x.m = (int)(range_start(p, x.cs, x.ce, c + 1) - x.r0);
    x.nu = 0;
    x.nu = sel_tables<D, G>(p, swb, x);
    sel_sums<D, G>(p, swb, x);
    if (!grid_round(p, ms, kSyncA, g, t)) { alive = false; break; }
    sel_zkeys<D, G>(p, swb, x);
    if (t == 0) dev::mbar_arrive(&rawfree[slot]);  // the consumers may reuse this raw slot
    if (!grid_round(p, ms, kSyncB, g, t)) { alive = false; break; }
    sel_bins<D, G>(p, swb, x);
    if (!grid_round(p, ms, kSyncC, g, t)) { alive = false; break; }
    sel_emit<D, G>(p, swb, x);
    if (!grid_round(p, ms, kSyncD, g, t)) { alive = false; break; }
    sel_stage<D, G>(p, swb, x);
    if (!grid_round(p, ms, kSyncE, g, t)) { alive = false; break; }
    sel_write<D, G>(p, swb, x);
    sw_sync();
  }
  // ------------------------------------------------------------------ leave
  sw_sync();
  if (t == 0) {
    __threadfence();
    const int32_t was = atomicAdd(sync_word(p, kSyncExit), 1);
    if (was == p.ncta - 1) {
      // the last CTA out: every other CTA is past its last synchronisation
      __threadfence();
      const bool aborted = ld_volatile(sync_word(p, kSyncAbort)) != 0;
      if (aborted) {
        // a group may have stopped half-way: clear what must be zero at rest
        for (int k = 0; k < 2 * kPruneMaxGroupUnits * kPruneHistBins; ++k) p.hist[k] = 0u;
        for (int k = 0; k < 2 * kPruneMaxGroupUnits; ++k) p.bcount[k] = 0;
      }
      for (int k = 0; k < kSyncWords; ++k) *sync_word(p, k) = 0;
      __threadfence();
    }
  }
}

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
  uint8_t *r1 = swb + SmemMap::R1;  // the local offset table of the weight prologue
  int32_t *seqlen_s = reinterpret_cast<int32_t *>(swb + SmemMap::SEQ);     // [B]
  int4 *tab = reinterpret_cast<int4 *>(swb + SmemMap::TAB);                // [32]
  int32_t *taby = reinterpret_cast<int32_t *>(swb + SmemMap::TABY);        // [32]
  int4 *desc = reinterpret_cast<int4 *>(swb + SmemMap::DESC);              // [NSLOT]
  uint64_t *full = reinterpret_cast<uint64_t *>(desc + NSLOT);
  uint64_t *empty = full + NSLOT;
  uint64_t *wfull = empty + NSLOT;     // [2]
  uint64_t *gdone = wfull + 2;         // [2] consumer warps finished a group
  uint64_t *rawfree = gdone + 2;       // [2] select warps done with a group's raw scores

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x;
  __shared__ int pro_ok;
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
    // keys are read once here: they leave the L2 first, ahead of the group scratch
    const uint64_t kpol = dev::l2_evict_first();
    uint32_t q = 0;
    bool failed = false;
    int cur_unit = -1, wslot = 1;
    bool wready = false;
    uint32_t wuse[2] = {0, 0};
    int64_t wlast[2] = {-1, -1};
    // Weight fills wait for the prologue (every CTA's share of the weights written);
    // until then they are held back, so that the key chunks stream in meanwhile.
    int npend = 0;
    int pend_slot[2] = {0, 0}, pend_unit[2] = {0, 0};
    auto flush = [&]() -> bool {
      if (npend == 0) return true;
      int okf = 1;
      if (!wready) {
        if (lane == 0) {
          okf = poll_counter(p, kSyncP2, p.ncta);
          asm volatile("fence.proxy.async.global;" ::: "memory");  // bulk copies read them
        }
        if (!__shfl_sync(0xffffffffu, okf, 0)) return false;
        wready = true;
      }
      if (lane == 0)
        for (int i = 0; i < npend; ++i) {
          dev::mbar_arrive_expect_tx(&wfull[pend_slot[i]], WB);
          dev::bulk_g2s(wring + pend_slot[i] * WB,
                        reinterpret_cast<const uint8_t *>(p.w) + (size_t)pend_unit[i] * WB, WB,
                        &wfull[pend_slot[i]]);
        }
      npend = 0;
      return true;
    };
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
              if (!flush()) { failed = true; break; }  // the chunks awaited below need theirs
              if (lane == 0)
                for (int64_t pp = (int64_t)q - NSLOT + 1; pp <= wlast[j] && ok; ++pp)
                  if (pp >= 0) ok = wait_bar(p, &empty[pp % NSLOT], (uint32_t)(pp / NSLOT) & 1);
              if (!__shfl_sync(0xffffffffu, ok, 0)) { failed = true; break; }
            }
            pend_slot[npend] = j;
            pend_unit[npend] = e.x;
            ++npend;
            if (wready && !flush()) { failed = true; break; }
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
              dev::tma_load_2d_hint(ring + (size_t)s * CB + bx * S::BOXB, &p.tmap, bx * 64, taby[i],
                                    &full[s], kpol);
          }
          ++q;
          // the ring is full: the producer waits for slots anyway, so wait for the weights
          if (q >= (uint32_t)NSLOT && npend && !flush()) { failed = true; break; }
        }
        __syncwarp();  // the table is read before it is rewritten
      }
    }
    if (!failed && !flush()) failed = true;
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
      if (!warm) {
        // per-chunk sums of s and s^2 per head (float64, fixed order), from which the
        // select warps form each unit's mean and variance
        constexpr int HG = G < 4 ? G : 4;  // heads per warp reduction
        constexpr int NV = 2 * HG;
        double *cs = p.csum + (((size_t)(g & 1) * p.ncta + c) * p.range_chunks + lchunk) * (2 * G);
#pragma unroll
        for (int h0 = 0; h0 < G; h0 += HG) {
          double v[NV];
#pragma unroll
          for (int h = 0; h < HG; ++h) {
            v[2 * h] = 0.0;
            v[2 * h + 1] = 0.0;
#pragma unroll
            for (int k = 0; k < KPT; ++k)
              if (lane + 32 * k < n) {
                const double x = (double)out[k][h0 + h];
                v[2 * h] += x;
                v[2 * h + 1] = fma(x, x, v[2 * h + 1]);
              }
          }
          const int idx = warp_sum_scatter<NV>(v, lane);
          if ((lane & (32 / NV - 1)) == 0) cs[2 * h0 + idx] = v[0];
        }
      }
      if (warm) {
        warm = false;
        dev::named_barrier_arrive(2, (NW + 1) * 32);  // the producer may start the stream
        if (!prologue_weights<D, G>(p, c, threadIdx.x, (NW + NSW) * 32, &pro_ok,
                                    reinterpret_cast<double2 *>(r1))) {
          failed = true;
          break;
        }
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
  select_role<D, G>(p, swb, gdone, rawfree, &pro_ok);
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
  // a CTA's share of a group: at most kPruneRangeKeys keys, and at most 32768 / G so
  // that the raw scores of two groups in flight (2 x ncta x share x G floats, about
  // 39 MB) stay small next to the L2
  const int range_cap = std::min(kPruneRangeKeys, 32768 / std::max(G, 1));
  const int64_t cap_chunks = (int64_t)pl.ncta * (range_cap / CH);
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
  // groups as large as the ranges allow (at most kPruneMaxGroupUnits units): a group's
  // selection is a chain of grid rounds whose latency hardly grows with its size, and
  // the next group's scoring hides it
  int64_t ug = std::max<int64_t>(1, std::min<int64_t>(units, kPruneMaxGroupUnits));
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
