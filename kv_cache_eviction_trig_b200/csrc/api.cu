// Host side of the C ABI declared in include/tria.h: argument validation,
// workspace layout and kernel launches.  No allocation, no host
// synchronisation (except tria_get_device_error), no global mutable state
// beyond per-device launch-configuration caches.
#include <cmath>
#include <cstring>
#include <vector>

#include "attention.cuh"
#include "tria_internal.cuh"

namespace tria {

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

ScoreGrid score_grid(const tria_config &cfg, const int64_t *seq_start) {
  ScoreGrid g{};
  const int G = cfg.n_kv_heads > 0 ? cfg.n_q_heads / cfg.n_kv_heads : 1;
  g.chunk_keys = score_chunk_keys(cfg.head_dim, G);
  const int ch = g.chunk_keys > 0 ? g.chunk_keys : 1;
  int64_t acc = 0, most = 0;
  for (int b = 0; b < cfg.batch; ++b) {
    const int64_t n = (seq_start[b + 1] - seq_start[b] + ch - 1) / ch;
    acc += n;
    if (n > most) most = n;
  }
  g.chunks_per_row = (int)acc;
  g.total = (int64_t)cfg.num_layers * cfg.n_kv_heads * acc;
  if (g.total == 0) return g;
  int64_t grid = device_sm_count();
  if (grid > g.total) grid = g.total;
  g.chunks_per_cta = (int)((g.total + grid - 1) / grid);
  g.grid = (int)((g.total + g.chunks_per_cta - 1) / g.chunks_per_cta);
  g.max_slots = (int)((most + g.chunks_per_cta - 1) / g.chunks_per_cta + 1);
  return g;
}

WsLayout ws_layout(const tria_config &cfg, const int64_t *seq_start, int64_t cap) {
  static_assert(kPruneMaxGroupUnits == 32 && kPruneHistBins == 4096, "prefix layout");
  static_assert(kWsBcount + 2 * kPruneMaxGroupUnits * 4 <= kWsHist, "prefix layout");
  WsLayout w{};
  const size_t F = (size_t)cfg.head_dim / 2;
  const size_t units = (size_t)cfg.num_layers * cfg.n_kv_heads * cfg.batch;
  const size_t G = cfg.n_kv_heads > 0 ? (size_t)(cfg.n_q_heads / cfg.n_kv_heads) : 1;
  w.max_slots = score_grid(cfg, seq_start).max_slots;
  w.err = kWsErr;
  size_t o = kWsPrefix;
  w.seqlen = o;   o = align_up(o + 4ull * (units > (size_t)cfg.batch ? units : cfg.batch), 256);
  w.w = o;        o = align_up(o + 4ull * units * (F / 2) * G * 6, 256);
  w.raw = o;      o = align_up(o + 4ull * cfg.num_layers * cfg.n_q_heads * (size_t)cap, 256);
  w.sel = o;      o = align_up(o + 4ull * units * cfg.budget, 256);
  w.partials = o;
  o = align_up(o + 16ull * units * (size_t)w.max_slots * kScoreMaxWarps * G, 256);
  size_t end = o;
  const PrunePlan pl = (cfg.flags & TRIA_FUSED_PRUNE) ? prune_plan(cfg, seq_start) : PrunePlan{};
  w.fused = pl.ok;
  if (pl.ok) {
    const size_t nc = (size_t)pl.ncta, ug = (size_t)pl.ug, rowb = 2ull * cfg.head_dim;
    o = kWsPrefix;
    w.f_ea = o;        o = align_up(o + 16ull * cfg.batch * F, 256);
    w.f_w = o;         o = align_up(o + 4ull * units * (F / 2) * G * 6, 256);
    w.f_raw = o;       o = align_up(o + 2ull * nc * pl.range_keys * G * 4, 256);
    w.f_csum = o;      o = align_up(o + 2ull * nc * (pl.range_keys / pl.chunk_keys) * G * 16, 256);
    w.f_partial = o;   o = align_up(o + 2ull * nc * ug * G * 16, 256);
    w.f_zk = o;        o = align_up(o + 2ull * (size_t)pl.zk_stride * 4, 256);
    w.f_bucket = o;    o = align_up(o + 2ull * ug * kPruneBucketMax * 8, 256);
    w.f_above = o;     o = align_up(o + 2ull * ug * nc * 4, 256);
    w.f_thr = o;       o = align_up(o + 2ull * ug * 8, 256);
    w.f_kcount = o;    o = align_up(o + 2ull * ug * nc * 4, 256);
    w.f_klist = o;     o = align_up(o + ug * (size_t)cfg.budget * 4, 256);
    w.f_khaz = o;      o = align_up(o + 2ull * kPruneMaxGroupUnits * 4, 256);
    w.f_stage_k = o;   o = align_up(o + ug * (size_t)cfg.budget * rowb, 256);
    w.f_stage_v = o;   o = align_up(o + ug * (size_t)cfg.budget * rowb, 256);
    w.f_stage_pos = o; o = align_up(o + ug * (size_t)cfg.budget * 4, 256);
    if (o > end) end = o;
  }
  w.total = end;
  return w;
}

int device_sm_count() {
  static int cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cache[dev]) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = n > 0 ? n : 148;
  }
  return cache[dev];
}

}  // namespace tria

using namespace tria;

namespace {

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

tria_status check_config(const tria_config *cfg, bool scoring) {
  if (!cfg) return TRIA_ERR_INVALID_ARG;
  if (cfg->num_layers < 1 || cfg->batch < 1 || cfg->n_kv_heads < 1 || cfg->n_q_heads < 1)
    return TRIA_ERR_INVALID_ARG;
  if (cfg->batch > TRIA_MAX_BATCH) return TRIA_ERR_UNSUPPORTED;
  if (cfg->n_q_heads % cfg->n_kv_heads != 0) return TRIA_ERR_INVALID_ARG;
  if (cfg->head_dim < 2 || cfg->head_dim % 2 != 0) return TRIA_ERR_INVALID_ARG;
  if (cfg->rope_layout != TRIA_ROPE_HALF_SPLIT && cfg->rope_layout != TRIA_ROPE_INTERLEAVED)
    return TRIA_ERR_INVALID_ARG;
  if (cfg->budget < 1) return TRIA_ERR_INVALID_ARG;
  if (cfg->budget > TRIA_MAX_SEGMENT) return TRIA_ERR_UNSUPPORTED;
  if (cfg->n_q_heads / cfg->n_kv_heads > 16) return TRIA_ERR_UNSUPPORTED;
  if (cfg->prune_window < 0) return TRIA_ERR_INVALID_ARG;
  if (scoring) {
    if (!(cfg->rope_theta > 1.0) || !std::isfinite(cfg->rope_theta)) return TRIA_ERR_INVALID_ARG;
    if (!cfg->offsets || cfg->n_offsets < 1) return TRIA_ERR_INVALID_ARG;
    if (cfg->n_offsets > TRIA_MAX_OFFSETS) return TRIA_ERR_UNSUPPORTED;
    for (int i = 0; i < cfg->n_offsets; ++i)
      if (cfg->offsets[i] < 1) return TRIA_ERR_INVALID_ARG;
    if (cfg->flags & ~(TRIA_NO_TRIG | TRIA_NO_CONC_WEIGHT | TRIA_FUSED_PRUNE))
      return TRIA_ERR_INVALID_ARG;
    if (!score_supported(cfg->head_dim, cfg->n_q_heads / cfg->n_kv_heads, cfg->rope_layout))
      return TRIA_ERR_UNSUPPORTED;
  } else {
    if (cfg->head_dim % 8 != 0) return TRIA_ERR_UNSUPPORTED;
  }
  return TRIA_OK;
}

tria_status check_cache(const tria_config *cfg, const tria_cache *c, bool need_kv) {
  if (!c) return TRIA_ERR_INVALID_ARG;
  if (!c->seq_start || c->cap_total < 0) return TRIA_ERR_INVALID_ARG;
  // lengths per sequence, or per unit (then seq_len may be null); head budgets need the latter
  if (!c->seq_len && !c->unit_len) return TRIA_ERR_INVALID_ARG;
  if (c->unit_len && !aligned(c->unit_len, 4)) return TRIA_ERR_INVALID_ARG;
  if (cfg->head_budgets && (!c->unit_len || !aligned(cfg->head_budgets, 4)))
    return TRIA_ERR_INVALID_ARG;
  if (need_kv) {
    if (!c->k || !c->v || !c->pos) return TRIA_ERR_INVALID_ARG;
    if (!aligned(c->k, 16) || !aligned(c->v, 16) || !aligned(c->pos, 16))
      return TRIA_ERR_INVALID_ARG;
  }
  if (c->seq_start[0] < 0) return TRIA_ERR_INVALID_ARG;
  for (int b = 0; b < cfg->batch; ++b) {
    const int64_t a = c->seq_start[b], e = c->seq_start[b + 1];
    if (e < a) return TRIA_ERR_INVALID_ARG;
    if (e - a > TRIA_MAX_SEGMENT) return TRIA_ERR_UNSUPPORTED;
  }
  if (c->seq_start[cfg->batch] > c->cap_total) return TRIA_ERR_INVALID_ARG;
  return TRIA_OK;
}

// The score kernel addresses keys by 32-bit tensor coordinates.
tria_status check_key_rows(const tria_config *cfg, const tria_cache *c) {
  const int64_t rows = (int64_t)cfg->num_layers * cfg->n_kv_heads * c->cap_total;
  return rows <= INT32_MAX ? TRIA_OK : TRIA_ERR_UNSUPPORTED;
}

tria_status check_stats(const tria_stats *s) {
  if (!s || !s->centre || !s->mean_norm || !s->mrl) return TRIA_ERR_INVALID_ARG;
  if (!aligned(s->centre, 8) || !aligned(s->mean_norm, 4) || !aligned(s->mrl, 4))
    return TRIA_ERR_INVALID_ARG;
  return TRIA_OK;
}

tria_status check_ws(const tria_config *cfg, const tria_cache *c, void *ws, size_t bytes) {
  if (!ws || !aligned(ws, 256)) return TRIA_ERR_WORKSPACE;
  if (bytes < ws_layout(*cfg, c->seq_start, c->cap_total).total) return TRIA_ERR_WORKSPACE;
  return TRIA_OK;
}

tria_status cuda_status(cudaError_t e) { return e == cudaSuccess ? TRIA_OK : TRIA_ERR_CUDA; }

// The shortest live length the prune acts on: budget + max(prune_window, 1).
int32_t prune_from(const tria_config *cfg) {
  const int64_t w = cfg->prune_window > 1 ? cfg->prune_window : 1;
  const int64_t t = (int64_t)cfg->budget + w;
  return t < INT32_MAX ? (int32_t)t : INT32_MAX;
}

// Mean over the offsets of e^{i w_f delta} for every RoPE pair (the part of the
// trigonometric weight that depends on neither the keys nor the current position),
// in float64 on the host.  The last problem's table is kept per host thread: a
// decode loop calls with the same offsets every time.
struct OffsetMean {
  double theta = 0.0;
  int32_t D = 0;
  std::vector<int32_t> offsets;
  std::vector<double> re, im;
};

const OffsetMean &offset_mean(const tria_config *cfg) {
  static thread_local OffsetMean m;
  const bool same = m.theta == cfg->rope_theta && m.D == cfg->head_dim &&
                    (int)m.offsets.size() == cfg->n_offsets &&
                    std::memcmp(m.offsets.data(), cfg->offsets, sizeof(int32_t) * cfg->n_offsets) == 0;
  if (!same) {
    const int F = cfg->head_dim / 2;
    m.theta = cfg->rope_theta;
    m.D = cfg->head_dim;
    m.offsets.assign(cfg->offsets, cfg->offsets + cfg->n_offsets);
    m.re.assign(F, 0.0);
    m.im.assign(F, 0.0);
    for (int f = 0; f < F; ++f) {
      const double w = std::pow(cfg->rope_theta, -2.0 * (double)f / (double)cfg->head_dim);
      double re = 0.0, im = 0.0;
      for (int j = 0; j < cfg->n_offsets; ++j) {
        re += std::cos(w * (double)cfg->offsets[j]);
        im += std::sin(w * (double)cfg->offsets[j]);
      }
      m.re[f] = re / (double)cfg->n_offsets;
      m.im[f] = im / (double)cfg->n_offsets;
    }
  }
  return m;
}

void fill_fold(FoldParams &fp, const tria_config *cfg, const tria_stats *st,
               const tria_cache *c, int32_t *seqlen_snap, float *w, int32_t *err) {
  std::memset(&fp, 0, sizeof fp);
  fp.cur_pos = c->cur_pos;
  fp.seq_len = c->seq_len;
  fp.unit_len = c->unit_len;
  fp.units = (int64_t)cfg->num_layers * cfg->n_kv_heads * cfg->batch;
  fp.seqlen_snap = seqlen_snap;
  fp.err = err;
  fp.centre = reinterpret_cast<const float2 *>(st->centre);
  fp.mean_norm = st->mean_norm;
  fp.mrl = st->mrl;
  fp.w = w;
  fp.theta = cfg->rope_theta;
  fp.D = cfg->head_dim;
  fp.B = cfg->batch;
  fp.L = cfg->num_layers;
  fp.Hkv = cfg->n_kv_heads;
  fp.Hq = cfg->n_q_heads;
  fp.G = cfg->n_q_heads / cfg->n_kv_heads;
  fp.flags = cfg->flags;
  for (int b = 0; b < cfg->batch; ++b) fp.seg_cap[b] = c->seq_start[b + 1] - c->seq_start[b];
  // the offset average does not depend on the call's positions: it is formed on the host
  // in float64 (once per offset set, then cached) and passed with the frequencies
  const OffsetMean &om = offset_mean(cfg);
  const bool no_trig = (cfg->flags & TRIA_NO_TRIG) != 0;
  for (int f = 0; f < cfg->head_dim / 2 && f < 128; ++f) {
    fp.omega[f] = std::pow(cfg->rope_theta, -2.0 * (double)f / (double)cfg->head_dim);
    fp.A[f] = no_trig ? make_double2(0.0, 0.0) : make_double2(om.re[f], om.im[f]);
  }
}

// Builds the score kernel parameters; *grid receives the grid size (0: nothing to launch).
cudaError_t fill_score(ScoreParams &sp, const tria_config *cfg, const tria_cache *c,
                       const float *w, float *raw, double *partials, int32_t *err, int skip_short,
                       int *grid) {
  std::memset(&sp, 0, sizeof sp);
  const ScoreGrid sg = score_grid(*cfg, c->seq_start);
  const int ch = sg.chunk_keys;
  sp.w = w;
  sp.seq_len = c->seq_len;
  sp.unit_len = c->unit_len;
  sp.head_budget = cfg->head_budgets;
  sp.budget = cfg->budget;
  sp.window = cfg->prune_window;
  sp.raw = raw;
  sp.partials = partials;
  sp.max_slots = sg.max_slots;
  sp.err = err;
  sp.cap = c->cap_total;
  sp.L = cfg->num_layers;
  sp.Hkv = cfg->n_kv_heads;
  sp.Hq = cfg->n_q_heads;
  sp.B = cfg->batch;
  sp.prune_from = prune_from(cfg);
  sp.skip_short = skip_short;
  int32_t acc = 0;
  for (int b = 0; b <= cfg->batch; ++b) {
    sp.seg_start[b] = c->seq_start[b];
    sp.chunk_prefix[b] = acc;
    if (b < cfg->batch) acc += (int32_t)((c->seq_start[b + 1] - c->seq_start[b] + ch - 1) / ch);
  }
  sp.chunks_per_row = acc;
  *grid = 0;
  if (sg.total > INT32_MAX - 64) return cudaErrorInvalidValue;  // excluded by check_key_rows
  sp.total_chunks = (int32_t)sg.total;
  sp.chunks_per_cta = sg.chunks_per_cta;
  sp.tc = score_uses_tc(cfg->head_dim, cfg->n_q_heads / cfg->n_kv_heads, sg.chunks_per_cta) ? 1 : 0;
  if (sg.total == 0) return cudaSuccess;
  const int64_t rows = (int64_t)cfg->num_layers * cfg->n_kv_heads * c->cap_total;
  cudaError_t e = make_key_tensor_map(&sp.tmap, c->k, cfg->head_dim, rows, ch);
  if (e != cudaSuccess) return e;
  *grid = sg.grid;
  return cudaSuccess;
}

// The unit kernel finds the score kernel's partial sums through its chunk decomposition.
void link_unit_to_score(UnitParams &up, const ScoreParams &sp) {
  up.partials = sp.partials;
  up.max_slots = sp.max_slots;
  up.chunks_per_cta = sp.chunks_per_cta > 0 ? sp.chunks_per_cta : 1;
  up.chunks_per_row = sp.chunks_per_row;
  up.score_warps = sp.tc ? kScoreTcWarps : kScoreConsumerWarps;
  for (int b = 0; b <= TRIA_MAX_BATCH; ++b) up.chunk_prefix[b] = sp.chunk_prefix[b];
}

void fill_unit(UnitParams &up, const tria_config *cfg, const tria_cache *c, int mode) {
  std::memset(&up, 0, sizeof up);
  up.k = static_cast<uint8_t *>(c->k);
  up.v = static_cast<uint8_t *>(c->v);
  up.pos = c->pos;
  up.cap = c->cap_total;
  up.L = cfg->num_layers;
  up.Hkv = cfg->n_kv_heads;
  up.Hq = cfg->n_q_heads;
  up.B = cfg->batch;
  up.G = cfg->n_q_heads / cfg->n_kv_heads;
  up.D = cfg->head_dim;
  up.budget = cfg->budget;
  up.prune_from = prune_from(cfg);
  up.unit_mode = c->unit_len != nullptr;
  up.head_budget = cfg->head_budgets;
  up.window = cfg->prune_window;
  up.mode = mode;
  int64_t most = 0;
  for (int b = 0; b <= cfg->batch; ++b) {
    up.seg_start[b] = c->seq_start[b];
    if (b < cfg->batch && c->seq_start[b + 1] - c->seq_start[b] > most)
      most = c->seq_start[b + 1] - c->seq_start[b];
  }
  up.smem_bytes = unit_smem_bytes();
  up.cluster = unit_cluster_size((int64_t)cfg->num_layers * cfg->n_kv_heads * cfg->batch, most);
}

struct Ws {
  WsLayout lay;
  uint8_t *base;
  int32_t *err() const { return reinterpret_cast<int32_t *>(base + lay.err); }
  int32_t *seqlen() const { return reinterpret_cast<int32_t *>(base + lay.seqlen); }
  float *w() const { return reinterpret_cast<float *>(base + lay.w); }
  double *partials() const { return reinterpret_cast<double *>(base + lay.partials); }
  float *raw() const { return reinterpret_cast<float *>(base + lay.raw); }
  int32_t *sel() const { return reinterpret_cast<int32_t *>(base + lay.sel); }
};

const char *kStageNames[] = {"fold_kernel", "score_kernel", "unit_kernel", "prune_kernel"};
enum StageId : int32_t { kStageFold = 0, kStageScore = 1, kStageUnit = 2, kStagePrune = 3 };


// Parameters of the fused prune kernel.
cudaError_t fill_prune(PruneParams &pp, const tria_config *cfg, const tria_stats *st,
                       const tria_cache *c, const WsLayout &lay, uint8_t *ws, int32_t *sel_out) {
  std::memset(&pp, 0, sizeof pp);
  const PrunePlan pl = prune_plan(*cfg, c->seq_start);
  if (!pl.ok) return cudaErrorInvalidValue;
  const int G = cfg->n_q_heads / cfg->n_kv_heads, F = cfg->head_dim / 2;
  pp.k = static_cast<uint8_t *>(c->k);
  pp.v = static_cast<uint8_t *>(c->v);
  pp.pos = c->pos;
  pp.seq_len = c->seq_len;
  pp.unit_len = c->unit_len;
  pp.head_budget = cfg->head_budgets;
  pp.cur_pos = c->cur_pos;
  pp.centre = reinterpret_cast<const float2 *>(st->centre);
  pp.mean_norm = st->mean_norm;
  pp.mrl = st->mrl;
  pp.sel_out = sel_out;
  pp.err = reinterpret_cast<int32_t *>(ws + kWsErr);
  pp.sync = reinterpret_cast<int32_t *>(ws + kWsSync);
  pp.bcount = reinterpret_cast<int32_t *>(ws + kWsBcount);
  pp.hist = reinterpret_cast<uint32_t *>(ws + kWsHist);
  pp.ea = reinterpret_cast<double2 *>(ws + lay.f_ea);
  pp.w = reinterpret_cast<float *>(ws + lay.f_w);
  pp.raw = reinterpret_cast<float *>(ws + lay.f_raw);
  pp.csum = reinterpret_cast<double *>(ws + lay.f_csum);
  pp.partial = reinterpret_cast<double *>(ws + lay.f_partial);
  pp.zk = reinterpret_cast<uint32_t *>(ws + lay.f_zk);
  pp.bucket = reinterpret_cast<unsigned long long *>(ws + lay.f_bucket);
  pp.above = reinterpret_cast<int32_t *>(ws + lay.f_above);
  pp.thr = reinterpret_cast<unsigned long long *>(ws + lay.f_thr);
  pp.kcount = reinterpret_cast<int32_t *>(ws + lay.f_kcount);
  pp.klist = reinterpret_cast<int32_t *>(ws + lay.f_klist);
  pp.khaz = reinterpret_cast<int32_t *>(ws + lay.f_khaz);
  pp.stage_k = ws + lay.f_stage_k;
  pp.stage_v = ws + lay.f_stage_v;
  pp.stage_pos = reinterpret_cast<int32_t *>(ws + lay.f_stage_pos);
  pp.cap = c->cap_total;
  pp.zk_stride = pl.zk_stride;
  pp.L = cfg->num_layers;
  pp.Hkv = cfg->n_kv_heads;
  pp.Hq = cfg->n_q_heads;
  pp.B = cfg->batch;
  pp.budget = cfg->budget;
  pp.window = cfg->prune_window;
  pp.write_short_sel = sel_out ? 1 : 0;
  pp.flags = (int32_t)cfg->flags;
  pp.units = cfg->num_layers * cfg->n_kv_heads * cfg->batch;
  pp.ug = pl.ug;
  pp.ngroups = pl.ngroups;
  pp.ncta = pl.ncta;
  pp.cpr = pl.cpr;
  pp.range_keys = pl.range_keys;
  pp.range_units = pl.range_units;
  pp.range_chunks = pl.range_keys / pl.chunk_keys;
  int32_t acc = 0;
  for (int b = 0; b <= cfg->batch; ++b) {
    pp.seg_start[b] = c->seq_start[b];
    pp.chunk_prefix[b] = acc;
    if (b < cfg->batch)
      acc += (int32_t)((c->seq_start[b + 1] - c->seq_start[b] + pl.chunk_keys - 1) / pl.chunk_keys);
  }
  const OffsetMean &om = offset_mean(cfg);
  const bool no_trig = (cfg->flags & TRIA_NO_TRIG) != 0;
  for (int f = 0; f < F && f < 128; ++f) {
    pp.omega[f] = std::pow(cfg->rope_theta, -2.0 * (double)f / (double)cfg->head_dim);
    pp.A[f] = no_trig ? make_double2(0.0, 0.0) : make_double2(om.re[f], om.im[f]);
  }
  (void)G;
  const int64_t rows = (int64_t)cfg->num_layers * cfg->n_kv_heads * c->cap_total;
  return make_key_tensor_map(&pp.tmap, c->k, cfg->head_dim, rows, pl.chunk_keys);
}

}  // namespace

extern "C" {

tria_status tria_workspace_size(const tria_config *cfg, const tria_cache *cache, size_t *bytes) {
  if (!bytes) return TRIA_ERR_INVALID_ARG;
  tria_status s = check_config(cfg, false);
  if (s != TRIA_OK) return s;
  if (!cache || cache->cap_total < 0) return TRIA_ERR_INVALID_ARG;
  if (!cache->seq_start) return TRIA_ERR_INVALID_ARG;
  *bytes = ws_layout(*cfg, cache->seq_start, cache->cap_total).total;
  return TRIA_OK;
}

tria_status tria_workspace_init(void *ws, size_t ws_bytes, void *stream) {
  if (!ws || ws_bytes < 256 || !aligned(ws, 256)) return TRIA_ERR_WORKSPACE;
  const size_t n = ws_bytes < kWsPrefix ? ws_bytes : kWsPrefix;
  return cuda_status(cudaMemsetAsync(ws, 0, n, static_cast<cudaStream_t>(stream)));
}

tria_status tria_calibrate(const tria_config *cfg, const void *q_pre, int32_t q_dtype,
                           int64_t n_samples, float *centre, float *mean_norm, float *mrl,
                           void *stream) {
  if (!cfg || !q_pre || !centre || !mean_norm || !mrl || n_samples < 1)
    return TRIA_ERR_INVALID_ARG;
  if (cfg->num_layers < 1 || cfg->n_q_heads < 1 || cfg->head_dim < 2 || cfg->head_dim % 2)
    return TRIA_ERR_INVALID_ARG;
  if (cfg->rope_layout != TRIA_ROPE_HALF_SPLIT && cfg->rope_layout != TRIA_ROPE_INTERLEAVED)
    return TRIA_ERR_INVALID_ARG;
  if (q_dtype != TRIA_DTYPE_F32 && q_dtype != TRIA_DTYPE_BF16) return TRIA_ERR_INVALID_ARG;
  if (cfg->head_dim / 2 > 256) return TRIA_ERR_UNSUPPORTED;
  if (!aligned(centre, 8) || !aligned(mean_norm, 4) || !aligned(mrl, 4) ||
      !aligned(q_pre, q_dtype == TRIA_DTYPE_F32 ? 4 : 2))
    return TRIA_ERR_INVALID_ARG;
  return cuda_status(launch_calibrate(q_pre, q_dtype, cfg->num_layers, n_samples, cfg->n_q_heads,
                                      cfg->head_dim, cfg->rope_layout, centre, mean_norm, mrl,
                                      static_cast<cudaStream_t>(stream)));
}

tria_status tria_score(const tria_config *cfg, const tria_stats *stats, const tria_cache *cache,
                       float *score, float *raw, void *ws, size_t ws_bytes, void *stream) {
  tria_status s;
  if ((s = check_config(cfg, true)) != TRIA_OK) return s;
  if ((s = check_cache(cfg, cache, false)) != TRIA_OK) return s;
  if (!cache->k || !aligned(cache->k, 16) || !cache->cur_pos) return TRIA_ERR_INVALID_ARG;
  if ((s = check_key_rows(cfg, cache)) != TRIA_OK) return s;
  if ((s = check_stats(stats)) != TRIA_OK) return s;
  if (!score || (raw && !aligned(raw, 4))) return TRIA_ERR_INVALID_ARG;
  if ((s = check_ws(cfg, cache, ws, ws_bytes)) != TRIA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Ws w{ws_layout(*cfg, cache->seq_start, cache->cap_total), static_cast<uint8_t *>(ws)};
  float *rawp = raw ? raw : w.raw();

  static thread_local FoldParams fp;
  fill_fold(fp, cfg, stats, cache, w.seqlen(), w.w(), w.err());
  ScoreParams sp;
  int grid = 0;
  if (fill_score(sp, cfg, cache, w.w(), rawp, w.partials(), w.err(), 0, &grid) != cudaSuccess)
    return TRIA_ERR_CUDA;
  if (launch_fold(fp, st) != cudaSuccess) return TRIA_ERR_CUDA;
  if (grid > 0 && launch_score(sp, cfg->head_dim, cfg->n_q_heads / cfg->n_kv_heads,
                               cfg->rope_layout, grid, st, true) != cudaSuccess)
    return TRIA_ERR_CUDA;
  UnitParams up;
  fill_unit(up, cfg, cache, kModeZmax);
  link_unit_to_score(up, sp);
  up.raw = rawp;
  up.score = score;
  up.seqlen = w.seqlen();
  up.err = w.err();
  return cuda_status(launch_unit(up, cfg->num_layers * cfg->n_kv_heads * cfg->batch, st, true));
}

tria_status tria_select(const tria_config *cfg, const tria_cache *cache, const float *score,
                        int32_t *sel, void *ws, size_t ws_bytes, void *stream) {
  tria_status s;
  if ((s = check_config(cfg, false)) != TRIA_OK) return s;
  if ((s = check_cache(cfg, cache, false)) != TRIA_OK) return s;
  if (!score || !sel || !aligned(score, 4) || !aligned(sel, 4)) return TRIA_ERR_INVALID_ARG;
  if ((s = check_ws(cfg, cache, ws, ws_bytes)) != TRIA_OK) return s;
  const Ws w{ws_layout(*cfg, cache->seq_start, cache->cap_total), static_cast<uint8_t *>(ws)};
  UnitParams up;
  fill_unit(up, cfg, cache, kModeSelect);
  up.score = const_cast<float *>(score);
  up.sel = sel;
  up.seqlen = cache->unit_len ? cache->unit_len : cache->seq_len;
  up.err = w.err();
  return cuda_status(launch_unit(up, cfg->num_layers * cfg->n_kv_heads * cfg->batch,
                                 static_cast<cudaStream_t>(stream), false));
}

tria_status tria_compact(const tria_config *cfg, const tria_cache *cache, const int32_t *sel,
                         void *ws, size_t ws_bytes, void *stream) {
  tria_status s;
  if ((s = check_config(cfg, false)) != TRIA_OK) return s;
  if ((s = check_cache(cfg, cache, true)) != TRIA_OK) return s;
  if (!sel || !aligned(sel, 4)) return TRIA_ERR_INVALID_ARG;
  if ((s = check_ws(cfg, cache, ws, ws_bytes)) != TRIA_OK) return s;
  const Ws w{ws_layout(*cfg, cache->seq_start, cache->cap_total), static_cast<uint8_t *>(ws)};
  UnitParams up;
  fill_unit(up, cfg, cache, kModeCompact);
  up.sel = const_cast<int32_t *>(sel);
  up.seq_len_out = cache->unit_len ? cache->unit_len : cache->seq_len;
  up.err = w.err();
  return cuda_status(launch_unit(up, cfg->num_layers * cfg->n_kv_heads * cfg->batch,
                                 static_cast<cudaStream_t>(stream), false));
}

tria_status tria_append(const tria_config *cfg, const tria_cache *cache, const void *k_new,
                        const void *v_new, void *ws, size_t ws_bytes, void *stream) {
  tria_status s;
  if ((s = check_config(cfg, false)) != TRIA_OK) return s;
  if ((s = check_cache(cfg, cache, true)) != TRIA_OK) return s;
  if (!cache->cur_pos) return TRIA_ERR_INVALID_ARG;
  if (!k_new || !v_new || !aligned(k_new, 16) || !aligned(v_new, 16)) return TRIA_ERR_INVALID_ARG;
  if (cfg->head_dim > 256) return TRIA_ERR_UNSUPPORTED;
  if ((s = check_ws(cfg, cache, ws, ws_bytes)) != TRIA_OK) return s;
  const Ws w{ws_layout(*cfg, cache->seq_start, cache->cap_total), static_cast<uint8_t *>(ws)};
  AppendParams ap;
  std::memset(&ap, 0, sizeof ap);
  ap.k_new = static_cast<const uint8_t *>(k_new);
  ap.v_new = static_cast<const uint8_t *>(v_new);
  ap.k = static_cast<uint8_t *>(cache->k);
  ap.v = static_cast<uint8_t *>(cache->v);
  ap.pos = cache->pos;
  ap.seq_len = cache->seq_len;
  ap.unit_len = cache->unit_len;
  ap.cur_pos = cache->cur_pos;
  ap.err = w.err();
  ap.cap = cache->cap_total;
  ap.L = cfg->num_layers;
  ap.Hkv = cfg->n_kv_heads;
  ap.B = cfg->batch;
  ap.D = cfg->head_dim;
  for (int b = 0; b <= cfg->batch; ++b) ap.seg_start[b] = cache->seq_start[b];
  return cuda_status(launch_append(ap, static_cast<cudaStream_t>(stream)));
}

tria_status tria_decode_attention(const tria_config *cfg, const tria_cache *cache, int32_t layer,
                                  const void *q, float scale, float *out, void *ws,
                                  size_t ws_bytes, void *stream) {
  tria_status s;
  if ((s = check_config(cfg, false)) != TRIA_OK) return s;
  if ((s = check_cache(cfg, cache, true)) != TRIA_OK) return s;
  if (layer < 0 || layer >= cfg->num_layers) return TRIA_ERR_INVALID_ARG;
  if (!q || !out || !aligned(q, 16) || !aligned(out, 4)) return TRIA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return TRIA_ERR_INVALID_ARG;
  if (!attention_supported(cfg->head_dim, cfg->n_q_heads / cfg->n_kv_heads))
    return TRIA_ERR_UNSUPPORTED;
  if ((s = check_ws(cfg, cache, ws, ws_bytes)) != TRIA_OK) return s;
  const Ws w{ws_layout(*cfg, cache->seq_start, cache->cap_total), static_cast<uint8_t *>(ws)};
  AttnParams ap;
  std::memset(&ap, 0, sizeof ap);
  ap.q = static_cast<const uint16_t *>(q);
  ap.k = static_cast<const uint16_t *>(cache->k);
  ap.v = static_cast<const uint16_t *>(cache->v);
  ap.seq_len = cache->seq_len;
  ap.unit_len = cache->unit_len;
  ap.out = out;
  ap.err = w.err();
  ap.cap = cache->cap_total;
  ap.layer = layer;
  ap.B = cfg->batch;
  ap.Hkv = cfg->n_kv_heads;
  ap.Hq = cfg->n_q_heads;
  ap.G = cfg->n_q_heads / cfg->n_kv_heads;
  ap.D = cfg->head_dim;
  ap.scale = scale > 0.0f ? scale : 1.0f / std::sqrt((float)cfg->head_dim);
  for (int b = 0; b <= cfg->batch; ++b) ap.seg_start[b] = cache->seq_start[b];
  // the tensor-core path reads K and V through TMA tensor maps (rows addressed as int32)
  const int64_t rows = (int64_t)cfg->num_layers * cfg->n_kv_heads * cache->cap_total;
  if (attention_mma_supported(cfg->head_dim, ap.G) && rows <= INT32_MAX && rows > 0 &&
      aligned(cache->k, 16) && aligned(cache->v, 16) &&
      make_key_tensor_map(&ap.tk, cache->k, cfg->head_dim, rows, 128) == cudaSuccess &&
      make_key_tensor_map(&ap.tv, cache->v, cfg->head_dim, rows, 128) == cudaSuccess) {
    ap.mma = 1;
    // Few (sequence, KV head) pairs: four clusters per pair when their partial results
    // fit the raw-score region of the workspace (unused by this call); the arrival
    // counters live in the workspace's zero-at-rest prefix.
    const int64_t units = (int64_t)cfg->batch * cfg->n_kv_heads;
    const size_t need = (size_t)units * 4 * (16 + 8 * (size_t)cfg->head_dim) * 4;
    const size_t have = 4ull * cfg->num_layers * cfg->n_q_heads * (size_t)cache->cap_total;
    int64_t most = 0;  // the longest segment: short ones are not worth the extra merge
    for (int b = 0; b < cfg->batch; ++b)
      most = std::max<int64_t>(most, cache->seq_start[b + 1] - cache->seq_start[b]);
    if (units * 16 <= 148 && most >= 8192 && need <= have &&
        (size_t)units * 4 <= kWsPrefix - kWsHist) {
      ap.split = 4;
      ap.scratch = w.raw();
      ap.counters = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(ws) + kWsHist);
    }
  }
  return cuda_status(launch_attention(ap, static_cast<cudaStream_t>(stream)));
}

tria_status tria_prune_profiled(const tria_config *cfg, const tria_stats *stats,
                                const tria_cache *cache, int32_t *sel_out, void *ws,
                                size_t ws_bytes, void *stream, void *const *events,
                                int32_t *n_stages, int32_t *stage_ids) {
  tria_status s;
  if ((s = check_config(cfg, true)) != TRIA_OK) return s;
  if ((s = check_cache(cfg, cache, true)) != TRIA_OK) return s;
  if (!cache->cur_pos) return TRIA_ERR_INVALID_ARG;
  if ((s = check_key_rows(cfg, cache)) != TRIA_OK) return s;
  if ((s = check_stats(stats)) != TRIA_OK) return s;
  if (sel_out && !aligned(sel_out, 4)) return TRIA_ERR_INVALID_ARG;
  if ((s = check_ws(cfg, cache, ws, ws_bytes)) != TRIA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const WsLayout lay = ws_layout(*cfg, cache->seq_start, cache->cap_total);
  const Ws w{lay, static_cast<uint8_t *>(ws)};
  int stage = 0;
  auto mark = [&](int32_t id) -> bool {
    if (events && cudaEventRecord(static_cast<cudaEvent_t>(events[stage]), st) != cudaSuccess)
      return false;
    if (stage_ids && id >= 0 && stage < TRIA_PRUNE_MAX_STAGES) stage_ids[stage] = id;
    ++stage;
    return true;
  };

  if (lay.fused) {
    // the whole step in one cooperative launch
    static thread_local PruneParams pp;
    if (fill_prune(pp, cfg, stats, cache, lay, static_cast<uint8_t *>(ws), sel_out) != cudaSuccess)
      return TRIA_ERR_CUDA;
    if (!mark(kStagePrune)) return TRIA_ERR_CUDA;
    if (launch_prune(pp, cfg->head_dim, cfg->n_q_heads / cfg->n_kv_heads, cfg->rope_layout, st) !=
        cudaSuccess)
      return TRIA_ERR_CUDA;
    if (!mark(-1)) return TRIA_ERR_CUDA;
    if (n_stages) *n_stages = stage - 1;
    return TRIA_OK;
  }

  static thread_local FoldParams fp;
  fill_fold(fp, cfg, stats, cache, w.seqlen(), w.w(), w.err());
  ScoreParams sp;
  int grid = 0;
  if (fill_score(sp, cfg, cache, w.w(), w.raw(), w.partials(), w.err(), 1, &grid) != cudaSuccess)
    return TRIA_ERR_CUDA;
  const bool pdl = events == nullptr;  // stage events between kernels would defeat the overlap
  if (!mark(kStageFold)) return TRIA_ERR_CUDA;
  if (launch_fold(fp, st) != cudaSuccess) return TRIA_ERR_CUDA;
  if (!mark(kStageScore)) return TRIA_ERR_CUDA;
  if (grid > 0 && launch_score(sp, cfg->head_dim, cfg->n_q_heads / cfg->n_kv_heads,
                               cfg->rope_layout, grid, st, pdl) != cudaSuccess)
    return TRIA_ERR_CUDA;
  UnitParams up;
  fill_unit(up, cfg, cache, kModePrune);
  link_unit_to_score(up, sp);
  up.raw = w.raw();
  up.sel = sel_out ? sel_out : w.sel();
  up.write_short_sel = sel_out ? 1 : 0;
  up.seqlen = w.seqlen();
  up.seq_len_out = cache->unit_len ? cache->unit_len : cache->seq_len;
  up.err = w.err();
  if (!mark(kStageUnit)) return TRIA_ERR_CUDA;
  if (launch_unit(up, cfg->num_layers * cfg->n_kv_heads * cfg->batch, st, pdl) != cudaSuccess)
    return TRIA_ERR_CUDA;
  if (!mark(-1)) return TRIA_ERR_CUDA;
  if (n_stages) *n_stages = stage - 1;
  return TRIA_OK;
}

tria_status tria_prune(const tria_config *cfg, const tria_stats *stats, const tria_cache *cache,
                       int32_t *sel_out, void *ws, size_t ws_bytes, void *stream) {
  return tria_prune_profiled(cfg, stats, cache, sel_out, ws, ws_bytes, stream, nullptr, nullptr,
                             nullptr);
}

const char *tria_prune_stage_name(int32_t i) {
  if (i < 0 || i >= (int32_t)(sizeof kStageNames / sizeof kStageNames[0])) return "";
  return kStageNames[i];
}

tria_status tria_get_device_error(const void *ws, int32_t *code, void *stream) {
  if (!ws || !code) return TRIA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t v = 0;
  if (cudaMemcpyAsync(&v, ws, sizeof v, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return TRIA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return TRIA_ERR_CUDA;
  *code = v;
  return v ? TRIA_ERR_DEVICE_FLAG : TRIA_OK;
}

const char *tria_status_string(tria_status s) {
  switch (s) {
    case TRIA_OK: return "TRIA_OK";
    case TRIA_ERR_INVALID_ARG: return "TRIA_ERR_INVALID_ARG";
    case TRIA_ERR_UNSUPPORTED: return "TRIA_ERR_UNSUPPORTED";
    case TRIA_ERR_WORKSPACE: return "TRIA_ERR_WORKSPACE";
    case TRIA_ERR_CUDA: return "TRIA_ERR_CUDA";
    case TRIA_ERR_DEVICE_FLAG: return "TRIA_ERR_DEVICE_FLAG";
  }
  return "TRIA_UNKNOWN_STATUS";
}

const char *tria_version(void) { return "tria 0.1 (sm_100a)"; }

}  // extern "C"
