/*
 * TriAttention prune-step oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, float64 CPU restatement of what the prune step computes, used
 * by the tests, by the smoke check and by the benchmark's CPU baseline.  The
 * product path never links, loads or calls it.  It shares no code, header,
 * table or helper with the CUDA library.
 *
 * Sources (the pages describing arXiv 2604.04921, "TriAttention: Efficient
 * Long Reasoning with Trigonometric KV Compression"):
 *   [R1 Method]   romaanj.github.io review, section "Method": calibration of
 *                 E[q_f], mean norm and MRL R_f; the trigonometric term
 *                 sum_f ||E[q_f]||*||k_f||*cos(w_f*Delta + phi_f); the norm term
 *                 weighted by (1 - R_f); averaging over future offsets; per-head
 *                 z-score then max over the GQA group; prune back to budget.
 *   [R2 2-2]      dimensionstp.github.io review, section 2-2, equation
 *                 a(i,j) = sum_f r_q,f r_k,f cos((i-j) theta_f + phi_f).
 *   [R2 2-1]      same page, section 2-1 step 3: keys are scored from their
 *                 position and pre-RoPE representation.
 *   [R2 3-2(2)-(6)] same page, section 3-2 items (2) trigonometric score,
 *                 (3) norm score, (4) adaptive weighting score = S_tri + S_norm,
 *                 (5) window pruning keeps the top-budget keys, (6) GQA
 *                 normalize-then-aggregate (z-score per query head, max).
 *
 * Readings where the pages are silent (each restated where it is used):
 *   R_f = |E[q_f]| / E|q_f|  (0 when E|q_f| = 0);
 *   pairs are half-split (x = v[f], y = v[f+D/2]) or interleaved (v[2f], v[2f+1]);
 *   w_f = theta^(-2f/D);  "current position" = position of the newest token;
 *   the mean (not the sum) over the offsets; score = S_trig + S_norm with no
 *   extra coefficient and no 1/sqrt(D); population standard deviation, z = 0
 *   when it is 0; ties go to the lower slot (= lower position); no protected
 *   sink or recent window.
 *
 * Every function here is pinned by a test against closed forms, special
 * cases, invariants or brute force (see tests/test_oracle_pins.py).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_NO_TRIG        1u  /* ablation: drop the trigonometric term        */
#define ORC_NO_CONC_WEIGHT 2u  /* ablation: norm term without the (1 - R_f)    */

typedef struct {
  int32_t L, B, Hq, Hkv, D, layout; /* layout 0 half-split, 1 interleaved */
  double theta;
  int32_t budget;
  int32_t n_offsets;
  const int32_t *offsets;           /* future query offsets delta >= 1 */
  uint32_t flags;
  int64_t cap;                      /* slots per (layer, kv head) */
  const int64_t *seq_start;         /* [B+1] */
  const int32_t *seq_len;           /* [B] */
  const int32_t *cur_pos;           /* [B] */
  const uint16_t *k;                /* bf16 bit patterns [L][Hkv][cap][D], post-RoPE */
  const int32_t *pos;               /* [L][Hkv][cap] */
  const double *centre;             /* [L][Hq][D/2][2] complex E[q_f] */
  const double *mean_norm;          /* [L][Hq][D/2] E|q_f| */
  const double *mrl;                /* [L][Hq][D/2] R_f */
  const int32_t *head_budget;       /* [L][Hkv] keys kept per unit of each KV head, or NULL */
  const int32_t *unit_len;          /* [L][Hkv][B] live keys per unit, or NULL (seq_len) */
} orc_problem;

/*
 * Head-specific budgets [R1 Future work: refined compression with budgets per
 * head]: the pages name the idea without a rule for choosing the budgets, so the
 * budgets are an input, one per (layer, KV head), each at most `budget` (the row
 * length of the selection lists).  Once heads keep different numbers of keys,
 * the units of one sequence have different lengths: unit_len holds them.
 */
static int64_t unit_T(const orc_problem *p, int32_t l, int32_t g, int32_t b) {
  return p->unit_len ? p->unit_len[((int64_t)l * p->Hkv + g) * p->B + b] : p->seq_len[b];
}
static int32_t unit_budget(const orc_problem *p, int32_t l, int32_t g) {
  return p->head_budget ? p->head_budget[(int64_t)l * p->Hkv + g] : p->budget;
}

/* bfloat16 bits -> double: the bf16 value is the top half of a float32. */
static double bf16_to_double(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Indices of the two real components of RoPE pair f. */
static void pair_index(int32_t D, int32_t layout, int32_t f, int32_t *xi, int32_t *yi) {
  if (layout == 0) { *xi = f; *yi = f + D / 2; }
  else             { *xi = 2 * f; *yi = 2 * f + 1; }
}

/* RoPE rotation frequency of pair f. */
static double rope_freq(double theta, int32_t D, int32_t f) {
  return pow(theta, -2.0 * (double)f / (double)D);
}

/*
 * Calibration [R1 Method; R2 3-1]: for every (layer, query head, pair f) over
 * the N pre-RoPE sample queries q^(n):
 *   centre_f = (1/N) sum_n q_f^(n)        (complex mean, E[q_f])
 *   mean_f   = (1/N) sum_n |q_f^(n)|      (mean norm, E|q_f|)
 *   R_f      = |centre_f| / mean_f        (mean resultant length; 0 if mean_f = 0)
 * q is [L][N][Hq][D] float64.
 */
void orc_calibrate(const double *q, int64_t L, int64_t N, int64_t Hq, int64_t D,
                   int32_t layout, double *centre, double *mean_norm, double *mrl) {
  const int64_t F = D / 2;
  for (int64_t l = 0; l < L; ++l)
    for (int64_t h = 0; h < Hq; ++h)
      for (int64_t f = 0; f < F; ++f) {
        int32_t xi, yi;
        pair_index((int32_t)D, layout, (int32_t)f, &xi, &yi);
        double sx = 0.0, sy = 0.0, sn = 0.0;
        for (int64_t n = 0; n < N; ++n) {
          const double *v = q + ((l * N + n) * Hq + h) * D;
          sx += v[xi];
          sy += v[yi];
          sn += hypot(v[xi], v[yi]);
        }
        const int64_t o = (l * Hq + h) * F + f;
        centre[2 * o + 0] = sx / (double)N;
        centre[2 * o + 1] = sy / (double)N;
        mean_norm[o] = sn / (double)N;
        mrl[o] = mean_norm[o] > 0.0 ? hypot(centre[2 * o], centre[2 * o + 1]) / mean_norm[o] : 0.0;
      }
}

/*
 * Raw score of one cached key for one query head, term by term
 * [R1 Method; R2 2-2; R2 3-2 (2)-(4)].
 *
 * The stored key is post-RoPE; its pre-RoPE pair k_f is recovered by rotating
 * back by the key's position p [R2 2-1 step 3]:  k_f = ktilde_f * e^{-i w_f p}.
 * With c_f the query centre of head h:
 *   S_trig = (1/|O|) sum_{delta in O} sum_f |c_f| |k_f| cos(w_f (cur + delta - p) + arg c_f - arg k_f)
 *   S_norm = sum_f (1 - R_f) * mean_f * |k_f|
 *   s      = S_trig + S_norm
 * where cur + delta is the position of a future query, so cur + delta - p is
 * the query-key distance and arg c_f - arg k_f the phase difference.
 * t is the slot within sequence b's segment.
 */
double orc_key_score(const orc_problem *p, int32_t l, int32_t h, int32_t b, int64_t t) {
  const int32_t D = p->D, F = D / 2, G = p->Hq / p->Hkv, g = h / G;
  const int64_t slot = ((int64_t)l * p->Hkv + g) * p->cap + p->seq_start[b] + t;
  const uint16_t *row = p->k + slot * D;
  const double kpos = (double)p->pos[slot];
  const double cur = (double)p->cur_pos[b];
  double s_trig = 0.0, s_norm = 0.0;
  for (int32_t f = 0; f < F; ++f) {
    int32_t xi, yi;
    pair_index(D, p->layout, f, &xi, &yi);
    const double w = rope_freq(p->theta, D, f);
    const double xt = bf16_to_double(row[xi]), yt = bf16_to_double(row[yi]);
    /* undo the rotation by the key's own position */
    const double ca = cos(w * kpos), sa = sin(w * kpos);
    const double kx = xt * ca + yt * sa;
    const double ky = -xt * sa + yt * ca;
    const double k_abs = hypot(kx, ky), k_arg = atan2(ky, kx);
    const int64_t o = ((int64_t)l * p->Hq + h) * F + f;
    const double cx = p->centre[2 * o], cy = p->centre[2 * o + 1];
    const double c_abs = hypot(cx, cy), c_arg = atan2(cy, cx);
    if (!(p->flags & ORC_NO_TRIG)) {
      double acc = 0.0;
      for (int32_t j = 0; j < p->n_offsets; ++j) {
        const double dist = cur + (double)p->offsets[j] - kpos;
        acc += c_abs * k_abs * cos(w * dist + c_arg - k_arg);
      }
      s_trig += acc / (double)p->n_offsets;
    }
    const double weight = (p->flags & ORC_NO_CONC_WEIGHT) ? 1.0 : (1.0 - p->mrl[o]);
    s_norm += weight * p->mean_norm[o] * k_abs;
  }
  return s_trig + s_norm;
}

/* Raw scores of every key of every segment: raw is [L][Hq][cap]; slots outside
 * the live part of a segment are left untouched.  Each key is scored on its
 * own; the work is shared out over (layer, head, sequence, block of 256 keys). */
void orc_raw_scores(const orc_problem *p, double *raw) {
  const int64_t blk = 256;
  const int32_t G = p->Hq / p->Hkv;
  int64_t most = 0;
  for (int32_t l = 0; l < p->L; ++l)
    for (int32_t g = 0; g < p->Hkv; ++g)
      for (int32_t b = 0; b < p->B; ++b)
        if (unit_T(p, l, g, b) > most) most = unit_T(p, l, g, b);
  const int64_t nblk = (most + blk - 1) / blk;
  const int64_t units = (int64_t)p->L * p->Hq * p->B;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t w = 0; w < units * nblk; ++w) {
    const int64_t u = w / nblk, kb = w % nblk;
    const int32_t b = (int32_t)(u % p->B);
    const int32_t h = (int32_t)((u / p->B) % p->Hq);
    const int32_t l = (int32_t)(u / ((int64_t)p->B * p->Hq));
    double *out = raw + ((int64_t)l * p->Hq + h) * p->cap + p->seq_start[b];
    const int64_t T = unit_T(p, l, h / G, b);
    const int64_t t1 = (kb + 1) * blk < T ? (kb + 1) * blk : T;
    for (int64_t t = kb * blk; t < t1; ++t) out[t] = orc_key_score(p, l, h, b, t);
  }
}

/*
 * The same raw scores through the angle-addition fold [R1 Method; R2 2-2]: the
 * key's position cancels between un-rotating the key and the query-key distance,
 * so with ktilde_f the stored (post-RoPE) pair,
 *   S_trig = Re sum_f conj(ktilde_f) * W_f,
 *   W_f    = c_f * (1/|O|) sum_{delta in O} e^{i w_f (cur + delta)},
 * and |k_f| = |ktilde_f| in the norm term.  One weight per (head, pair) per
 * sequence, then one pass over each key.  This is not a second reference for the
 * scores: tests pin it to orc_key_score, and the benchmark times it as the CPU
 * baseline that does the same arithmetic per key as the GPU path.
 */
void orc_raw_scores_folded(const orc_problem *p, double *raw) {
  const int32_t D = p->D, F = D / 2, G = p->Hq / p->Hkv;
  const int64_t units = (int64_t)p->L * p->Hq * p->B;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t u = 0; u < units; ++u) {
    const int32_t b = (int32_t)(u % p->B);
    const int32_t h = (int32_t)((u / p->B) % p->Hq);
    const int32_t l = (int32_t)(u / ((int64_t)p->B * p->Hq));
    const int32_t g = h / G;
    double *wx = (double *)malloc(sizeof(double) * (size_t)F * 3);
    double *wy = wx + F, *wn = wx + 2 * F;
    for (int32_t f = 0; f < F; ++f) {
      const double w = rope_freq(p->theta, D, f);
      double er = 0.0, ei = 0.0;
      if (!(p->flags & ORC_NO_TRIG)) {
        for (int32_t j = 0; j < p->n_offsets; ++j) {
          const double a = w * ((double)p->cur_pos[b] + (double)p->offsets[j]);
          er += cos(a);
          ei += sin(a);
        }
        er /= (double)p->n_offsets;
        ei /= (double)p->n_offsets;
      }
      const int64_t o = ((int64_t)l * p->Hq + h) * F + f;
      const double *cf = p->centre + 2 * o; /* (re, im) of c_f */
      wx[f] = cf[0] * er - cf[1] * ei;      /* W_f = c_f * e */
      wy[f] = cf[0] * ei + cf[1] * er;
      /* norm weight: E|q_f| less the part that the trig term carries, R_f E|q_f| */
      wn[f] = (p->flags & ORC_NO_CONC_WEIGHT) ? p->mean_norm[o]
                                              : p->mean_norm[o] - p->mrl[o] * p->mean_norm[o];
    }
    const int64_t row = ((int64_t)l * p->Hkv + g) * p->cap + p->seq_start[b];
    double *out = raw + ((int64_t)l * p->Hq + h) * p->cap + p->seq_start[b];
    for (int64_t t = 0; t < unit_T(p, l, g, b); ++t) {
      const uint16_t *k = p->k + (row + t) * D;
      double s = 0.0;
      for (int32_t f = 0; f < F; ++f) {
        int32_t xi, yi;
        pair_index(D, p->layout, f, &xi, &yi);
        const double x = bf16_to_double(k[xi]), y = bf16_to_double(k[yi]);
        /* Re(conj(x + iy) * (wx + i wy)) = x wx + y wy */
        s += x * wx[f] + y * wy[f] + wn[f] * hypot(x, y);
      }
      out[t] = s;
    }
    free(wx);
  }
}

/* Sets the number of threads the oracle's parallel loops use (>= 1). */
void orc_set_num_threads(int32_t n) {
#ifdef _OPENMP
  if (n >= 1) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/*
 * GQA normalize-then-aggregate [R1 Method; R2 3-2 (6)]: for each (layer,
 * sequence, query head) the raw scores of the sequence's T keys are z-scored
 *   mu = (1/T) sum_t s(t),  sigma = sqrt((1/T) sum_t (s(t) - mu)^2)   (two passes)
 *   z(t) = (s(t) - mu) / sigma,  z = 0 when sigma = 0,
 * and the key's score is the max of z over the query heads sharing its KV head.
 * z may be NULL ([L][Hq][cap]); score is [L][Hkv][cap].
 */
void orc_zmax(const orc_problem *p, const double *raw, double *z, double *score) {
  const int32_t G = p->Hq / p->Hkv;
  const int64_t units = (int64_t)p->L * p->Hkv * p->B;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t u = 0; u < units; ++u) {
    const int32_t b = (int32_t)(u % p->B);
    const int32_t g = (int32_t)((u / p->B) % p->Hkv);
    const int32_t l = (int32_t)(u / ((int64_t)p->B * p->Hkv));
    const int64_t T = unit_T(p, l, g, b), s0 = p->seq_start[b];
    double *sc = score + ((int64_t)l * p->Hkv + g) * p->cap + s0;
    for (int64_t t = 0; t < T; ++t) sc[t] = -INFINITY;
    for (int32_t j = 0; j < G; ++j) {
      const int32_t h = g * G + j;
      const double *s = raw + ((int64_t)l * p->Hq + h) * p->cap + s0;
      double mu = 0.0, var = 0.0;
      for (int64_t t = 0; t < T; ++t) mu += s[t];
      mu /= (double)(T > 0 ? T : 1);
      for (int64_t t = 0; t < T; ++t) var += (s[t] - mu) * (s[t] - mu);
      var /= (double)(T > 0 ? T : 1);
      const double sigma = sqrt(var);
      for (int64_t t = 0; t < T; ++t) {
        const double zt = sigma > 0.0 ? (s[t] - mu) / sigma : 0.0;
        if (z) z[((int64_t)l * p->Hq + h) * p->cap + s0 + t] = zt;
        if (zt > sc[t]) sc[t] = zt;
      }
    }
  }
}

typedef struct { double score; int64_t slot; } orc_key;

/* Order for selection: higher score first, then lower slot. */
static int by_score_then_slot(const void *a, const void *b) {
  const orc_key *x = (const orc_key *)a, *y = (const orc_key *)b;
  if (x->score > y->score) return -1;
  if (x->score < y->score) return 1;
  return (x->slot > y->slot) - (x->slot < y->slot);
}

static int by_value(const void *a, const void *b) {
  const int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
  return (x > y) - (x < y);
}

/*
 * Top-budget selection [R1 Method; R2 3-2 (5)]: per (layer, KV head,
 * sequence), sort the keys by (score descending, slot ascending), keep the
 * first `budget` (the unit's head budget when budgets are per head), and list
 * them by ascending slot.  A unit of at most that many keys keeps every key.
 * sel is [L][Hkv][B][budget], padded with -1.
 */
void orc_select(const orc_problem *p, const double *score, int32_t *sel) {
  const int64_t units = (int64_t)p->L * p->Hkv * p->B;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t u = 0; u < units; ++u) {
    const int32_t b = (int32_t)(u % p->B);
    const int32_t g = (int32_t)((u / p->B) % p->Hkv);
    const int32_t l = (int32_t)(u / ((int64_t)p->B * p->Hkv));
    const int64_t T = unit_T(p, l, g, b);
    const int32_t keep = unit_budget(p, l, g);
    int32_t *out = sel + (((int64_t)l * p->Hkv + g) * p->B + b) * p->budget;
    for (int32_t j = 0; j < p->budget; ++j) out[j] = -1;
    if (T <= keep) {
      for (int64_t t = 0; t < T; ++t) out[t] = (int32_t)t;
      continue;
    }
    const double *sc = score + ((int64_t)l * p->Hkv + g) * p->cap + p->seq_start[b];
    orc_key *keys = (orc_key *)malloc((size_t)T * sizeof(orc_key));
    for (int64_t t = 0; t < T; ++t) { keys[t].score = sc[t]; keys[t].slot = t; }
    qsort(keys, (size_t)T, sizeof(orc_key), by_score_then_slot);
    for (int32_t j = 0; j < keep; ++j) out[j] = (int32_t)keys[j].slot;
    qsort(out, (size_t)keep, sizeof(int32_t), by_value);
    free(keys);
  }
}

/*
 * Eviction by compaction [R1 Method; R2 3-2 (5)]: the selected rows of K, V and
 * pos move to the front of the segment in ascending slot order and the
 * sequence length becomes the number kept.  k, v ([L][Hkv][cap][D] bf16 bits)
 * and pos ([L][Hkv][cap]) are updated in place through a temporary copy;
 * seq_len_out[b] receives the new length (the one all units of sequence b share
 * when there is a single budget), unit_len_out[L][Hkv][B] every unit's.
 */
void orc_compact(const orc_problem *p, const int32_t *sel, uint16_t *k, uint16_t *v,
                 int32_t *pos, int32_t *seq_len_out, int32_t *unit_len_out) {
  const int32_t D = p->D;
  for (int32_t b = 0; b < p->B; ++b)
    seq_len_out[b] = p->seq_len[b] < p->budget ? p->seq_len[b] : p->budget;
  const int64_t units = (int64_t)p->L * p->Hkv * p->B;
  for (int64_t u = 0; u < units; ++u) {
    const int32_t b = (int32_t)(u % p->B);
    const int32_t g = (int32_t)((u / p->B) % p->Hkv);
    const int32_t l = (int32_t)(u / ((int64_t)p->B * p->Hkv));
    const int64_t T = unit_T(p, l, g, b);
    const int32_t kept_max = unit_budget(p, l, g);
    unit_len_out[u] = (int32_t)(T < kept_max ? T : kept_max);
  }
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t u = 0; u < units; ++u) {
    const int32_t b = (int32_t)(u % p->B);
    const int32_t g = (int32_t)((u / p->B) % p->Hkv);
    const int32_t l = (int32_t)(u / ((int64_t)p->B * p->Hkv));
    const int64_t n = unit_len_out[u];
    const int64_t base = ((int64_t)l * p->Hkv + g) * p->cap + p->seq_start[b];
    const int32_t *s = sel + (((int64_t)l * p->Hkv + g) * p->B + b) * p->budget;
    uint16_t *tk = (uint16_t *)malloc((size_t)(n > 0 ? n : 1) * D * sizeof(uint16_t));
    uint16_t *tv = (uint16_t *)malloc((size_t)(n > 0 ? n : 1) * D * sizeof(uint16_t));
    int32_t *tp = (int32_t *)malloc((size_t)(n > 0 ? n : 1) * sizeof(int32_t));
    for (int64_t j = 0; j < n; ++j) {
      const int64_t src = base + s[j];
      memcpy(tk + j * D, k + src * D, (size_t)D * sizeof(uint16_t));
      memcpy(tv + j * D, v + src * D, (size_t)D * sizeof(uint16_t));
      tp[j] = pos[src];
    }
    for (int64_t j = 0; j < n; ++j) {
      memcpy(k + (base + j) * D, tk + j * D, (size_t)D * sizeof(uint16_t));
      memcpy(v + (base + j) * D, tv + j * D, (size_t)D * sizeof(uint16_t));
      pos[base + j] = tp[j];
    }
    free(tk); free(tv); free(tp);
  }
}

/* Threads the OpenMP runtime will use (1 without OpenMP). */
int32_t orc_num_threads(void) {
#ifdef _OPENMP
  return (int32_t)omp_get_max_threads();
#else
  return 1;
#endif
}
