/*
 * qsa_oracle.c -- plain, slow, obviously correct CPU oracle for the QSA hot
 * path.  TEST INFRASTRUCTURE ONLY: loaded by the tests, the smoke check and
 * the benchmark's CPU-baseline leg, never by the product path.
 *
 * Every function follows the statement of the method one step at a time:
 * decode the stored values, accumulate in double, round once at the end.
 * The only parallelism is an OpenMP loop over independent query tokens.
 */
#include "qsa_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---- value decoders -------------------------------------------------------- */

/* bfloat16: the upper 16 bits of an IEEE-754 binary32. */
double orc_bf16_to_f64(uint16_t bits) {
  uint32_t u = (uint32_t)bits << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* FP8 E4M3FN (OCP 8-bit floating point, E4M3 variant): 1 sign bit, 4 exponent
 * bits with bias 7, 3 mantissa bits; exponent field 0 encodes subnormals
 * (mantissa/8 * 2^-6); there are no infinities; S.1111.111 is NaN. */
double orc_e4m3_to_f64(uint8_t code) {
  int sign = (code >> 7) & 1;
  int e = (code >> 3) & 0xF;
  int m = code & 0x7;
  double v;
  if (e == 0xF && m == 0x7) return NAN;
  if (e == 0)
    v = ldexp((double)m / 8.0, -6);
  else
    v = ldexp(1.0 + (double)m / 8.0, e - 7);
  return sign ? -v : v;
}

static double load_val(const void* base, int dt, long idx) {
  switch (dt) {
    case ORC_F32: return (double)((const float*)base)[idx];
    case ORC_BF16: return orc_bf16_to_f64(((const uint16_t*)base)[idx]);
    case ORC_FP8_E4M3: return orc_e4m3_to_f64(((const uint8_t*)base)[idx]);
    default: return NAN;
  }
}

void orc_set_max_threads(int n) {
#ifdef _OPENMP
  if (n >= 1) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

int orc_threads_for(int T) {
#ifdef _OPENMP
  int n = omp_get_max_threads();
  return T < n ? (T < 1 ? 1 : T) : n;
#else
  (void)T;
  return 1;
#endif
}

/* ---- stage 1: indexer scores ----------------------------------------------- */

long orc_index_scores(const void* q_idx, int q_dt, const float* w_idx,
                      const void* k_idx_pages, int k_dt, int num_pages,
                      const int32_t* page_table, int pt_stride,
                      const int32_t* q_req, const int32_t* q_pos,
                      int T, int H_I, int D_I, float* scores, int score_stride) {
  if (T < 0 || H_I < 1 || D_I < 1 || pt_stride < 1 || score_stride < 0) return -1;
  if (q_dt != ORC_F32 && q_dt != ORC_BF16) return -2;
  if (k_dt != ORC_F32 && k_dt != ORC_BF16) return -2;
  long skipped = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : skipped) num_threads(orc_threads_for(T))
  for (int t = 0; t < T; ++t) {
    const int r = q_req ? q_req[t] : t;
    const int p = q_pos[t];
    const int c = p >= 0 ? p / ORC_GROUP_TOKENS : 0; /* complete groups before the current block */
    float* row = scores + (long)t * score_stride;
    for (int g = 0; g < score_stride; ++g) row[g] = -INFINITY;
    for (int g = 0; g < c && g < score_stride; ++g) {
      const int lp = g / ORC_PAGE_GROUPS; /* logical page holding group g */
      if (lp >= pt_stride) { ++skipped; continue; }
      const int page = page_table[(long)r * pt_stride + lp];
      if (page < 0 || page >= num_pages) { ++skipped; continue; }
      const long kbase = ((long)page * ORC_PAGE_GROUPS + g % ORC_PAGE_GROUPS) * D_I;
      double s = 0.0;
      for (int h = 0; h < H_I; ++h) {
        double dot = 0.0;
        for (int d = 0; d < D_I; ++d)
          dot += load_val(q_idx, q_dt, ((long)t * H_I + h) * D_I + d) *
                 load_val(k_idx_pages, k_dt, kbase + d);
        const double relu = dot > 0.0 ? dot : 0.0;
        s += (double)w_idx[(long)t * H_I + h] * relu;
      }
      row[g] = (float)s;
    }
  }
  return skipped;
}

/* ---- stage 2: exact top-K over groups -------------------------------------- */

typedef struct {
  float key;
  int32_t id;
} cand_t;

/* (score desc, id asc): the unique strict total order the selection uses. */
static int cand_cmp(const void* a, const void* b) {
  const cand_t* x = (const cand_t*)a;
  const cand_t* y = (const cand_t*)b;
  if (x->key > y->key) return -1;
  if (x->key < y->key) return 1;
  return (x->id > y->id) - (x->id < y->id);
}

static int int_cmp(const void* a, const void* b) {
  int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
  return (x > y) - (x < y);
}

long orc_topk_groups(const float* scores, int score_stride, const int32_t* q_pos,
                     int T, int K, int32_t* sel, int32_t* n_sel) {
  if (T < 0 || K < 1 || score_stride < 0) return -1;
  long bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : bad) num_threads(orc_threads_for(T))
  for (int t = 0; t < T; ++t) {
    const int p = q_pos[t];
    int c = p >= 0 ? p / ORC_GROUP_TOKENS : 0;
    if (c > score_stride) c = score_stride;
    const int n = c < K ? c : K;
    int32_t* out = sel + (long)t * K;
    cand_t* cand = (cand_t*)malloc(sizeof(cand_t) * (size_t)(c > 0 ? c : 1));
    for (int g = 0; g < c; ++g) {
      float v = scores[(long)t * score_stride + g];
      if (v != v) ++bad;
      if (v == 0.0f) v = 0.0f; /* -0 and +0 rank as the same value */
      cand[g].key = v;
      cand[g].id = g;
    }
    qsort(cand, (size_t)c, sizeof(cand_t), cand_cmp);
    for (int i = 0; i < n; ++i) out[i] = cand[i].id;
    qsort(out, (size_t)n, sizeof(int32_t), int_cmp);
    for (int i = n; i < K; ++i) out[i] = -1;
    n_sel[t] = n;
    free(cand);
  }
  return bad ? -3 : 0;
}

/* ---- stage 3: expansion to token ids --------------------------------------- */

long orc_expand_select(const int32_t* sel, const int32_t* n_sel, int K,
                       const int32_t* q_pos, const int32_t* capture_pos, int T,
                       int32_t* tok, int32_t* n_tok, int W) {
  if (T < 0 || K < 1 || W < 1) return -1;
  long bad = 0, overflow = 0;
  for (int t = 0; t < T; ++t) {
    const int p = q_pos[t];
    const int c = p >= 0 ? p / ORC_GROUP_TOKENS : 0;
    int p0 = capture_pos ? capture_pos[t] : p;
    if (p0 > p) p0 = p;
    const int c0 = p0 >= 0 ? p0 / ORC_GROUP_TOKENS : 0;
    int ns = n_sel[t];
    if (ns < 0) ns = 0;
    if (ns > K) ns = K;
    int32_t* row = tok + (long)t * W;
    int n = 0;
    /* kept groups, in the order the selection lists them (ascending) */
    for (int i = 0; i < ns; ++i) {
      const int g = sel[(long)t * K + i];
      const int ok = g >= 0 && g < c0;
      if (!ok) ++bad;
      for (int j = 0; j < ORC_GROUP_TOKENS; ++j) {
        if (n < W) row[n] = ok ? ORC_GROUP_TOKENS * g + j : -1;
        ++n;
      }
    }
    /* groups completed between the capture position and the query (MTP reuse) */
    for (int g = c0; g < c; ++g)
      for (int j = 0; j < ORC_GROUP_TOKENS; ++j) {
        if (n < W) row[n] = ORC_GROUP_TOKENS * g + j;
        ++n;
      }
    /* the current block: always attended, outside the budget */
    if (p >= 0)
      for (int j = ORC_GROUP_TOKENS * c; j <= p; ++j) {
        if (n < W) row[n] = j;
        ++n;
      }
    if (n > W) ++overflow;
    n_tok[t] = n < W ? n : W;
    for (int i = n; i < W; ++i) row[i] = -1;
  }
  if (overflow) return -4;
  return bad;
}

/* ---- stage 4: attention over the selected tokens --------------------------- */

long orc_sparse_attn(const void* q, int q_dt, const void* k_pages,
                     const void* v_pages, int kv_dt, float k_scale, float v_scale,
                     int num_pages, const int32_t* page_table, int pt_stride,
                     const int32_t* q_req, const int32_t* tok,
                     const int32_t* n_tok, int W, int T, int Hq, int Hkv, int D,
                     float sm_scale, double* out, double* lse) {
  if (T < 0 || Hq < 1 || Hkv < 1 || D < 1 || W < 0 || pt_stride < 1) return -1;
  if (Hq % Hkv != 0) return -1;
  if (q_dt != ORC_F32 && q_dt != ORC_BF16) return -2;
  if (kv_dt != ORC_F32 && kv_dt != ORC_BF16 && kv_dt != ORC_FP8_E4M3) return -2;
  const double scale = sm_scale > 0.0f ? (double)sm_scale : 1.0 / sqrt((double)D);
  const double ks = kv_dt == ORC_FP8_E4M3 ? (double)k_scale : 1.0;
  const double vs = kv_dt == ORC_FP8_E4M3 ? (double)v_scale : 1.0;
  const int group = Hq / Hkv;
  long skipped = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : skipped) num_threads(orc_threads_for(T))
  for (int t = 0; t < T; ++t) {
    const int r = q_req ? q_req[t] : t;
    int n = n_tok[t];
    if (n < 0) n = 0;
    if (n > W) n = W;
    /* physical row (page*64 + slot) of every usable entry; -1 = skip */
    long* slot = (long*)malloc(sizeof(long) * (size_t)(n > 0 ? n : 1));
    double* logit = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    for (int i = 0; i < n; ++i) {
      const int j = tok[(long)t * W + i];
      slot[i] = -1;
      if (j == -1) continue;
      if (j < -1 || j / ORC_PAGE_TOKENS >= pt_stride) { ++skipped; continue; }
      const int page = page_table[(long)r * pt_stride + j / ORC_PAGE_TOKENS];
      if (page < 0 || page >= num_pages) { ++skipped; continue; }
      slot[i] = (long)page * ORC_PAGE_TOKENS + j % ORC_PAGE_TOKENS;
    }
    for (int h = 0; h < Hq; ++h) {
      const int kvh = h / group;
      double* o = out + ((long)t * Hq + h) * D;
      for (int d = 0; d < D; ++d) o[d] = 0.0;
      /* pass 1: logits and their maximum */
      double m = -INFINITY;
      for (int i = 0; i < n; ++i) {
        if (slot[i] < 0) continue;
        const long kb = (slot[i] * Hkv + kvh) * D;
        double dot = 0.0;
        for (int d = 0; d < D; ++d)
          dot += load_val(q, q_dt, ((long)t * Hq + h) * D + d) * (load_val(k_pages, kv_dt, kb + d) * ks);
        logit[i] = scale * dot;
        if (logit[i] > m) m = logit[i];
      }
      if (m == -INFINITY) { /* nothing to attend: zero output */
        if (lse) lse[(long)t * Hq + h] = -INFINITY;
        continue;
      }
      /* pass 2: normaliser and weighted sum of values */
      double l = 0.0;
      for (int i = 0; i < n; ++i) {
        if (slot[i] < 0) continue;
        const double e = exp(logit[i] - m);
        l += e;
        const long vb = (slot[i] * Hkv + kvh) * D;
        for (int d = 0; d < D; ++d) o[d] += e * (load_val(v_pages, kv_dt, vb + d) * vs);
      }
      for (int d = 0; d < D; ++d) o[d] /= l;
      if (lse) lse[(long)t * Hq + h] = m + log(l);
    }
    free(slot);
    free(logit);
  }
  return skipped;
}

/* ---- before stage 1: the indexer projection --------------------------------- */

long orc_indexer_project(const void* x, int x_dt, const void* w, int w_dt, int T, int H, int N,
                         float* y) {
  if (T < 0 || H < 1 || N < 1) return -1;
  if ((x_dt != ORC_F32 && x_dt != ORC_BF16) || (w_dt != ORC_F32 && w_dt != ORC_BF16)) return -2;
#pragma omp parallel for schedule(dynamic, 1) num_threads(orc_threads_for(T))
  for (int t = 0; t < T; ++t)
    for (int n = 0; n < N; ++n) {
      double acc = 0.0;
      for (int h = 0; h < H; ++h)
        acc += load_val(x, x_dt, (long)t * H + h) * load_val(w, w_dt, (long)n * H + h);
      y[(long)t * N + n] = (float)acc;
    }
  return 0;
}

/* ---- before stage 1: the C4 compressed-key write ----------------------------- */

/* bfloat16 bits of a float, round to nearest even (finite inputs). */
static uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  const uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

long orc_compress_keys(const float* k_tok, int n_groups, const int32_t* g_req, const int32_t* g_id,
                       const float* wphi, const float* bias, int D_I, void* k_idx_pages, int k_dt,
                       int num_pages, const int32_t* page_table, int pt_rows, int pt_stride) {
  if (n_groups < 0 || D_I < 1 || pt_rows < 1 || pt_stride < 1) return -1;
  if (k_dt != ORC_F32 && k_dt != ORC_BF16) return -2;
  long skipped = 0;
  for (int i = 0; i < n_groups; ++i) {
    const int r = g_req ? g_req[i] : 0;
    const int g = g_id[i];
    if (r < 0 || r >= pt_rows || g < 0 || g / ORC_PAGE_GROUPS >= pt_stride) { ++skipped; continue; }
    const int page = page_table[(long)r * pt_stride + g / ORC_PAGE_GROUPS];
    if (page < 0 || page >= num_pages) { ++skipped; continue; }
    const long row = ((long)page * ORC_PAGE_GROUPS + g % ORC_PAGE_GROUPS) * D_I;
    /* khat[d] = bias[d] + sum over the group's four tokens j and dims e of
       wphi[d][j * D_I + e] * k_tok[i][j][e] */
    for (int d = 0; d < D_I; ++d) {
      double acc = bias ? (double)bias[d] : 0.0;
      for (int j = 0; j < ORC_GROUP_TOKENS; ++j)
        for (int e = 0; e < D_I; ++e)
          acc += (double)wphi[((long)d * ORC_GROUP_TOKENS + j) * D_I + e] *
                 (double)k_tok[((long)i * ORC_GROUP_TOKENS + j) * D_I + e];
      const float v = (float)acc;
      if (k_dt == ORC_F32) ((float*)k_idx_pages)[row + d] = v;
      else ((uint16_t*)k_idx_pages)[row + d] = f32_to_bf16_rne(v);
    }
  }
  return skipped;
}
