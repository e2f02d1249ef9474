/*
 * oracle.c -- plain fp64 CPU oracle for paged mixed-length decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path calls, links or
 * loads this file: only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header, table or helper with the
 * CUDA library.
 *
 * What it computes (the plain definitions the fast path must reproduce):
 *   - decode attention over a paged KV cache: for sequence b and query head h
 *     (KV head g = h / G), o = sum_j softmax_j(scale * <q, K_b[j,g]>) V_b[j,g]
 *     over the sequence's live tokens, K_b[j,g] being row j mod 64 of physical
 *     page page_table[b][j / 64].  (xiaodao.ai "HPC-Ops TPOT -48.8%", Attention
 *     section: KV cut into 64-token tiles; bitbyai.com "vLLM x HPC-Ops",
 *     Attention Backend: the schedule changes only where work runs, so the
 *     result is the unsplit softmax.)
 *   - a partial over a token range and the log-sum-exp merge of partials
 *     (the split-KV decomposition named in the xiaodao.ai Attention section);
 *   - RMSNorm of q/k per head, rotate-half RoPE, and the KV slot write of the
 *     fused prologue (bitbyai.com, Attention Backend: "RoPE, query-key
 *     normalization, and KV-write" fused into a prologue);
 *   - the OCP FP8 E4M3FN codec and a per-(page, kv-head) amax quantiser for
 *     FP8 caches (aipuzi.cn HPC-Ops, section 2.3: native BF16/FP8);
 *   - the tile planner: the global list of (sequence, kv-head, tile) units
 *     spread over CTAs (xiaodao.ai Attention section: 64-token tiles spread as
 *     evenly as possible over persistent CTAs), and the two static split-KV
 *     plans it is compared with (same section: fixed split count, or fixed
 *     split size with the grid reserved for the longest request).
 *
 * Everything is fp64 (bf16 and e4m3 inputs convert to fp64 exactly), written
 * as straight loops in the order of the definitions.  OpenMP only spreads
 * independent (sequence, head) outputs over host threads; it never reorders
 * a sum.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_OK = 0, ORC_BAD_ARG = 1, ORC_BAD_PAGE = 2 };

/* ------------------------------------------------------------------ */
/* bf16                                                                */
/* ------------------------------------------------------------------ */

/* bf16 bit pattern -> fp64, exact (bf16 is the top half of an fp32). */
double oracle_bf16_to_f64(uint16_t bits) {
  uint32_t u = (uint32_t)bits << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* fp64 -> bf16 bit pattern, round to nearest, ties to even.
 * bf16: 8 exponent bits (bias 127), 7 stored mantissa bits, subnormals down to
 * 2^-133.  The value is scaled so its rounding quantum is 1, rounded with
 * rint() (ties-to-even in the default rounding mode), and scaled back. */
uint16_t oracle_bf16_from_f64(double x) {
  if (isnan(x)) return 0x7FC0;
  uint16_t sign = signbit(x) ? 0x8000 : 0;
  double ax = fabs(x);
  if (isinf(ax)) return sign | 0x7F80;
  if (ax == 0.0) return sign;
  int ex;
  frexp(ax, &ex);                    /* ax = f * 2^ex, f in [0.5, 1) */
  int lead = ex - 1;                 /* exponent of the leading bit */
  int qexp = lead - 7;               /* 7 mantissa bits below the leading one */
  if (qexp < -133) qexp = -133;      /* subnormal quantum */
  double n = rint(ldexp(ax, -qexp));
  double y = ldexp(n, qexp);
  if (y >= ldexp(1.0, 128)) return sign | 0x7F80; /* overflow to inf */
  float yf = (float)y;                /* exact: y is a bf16 value */
  uint32_t u;
  memcpy(&u, &yf, sizeof u);
  return sign | (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------ */
/* OCP FP8 E4M3FN: 1 sign, 4 exponent (bias 7), 3 mantissa bits; no      */
/* infinities; S.1111.111 is NaN; max finite 448; subnormals m * 2^-9.   */
/* ------------------------------------------------------------------ */

double oracle_e4m3_decode(uint8_t code) {
  int s = code >> 7, e = (code >> 3) & 0xF, m = code & 7;
  double v;
  if (e == 0xF && m == 7) return NAN;
  if (e == 0)
    v = ldexp((double)m, -9);
  else
    v = ldexp(1.0 + m / 8.0, e - 7);
  return s ? -v : v;
}

/* Round to nearest even, saturating to +-448 (satfinite); NaN -> 0x7F. */
uint8_t oracle_e4m3_encode(double x) {
  if (isnan(x)) return 0x7F;
  uint8_t sign = signbit(x) ? 0x80 : 0;
  double ax = fabs(x);
  if (ax == 0.0) return sign;
  double y;
  if (isinf(ax)) {
    y = 448.0;
  } else {
    int ex;
    frexp(ax, &ex);
    int lead = ex - 1;
    int qexp = lead - 3;            /* 3 mantissa bits */
    if (qexp < -9) qexp = -9;       /* subnormal quantum 2^-9 */
    y = ldexp(rint(ldexp(ax, -qexp)), qexp);
    if (y > 448.0) y = 448.0;
  }
  if (y == 0.0) return sign;
  if (y < ldexp(1.0, -6)) {          /* subnormal: m * 2^-9, m in 1..7 */
    int m = (int)ldexp(y, 9);
    return sign | (uint8_t)m;
  }
  int ex;
  frexp(y, &ex);
  int lead = ex - 1;                 /* -6 .. 8 */
  int m = (int)((ldexp(y, -lead) - 1.0) * 8.0);
  return sign | (uint8_t)(((lead + 7) << 3) | m);
}

/* Per-(page, kv-head) FP8 quantiser for a cache given as fp32 values
 * [num_pages][Hkv][page_size][D].  live[p] = live tokens of page p.
 * scale = fp32(amax / 448) over the live tokens of that (page, kv-head)
 * (amax == 0 -> scale 1); code = encode(value / scale); dead slots get
 * dead_code. */
void oracle_quantize_kv_e4m3(const float* values, const int32_t* live, int num_pages,
                             int num_kv_heads, int page_size, int head_dim,
                             uint8_t dead_code, uint8_t* codes, float* scales) {
#pragma omp parallel for schedule(static)
  for (long pg = 0; pg < (long)num_pages * num_kv_heads; ++pg) {
    long p = pg / num_kv_heads;
    const float* blk = values + pg * (long)page_size * head_dim;
    uint8_t* out = codes + pg * (long)page_size * head_dim;
    int nlive = live[p];
    double amax = 0.0;
    for (int t = 0; t < nlive; ++t)
      for (int d = 0; d < head_dim; ++d) {
        double a = fabs((double)blk[(long)t * head_dim + d]);
        if (a > amax) amax = a;
      }
    float sc = amax > 0.0 ? (float)(amax / 448.0) : 1.0f;
    scales[pg] = sc;
    for (int t = 0; t < page_size; ++t)
      for (int d = 0; d < head_dim; ++d) {
        long i = (long)t * head_dim + d;
        out[i] = t < nlive ? oracle_e4m3_encode((double)blk[i] / (double)sc) : dead_code;
      }
  }
}

/* ------------------------------------------------------------------ */
/* Prologue pieces (bitbyai.com "vLLM x HPC-Ops", Attention Backend)     */
/* ------------------------------------------------------------------ */

/* RMSNorm over one head vector: y_i = x_i / sqrt(mean_k x_k^2 + eps) * gamma_i */
void oracle_rmsnorm(const double* x, const double* gamma, int n, double eps, double* y) {
  double ss = 0.0;
  for (int i = 0; i < n; ++i) ss += x[i] * x[i];
  double r = 1.0 / sqrt(ss / n + eps);
  for (int i = 0; i < n; ++i) y[i] = x[i] * r * gamma[i];
}

/* Rotary embedding, rotate-half pairing over the full head:
 * for i < D/2, w_i = theta^(-2i/D), phi = pos * w_i,
 *   y_i       = x_i cos phi - x_{i+D/2} sin phi
 *   y_{i+D/2} = x_{i+D/2} cos phi + x_i sin phi */
void oracle_rope(const double* x, int n, double pos, double theta, double* y) {
  int h = n / 2;
  for (int i = 0; i < h; ++i) {
    double w = pow(theta, -2.0 * i / n);
    double phi = pos * w;
    double c = cos(phi), s = sin(phi);
    y[i] = x[i] * c - x[i + h] * s;
    y[i + h] = x[i + h] * c + x[i] * s;
  }
}

/* Fused prologue for one decode step, on host copies of the caches.
 * Per sequence b with position pos = positions[b] (the pre-append length):
 *   q_h <- RoPE(RMSNorm(q_raw_h; gq), pos) for every query head (fp64 out),
 *   k_g <- RoPE(RMSNorm(k_raw_g; gk), pos), rounded to bf16 and written,
 *   v_g  = v_raw_g written unchanged,
 * into slot (page_table[b][pos / page_size], g, pos % page_size). */
int oracle_prologue(const uint16_t* q_raw, const uint16_t* k_raw, const uint16_t* v_raw,
                    const float* q_gamma, const float* k_gamma, double eps, double theta,
                    const int32_t* positions, const int32_t* page_table, int pt_stride,
                    uint16_t* k_cache, uint16_t* v_cache, double* q_out, int B, int Hq,
                    int Hkv, int D, int page_size, int num_pages) {
  if (D <= 0 || D % 2 || Hq <= 0 || Hkv <= 0 || page_size <= 0) return ORC_BAD_ARG;
  double* gq = malloc(sizeof(double) * D);
  double* gk = malloc(sizeof(double) * D);
  double* x = malloc(sizeof(double) * D);
  double* t = malloc(sizeof(double) * D);
  double* y = malloc(sizeof(double) * D);
  int rc = ORC_OK;
  for (int i = 0; i < D; ++i) {
    gq[i] = q_gamma[i];
    gk[i] = k_gamma[i];
  }
  for (int b = 0; b < B && rc == ORC_OK; ++b) {
    int pos = positions[b];
    for (int h = 0; h < Hq; ++h) {
      const uint16_t* src = q_raw + ((long)b * Hq + h) * D;
      for (int i = 0; i < D; ++i) x[i] = oracle_bf16_to_f64(src[i]);
      oracle_rmsnorm(x, gq, D, eps, t);
      oracle_rope(t, D, (double)pos, theta, y);
      memcpy(q_out + ((long)b * Hq + h) * D, y, sizeof(double) * D);
    }
    if (pos < 0 || pos / page_size >= pt_stride) { rc = ORC_BAD_ARG; break; }
    int page = page_table[(long)b * pt_stride + pos / page_size];
    if (page < 0 || page >= num_pages) { rc = ORC_BAD_PAGE; break; }
    int slot = pos % page_size;
    for (int g = 0; g < Hkv; ++g) {
      const uint16_t* ks = k_raw + ((long)b * Hkv + g) * D;
      const uint16_t* vs = v_raw + ((long)b * Hkv + g) * D;
      long dst = (((long)page * Hkv + g) * page_size + slot) * D;
      for (int i = 0; i < D; ++i) x[i] = oracle_bf16_to_f64(ks[i]);
      oracle_rmsnorm(x, gk, D, eps, t);
      oracle_rope(t, D, (double)pos, theta, y);
      for (int i = 0; i < D; ++i) {
        k_cache[dst + i] = oracle_bf16_from_f64(y[i]);
        v_cache[dst + i] = vs[i];
      }
    }
  }
  free(gq); free(gk); free(x); free(t); free(y);
  return rc;
}

/* ------------------------------------------------------------------ */
/* Paged decode attention                                              */
/* ------------------------------------------------------------------ */

typedef struct {
  const void* k_cache;
  const void* v_cache;
  int kv_fp8;               /* 0: bf16 bits, 1: e4m3 codes */
  const float* k_scale;     /* [num_pages][Hkv] (fp8 only) */
  const float* v_scale;
  const int32_t* page_table;
  int pt_stride;
  int Hkv, D, page_size, num_pages;
} orc_cache;

/* Element d of token j of sequence b, kv head g, K (which = 0) or V (1), in
 * fp64.  Returns 0 and sets *ok = 0 if the page id is out of range. */
static double cache_elem(const orc_cache* c, int b, int g, long j, int d, int which, int* ok) {
  int page = c->page_table[(long)b * c->pt_stride + j / c->page_size];
  if (page < 0 || page >= c->num_pages) { *ok = 0; return 0.0; }
  long idx = (((long)page * c->Hkv + g) * c->page_size + j % c->page_size) * c->D + d;
  const void* base = which ? c->v_cache : c->k_cache;
  if (!c->kv_fp8) return oracle_bf16_to_f64(((const uint16_t*)base)[idx]);
  const float* sc = which ? c->v_scale : c->k_scale;
  return oracle_e4m3_decode(((const uint8_t*)base)[idx]) * (double)sc[(long)page * c->Hkv + g];
}

/* Partial attention of one (b, h) over tokens [t0, t1):
 *   m = max_j s_j, l = sum_j exp(s_j - m), acc = sum_j exp(s_j - m) v_j
 * with s_j = scale * <q, k_j>.  Natural-exp units.  Empty range -> m = -inf,
 * l = 0, acc = 0. */
static int partial_one(const orc_cache* c, const double* q, int b, int g, long t0, long t1,
                       double scale, double* s_buf, double* acc, double* m_out, double* l_out) {
  int ok = 1;
  int D = c->D;
  double m = -INFINITY;
  for (long j = t0; j < t1; ++j) {
    double dot = 0.0;
    for (int d = 0; d < D; ++d) dot += q[d] * cache_elem(c, b, g, j, d, 0, &ok);
    s_buf[j - t0] = scale * dot;
    if (s_buf[j - t0] > m) m = s_buf[j - t0];
  }
  double l = 0.0;
  for (int d = 0; d < D; ++d) acc[d] = 0.0;
  for (long j = t0; j < t1; ++j) {
    double w = exp(s_buf[j - t0] - m);
    l += w;
    for (int d = 0; d < D; ++d) acc[d] += w * cache_elem(c, b, g, j, d, 1, &ok);
  }
  *m_out = m;
  *l_out = l;
  return ok ? ORC_OK : ORC_BAD_PAGE;
}

static void load_q(const uint16_t* q16, const double* q64, long off, int D, double* q) {
  for (int d = 0; d < D; ++d) q[d] = q64 ? q64[off + d] : oracle_bf16_to_f64(q16[off + d]);
}

/* Multi-token decode attention (speculative / multi-token-prediction decode:
 * T new query tokens per sequence, already appended to the cache, causal
 * among themselves).  Query token i of sequence b sits at position
 * L_b - T + i and attends to positions [0, L_b - T + i], i.e. it is the
 * single-token decode of that query over the first L_b - T + i + 1 tokens.
 * For the sequences listed in rows[0..n_rows) (all B if rows is NULL); q is
 * [B][T][Hq][D] as bf16 bits (q16) or fp64 (q64); out is [B][T][Hq][D] fp64.
 * A query that sees no token (L_b - T + i + 1 <= 0, e.g. an empty sequence)
 * gets a zero output (softmax over an empty set is undefined; zero is this
 * library's convention). */
int oracle_paged_decode_multi(const uint16_t* q16, const double* q64, const void* k_cache,
                              const void* v_cache, int kv_fp8, const float* k_scale,
                              const float* v_scale, const int32_t* page_table, int pt_stride,
                              const int32_t* seq_lens, int B, int T, int Hq, int Hkv, int D,
                              int page_size, int num_pages, double scale, const int32_t* rows,
                              int n_rows, double* out, int num_threads) {
  if (Hkv <= 0 || Hq % Hkv || D <= 0 || page_size <= 0 || T <= 0) return ORC_BAD_ARG;
  orc_cache c = {k_cache, v_cache, kv_fp8, k_scale, v_scale, page_table, pt_stride,
                 Hkv, D, page_size, num_pages};
  int G = Hq / Hkv;
  int nr = rows ? n_rows : B;
  long total = (long)nr * T * Hq;
  int rc = ORC_OK;
#ifdef _OPENMP
  if (num_threads > 0) omp_set_num_threads(num_threads);
#endif
#pragma omp parallel
  {
    long maxL = 0;
    for (int r = 0; r < nr; ++r) {
      int b = rows ? rows[r] : r;
      if (seq_lens[b] > maxL) maxL = seq_lens[b];
    }
    double* s_buf = malloc(sizeof(double) * (maxL > 0 ? maxL : 1));
    double* q = malloc(sizeof(double) * D);
    double* acc = malloc(sizeof(double) * D);
#pragma omp for schedule(dynamic, 1)
    for (long it = 0; it < total; ++it) {
      int b = rows ? rows[it / ((long)T * Hq)] : (int)(it / ((long)T * Hq));
      int i = (int)(it / Hq % T);
      int h = (int)(it % Hq);
      int g = h / G;
      long L = seq_lens[b];
      long row = ((long)b * T + i) * Hq + h;
      double* o = out + row * D;
      long Li = L - T + i + 1; /* tokens this query sees */
      if (L > 0 && (L + page_size - 1) / page_size > pt_stride) {
        for (int d = 0; d < D; ++d) o[d] = 0.0;
#pragma omp atomic write
        rc = ORC_BAD_ARG;
        continue;
      }
      if (Li <= 0) {
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        continue;
      }
      load_q(q16, q64, row * D, D, q);
      double m, l;
      int e = partial_one(&c, q, b, g, 0, Li, scale, s_buf, acc, &m, &l);
      if (e != ORC_OK) {
#pragma omp atomic write
        rc = e;
      }
      for (int d = 0; d < D; ++d) o[d] = acc[d] / l;
    }
    free(s_buf); free(q); free(acc);
  }
  return rc;
}

/* Decode attention of one query token per sequence: the T = 1 case above.
 * q and out are [B][Hq][D]. */
int oracle_paged_decode(const uint16_t* q16, const double* q64, const void* k_cache,
                        const void* v_cache, int kv_fp8, const float* k_scale,
                        const float* v_scale, const int32_t* page_table, int pt_stride,
                        const int32_t* seq_lens, int B, int Hq, int Hkv, int D, int page_size,
                        int num_pages, double scale, const int32_t* rows, int n_rows,
                        double* out, int num_threads) {
  return oracle_paged_decode_multi(q16, q64, k_cache, v_cache, kv_fp8, k_scale, v_scale,
                                   page_table, pt_stride, seq_lens, B, 1, Hq, Hkv, D, page_size,
                                   num_pages, scale, rows, n_rows, out, num_threads);
}

/* Partial (acc[D], m, l) of one (b, h) over tokens [t0, t1). */
int oracle_partial(const uint16_t* q16, const double* q64, const void* k_cache,
                   const void* v_cache, int kv_fp8, const float* k_scale, const float* v_scale,
                   const int32_t* page_table, int pt_stride, int Hq, int Hkv, int D,
                   int page_size, int num_pages, double scale, int b, int h, long t0, long t1,
                   double* acc, double* m, double* l) {
  if (Hkv <= 0 || Hq % Hkv || t1 < t0) return ORC_BAD_ARG;
  orc_cache c = {k_cache, v_cache, kv_fp8, k_scale, v_scale, page_table, pt_stride,
                 Hkv, D, page_size, num_pages};
  double* q = malloc(sizeof(double) * D);
  double* s_buf = malloc(sizeof(double) * (t1 > t0 ? t1 - t0 : 1));
  load_q(q16, q64, ((long)b * Hq + h) * D, D, q);
  int rc = partial_one(&c, q, b, h / (Hq / Hkv), t0, t1, scale, s_buf, acc, m, l);
  free(q); free(s_buf);
  return rc;
}

/* Log-sum-exp merge of n partials (acc_i[D], m_i, l_i), folded in index order:
 *   M = max_i m_i, Lambda = sum_i l_i e^{m_i - M}, o = sum_i acc_i e^{m_i - M} / Lambda.
 * A partial with m_i = -inf (empty range) contributes nothing. */
void oracle_lse_merge(const double* acc, const double* m, const double* l, int n, int D,
                      double* out) {
  double M = -INFINITY;
  for (int i = 0; i < n; ++i)
    if (m[i] > M) M = m[i];
  double lam = 0.0;
  for (int d = 0; d < D; ++d) out[d] = 0.0;
  for (int i = 0; i < n; ++i) {
    if (m[i] == -INFINITY) continue;
    double w = exp(m[i] - M);
    lam += l[i] * w;
    for (int d = 0; d < D; ++d) out[d] += acc[(long)i * D + d] * w;
  }
  for (int d = 0; d < D; ++d) out[d] /= lam;
}

/* ------------------------------------------------------------------ */
/* Tile planner (xiaodao.ai "HPC-Ops TPOT -48.8%", Attention section)   */
/* ------------------------------------------------------------------ */
/*
 * A unit is one (sequence b, kv head g, 64-token tile t).  The global list
 * orders units by b, then g, then t.  A "segment" is the run of units of one
 * (b, g).  Three plans give every CTA a contiguous range of that list:
 *
 *   kind 0, dynamic: P persistent CTAs.  If U <= P, CTA c < U takes unit c
 *     and the rest take nothing.  Otherwise the unit list is spread as evenly
 *     as possible over P primary ranges, except for a tail of Ut units that
 *     is spread as evenly as possible over M smaller chunks which CTAs take
 *     at run time as they finish (bitbyai.com "vLLM x HPC-Ops", Attention
 *     Backend: progress is evaluated dynamically).  The pages fix the even
 *     spread but not the size of the tail, so this is a FAMILY of plans with
 *     three parameters given by the caller: the tail divisor den, the chunks
 *     per CTA k and the least units per CTA mn for a tail.  If den > 0 and
 *     U >= mn P, Ut = min(floor(U / den), U - P) (every primary range keeps
 *     at least one unit); otherwise there is no tail, Ut = 0.  M = min(k P, Ut).
 *     With U1 = U - Ut, range P + j is [U1 + floor(j Ut / M),
 *     U1 + floor((j+1) Ut / M)).  The P primary ranges split the first U1
 *     units so that each carries an even share of their cost, two more
 *     parameters of the family: every unit costs q (unit_cost) and the last
 *     unit of each segment e (end_cost) more.  With K(x) the summed cost of
 *     units [0, x), primary range c starts at the largest x <= U1 with
 *     P K(x) <= c K(U1), and ends where range c + 1 starts (range P - 1 at
 *     U1).  The weights apply only if K(U1) >= (q + e) P, so that no primary
 *     range is empty; otherwise, and always with e = 0, range c is
 *     [floor(c U1 / P), floor((c+1) U1 / P)) -- with den = 0 too, the plain
 *     even partition [floor(c U / P), floor((c+1) U / P)).  Grid = P;
 *     V = P + M ranges.
 *   kind 1, static fixed split count S (param, default ceil(P / (B Hkv))):
 *     one CTA per (segment, split i); each segment's n tiles cut into
 *     chunks of ceil(n / S) tiles, chunk i = [i C, min((i+1) C, n)).
 *     Grid = B * Hkv * S.
 *   kind 2, static fixed split size C tiles (param, default
 *     ceil(T_max / ceil(P / Hkv)) with T_max = ceil(max_seq_len / 64)):
 *     NC = ceil(T_max / C) chunks reserved for every segment, as if every
 *     sequence were the longest; chunk i = [i C, min((i+1) C, n)), empty past
 *     the segment's end.  Grid = B * Hkv * NC.
 *   kind 3, length-aware with smallest piece m tiles (param, default 4): the
 *     ranges of kind 0 with every range end moved by snap_cut, so that a
 *     segment of fewer than 2m tiles is never cut and the first and last
 *     pieces of a cut segment have at least m tiles (cuts further inside
 *     stay, so the ranges holding a segment remain consecutive).  Grid = P.
 *
 * For each range the plan records (u_begin, u_end).  A segment whose units
 * lie in more than one range is computed in pieces, one per range, each
 * leaving a partial (acc, m, l) that a log-sum-exp merge combines; the piece
 * a range holds of its first segment goes to partial slot 2c, that of its
 * last segment to slot 2c + 1 (a segment strictly inside a range is whole
 * there).  For each segment the plan records split_count (ranges holding
 * its units) and first_slot (the slot of its first piece, -1 if the
 * segment is not split).  The static kinds have one range per CTA (V =
 * grid).
 *
 * This implementation enumerates every unit explicitly and assigns it, then
 * counts; it does not use any closed form.
 */
long oracle_plan_grid(int kind, int B, int Hkv, int num_ctas, int param, int max_seq_len,
                      int page_size) {
  if (kind == 0 || kind == 3) return num_ctas;
  if (kind == 1) {
    long S = param > 0 ? param : (num_ctas + (long)B * Hkv - 1) / ((long)B * Hkv);
    if (S < 1) S = 1;
    return (long)B * Hkv * S;
  }
  long tmax = (max_seq_len + page_size - 1) / page_size;
  long per_seg = (num_ctas + Hkv - 1) / Hkv;
  long C = param > 0 ? param : (tmax + per_seg - 1) / per_seg;
  if (C < 1) C = 1;
  long NC = (tmax + C - 1) / C;
  if (NC < 1) NC = 1;
  return (long)B * Hkv * NC;
}

/* Length-aware plan (bitbyai.com "vLLM x HPC-Ops", Attention Backend: short
 * requests finish first, long ones are spread over the grid): the cut point
 * x between units x-1 and x.  If x lies strictly inside a segment of n tiles,
 * a = tiles of the segment before x, r = n - a after it.  When a < m or
 * r < m the cut moves to the segment's start (a <= r) or end (a > r);
 * otherwise it stays. */
static long snap_cut(long x, long U, long m, const int32_t* unit_seg, const int32_t* unit_tile,
                     const long* ntile, int Hkv) {
  if (x <= 0 || x >= U) return x;
  long a = unit_tile[x];
  if (a == 0) return x; /* already between two segments */
  long n = ntile[unit_seg[x] / Hkv];
  long r = n - a;
  if (a < m || r < m) return a <= r ? x - a : x + r;
  return x;
}

int oracle_plan(const int32_t* seq_lens, int B, int Hkv, int page_size, int capacity_tokens,
                int kind, int num_ctas, int param, int max_seq_len, int tail_den,
                int tail_chunks, int tail_min, int unit_cost, int end_cost, int32_t* lens_out,
                int32_t* tile_start, int32_t* cta_desc /* [<= 5*grid][2] */,
                int32_t* split_count /* [B*Hkv] */, int32_t* first_slot /* [B*Hkv] */,
                int32_t* n_units_out, int32_t* n_ranges_out) {
  if (B <= 0 || Hkv <= 0 || page_size <= 0 || num_ctas <= 0 || kind < 0 || kind > 3)
    return ORC_BAD_ARG;
  if (tail_den < 0 || tail_chunks < 1 || tail_min < 0 || unit_cost < 1 || end_cost < 0)
    return ORC_BAD_ARG;
  long grid = oracle_plan_grid(kind, B, Hkv, num_ctas, param, max_seq_len, page_size);
  int S = B * Hkv;
  /* 1. lengths clamped to [0, capacity], tiles per sequence, tile offsets */
  long* ntile = calloc(B, sizeof(long));
  tile_start[0] = 0;
  for (int b = 0; b < B; ++b) {
    long L = seq_lens[b];
    if (L < 0) L = 0;
    if (L > capacity_tokens) L = capacity_tokens;
    lens_out[b] = (int32_t)L;
    ntile[b] = (L + page_size - 1) / page_size;
    tile_start[b + 1] = (int32_t)(tile_start[b] + ntile[b]);
  }
  /* 2. enumerate the global unit list: unit -> segment */
  long U = (long)tile_start[B] * Hkv;
  *n_units_out = (int32_t)U;
  int32_t* unit_seg = malloc(sizeof(int32_t) * (U > 0 ? U : 1));
  int32_t* unit_tile = malloc(sizeof(int32_t) * (U > 0 ? U : 1));
  long* seg_first_unit = malloc(sizeof(long) * S);
  long u = 0;
  for (int b = 0; b < B; ++b)
    for (int g = 0; g < Hkv; ++g) {
      seg_first_unit[b * Hkv + g] = u;
      for (long t = 0; t < ntile[b]; ++t) {
        unit_seg[u] = b * Hkv + g;
        unit_tile[u] = (int32_t)t;
        ++u;
      }
    }
  /* 3. ranges */
  long nranges = grid;
  long* beg = malloc(sizeof(long) * grid * 5);
  long* end = malloc(sizeof(long) * grid * 5);
  if (kind == 0 || kind == 3) {
    long P = num_ctas;
    if (U <= P) {
      for (long c = 0; c < P; ++c) {
        beg[c] = c < U ? c : U;
        end[c] = c < U ? c + 1 : U;
      }
    } else {
      long Ut = 0; /* tail units: none when den = 0 or U < mn P */
      if (tail_den > 0 && U >= (long)tail_min * P) Ut = U / tail_den < U - P ? U / tail_den : U - P;
      long U1 = U - Ut;
      long M = (long)tail_chunks * P < Ut ? (long)tail_chunks * P : Ut;
      /* K[x] = cost of units [0, x): q per unit, e more for a segment's last */
      long* K = malloc(sizeof(long) * (U1 + 1));
      K[0] = 0;
      for (long x = 0; x < U1; ++x) {
        int last = (x + 1 == U) || unit_seg[x + 1] != unit_seg[x];
        K[x + 1] = K[x] + unit_cost + (last ? end_cost : 0);
      }
      if (end_cost > 0 && K[U1] >= (long)(unit_cost + end_cost) * P) {
        /* start of range c: the largest x <= U1 with P K[x] <= c K[U1]; the
         * starts do not decrease in c, so one forward scan finds them all */
        long x = 0;
        for (long c = 0; c <= P; ++c) {
          while (x < U1 && P * K[x + 1] <= c * K[U1]) ++x;
          if (c < P) beg[c] = x;
          if (c > 0) end[c - 1] = x;
        }
      } else {
        for (long c = 0; c < P; ++c) {
          beg[c] = c * U1 / P;
          end[c] = (c + 1) * U1 / P;
        }
      }
      free(K);
      for (long j = 0; j < M; ++j) {
        beg[P + j] = U1 + j * Ut / M;
        end[P + j] = U1 + (j + 1) * Ut / M;
      }
      nranges = P + M;
    }
  } else {
    long per = grid / S; /* chunks reserved per segment */
    for (int s = 0; s < S; ++s) {
      long n = ntile[s / Hkv];
      long C;
      if (kind == 1) {
        C = (n + per - 1) / per;
      } else {
        long tmax = (max_seq_len + page_size - 1) / page_size;
        long per_seg = (num_ctas + Hkv - 1) / Hkv;
        C = param > 0 ? param : (tmax + per_seg - 1) / per_seg;
        if (C < 1) C = 1;
      }
      for (long i = 0; i < per; ++i) {
        long t0 = i * C, t1 = (i + 1) * C;
        if (t0 > n) t0 = n;
        if (t1 > n) t1 = n;
        long c = (long)s * per + i;
        beg[c] = seg_first_unit[s] + t0;
        end[c] = seg_first_unit[s] + t1;
      }
    }
  }
  /* 3b. length-aware kind: move every cut point that would leave a piece of
   *     fewer than m tiles to the nearer end of its segment (the start on a
   *     tie).  Every range end is the next range's start, so moving both ends
   *     of every range by the same rule keeps the ranges contiguous. */
  if (kind == 3) {
    long m = param > 0 ? param : 4;
    for (long c = 0; c < nranges; ++c) {
      beg[c] = snap_cut(beg[c], U, m, unit_seg, unit_tile, ntile, Hkv);
      end[c] = snap_cut(end[c], U, m, unit_seg, unit_tile, ntile, Hkv);
    }
  }
  /* 4. walk each range's units: list its segments in order, count the
   *    ranges holding each segment, and give every cut piece its slot */
  int32_t* holders = calloc(S, sizeof(int32_t));
  long* seg_units = calloc(S, sizeof(long)); /* units of each segment */
  for (long v = 0; v < U; ++v) seg_units[unit_seg[v]] += 1;
  for (int s = 0; s < S; ++s) first_slot[s] = -1;
  int32_t* segs = malloc(sizeof(int32_t) * (U > 0 ? U : 1));
  long* held = malloc(sizeof(long) * (U > 0 ? U : 1));
  for (long c = 0; c < nranges; ++c) {
    long nseg = 0;
    for (long v = beg[c]; v < end[c]; ++v) {
      int s = unit_seg[v];
      if (nseg == 0 || segs[nseg - 1] != s) {
        segs[nseg] = s;
        held[nseg] = 0;
        ++nseg;
      }
      held[nseg - 1] += 1;
    }
    for (long i = 0; i < nseg; ++i) {
      int s = segs[i];
      if (holders[s] == 0 && held[i] < seg_units[s]) /* first piece of a cut segment */
        first_slot[s] = (int32_t)(2 * c + (i == 0 ? 0 : 1));
      holders[s] += 1;
    }
    cta_desc[c * 2 + 0] = (int32_t)beg[c];
    cta_desc[c * 2 + 1] = (int32_t)end[c];
  }
  *n_ranges_out = (int32_t)nranges;
  for (int s = 0; s < S; ++s) split_count[s] = holders[s];
  free(seg_units); free(segs); free(held);
  free(ntile); free(unit_seg); free(unit_tile); free(seg_first_unit);
  free(beg); free(end); free(holders);
  return ORC_OK;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
