/*
 * svg_oracle.c — plain, slow fp64 CPU oracle for the Sparse VideoGen attention step.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's
 * cpu_baseline / reference arm may load this library.  It shares no code, header,
 * table or constant with the CUDA library; neither includes or calls the other.
 *
 * Every routine is the textbook definition of its stage, written out with plain
 * loops in double precision (OpenMP only distributes independent rows).
 * Sources (page title, section):
 *   [A] "Sparse VideoGen" WeChat article (dtcms.com repost): sections
 *       "Spatial Head", "Temporal Head", "Online Profiling Strategy",
 *       "硬件高效的 Layout Transformation", "其他优化方法".
 *   [B] "ICML 2025 | 视频生成模型无损加速两倍…" (机器之心 report): sections
 *       "Sparse VideoGen 的核心设计", "动态自适应的稀疏策略" (steps 1-3),
 *       "Layout Transformation + Kernel 加速".
 * The pages give no formulas; where they are silent the plainest reading is
 * taken (RMSNorm y = x / sqrt(mean(x^2) + eps) * gamma; interleaved-pair 3D RoPE
 * over t/h/w sections; boolean masks; masked softmax attention; MSE over the
 * sampled rows).  Each reading is listed in the repository design notes.
 *
 * Parity: every function here is pinned by tests in tests/test_oracle_*.py
 * (closed forms, invariants, brute force on tiny inputs, numpy textbook routes).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
  int B, H, L, d;   /* batch, heads, sequence length, head dim            */
  int F, Hs, Ws;    /* latent frames and per-frame spatial grid           */
  int T;            /* text tokens, stored after the F*Hs*Ws video tokens */
} ora_shape;

typedef struct {
  int w;            /* spatial window: keep keys with |frame delta| <= w          */
  int r;            /* temporal radius: keep keys with |spatial-index delta| <= r */
  int bq, bk;       /* tile sizes of the block list (query rows, key columns)    */
  double eps;       /* RMSNorm epsilon                                            */
  double base;      /* RoPE base                                                  */
  double scale;     /* softmax scale (1/sqrt(d) unless given)                     */
  int split[3];     /* RoPE widths of the t, h, w sections (sum = d)              */
} ora_params;

enum { ORA_SPATIAL = 0, ORA_TEMPORAL = 1, ORA_DENSE = 2 };

/* ---------------------------------------------------------------- bf16 ---- */

double ora_bf16_to_f64(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* Round a double to the nearest bfloat16 (ties to even), computed on the
 * double itself: bf16 keeps 8 significant bits and fp32's exponent range. */
uint16_t ora_f64_to_bf16(double x) {
  if (isnan(x)) return 0x7FC0;
  double ax = fabs(x);
  double r;
  if (ax < ldexp(1.0, -126)) {
    /* bf16 subnormal range: spacing 2^-133, round half to even */
    r = nearbyint(ldexp(x, 133));
    r = ldexp(r, -133);
  } else {
    int e;
    double m = frexp(x, &e);          /* x = m * 2^e, 0.5 <= |m| < 1 */
    double s = ldexp(m, 8);            /* 8 significant bits          */
    double t = nearbyint(s);           /* default mode: ties to even  */
    r = ldexp(t, e - 8);
  }
  if (fabs(r) > 3.3895313892515355e38) r = copysign(INFINITY, x);
  float f = (float)r;                  /* exact: r has <= 8 significant bits */
  uint32_t u;
  memcpy(&u, &f, 4);
  return (uint16_t)(u >> 16);
}

void ora_round_bf16(int64_t n, const double* x, uint16_t* y) {
  for (int64_t i = 0; i < n; i++) y[i] = ora_f64_to_bf16(x[i]);
}

/* ------------------------------------------------------- token geometry ---- */

static int64_t video_len(const ora_shape* s) { return (int64_t)s->F * s->Hs * s->Ws; }

/* Position of frame-major token i in the head's layout.  Temporal heads use the
 * token-major order (all frames of one spatial location are adjacent), [A]
 * "硬件高效的 Layout Transformation", [B] "Layout Transformation + Kernel 加速":
 * video token f*S+s moves to s*F+f.  Text tokens and other heads stay put. */
int64_t ora_perm(const ora_shape* sh, int kind, int64_t i) {
  int64_t S = (int64_t)sh->Hs * sh->Ws, Lv = video_len(sh);
  if (kind != ORA_TEMPORAL || i >= Lv) return i;
  int64_t f = i / S, s = i % S;
  return s * sh->F + f;
}

/* Inverse of ora_perm: frame-major index of the token at layout position p. */
int64_t ora_perm_inv(const ora_shape* sh, int kind, int64_t p) {
  int64_t S = (int64_t)sh->Hs * sh->Ws, Lv = video_len(sh);
  if (kind != ORA_TEMPORAL || p >= Lv) return p;
  int64_t s = p / sh->F, f = p % sh->F;
  return f * S + s;
}

/* Boolean attention mask on frame-major indices ([A] "Spatial Head",
 * "Temporal Head"; [B] "Sparse VideoGen 的核心设计"):
 *   text query or text key -> kept;
 *   spatial head  -> kept iff the frames differ by at most w;
 *   temporal head -> kept iff the spatial indices s = y*Ws + x differ by at most r;
 *   dense         -> kept. */
int ora_keep(const ora_shape* sh, const ora_params* pr, int kind, int64_t q, int64_t k) {
  int64_t S = (int64_t)sh->Hs * sh->Ws, Lv = video_len(sh);
  if (q >= Lv || k >= Lv) return 1;
  if (kind == ORA_SPATIAL) {
    int64_t df = q / S - k / S;
    if (df < 0) df = -df;
    return df <= pr->w;
  }
  if (kind == ORA_TEMPORAL) {
    int64_t ds = q % S - k % S;
    if (ds < 0) ds = -ds;
    return ds <= pr->r;
  }
  return 1;
}

/* ----------------------------------------------------- QK-Norm + 3D RoPE ---- */

/* One row: RMSNorm then (video rows only) 3D RoPE, all in double.
 * [A] "其他优化方法" and [B] "Layout Transformation + Kernel 加速" name the two
 * operations (QK-Norm, RoPE) without formulas; the textbook forms are used:
 *   y_c = x_c / sqrt(mean_c x_c^2 + eps) * gamma_c
 *   for section a in (t, h, w) with width n_a, offset o_a, position p_a in (f, y, x):
 *     theta_j = p_a * base^(-2j/n_a),  j < n_a/2
 *     (y[o_a+2j], y[o_a+2j+1]) <- rotation of that pair by theta_j. */
void ora_norm_rope_row(const ora_shape* sh, const ora_params* pr, int64_t token,
                       const uint16_t* x, const float* gamma, double* y) {
  int d = sh->d;
  double ss = 0.0;
  for (int c = 0; c < d; c++) {
    double v = ora_bf16_to_f64(x[c]);
    ss += v * v;
  }
  double inv = 1.0 / sqrt(ss / d + pr->eps);
  for (int c = 0; c < d; c++) y[c] = ora_bf16_to_f64(x[c]) * inv * (double)gamma[c];
  if (token >= video_len(sh)) return;  /* text rows carry no RoPE */
  int64_t S = (int64_t)sh->Hs * sh->Ws;
  int64_t f = token / S, s = token % S;
  int64_t pos[3] = {f, s / sh->Ws, s % sh->Ws};
  int off = 0;
  for (int a = 0; a < 3; a++) {
    int n = pr->split[a];
    for (int j = 0; j < n / 2; j++) {
      double theta = (double)pos[a] * pow(pr->base, -2.0 * j / n);
      double c = cos(theta), sn = sin(theta);
      double u = y[off + 2 * j], v = y[off + 2 * j + 1];
      y[off + 2 * j] = u * c - v * sn;
      y[off + 2 * j + 1] = u * sn + v * c;
    }
    off += n;
  }
}

/* Rows given by global index g = (b*H + h)*L + token of a [B,H,L,d] tensor;
 * rows == NULL means all B*H*L rows in order.  Output fp64 [nrows][d]. */
void ora_qknorm_rope_f64(const ora_shape* sh, const ora_params* pr, const uint16_t* x,
                         const float* gamma, int64_t nrows, const int64_t* rows, double* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < nrows; i++) {
    int64_t g = rows ? rows[i] : i;
    ora_norm_rope_row(sh, pr, g % sh->L, x + g * sh->d, gamma, out + i * sh->d);
  }
}

/* Whole tensor, bf16 in -> bf16 out (rounded to nearest even from double). */
void ora_qknorm_rope_bf16(const ora_shape* sh, const ora_params* pr, const uint16_t* x,
                          const float* gamma, uint16_t* out) {
  int64_t nrows = (int64_t)sh->B * sh->H * sh->L;
#pragma omp parallel
  {
    double* y = (double*)malloc(sizeof(double) * sh->d);
#pragma omp for schedule(static)
    for (int64_t g = 0; g < nrows; g++) {
      ora_norm_rope_row(sh, pr, g % sh->L, x + g * sh->d, gamma, y);
      for (int c = 0; c < sh->d; c++) out[g * sh->d + c] = ora_f64_to_bf16(y[c]);
    }
    free(y);
  }
}

/* ------------------------------------------------------------ layout ---- */

/* Applies the head's layout to a [B,H,L,d] bf16 tensor: dst[perm(i)] = src[i].
 * inverse != 0 applies the inverse: dst[i] = src[perm(i)]. */
void ora_layout(const ora_shape* sh, const uint8_t* kinds, int inverse, const uint16_t* src, uint16_t* dst) {
  int64_t L = sh->L, d = sh->d;
  int64_t nbh = (int64_t)sh->B * sh->H;
#pragma omp parallel for schedule(static)
  for (int64_t bh = 0; bh < nbh; bh++) {
    const uint16_t* s = src + bh * L * d;
    uint16_t* t = dst + bh * L * d;
    for (int64_t i = 0; i < L; i++) {
      int64_t p = ora_perm(sh, kinds[bh], i);
      if (!inverse)
        memcpy(t + p * d, s + i * d, sizeof(uint16_t) * d);
      else
        memcpy(t + i * d, s + p * d, sizeof(uint16_t) * d);
    }
  }
}

/* ---------------------------------------------------------- attention ---- */

/* Masked softmax attention of one query row against every key of its head:
 *   o = sum_k softmax_k(scale * q.k | keep) v_k,   lse = log sum_k exp(scale*q.k) over kept k.
 * `layout` = 0: q_tok and key rows are frame-major tokens (the model's order).
 * `layout` = 1: q_tok and key rows are positions in the head's layout and the
 *               mask is evaluated on the frame-major tokens they hold.
 * Returns the number of kept keys. */
int64_t ora_attention_row(const ora_shape* sh, const ora_params* pr, int kind, int layout,
                          const uint16_t* Qh, const uint16_t* Kh, const uint16_t* Vh,
                          int64_t q_tok, double* o, double* lse, double* sbuf) {
  int64_t L = sh->L;
  int d = sh->d;
  const uint16_t* q = Qh + q_tok * d;
  int64_t qi = layout ? ora_perm_inv(sh, kind, q_tok) : q_tok;
  double m = -INFINITY;
  int64_t kept = 0;
  for (int64_t k = 0; k < L; k++) {
    int64_t ki = layout ? ora_perm_inv(sh, kind, k) : k;
    if (!ora_keep(sh, pr, kind, qi, ki)) {
      sbuf[k] = -INFINITY;
      continue;
    }
    const uint16_t* kr = Kh + k * d;
    double s = 0.0;
    for (int c = 0; c < d; c++) s += ora_bf16_to_f64(q[c]) * ora_bf16_to_f64(kr[c]);
    s *= pr->scale;
    sbuf[k] = s;
    if (s > m) m = s;
    kept++;
  }
  for (int c = 0; c < d; c++) o[c] = 0.0;
  if (kept == 0) {
    if (lse) *lse = -INFINITY;
    return 0;
  }
  double l = 0.0;
  for (int64_t k = 0; k < L; k++) {
    if (sbuf[k] == -INFINITY) continue;
    double p = exp(sbuf[k] - m);
    l += p;
    const uint16_t* vr = Vh + k * d;
    for (int c = 0; c < d; c++) o[c] += p * ora_bf16_to_f64(vr[c]);
  }
  for (int c = 0; c < d; c++) o[c] /= l;
  if (lse) *lse = m + log(l);
  return kept;
}

/* Attention for a list of rows.  rows[i] = (b*H + h)*L + token (token in the
 * order given by `layout`); kinds[b*H+h] selects the mask of that head.
 * out: [nrows][d] fp64; lse: [nrows] or NULL; kept: [nrows] or NULL. */
void ora_attention_rows(const ora_shape* sh, const ora_params* pr, const uint8_t* kinds, int layout,
                        const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                        int64_t nrows, const int64_t* rows, double* out, double* lse, int64_t* kept) {
  int64_t L = sh->L, d = sh->d;
#pragma omp parallel
  {
    double* sbuf = (double*)malloc(sizeof(double) * L);
#pragma omp for schedule(dynamic, 4)
    for (int64_t i = 0; i < nrows; i++) {
      int64_t bh = rows[i] / L, tok = rows[i] % L;
      int64_t kk = ora_attention_row(sh, pr, kinds[bh], layout, Q + bh * L * d, K + bh * L * d,
                                     V + bh * L * d, tok, out + i * d, lse ? lse + i : NULL, sbuf);
      if (kept) kept[i] = kk;
    }
    free(sbuf);
  }
}

/* ---------------------------------------------------------- profiling ---- */

/* Online profiling ([A] "Online Profiling Strategy"; [B] "动态自适应的稀疏策略"
 * steps 1-3): for each head, the n sampled query tokens (frame-major video
 * indices, the same set for every head) are attended densely, with the spatial
 * mask and with the temporal mask; the error of each sparse pattern is
 *   MSE_m = (1/(n*d)) * sum_{q in sample} sum_c (O_m[q][c] - O_dense[q][c])^2
 * and the head takes the pattern with the smaller error (spatial on a tie).
 * mse: [B*H][2] = (MSE_spatial, MSE_temporal); choice: [B*H]. */
void ora_profile(const ora_shape* sh, const ora_params* pr, const uint16_t* Qn, const uint16_t* Kn,
                 const uint16_t* V, int n, const int32_t* sample, double* mse, uint8_t* choice) {
  int64_t L = sh->L, d = sh->d;
  int64_t nbh = (int64_t)sh->B * sh->H;
  double* part = (double*)calloc((size_t)(nbh * n * 2), sizeof(double));
#pragma omp parallel
  {
    double* sbuf = (double*)malloc(sizeof(double) * L);
    double* od = (double*)malloc(sizeof(double) * d);
    double* os = (double*)malloc(sizeof(double) * d);
    double* ot = (double*)malloc(sizeof(double) * d);
#pragma omp for schedule(dynamic, 1)
    for (int64_t t = 0; t < nbh * n; t++) {
      int64_t bh = t / n, i = t % n;
      const uint16_t *Qh = Qn + bh * L * d, *Kh = Kn + bh * L * d, *Vh = V + bh * L * d;
      ora_attention_row(sh, pr, ORA_DENSE, 0, Qh, Kh, Vh, sample[i], od, NULL, sbuf);
      ora_attention_row(sh, pr, ORA_SPATIAL, 0, Qh, Kh, Vh, sample[i], os, NULL, sbuf);
      ora_attention_row(sh, pr, ORA_TEMPORAL, 0, Qh, Kh, Vh, sample[i], ot, NULL, sbuf);
      double es = 0.0, et = 0.0;
      for (int c = 0; c < d; c++) {
        es += (os[c] - od[c]) * (os[c] - od[c]);
        et += (ot[c] - od[c]) * (ot[c] - od[c]);
      }
      part[(bh * n + i) * 2 + 0] = es;
      part[(bh * n + i) * 2 + 1] = et;
    }
    free(sbuf); free(od); free(os); free(ot);
  }
  for (int64_t bh = 0; bh < nbh; bh++) {
    double es = 0.0, et = 0.0;
    for (int i = 0; i < n; i++) {
      es += part[(bh * n + i) * 2 + 0];
      et += part[(bh * n + i) * 2 + 1];
    }
    mse[bh * 2 + 0] = es / ((double)n * d);
    mse[bh * 2 + 1] = et / ((double)n * d);
    choice[bh] = (mse[bh * 2 + 0] <= mse[bh * 2 + 1]) ? ORA_SPATIAL : ORA_TEMPORAL;
  }
  free(part);
}

/* -------------------------------------------------------- block list ---- */

/* Brute force over the explicit mask: in the head's layout, the tile
 * (query rows [qb*bq, +bq), key columns [kb*bk, +bk)) is listed iff at least
 * one (query, key) pair in it is kept; `full` is 1 iff every pair is kept.
 * Rows and columns at or beyond L are not part of any tile.  The list of one
 * (b, h, qb) is in ascending kb.  Counts per kind are computed once. */
static void tile_scan(const ora_shape* sh, const ora_params* pr, int kind, int64_t qb, int64_t kb,
                      const int64_t* inv, int* any, int* all) {
  int64_t L = sh->L;
  int64_t q0 = qb * pr->bq, q1 = q0 + pr->bq < L ? q0 + pr->bq : L;
  int64_t k0 = kb * pr->bk, k1 = k0 + pr->bk < L ? k0 + pr->bk : L;
  int a = 0, n = 0;
  for (int64_t q = q0; q < q1; q++) {
    for (int64_t k = k0; k < k1; k++) {
      if (ora_keep(sh, pr, kind, inv[q], inv[k])) a = 1; else n = 1;
      if (a && n) { *any = 1; *all = 0; return; }
    }
  }
  *any = a;
  *all = a && !n;
}

/* Per-kind tile table: flags[qb*nkb + kb] = 0 (not listed), 1 (listed, partial), 3 (listed, full). */
static uint8_t* kind_tiles(const ora_shape* sh, const ora_params* pr, int kind) {
  int64_t L = sh->L;
  int64_t nqb = (L + pr->bq - 1) / pr->bq, nkb = (L + pr->bk - 1) / pr->bk;
  int64_t* inv = (int64_t*)malloc(sizeof(int64_t) * L);
  for (int64_t p = 0; p < L; p++) inv[p] = ora_perm_inv(sh, kind, p);
  uint8_t* flags = (uint8_t*)calloc((size_t)(nqb * nkb), 1);
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t qb = 0; qb < nqb; qb++) {
    for (int64_t kb = 0; kb < nkb; kb++) {
      int any, all;
      tile_scan(sh, pr, kind, qb, kb, inv, &any, &all);
      flags[qb * nkb + kb] = (uint8_t)(any ? (all ? 3 : 1) : 0);
    }
  }
  free(inv);
  return flags;
}

/* CSR over (b, h, qb): row_ptr [B*H*nqb + 1], col [nnz], full [nnz].
 * Pass col == NULL to get only row_ptr (and the return value nnz). */
int64_t ora_block_list(const ora_shape* sh, const ora_params* pr, const uint8_t* kinds,
                       int32_t* row_ptr, int32_t* col, uint8_t* full) {
  int64_t L = sh->L;
  int64_t nqb = (L + pr->bq - 1) / pr->bq, nkb = (L + pr->bk - 1) / pr->bk;
  int64_t nbh = (int64_t)sh->B * sh->H;
  uint8_t* tab[3] = {NULL, NULL, NULL};
  for (int64_t bh = 0; bh < nbh; bh++)
    if (!tab[kinds[bh]]) tab[kinds[bh]] = kind_tiles(sh, pr, kinds[bh]);
  int64_t nnz = 0;
  row_ptr[0] = 0;
  for (int64_t bh = 0; bh < nbh; bh++) {
    const uint8_t* t = tab[kinds[bh]];
    for (int64_t qb = 0; qb < nqb; qb++) {
      for (int64_t kb = 0; kb < nkb; kb++) {
        uint8_t f = t[qb * nkb + kb];
        if (!f) continue;
        if (col) {
          col[nnz] = (int32_t)kb;
          full[nnz] = (uint8_t)(f == 3);
        }
        nnz++;
      }
      row_ptr[bh * nqb + qb + 1] = (int32_t)nnz;
    }
  }
  for (int i = 0; i < 3; i++) free(tab[i]);
  return nnz;
}
