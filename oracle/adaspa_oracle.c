/*
 * adaspa_oracle.c — plain CPU oracle for the blockified, LSE-cached search of
 * AdaSpa ("AdaSpa" abstract: a blockified sparse pattern; "Fused LSE-Cached
 * Search with Head-adaptive Hierarchical Block Sparse Attention"; the sparse
 * pattern and the LSE stay the same across denoising steps).
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's
 * cpu_baseline / reference arm may load this library.  It shares no code, header,
 * table or constant with the CUDA library.
 *
 * The abstract gives the ideas, not the arithmetic.  Readings (also in the
 * design notes):
 *   - the pattern is a set of (query tile, key tile) blocks in the model's
 *     token order, tiles bq x bk;
 *   - the search is exact ("precise") given the cached LSE: with lse_q the
 *     log-sum-exp of row q over all keys, taken from an earlier step, the
 *     attention weight of a pair is exp(scale * q.k - lse_q), and the mass of
 *     a block is the sum of its weights.  One pass over Q K^T gives every
 *     block's mass, with no normalisation pass ("fused");
 *   - head-adaptive: every head, and every query tile in it, keeps the
 *     smallest set of video key tiles, heaviest first, whose mass reaches p
 *     times the mass of all its video key tiles, so the density follows the
 *     head.  At least the heaviest video key tile is kept.  The running sum and
 *     the total are plain double sums of the masses in the heaviest-first order;
 *     ties in mass go to the lower tile index;
 *   - hierarchical between modalities: key tiles holding text keys are kept
 *     by every query tile, and query tiles holding text rows keep every key
 *     tile, as in the rest of this library;
 *   - a kept block is computed whole: a query attends to exactly the keys of
 *     its tile's kept key tiles.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double bf16_to_f64_3(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Block masses.  Q, K: bf16 [BH][L][d]; lse: float [BH][L] (natural log).
 * mass[bh][qb][kb] = sum over rows q < L of tile qb and keys k < L of tile kb
 * of exp(scale * q.k - lse[q]), nqb = ceil(L / bq), nkb = ceil(L / bk).
 * With tiles == NULL, mass is double [BH][nqb][nkb]; otherwise only the
 * ntiles query tiles tiles[i] = bh * nqb + qb, into mass [ntiles][nkb]. */
void ora3_block_mass(int BH, int64_t L, int d, int bq, int bk, double scale, const uint16_t* Q,
                     const uint16_t* K, const float* lse, int64_t ntiles, const int64_t* tiles, double* mass) {
  int64_t nqb = (L + bq - 1) / bq, nkb = (L + bk - 1) / bk;
  int64_t nt = tiles ? ntiles : (int64_t)BH * nqb;
  memset(mass, 0, sizeof(double) * (size_t)nt * nkb);
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < nt; i++) {
    int64_t t = tiles ? tiles[i] : i;
    int64_t bh = t / nqb, qb = t % nqb;
    double* m = mass + i * nkb;
    for (int64_t q = qb * bq; q < (qb + 1) * bq && q < L; q++) {
      const uint16_t* qr = Q + (bh * L + q) * d;
      double lq = (double)lse[bh * L + q];
      for (int64_t k = 0; k < L; k++) {
        const uint16_t* kr = K + (bh * L + k) * d;
        double s = 0.0;
        for (int e = 0; e < d; e++) s += bf16_to_f64_3(qr[e]) * bf16_to_f64_3(kr[e]);
        m[k / bk] += exp(scale * s - lq);
      }
    }
  }
}

/* Kept key tiles of every (head, query tile), from float masses
 * mass: float [BH][nqb][nkb].  Returns the entry count; row_ptr [BH*nqb+1],
 * col (increasing within a tile) and full (all 1) written up to `capacity`.
 * margin (nullable): double [BH*nqb], how far the cut is from moving: the
 * smaller of (goal - running sum before the last kept tile) and (running sum
 * with it - goal); +inf where no cut is made (text rows, no video tiles). */
int64_t ora3_select(int BH, int64_t L, int64_t Lv, int bq, int bk, const float* mass, double p,
                    int32_t* row_ptr, int32_t* col, uint8_t* full, int64_t capacity, double* margin) {
  int64_t nqb = (L + bq - 1) / bq, nkb = (L + bk - 1) / bk;
  int* order = (int*)malloc(sizeof(int) * (size_t)nkb);
  uint8_t* keep = (uint8_t*)malloc((size_t)nkb);
  int64_t e = 0;
  row_ptr[0] = 0;
  for (int64_t t = 0; t < (int64_t)BH * nqb; t++) {
    int64_t qb = t % nqb;
    const float* m = mass + t * nkb;
    int64_t q1 = (qb + 1) * bq < L ? (qb + 1) * bq : L;
    int text_q = q1 > Lv;                       /* the tile holds a text row */
    int nv = 0;                                 /* video key tiles: every key of the tile < Lv */
    for (int64_t kb = 0; kb < nkb; kb++) {
      int64_t k1 = (kb + 1) * bk < L ? (kb + 1) * bk : L;
      int text_k = k1 > Lv;                     /* the tile holds a text key */
      keep[kb] = (uint8_t)(text_q || text_k);
      if (!text_k) order[nv++] = (int)kb;
    }
    if (margin) margin[t] = INFINITY;
    if (!text_q && nv > 0) {
      /* insertion sort of the video tiles: mass descending, lower index first */
      for (int a = 1; a < nv; a++) {
        int x = order[a], b = a - 1;
        while (b >= 0 && (m[order[b]] < m[x] || (m[order[b]] == m[x] && order[b] > x))) {
          order[b + 1] = order[b];
          b--;
        }
        order[b + 1] = x;
      }
      double total = 0.0;
      for (int a = 0; a < nv; a++) total += (double)m[order[a]];
      /* the heaviest tile, then more until the running sum reaches the goal */
      double goal = p * total, run = 0.0, before = 0.0;
      for (int a = 0; a < nv; a++) {
        keep[order[a]] = 1;
        before = run;
        run += (double)m[order[a]];
        if (run >= goal) break;
      }
      if (margin) margin[t] = fmin(goal - before, run - goal);
    }
    for (int64_t kb = 0; kb < nkb; kb++)
      if (keep[kb]) {
        if (e < capacity) {
          col[e] = (int32_t)kb;
          full[e] = 1;
        }
        e++;
      }
    row_ptr[t + 1] = (int32_t)e;
  }
  free(order);
  free(keep);
  return e;
}

/* Attention with a block list: row q of head bh attends to the keys of the
 * kept key tiles of its query tile.  rows[i] = bh * L + q; out: double
 * [nrows][d]; lse optional. */
void ora3_attention_rows(int BH, int64_t L, int d, int bq, int bk, double scale, const uint16_t* Q,
                         const uint16_t* K, const uint16_t* V, const int32_t* row_ptr, const int32_t* col,
                         int64_t nrows, const int64_t* rows, double* out, double* lse) {
  int64_t nqb = (L + bq - 1) / bq;
  (void)BH;
#pragma omp parallel
  {
    double* sb = (double*)malloc(sizeof(double) * (size_t)L);
#pragma omp for schedule(dynamic, 4)
    for (int64_t n = 0; n < nrows; n++) {
      int64_t bh = rows[n] / L, q = rows[n] % L;
      int64_t t = bh * nqb + q / bq;
      const uint16_t* qr = Q + (bh * L + q) * d;
      for (int64_t k = 0; k < L; k++) sb[k] = -INFINITY;
      double mx = -INFINITY;
      for (int32_t i = row_ptr[t]; i < row_ptr[t + 1]; i++)
        for (int64_t k = (int64_t)col[i] * bk; k < ((int64_t)col[i] + 1) * bk && k < L; k++) {
          const uint16_t* kr = K + (bh * L + k) * d;
          double s = 0.0;
          for (int e = 0; e < d; e++) s += bf16_to_f64_3(qr[e]) * bf16_to_f64_3(kr[e]);
          sb[k] = s * scale;
          if (sb[k] > mx) mx = sb[k];
        }
      double* o = out + n * d;
      for (int e = 0; e < d; e++) o[e] = 0.0;
      double l = 0.0;
      for (int64_t k = 0; k < L; k++) {
        if (sb[k] == -INFINITY) continue;
        double pk = exp(sb[k] - mx);
        l += pk;
        const uint16_t* vr = V + (bh * L + k) * d;
        for (int e = 0; e < d; e++) o[e] += pk * bf16_to_f64_3(vr[e]);
      }
      for (int e = 0; e < d; e++) o[e] = (l > 0.0) ? o[e] / l : 0.0;
      if (lse) lse[n] = (l > 0.0) ? mx + log(l) : -INFINITY;
    }
    free(sb);
  }
}
