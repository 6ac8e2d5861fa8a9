/*
 * svg2_oracle.c — plain CPU oracle for the semantic-aware permutation of
 * "Sparse VideoGen2" (gist.science explainer: "A. 语义感知排列", "B. 基于质心的
 * Top-p 选择"), the second workload of the attention step.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's
 * cpu_baseline / reference arm may load this library.  It shares no code, header,
 * table or constant with the CUDA library.
 *
 * The steps, in the page's order:
 *   1. k-means clustering of the video rows of Q and, separately, of K, per head
 *      (Lloyd's iteration: assign every row to its nearest centroid, then move
 *      each centroid to the mean of its rows);
 *   2. a permutation that makes every cluster contiguous;
 *   3. the attention of query cluster i to key cluster j estimated from the
 *      centroids, weighted by the key cluster's size, and the top-p set of key
 *      clusters per query cluster;
 *   4. attention of each query row to the keys of its selected clusters.
 * The page gives no numbers or precisions.  Readings (also in the design notes):
 *   - init: centroid c = row floor(c * Lv / C); text rows are not clustered;
 *   - the nearest centroid minimises the squared Euclidean distance
 *     sum_i (x_i - c_i)^2, evaluated in double; the lowest index wins a tie;
 *   - a centroid is the mean of its rows: the sum in double over the rows in
 *     their order, divided by the count, rounded once to float; an empty
 *     cluster keeps its centroid;
 *   - the permutation is a stable counting sort by cluster;
 *   - score s_ij = scale * (c^q_i . c^k_j) in double; weight
 *     w_ij = n^k_j * exp(s_ij - max_j s_ij); key clusters sorted by weight
 *     (descending, lower index first on a tie); the selected set is the
 *     shortest prefix whose running sum reaches p * (sum of all weights);
 *   - text keys are kept for every query and text queries keep every key.
 * A library that takes the nearest-centroid decision in float may disagree
 * with this one where the two nearest centroids are almost equally far; the
 * assignment can report, per row, how far the decision is from such a tie.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double bf16_to_f64(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

static float bf16_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* Centroid c = row floor(c * Lv / C) of the head, as float.
 * x: bf16 [BH][L][d]; cent: float [BH][C][d]. */
void ora2_kmeans_init(const uint16_t* x, int BH, int64_t L, int64_t Lv, int d, int C, float* cent) {
  for (int bh = 0; bh < BH; bh++)
    for (int c = 0; c < C; c++) {
      int64_t r = (int64_t)c * Lv / C;
      for (int i = 0; i < d; i++) cent[((int64_t)bh * C + c) * d + i] = bf16_to_f32(x[((int64_t)bh * L + r) * d + i]);
    }
}

/* Nearest centroid of every video row (step 1, assignment).  assign: uint8
 * [BH][Lv].  margin (nullable): double [BH][Lv], the gap between the second
 * nearest and the nearest squared distance over |x|^2 + |c1|^2 + |c2|^2 (the
 * scale of the terms a distance is formed from); +inf with one centroid. */
void ora2_assign(const uint16_t* x, int BH, int64_t L, int64_t Lv, int d, int C, const float* cent,
                 uint8_t* assign, double* margin) {
#pragma omp parallel for schedule(static)
  for (int64_t g = 0; g < (int64_t)BH * Lv; g++) {
    int64_t bh = g / Lv, r = g % Lv;
    const uint16_t* xr = x + (bh * L + r) * d;
    int best = 0, second = -1;
    double bestd = INFINITY, secondd = INFINITY;
    for (int c = 0; c < C; c++) {
      const float* cc = cent + (bh * C + c) * d;
      double dist = 0.0;
      for (int i = 0; i < d; i++) {
        double diff = bf16_to_f64(xr[i]) - (double)cc[i];
        dist += diff * diff;
      }
      if (dist < bestd) {
        second = best;
        secondd = bestd;
        bestd = dist;
        best = c;
      } else if (dist < secondd) {
        secondd = dist;
        second = c;
      }
    }
    assign[g] = (uint8_t)best;
    if (margin) {
      if (second < 0) {
        margin[g] = INFINITY;
      } else {
        double n = 0.0;
        for (int i = 0; i < d; i++) {
          double xi = bf16_to_f64(xr[i]), a = cent[(bh * C + best) * d + i], b = cent[(bh * C + second) * d + i];
          n += xi * xi + a * a + b * b;
        }
        margin[g] = (secondd - bestd) / n;
      }
    }
  }
}

/* Centroids as the means of their rows (step 1, update); counts: int32 [BH][C]. */
void ora2_update(const uint16_t* x, int BH, int64_t L, int64_t Lv, int d, int C, const uint8_t* assign,
                 float* cent, int32_t* counts) {
  double* sum = (double*)calloc((size_t)C * d, sizeof(double));
  for (int bh = 0; bh < BH; bh++) {
    memset(sum, 0, sizeof(double) * (size_t)C * d);
    for (int c = 0; c < C; c++) counts[bh * C + c] = 0;
    for (int64_t r = 0; r < Lv; r++) {
      int c = assign[(int64_t)bh * Lv + r];
      counts[bh * C + c]++;
      const uint16_t* xr = x + ((int64_t)bh * L + r) * d;
      for (int i = 0; i < d; i++) sum[(int64_t)c * d + i] += bf16_to_f64(xr[i]);
    }
    for (int c = 0; c < C; c++) {
      int n = counts[bh * C + c];
      if (n == 0) continue;
      for (int i = 0; i < d; i++) cent[((int64_t)bh * C + c) * d + i] = (float)(sum[(int64_t)c * d + i] / (double)n);
    }
  }
  free(sum);
}

/* `iters` rounds of (assign, update), then a final assignment. */
void ora2_kmeans(const uint16_t* x, int BH, int64_t L, int64_t Lv, int d, int C, int iters, float* cent,
                 uint8_t* assign, int32_t* counts) {
  for (int t = 0; t < iters; t++) {
    ora2_assign(x, BH, L, Lv, d, C, cent, assign, NULL);
    ora2_update(x, BH, L, Lv, d, C, assign, cent, counts);
  }
  ora2_assign(x, BH, L, Lv, d, C, cent, assign, NULL);
  /* the counts of the final assignment */
  for (int bh = 0; bh < BH; bh++) {
    for (int c = 0; c < C; c++) counts[bh * C + c] = 0;
    for (int64_t r = 0; r < Lv; r++) counts[bh * C + assign[(int64_t)bh * Lv + r]]++;
  }
}

/* Step 2: stable counting sort.  perm[bh][p] = the video row placed at position p;
 * off[bh][c] = first position of cluster c (off[bh][C] = Lv). */
void ora2_permutation(const uint8_t* assign, int BH, int64_t Lv, int C, int32_t* perm, int32_t* off) {
  for (int bh = 0; bh < BH; bh++) {
    int32_t* o = off + (int64_t)bh * (C + 1);
    for (int c = 0; c <= C; c++) o[c] = 0;
    for (int64_t r = 0; r < Lv; r++) o[assign[(int64_t)bh * Lv + r] + 1]++;
    for (int c = 0; c < C; c++) o[c + 1] += o[c];
    int32_t* next = (int32_t*)malloc(sizeof(int32_t) * (size_t)C);
    for (int c = 0; c < C; c++) next[c] = o[c];
    for (int64_t r = 0; r < Lv; r++) {
      int c = assign[(int64_t)bh * Lv + r];
      perm[(int64_t)bh * Lv + next[c]++] = (int32_t)r;
    }
    free(next);
  }
}

/* Step 3: top-p key clusters of every query cluster.  cq: float [BH][Cq][d],
 * ck: float [BH][Ck][d], nk: int32 [BH][Ck] (key cluster sizes).
 * sel: uint64 [BH][Cq], bit j = key cluster j selected (Ck <= 64).
 * weight (optional): double [BH][Cq][Ck], the normalised weights. */
void ora2_select(const float* cq, const float* ck, const int32_t* nk, int BH, int Cq, int Ck, int d, double scale,
                 double p, uint64_t* sel, double* weight) {
  for (int bh = 0; bh < BH; bh++)
    for (int i = 0; i < Cq; i++) {
      double s[64], w[64];
      int order[64];
      double smax = -INFINITY;
      for (int j = 0; j < Ck; j++) {
        double acc = 0.0;
        for (int e = 0; e < d; e++)
          acc += (double)cq[((int64_t)bh * Cq + i) * d + e] * (double)ck[((int64_t)bh * Ck + j) * d + e];
        s[j] = scale * acc;
        if (nk[bh * Ck + j] > 0 && s[j] > smax) smax = s[j];
      }
      double total = 0.0;
      for (int j = 0; j < Ck; j++) {
        w[j] = nk[bh * Ck + j] > 0 ? (double)nk[bh * Ck + j] * exp(s[j] - smax) : 0.0;
        total += w[j];
        order[j] = j;
      }
      /* insertion sort: weight descending, lower index first */
      for (int a = 1; a < Ck; a++) {
        int t = order[a], b = a - 1;
        while (b >= 0 && (w[order[b]] < w[t] || (w[order[b]] == w[t] && order[b] > t))) {
          order[b + 1] = order[b];
          b--;
        }
        order[b + 1] = t;
      }
      uint64_t m = 0;
      double run = 0.0;
      for (int a = 0; a < Ck; a++) {
        int j = order[a];
        if (w[j] <= 0.0) break;
        m |= (uint64_t)1 << j;
        run += w[j];
        if (run >= p * total) break;
      }
      sel[(int64_t)bh * Cq + i] = m;
      if (weight)
        for (int j = 0; j < Ck; j++) weight[((int64_t)bh * Cq + i) * Ck + j] = total > 0.0 ? w[j] / total : 0.0;
    }
}

/* Step 4 in model order: rows[i] = bh * L + token.  A video query of cluster i
 * keeps the video keys of its selected key clusters and every text key; a text
 * query keeps every key.  out: double [nrows][d]; lse optional. */
void ora2_attention_rows(int BH, int64_t L, int64_t Lv, int d, int Cq, int Ck, double scale, const uint16_t* Q,
                         const uint16_t* K, const uint16_t* V, const uint8_t* aq, const uint8_t* ak,
                         const uint64_t* sel, int64_t nrows, const int64_t* rows, double* out, double* lse) {
#pragma omp parallel
  {
    double* sb = (double*)malloc(sizeof(double) * (size_t)L);
#pragma omp for schedule(dynamic, 4)
    for (int64_t n = 0; n < nrows; n++) {
      int64_t bh = rows[n] / L, q = rows[n] % L;
      const uint16_t* qr = Q + (bh * L + q) * d;
      uint64_t m = (q < Lv) ? sel[bh * Cq + aq[bh * Lv + q]] : ~(uint64_t)0;
      double mx = -INFINITY;
      for (int64_t k = 0; k < L; k++) {
        int keep = (q >= Lv) || (k >= Lv) || ((m >> ak[bh * Lv + k]) & 1u);
        if (!keep) {
          sb[k] = -INFINITY;
          continue;
        }
        const uint16_t* kr = K + (bh * L + k) * d;
        double s = 0.0;
        for (int e = 0; e < d; e++) s += bf16_to_f64(qr[e]) * bf16_to_f64(kr[e]);
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
        for (int e = 0; e < d; e++) o[e] += pk * bf16_to_f64(vr[e]);
      }
      for (int e = 0; e < d; e++) o[e] /= l;
      if (lse) lse[n] = mx + log(l);
    }
    free(sb);
  }
  (void)Ck;
}

/* Tile list over the permuted order, by brute force: position p < Lv holds video
 * row perm[p] (query or key permutation), positions >= Lv the text tokens.  Tile
 * (qb, kb) is listed iff some (query, key) pair in it is kept; full iff all pairs
 * with both indices < L are kept.  row_ptr: [BH*nqb+1]; col/full sized by the
 * caller (capacity); returns the entry count. */
int64_t ora2_block_list(int BH, int64_t L, int64_t Lv, int Cq, int Ck, int bq, int bk, const uint8_t* aq,
                        const uint8_t* ak, const int32_t* perm_q, const int32_t* perm_k, const uint64_t* sel,
                        int32_t* row_ptr, int32_t* col, uint8_t* full, int64_t capacity) {
  int64_t nqb = (L + bq - 1) / bq, nkb = (L + bk - 1) / bk;
  int64_t e = 0;
  row_ptr[0] = 0;
  for (int bh = 0; bh < BH; bh++)
    for (int64_t qb = 0; qb < nqb; qb++) {
      for (int64_t kb = 0; kb < nkb; kb++) {
        int any = 0, all = 1;
        for (int64_t q = qb * bq; q < (qb + 1) * bq && q < L; q++) {
          uint64_t m = ~(uint64_t)0;
          int qtext = q >= Lv;
          if (!qtext) m = sel[(int64_t)bh * Cq + aq[(int64_t)bh * Lv + perm_q[(int64_t)bh * Lv + q]]];
          for (int64_t k = kb * bk; k < (kb + 1) * bk && k < L; k++) {
            int keep = qtext || (k >= Lv) ||
                       ((m >> ak[(int64_t)bh * Lv + perm_k[(int64_t)bh * Lv + k]]) & 1u);
            any |= keep;
            all &= keep;
          }
        }
        if (any) {
          if (e < capacity) {
            col[e] = (int32_t)kb;
            full[e] = (uint8_t)all;
          }
          e++;
        }
      }
      row_ptr[(int64_t)bh * nqb + qb + 1] = (int32_t)e;
    }
  (void)Ck;
  return e;
}
