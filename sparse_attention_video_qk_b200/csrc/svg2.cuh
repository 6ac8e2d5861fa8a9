// svg2.cuh — the semantic-aware permutation of "Sparse VideoGen2" (gist.science
// explainer, "A. 语义感知排列" and "B. 基于质心的 Top-p 选择"): k-means of the
// video rows of Q and of K per head, a stable counting sort that makes every
// cluster contiguous, and the top-p key clusters of every query cluster from
// size-weighted centroid scores.  The block index over the permuted order and
// the cluster mask of the attention kernel build on these.
//
// Decisions made from floating point (nearest centroid, top-p set) are taken
// with a fixed operation order so that they do not depend on scheduling:
//   * a distance is sum_i (x_i - c_i)^2 in float, i = 0..d-1, each step one
//     subtraction and one fused multiply-add (packed over two centroids);
//   * centroid sums are 64-bit fixed point (value * 2^40, truncated toward
//     zero), so atomics in any order give the same sum; the mean is
//     ((double)sum / 2^40) / count rounded to float; an empty cluster keeps
//     its centroid;
//   * a score is scale * sum_e cq_e * ck_e in double with separate multiply
//     and add in the order e = 0..d-1; weights n_j * exp(s_j - max s), their
//     total summed in index order, the running sum in weight order.
#pragma once

#include "norm_rope.cuh"
#include "svg_common.cuh"

namespace svg {

constexpr int kMaxClusters = 64;            // a query cluster's key set is one 64-bit mask
constexpr double kFix = 1099511627776.0;    // 2^40

struct KmArgs {
  int BH, L, Lv, C;
  const uint16_t* x;       // bf16 [BH][L][D]
  float* cent;             // [BH][C][D]
  uint8_t* assign;         // [BH][Lv]
  int32_t* counts;         // [BH][C]
  unsigned long long* sum; // [BH][C][D] fixed-point sums
};

// Centroid c = video row floor(c * Lv / C) of the head.
template <int D>
__global__ void km_init_kernel(const KmArgs a) {
  const int bh = blockIdx.y, c = blockIdx.x;
  const int64_t r = static_cast<int64_t>(c) * a.Lv / a.C;
  const uint16_t* xr = a.x + (static_cast<int64_t>(bh) * a.L + r) * D;
  for (int i = threadIdx.x; i < D; i += blockDim.x)
    a.cent[(static_cast<int64_t>(bh) * a.C + c) * D + i] = __uint_as_float(static_cast<uint32_t>(xr[i]) << 16);
}

// Nearest centroid of every video row, and the cluster sizes.  One thread per
// row; the head's centroids sit in shared memory (C*D floats).
template <int D>
__global__ void __launch_bounds__(256) km_assign_kernel(const KmArgs a) {
  extern __shared__ float cs[];                       // [C][D]
  __shared__ int cnt[kMaxClusters];
  const int bh = blockIdx.y;
  const int C = a.C;
  for (int i = threadIdx.x; i < C * D; i += blockDim.x) cs[i] = a.cent[static_cast<int64_t>(bh) * C * D + i];
  if (threadIdx.x < kMaxClusters) cnt[threadIdx.x] = 0;
  __syncthreads();
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r < a.Lv) {
    const uint4* xr = reinterpret_cast<const uint4*>(a.x + (static_cast<int64_t>(bh) * a.L + r) * D);
    uint32_t xw[D / 2];                                 // the row as packed bf16 pairs
#pragma unroll
    for (int v = 0; v < D / 8; v++) {
      const uint4 u = __ldg(xr + v);
      xw[4 * v] = u.x;
      xw[4 * v + 1] = u.y;
      xw[4 * v + 2] = u.z;
      xw[4 * v + 3] = u.w;
    }
    int best = 0;
    float bestd = INFINITY;
    for (int c = 0; c < C; c += 2) {
      // two centroids at once: lanes (c, c+1) of packed pairs, same order as one at a time
      const float* c0 = cs + c * D;
      const float* c1 = cs + min(c + 1, C - 1) * D;
      uint64_t acc = pack_f2(0.f, 0.f);
#pragma unroll
      for (int i = 0; i < D; i++) {
        const float xi = (i & 1) ? bf16_hi(xw[i >> 1]) : bf16_lo(xw[i >> 1]);
        uint64_t t;
        asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(t) : "l"(pack_f2(xi, xi)), "l"(pack_f2(c0[i], c1[i])));
        acc = fma_f2(t, t, acc);
      }
      float d0, d1;
      unpack_f2(acc, d0, d1);
      if (d0 < bestd) {
        bestd = d0;
        best = c;
      }
      if (c + 1 < C && d1 < bestd) {
        bestd = d1;
        best = c + 1;
      }
    }
    a.assign[static_cast<int64_t>(bh) * a.Lv + r] = static_cast<uint8_t>(best);
    atomicAdd(&cnt[best], 1);
  }
  __syncthreads();
  if (threadIdx.x < C && cnt[threadIdx.x]) atomicAdd(&a.counts[bh * C + threadIdx.x], cnt[threadIdx.x]);
}

// Fixed-point sums of the rows of every cluster: a block sums a run of rows of
// one head in shared memory, then adds its sums to the head's global sums.
constexpr int kKmUpdateRows = 2048;

template <int D>
__global__ void __launch_bounds__(256) km_sum_kernel(const KmArgs a) {
  extern __shared__ unsigned long long ss[];          // [C][D]
  const int bh = blockIdx.y, C = a.C;
  for (int i = threadIdx.x; i < C * D; i += blockDim.x) ss[i] = 0ull;
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r0 = blockIdx.x * kKmUpdateRows, r1 = min(a.Lv, r0 + kKmUpdateRows);
  for (int r = r0 + warp; r < r1; r += blockDim.x / 32) {
    const int c = a.assign[static_cast<int64_t>(bh) * a.Lv + r];
    const uint16_t* xr = a.x + (static_cast<int64_t>(bh) * a.L + r) * D;
    for (int i = lane; i < D; i += 32) {
      const double xv = static_cast<double>(__uint_as_float(static_cast<uint32_t>(xr[i]) << 16));
      atomicAdd(&ss[c * D + i], static_cast<unsigned long long>(static_cast<long long>(xv * kFix)));
    }
  }
  __syncthreads();
  unsigned long long* gs = a.sum + static_cast<int64_t>(bh) * C * D;
  for (int i = threadIdx.x; i < C * D; i += blockDim.x)
    if (ss[i]) atomicAdd(&gs[i], ss[i]);
}

// Means from the sums; clears the sums and the counts of the next assignment.
template <int D>
__global__ void km_mean_kernel(const KmArgs a) {
  const int bh = blockIdx.y, c = blockIdx.x, C = a.C;
  const int n = a.counts[bh * C + c];
  const int64_t base = (static_cast<int64_t>(bh) * C + c) * D;
  for (int i = threadIdx.x; i < D; i += blockDim.x) {
    const long long s = static_cast<long long>(a.sum[base + i]);
    if (n > 0) a.cent[base + i] = static_cast<float>((static_cast<double>(s) / kFix) / static_cast<double>(n));
    a.sum[base + i] = 0ull;
  }
  __syncthreads();
  if (threadIdx.x == 0) a.counts[bh * C + c] = 0;
}

// Stable counting sort of one head's rows by cluster: perm[p] = row at position
// p, off[c] = first position of cluster c (off[C] = Lv).  One block of 1024
// threads per head walks the rows in chunks of 1024; inside a chunk a row's
// rank among equal clusters comes from warp matching and per-warp counts.
__global__ void __launch_bounds__(1024) km_perm_kernel(const uint8_t* __restrict__ assign, int Lv, int C,
                                                      int32_t* __restrict__ perm, int32_t* __restrict__ off) {
  __shared__ int base[kMaxClusters + 1];
  __shared__ int wcount[32][kMaxClusters];
  const int bh = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint8_t* as = assign + static_cast<int64_t>(bh) * Lv;
  // cluster sizes -> first positions
  if (tid <= kMaxClusters) base[tid] = 0;
  __syncthreads();
  for (int r = tid; r < Lv; r += 1024) atomicAdd(&base[as[r] + 1], 1);
  __syncthreads();
  if (tid == 0) {
    for (int c = 0; c < C; c++) base[c + 1] += base[c];
    for (int c = 0; c <= C; c++) off[static_cast<int64_t>(bh) * (C + 1) + c] = base[c];
  }
  __syncthreads();
  for (int r0 = 0; r0 < Lv; r0 += 1024) {
    const int r = r0 + tid;
    const int c = (r < Lv) ? as[r] : -1;
    const unsigned same = __match_any_sync(0xffffffffu, c);
    const int rank = __popc(same & ((1u << lane) - 1u));
    for (int i = tid; i < 32 * kMaxClusters; i += 1024) (&wcount[0][0])[i] = 0;
    __syncthreads();
    if (c >= 0 && rank == 0) wcount[warp][c] = __popc(same);
    __syncthreads();
    if (c >= 0) {
      int before = 0;
      for (int w = 0; w < warp; w++) before += wcount[w][c];
      perm[static_cast<int64_t>(bh) * Lv + base[c] + before + rank] = r;
    }
    __syncthreads();
    if (tid < C) {
      int tot = 0;
      for (int w = 0; w < 32; w++) tot += wcount[w][tid];
      base[tid] += tot;
    }
    __syncthreads();
  }
}

// Top-p key clusters of one query cluster (block of 64 threads; thread j =
// key cluster j).  sel[bh][i] bit j = key cluster j selected.
__global__ void __launch_bounds__(64) km_select_kernel(const float* __restrict__ cq, const float* __restrict__ ck,
                                                      const int32_t* __restrict__ nk, int Cq, int Ck, int D,
                                                      double scale, double p, uint64_t* __restrict__ sel) {
  __shared__ double w[kMaxClusters];
  __shared__ double s[kMaxClusters];
  __shared__ int order[kMaxClusters];
  __shared__ double smax_s;
  const int bh = blockIdx.y, i = blockIdx.x, j = threadIdx.x;
  const float* q = cq + (static_cast<int64_t>(bh) * Cq + i) * D;
  if (j < Ck) {
    const float* k = ck + (static_cast<int64_t>(bh) * Ck + j) * D;
    double acc = 0.0;
    for (int e = 0; e < D; e++) acc = __dadd_rn(acc, __dmul_rn(static_cast<double>(q[e]), static_cast<double>(k[e])));
    s[j] = __dmul_rn(scale, acc);
  }
  __syncthreads();
  if (j == 0) {
    double m = -INFINITY;
    for (int t = 0; t < Ck; t++)
      if (nk[bh * Ck + t] > 0 && s[t] > m) m = s[t];
    smax_s = m;
  }
  __syncthreads();
  if (j < Ck) {
    const int n = nk[bh * Ck + j];
    w[j] = n > 0 ? __dmul_rn(static_cast<double>(n), exp(__dsub_rn(s[j], smax_s))) : 0.0;
  }
  __syncthreads();
  if (j < Ck) {
    // rank: heavier first, the lower index first on equal weights
    int rank = 0;
    for (int t = 0; t < Ck; t++) rank += (w[t] > w[j]) || (w[t] == w[j] && t < j);
    order[rank] = j;
  }
  __syncthreads();
  if (j == 0) {
    double total = 0.0;
    for (int t = 0; t < Ck; t++) total = __dadd_rn(total, w[t]);
    const double goal = __dmul_rn(p, total);
    uint64_t m = 0;
    double run = 0.0;
    for (int t = 0; t < Ck; t++) {
      const int jj = order[t];
      if (w[jj] <= 0.0) break;
      m |= 1ull << jj;
      run = __dadd_rn(run, w[jj]);
      if (run >= goal) break;
    }
    sel[static_cast<int64_t>(bh) * Cq + i] = m;
  }
}

// ------------------------------------------------ block index, permuted order

struct Km2Geom {
  int BH, L, Lv, bq, bk, nqb, nkb, Cq, Ck;
  const int32_t* qoff;     // [BH][Cq+1]
  const int32_t* koff;     // [BH][Ck+1]
  const uint64_t* sel;     // [BH][Cq]
};

// Walks the key blocks of one query tile and calls f(kb, full) for every
// listed one.  In the permuted order a query tile covers a run of query
// clusters and a key block a run of key clusters; a pair (i, j) is kept iff bit
// j of sel[i] is set, text keys are kept by every query, text queries keep
// every key.  U / I = OR / AND of sel over the tile's query clusters.
template <typename Fn>
__device__ __forceinline__ void km2_tile_walk(const Km2Geom& g, int bh, int qb, Fn f) {
  const int32_t* qo = g.qoff + static_cast<int64_t>(bh) * (g.Cq + 1);
  const int32_t* ko = g.koff + static_cast<int64_t>(bh) * (g.Ck + 1);
  const uint64_t* sl = g.sel + static_cast<int64_t>(bh) * g.Cq;
  const int q0 = qb * g.bq, q1 = min(g.L, q0 + g.bq);
  const bool text_q = q1 > g.Lv, video_q = q0 < g.Lv;
  uint64_t U = 0, I = ~0ull;
  if (video_q) {
    const int i0 = cluster_of(qo, g.Cq, q0), i1 = cluster_of(qo, g.Cq, min(q1, g.Lv) - 1);
    for (int i = i0; i <= i1; i++)
      if (qo[i + 1] > qo[i]) {
        U |= sl[i];
        I &= sl[i];
      }
  }
  if (text_q) U = ~0ull;
  int j = 0;                                   // key cluster of the current block's first video key
  for (int kb = 0; kb < g.nkb; kb++) {
    const int k0 = kb * g.bk, k1 = min(g.L, k0 + g.bk);
    const bool text_k = k1 > g.Lv;
    uint64_t R = 0;                            // non-empty key clusters in the block
    if (k0 < g.Lv) {
      while (ko[j + 1] <= k0) j++;
      for (int t = j; t < g.Ck && ko[t] < min(k1, g.Lv); t++)
        if (ko[t + 1] > ko[t]) R |= 1ull << t;
    }
    const bool listed = text_k || (U & R) != 0;
    if (listed) f(kb, (!video_q || (I & R) == R) ? 1 : 0);
  }
}

__global__ void km2_count_kernel(const Km2Geom g, int32_t* __restrict__ row_ptr) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t n = static_cast<int64_t>(g.BH) * g.nqb;
  if (i >= n) return;
  int cnt = 0;
  km2_tile_walk(g, static_cast<int>(i / g.nqb), static_cast<int>(i % g.nqb), [&](int, int) { cnt++; });
  row_ptr[i + 1] = cnt;
  if (i == 0) row_ptr[0] = 0;
}

__global__ void km2_fill_kernel(const Km2Geom g, const int32_t* __restrict__ row_ptr, int32_t* __restrict__ col,
                                uint8_t* __restrict__ full, int64_t capacity) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t n = static_cast<int64_t>(g.BH) * g.nqb;
  if (i >= n) return;
  int64_t e = row_ptr[i];
  km2_tile_walk(g, static_cast<int>(i / g.nqb), static_cast<int>(i % g.nqb), [&](int kb, int fl) {
    if (e < capacity) {
      col[e] = kb;
      full[e] = static_cast<uint8_t>(fl);
    }
    e++;
  });
}

}  // namespace svg

