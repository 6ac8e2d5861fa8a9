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
// row, the row held in registers as packed bf16 pairs.  The head's centroids
// sit in shared memory as interleaved pairs, cp[pair][i] = (c_{2 pair}[i],
// c_{2 pair + 1}[i]), so one 16-byte broadcast load gives two dimensions of
// two centroids; a pass covers kKmGroup pairs (8 centroids) with one
// unpacking of each x_i.  Per centroid the distance is still summed over
// i = 0..D-1 in order, and centroids are compared in index order.
constexpr int kKmGroup = 4;                              // centroid pairs per pass

__host__ __device__ constexpr int km_assign_pairs(int C) {
  return (C + 2 * kKmGroup - 1) / (2 * kKmGroup) * kKmGroup;   // padded to whole passes
}

template <int D>
__global__ void __launch_bounds__(256, D == 128 ? 1 : 2) km_assign_kernel(const KmArgs a) {
  extern __shared__ float4 cp4[];                     // [pairs][D/2] of (c0[i], c1[i], c0[i+1], c1[i+1])
  __shared__ int cnt[kMaxClusters];
  float* cpf = reinterpret_cast<float*>(cp4);
  const int bh = blockIdx.y;
  const int C = a.C, npair = km_assign_pairs(C);
  const float* cg = a.cent + static_cast<int64_t>(bh) * C * D;
  for (int e = threadIdx.x; e < npair * D * 2; e += blockDim.x) {
    const int pr = e / (2 * D), rem = e - pr * 2 * D, i = rem >> 1, side = rem & 1;
    const int c = min(2 * pr + side, C - 1);           // padding repeats the last centroid
    cpf[e] = cg[c * D + i];
  }
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
    for (int g = 0; g < npair; g += kKmGroup) {
      uint64_t acc[kKmGroup];
#pragma unroll
      for (int p = 0; p < kKmGroup; p++) acc[p] = pack_f2(0.f, 0.f);
      const float4* base = cp4 + g * (D / 2);
#pragma unroll
      for (int j = 0; j < D / 2; j++) {                 // dimensions 2j, 2j+1
        const float xa = bf16_lo(xw[j]), xb = bf16_hi(xw[j]);
        const uint64_t xa2 = pack_f2(xa, xa), xb2 = pack_f2(xb, xb);
#pragma unroll
        for (int p = 0; p < kKmGroup; p++) {
          const float4 c = base[p * (D / 2) + j];
          uint64_t t;
          asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(t) : "l"(xa2), "l"(pack_f2(c.x, c.y)));
          acc[p] = fma_f2(t, t, acc[p]);
          asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(t) : "l"(xb2), "l"(pack_f2(c.z, c.w)));
          acc[p] = fma_f2(t, t, acc[p]);
        }
      }
#pragma unroll
      for (int p = 0; p < kKmGroup; p++) {
        const int c = 2 * (g + p);
        float d0, d1;
        unpack_f2(acc[p], d0, d1);
        if (c < C && d0 < bestd) {
          bestd = d0;
          best = c;
        }
        if (c + 1 < C && d1 < bestd) {
          bestd = d1;
          best = c + 1;
        }
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

// ------------------------------------------------------- permutation of Q, K, V

struct KmGatherArgs {
  int BH, L, Lv;
  FastDiv divL;
  const uint16_t* src[3];
  uint16_t* dst[3];
  const int32_t* perm[3];  // [BH][Lv]: video position p of dst takes row perm[p] of src
};

// dst row p <- src row perm[p] (video rows), text rows copied in place.
// One 16-byte chunk per thread and step, kKmGatherU steps in flight; the
// stores are coalesced, a source row is read whole (D*2 contiguous bytes).
// blockIdx.y = tensor.
constexpr int kKmGatherU = 4;

template <int D>
__global__ void __launch_bounds__(256) km_gather_kernel(const KmGatherArgs a) {
  constexpr int CH = D / 8;                           // 16-byte chunks per row
  constexpr int SH = (D == 128) ? 4 : 3;
  static_assert((1 << SH) == CH, "chunks per row");
  // select the tensor without indexing the parameter arrays dynamically (that
  // would copy them to local memory)
  const int t = blockIdx.y;
  const uint4* __restrict__ src = reinterpret_cast<const uint4*>(t == 0 ? a.src[0] : t == 1 ? a.src[1] : a.src[2]);
  uint4* __restrict__ dst = reinterpret_cast<uint4*>(t == 0 ? a.dst[0] : t == 1 ? a.dst[1] : a.dst[2]);
  const int32_t* __restrict__ perm = t == 0 ? a.perm[0] : t == 1 ? a.perm[1] : a.perm[2];
  const int64_t n = static_cast<int64_t>(a.BH) * a.L * CH;
  const int64_t step = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i0 < n; i0 += step * kKmGatherU) {
    uint4 x[kKmGatherU];
#pragma unroll
    for (int u = 0; u < kKmGatherU; u++) {
      const int64_t i = i0 + u * step;
      if (i < n) {
        const int row = static_cast<int>(i >> SH), c = static_cast<int>(i & (CH - 1));
        const int bh = fdiv(row, a.divL), p = row - bh * a.L;
        const int sp = (p < a.Lv) ? __ldg(perm + static_cast<int64_t>(bh) * a.Lv + p) : p;
        x[u] = __ldg(src + (static_cast<int64_t>(bh) * a.L + sp) * CH + c);
      }
    }
#pragma unroll
    for (int u = 0; u < kKmGatherU; u++) {
      const int64_t i = i0 + u * step;
      if (i < n) dst[i] = x[u];
    }
  }
}

// ------------------------------------------------ block index, permuted order

struct Km2Geom {
  int BH, L, Lv, bq, bk, nqb, nkb, Cq, Ck;
  const int32_t* qoff;     // [BH][Cq+1]
  const int32_t* koff;     // [BH][Ck+1]
  const uint64_t* sel;     // [BH][Cq]
};

// One warp per (head, query tile).  In the permuted order a query tile covers a
// run of query clusters and a key block a run of key clusters; a pair (i, j)
// is kept iff bit j of sel[i] is set, text keys are kept by every query and
// text queries keep every key.  With U / I = OR / AND of sel over the tile's
// non-empty query clusters and R = the key clusters present in a block, the
// block is listed iff it holds a text key or U & R != 0, and full iff every
// pair is kept: the tile has no video query or I covers R.  The lanes take
// the key blocks 32 apart; ballots give the count and each entry's slot, so
// the list comes out in increasing block order.
struct Km2Tile {
  uint64_t U, I;
  bool video_q;
};

__device__ __forceinline__ Km2Tile km2_tile(const Km2Geom& g, int bh, int qb) {
  const int32_t* qo = g.qoff + static_cast<int64_t>(bh) * (g.Cq + 1);
  const uint64_t* sl = g.sel + static_cast<int64_t>(bh) * g.Cq;
  const int q0 = qb * g.bq, q1 = min(g.L, q0 + g.bq);
  Km2Tile t{0ull, ~0ull, q0 < g.Lv};
  if (t.video_q) {
    const int i0 = cluster_of(qo, g.Cq, q0), i1 = cluster_of(qo, g.Cq, min(q1, g.Lv) - 1);
    for (int i = i0; i <= i1; i++)
      if (__ldg(qo + i + 1) > __ldg(qo + i)) {
        const uint64_t m = __ldg(reinterpret_cast<const unsigned long long*>(sl) + i);
        t.U |= m;
        t.I &= m;
      }
  }
  if (q1 > g.Lv) t.U = ~0ull;                   // a text query keeps every key
  return t;
}

// Key clusters present in video keys [k0, k1) of one head (0 if none).
__device__ __forceinline__ uint64_t km2_block_clusters(const Km2Geom& g, const int32_t* ko, int k0, int k1) {
  uint64_t R = 0;
  const int e = min(k1, g.Lv);
  if (k0 < e)
    for (int j = cluster_of(ko, g.Ck, k0); j < g.Ck && __ldg(ko + j) < e; j++)
      if (__ldg(ko + j + 1) > __ldg(ko + j)) R |= 1ull << j;
  return R;
}

template <bool FILL>
__global__ void __launch_bounds__(256, 4) km2_list_kernel(const Km2Geom g, int32_t* __restrict__ row_ptr,
                                                       int32_t* __restrict__ col, uint8_t* __restrict__ full,
                                                       int64_t capacity) {
  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t n = static_cast<int64_t>(g.BH) * g.nqb;
  if (wid >= n) return;                          // whole warps leave together
  const int bh = static_cast<int>(wid / g.nqb), qb = static_cast<int>(wid % g.nqb);
  const Km2Tile t = km2_tile(g, bh, qb);
  const int32_t* ko = g.koff + static_cast<int64_t>(bh) * (g.Ck + 1);
  int64_t e = FILL ? static_cast<int64_t>(row_ptr[wid]) : 0;
  for (int kb0 = 0; kb0 < g.nkb; kb0 += 32) {
    const int kb = kb0 + lane;
    bool listed = false, fl = false;
    if (kb < g.nkb) {
      const int k0 = kb * g.bk, k1 = min(g.L, k0 + g.bk);
      const uint64_t R = km2_block_clusters(g, ko, k0, k1);
      listed = (k1 > g.Lv) || (t.U & R) != 0;
      fl = !t.video_q || (t.I & R) == R;
    }
    const unsigned b = __ballot_sync(0xffffffffu, listed);
    if (FILL && listed) {
      const int64_t slot = e + __popc(b & ((1u << lane) - 1u));
      if (slot < capacity) {
        col[slot] = kb;
        full[slot] = fl ? 1 : 0;
      }
    }
    e += __popc(b);
  }
  if (!FILL && lane == 0) {
    row_ptr[wid + 1] = static_cast<int32_t>(e);
    if (wid == 0) row_ptr[0] = 0;
  }
}

}  // namespace svg

