// svg2.cuh — the semantic-aware permutation of "Sparse VideoGen2" (gist.science
// explainer, "A. 语义感知排列" and "B. 基于质心的 Top-p 选择"): k-means of the
// video rows of Q and of K per head, a stable counting sort that makes every
// cluster contiguous, and the top-p key clusters of every query cluster from
// size-weighted centroid scores.  The block index over the permuted order and
// the cluster mask of the attention kernel build on these.
//
// Decisions made from floating point (nearest centroid, top-p set) are taken
// with a fixed operation order so that they do not depend on scheduling:
//   * the nearest centroid minimises |c|^2 - 2 x.c, both sums in float over
//     i = 0..d-1 with fused multiply-adds (packed over two centroids), then
//     one rounding of |c|^2 - 2 (x.c);
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
  double xmax;             // values must satisfy |x| < xmax (km_value_bound)
};

// Largest |x| the fixed-point sums take exactly: a cluster of up to Lv rows
// must keep its sum of |x| below 2^23 (x * 2^40 in a signed 64-bit word), and a
// block's 2,048-row high-word sums must fit a signed 32-bit word (|x| < 2^12).
__host__ __device__ inline double km_value_bound(int Lv) {
  const double b = 8388608.0 / (Lv > 0 ? Lv : 1);
  return b < 4096.0 ? b : 4096.0;
}

// Centroid c = video row floor(c * Lv / C) of the head.
template <int D>
__global__ void km_init_kernel(const KmArgs a) {
  const int bh = blockIdx.y, c = blockIdx.x;
  const int64_t r = static_cast<int64_t>(c) * a.Lv / a.C;
  const uint16_t* xr = a.x + (static_cast<int64_t>(bh) * a.L + r) * D;
  for (int i = threadIdx.x; i < D; i += blockDim.x)
    a.cent[(static_cast<int64_t>(bh) * a.C + c) * D + i] = __uint_as_float(static_cast<uint32_t>(xr[i]) << 16);
}

// Nearest centroid of every video row, and the cluster sizes.  The nearest
// centroid minimises |c|^2 - 2 x.c (the squared distance without |x|^2, the
// same for every centroid): |c|^2 and x.c are each summed in fp32 over
// i = 0..D-1 with fused multiply-adds, then |c|^2 - 2 (x.c) is rounded once;
// centroids are compared in index order, the lowest index winning a tie.
// Two rows per thread, held in registers as packed bf16 pairs.  The
// head's centroids sit in shared memory as interleaved pairs,
// cp[pair][i] = (c_{2 pair}[i], c_{2 pair + 1}[i]), so a 16-byte broadcast
// load gives two dimensions of two centroids and one packed FMA advances two
// dot products; a pass covers kKmGroup pairs (8 centroids) with one unpacking
// of each x_i.
constexpr int kKmGroup = 4;                              // centroid pairs per pass

__host__ __device__ constexpr int km_assign_pairs(int C) {
  return (C + 2 * kKmGroup - 1) / (2 * kKmGroup) * kKmGroup;   // padded to whole passes
}

// shared memory of km_assign_kernel: the pairs, then |c|^2 of every (padded) centroid
__host__ __device__ constexpr int km_assign_smem(int C, int D) {
  return km_assign_pairs(C) * 2 * D * 4 + km_assign_pairs(C) * 2 * 4;
}

// (lo, lo) and (hi, hi) as packed fp32 pairs from one packed bf16 pair.  The
// asm is volatile so that the unpacking stays inside the centroid loop:
// hoisted out of it, the unpacked rows would need 2*D registers per row.
__device__ __forceinline__ void bf16x2_dup(uint32_t w, uint64_t& lo2, uint64_t& hi2) {
  asm volatile(
      "{\n\t.reg .b32 l, h;\n\t"
      "shl.b32 l, %2, 16;\n\t"
      "and.b32 h, %2, 0xFFFF0000;\n\t"
      "mov.b64 %0, {l, l};\n\t"
      "mov.b64 %1, {h, h};\n\t}"
      : "=l"(lo2), "=l"(hi2)
      : "r"(w));
}

constexpr int kKmAssignThreads = 128;                  // each thread takes two rows
constexpr int kKmAssignRows = 2 * kKmAssignThreads;     // rows per block

template <int D>
__device__ __forceinline__ void km_load_row(const KmArgs& a, int bh, int r, uint32_t* xw) {
  if (r < a.Lv) {
    const uint4* xr = reinterpret_cast<const uint4*>(a.x + (static_cast<int64_t>(bh) * a.L + r) * D);
#pragma unroll
    for (int v = 0; v < D / 8; v++) {
      const uint4 u = __ldg(xr + v);
      xw[4 * v] = u.x;
      xw[4 * v + 1] = u.y;
      xw[4 * v + 2] = u.z;
      xw[4 * v + 3] = u.w;
    }
  } else {
#pragma unroll
    for (int v = 0; v < D / 2; v++) xw[v] = 0u;
  }
}

template <int D>
__global__ void __launch_bounds__(kKmAssignThreads, 1) km_assign_kernel(const KmArgs a) {
  extern __shared__ float4 cp4[];                     // [pairs][D/2] of (c0[i], c1[i], c0[i+1], c1[i+1])
  __shared__ int cnt[kMaxClusters];
  float* cpf = reinterpret_cast<float*>(cp4);
  const int bh = blockIdx.y;
  const int C = a.C, npair = km_assign_pairs(C);
  float* cn = cpf + npair * 2 * D;                    // [2 * npair]
  const float* cg = a.cent + static_cast<int64_t>(bh) * C * D;
  for (int e = threadIdx.x; e < npair * D * 2; e += blockDim.x) {
    const int pr = e / (2 * D), rem = e - pr * 2 * D, i = rem >> 1, side = rem & 1;
    const int c = min(2 * pr + side, C - 1);           // padding repeats the last centroid
    cpf[e] = cg[c * D + i];
  }
  for (int c = threadIdx.x; c < 2 * npair; c += blockDim.x) {
    const float* cc = cg + min(c, C - 1) * D;
    float acc = 0.f;
    for (int i = 0; i < D; i++) acc = fmaf(cc[i], cc[i], acc);
    cn[c] = acc;
  }
  if (threadIdx.x < kMaxClusters) cnt[threadIdx.x] = 0;
  __syncthreads();
  // two rows per thread: every centroid value loaded from shared memory feeds both
  const int r0 = blockIdx.x * kKmAssignRows + threadIdx.x, r1 = r0 + kKmAssignThreads;
  if (r0 < a.Lv) {
    uint32_t xw0[D / 2], xw1[D / 2];                    // the rows as packed bf16 pairs
    km_load_row<D>(a, bh, r0, xw0);
    km_load_row<D>(a, bh, r1, xw1);
    int best0 = 0, best1 = 0;
    float bestd0 = INFINITY, bestd1 = INFINITY;
    constexpr int G = kKmGroup;
    for (int g = 0; g < npair; g += G) {
      uint64_t acc0[G], acc1[G];
#pragma unroll
      for (int p = 0; p < G; p++) acc0[p] = acc1[p] = pack_f2(0.f, 0.f);
      const float4* base = cp4 + g * (D / 2);
#pragma unroll
      for (int j = 0; j < D / 2; j++) {                 // dimensions 2j, 2j+1
        uint64_t xa02, xb02, xa12, xb12;
        bf16x2_dup(xw0[j], xa02, xb02);
        bf16x2_dup(xw1[j], xa12, xb12);
#pragma unroll
        for (int p = 0; p < G; p++) {
          const float4 c = base[p * (D / 2) + j];
          const uint64_t ca = pack_f2(c.x, c.y), cb = pack_f2(c.z, c.w);
          acc0[p] = fma_f2(xa02, ca, acc0[p]);
          acc1[p] = fma_f2(xa12, ca, acc1[p]);
          acc0[p] = fma_f2(xb02, cb, acc0[p]);
          acc1[p] = fma_f2(xb12, cb, acc1[p]);
        }
      }
#pragma unroll
      for (int p = 0; p < G; p++) {
        const int c = 2 * (g + p);
        float u0, u1, w0, w1;
        unpack_f2(acc0[p], u0, u1);
        unpack_f2(acc1[p], w0, w1);
        const float du0 = fmaf(-2.f, u0, cn[c]), du1 = fmaf(-2.f, u1, cn[c + 1]);
        const float dw0 = fmaf(-2.f, w0, cn[c]), dw1 = fmaf(-2.f, w1, cn[c + 1]);
        if (c < C) {
          if (du0 < bestd0) { bestd0 = du0; best0 = c; }
          if (dw0 < bestd1) { bestd1 = dw0; best1 = c; }
        }
        if (c + 1 < C) {
          if (du1 < bestd0) { bestd0 = du1; best0 = c + 1; }
          if (dw1 < bestd1) { bestd1 = dw1; best1 = c + 1; }
        }
      }
    }
    a.assign[static_cast<int64_t>(bh) * a.Lv + r0] = static_cast<uint8_t>(best0);
    atomicAdd(&cnt[best0], 1);
    if (r1 < a.Lv) {
      a.assign[static_cast<int64_t>(bh) * a.Lv + r1] = static_cast<uint8_t>(best1);
      atomicAdd(&cnt[best1], 1);
    }
  }
  __syncthreads();
  if (threadIdx.x < C && cnt[threadIdx.x]) atomicAdd(&a.counts[bh * C + threadIdx.x], cnt[threadIdx.x]);
}

// Fixed-point sums of the rows of every cluster: a block sums a run of rows of
// one head in shared memory, then adds its sums to the head's global 64-bit
// sums.  Each warp walks its own contiguous share of the block's rows (four
// rows in flight), keeping the running sums of its current cluster in
// registers and flushing them to shared memory when the cluster changes, so
// a run of rows in one cluster costs one flush.  A flushed 64-bit value v is
// split as v = hi * 2^32 + mid * 2^16 + lo (hi = v >> 32 signed, mid and lo
// 16-bit) and the three parts are summed with 32-bit shared atomics: over
// kKmUpdateRows rows the mid and lo sums stay below 2^27, and the hi sum below
// 2^31 while the block's sum of |x| in one cluster stays below 2^23.  The
// recombined total is exact, so neither the order of the atomics nor the
// grouping into runs changes it.
constexpr int kKmUpdateRows = 2048;

template <int D>
__global__ void __launch_bounds__(256) km_sum_kernel(const KmArgs a) {
  extern __shared__ uint32_t s32[];                   // [3][C][D]: hi, mid, lo
  constexpr int E = D / 32;                           // dimensions per lane: lane + 32 e
  constexpr int U = 4;                                // rows in flight per warp
  const int bh = blockIdx.y, C = a.C, n = C * D;
  uint32_t* s_hi = s32;
  uint32_t* s_mid = s32 + n;
  uint32_t* s_lo = s32 + 2 * n;
  for (int i = threadIdx.x; i < 3 * n; i += blockDim.x) s32[i] = 0u;
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarp = blockDim.x >> 5;
  const int r0 = blockIdx.x * kKmUpdateRows, r1 = min(a.Lv, r0 + kKmUpdateRows);
  const int per = (r1 - r0 + nwarp - 1) / nwarp;
  const int w0 = r0 + warp * per, w1 = min(r1, w0 + per);
  const uint8_t* as = a.assign + static_cast<int64_t>(bh) * a.Lv;
  const uint16_t* xh = a.x + static_cast<int64_t>(bh) * a.L * D;
  long long acc[E];
#pragma unroll
  for (int e = 0; e < E; e++) acc[e] = 0;
  int cur = -1;
  bool out_of_range = false;
  auto flush = [&]() {
    if (cur < 0) return;
#pragma unroll
    for (int e = 0; e < E; e++) {
      const int i = cur * D + lane + 32 * e;
      const unsigned long long u = static_cast<unsigned long long>(acc[e]);
      atomicAdd(&s_hi[i], static_cast<uint32_t>(static_cast<int32_t>(acc[e] >> 32)));
      atomicAdd(&s_mid[i], static_cast<uint32_t>((u >> 16) & 0xFFFFu));
      atomicAdd(&s_lo[i], static_cast<uint32_t>(u & 0xFFFFu));
      acc[e] = 0;
    }
  };
  for (int r = w0; r < w1; r += U) {
    int cc[U];
    uint16_t xv[U][E];
#pragma unroll
    for (int u = 0; u < U; u++) {
      const int rr = r + u;
      cc[u] = (rr < w1) ? static_cast<int>(__ldg(as + rr)) : -1;
#pragma unroll
      for (int e = 0; e < E; e++) xv[u][e] = (rr < w1) ? __ldg(xh + static_cast<int64_t>(rr) * D + lane + 32 * e) : 0;
    }
#pragma unroll
    for (int u = 0; u < U; u++) {
      if (cc[u] < 0) continue;                        // warp-uniform: one row per step
      if (cc[u] != cur) {
        flush();
        cur = cc[u];
      }
#pragma unroll
      for (int e = 0; e < E; e++) {
        const double xd = static_cast<double>(__uint_as_float(static_cast<uint32_t>(xv[u][e]) << 16));
        // a value the sums cannot take exactly (or inf / NaN) is reported and left out
        const bool ok = fabs(xd) < a.xmax;
        out_of_range |= !ok;
        acc[e] += ok ? static_cast<long long>(xd * kFix) : 0ll;
      }
    }
  }
  flush();
  if (out_of_range) atomicOr(&g_error_word, kErrBadIndex);
  __syncthreads();
  unsigned long long* gs = a.sum + static_cast<int64_t>(bh) * n;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const long long hi = static_cast<int32_t>(s_hi[i]);
    const unsigned long long t = (static_cast<unsigned long long>(hi) << 32) +
                                 (static_cast<unsigned long long>(s_mid[i]) << 16) + s_lo[i];
    if (t) atomicAdd(&gs[i], t);
  }
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
  // a cluster id outside [0, C) (a caller's assignment) is reported and its row left out
  for (int r = tid; r < Lv; r += 1024) {
    const int c = as[r];
    if (c < C) atomicAdd(&base[c + 1], 1);
    else atomicOr(&g_error_word, kErrBadIndex);
  }
  __syncthreads();
  if (tid == 0) {
    for (int c = 0; c < C; c++) base[c + 1] += base[c];
    for (int c = 0; c <= C; c++) off[static_cast<int64_t>(bh) * (C + 1) + c] = base[c];
  }
  __syncthreads();
  for (int r0 = 0; r0 < Lv; r0 += 1024) {
    const int r = r0 + tid;
    const int c = (r < Lv && as[r] < C) ? as[r] : -1;
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
        int sp = (p < a.Lv) ? __ldg(perm + static_cast<int64_t>(bh) * a.Lv + p) : p;
        if (p < a.Lv && static_cast<unsigned>(sp) >= static_cast<unsigned>(a.Lv)) {   // a caller's entry out of range
          atomicOr(&g_error_word, kErrBadIndex);
          sp = p;
        }
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

