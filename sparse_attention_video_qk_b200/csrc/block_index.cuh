// block_index.cuh — CSR list of the key tiles each query tile must visit.
// Not on the pages: the block-sparse attention kernel they describe ("Sparse
// VideoGen" WeChat article, "其他优化方法"; ICML 2025 report, "Layout
// Transformation + Kernel 加速") needs it.
//
// In its head's layout every video query keeps one contiguous run of video
// keys plus every text key (see row_interval), and the runs grow with the
// row.  So a query tile keeps the key run [lo(first row), hi(last row)) and
// the text keys: at most two ranges of key tiles, counted and written in
// closed form.  A tile is "full" (no token-level predicate needed) when its
// video keys lie inside every video row's run: lo(last video row) <= k0 and
// end <= hi(first row).
// Three launches: count per (b, h, qb) into row_ptr[1..], an in-place scan
// (one block), and the fill.
#pragma once

#include "svg_common.cuh"

namespace svg {

struct TileRanges {
  int a0, a1;  // first key-tile range [a0, a1)
  int b0, b1;  // second key-tile range [b0, b1), b0 >= a1
  int r0, rv1; // query rows [r0, rv1) that are video rows
  int lo_last, hi_first;
};

__device__ __forceinline__ TileRanges tile_ranges(const Geometry& g, int kind, int qb) {
  TileRanges t;
  const int r0 = qb * g.bq;
  const int r1 = min(g.L, r0 + g.bq);
  t.r0 = r0;
  t.rv1 = min(r1, g.Lv);
  t.lo_last = 0;
  t.hi_first = g.L;
  if (t.rv1 > r0) {
    int lo, hi;
    row_interval(g, kind, t.rv1 - 1, lo, hi);
    t.lo_last = lo;
    row_interval(g, kind, r0, lo, hi);
    t.hi_first = hi;
  }
  if (kind == SVG_HEAD_DENSE || r1 > g.Lv) {  // dense head or a text row present: every key tile
    t.a0 = 0;
    t.a1 = g.nkb;
    t.b0 = t.b1 = g.nkb;
    return t;
  }
  int lo0, hi0, lo1, hi1;
  row_interval(g, kind, r0, lo0, hi0);
  row_interval(g, kind, r1 - 1, lo1, hi1);
  t.a0 = lo0 / g.bk;
  t.a1 = (hi1 - 1) / g.bk + 1;
  if (g.T > 0) {
    t.b0 = max(g.Lv / g.bk, t.a1);
    t.b1 = g.nkb;
    if (t.b0 > t.b1) t.b0 = t.b1;
  } else {
    t.b0 = t.b1 = t.a1;
  }
  return t;
}

__device__ __forceinline__ uint8_t tile_full(const Geometry& g, const TileRanges& t, int kb) {
  const int k0 = kb * g.bk;
  const int kv_end = min(min(k0 + g.bk, g.L), g.Lv);
  if (k0 >= g.Lv || t.rv1 <= t.r0) return 1;     // only text keys, or only text queries
  return (t.lo_last <= k0 && kv_end <= t.hi_first) ? 1 : 0;
}

__global__ void block_count_kernel(const Geometry g, const uint8_t* __restrict__ kind, int32_t* __restrict__ row_ptr) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t n = static_cast<int64_t>(g.BH) * g.nqb;
  if (i >= n) return;
  const int bh = static_cast<int>(i / g.nqb), qb = static_cast<int>(i % g.nqb);
  const TileRanges t = tile_ranges(g, kind[bh], qb);
  row_ptr[i + 1] = (t.a1 - t.a0) + (t.b1 - t.b0);
  if (i == 0) row_ptr[0] = 0;
}

// In-place inclusive scan of row_ptr[1..n] by one block of 1024 threads.
__global__ void __launch_bounds__(1024) block_scan_kernel(int32_t* __restrict__ row_ptr, int64_t n, int64_t capacity) {
  __shared__ long long part[1024];
  const int tid = threadIdx.x;
  const int64_t per = (n + 1023) / 1024;
  const int64_t b = tid * per, e = min(n, b + per);
  long long s = 0;
  for (int64_t i = b; i < e; i++) s += row_ptr[i + 1];
  part[tid] = s;
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {
    long long v = (tid >= off) ? part[tid - off] : 0;
    __syncthreads();
    part[tid] += v;
    __syncthreads();
  }
  long long run = (tid > 0) ? part[tid - 1] : 0;
  for (int64_t i = b; i < e; i++) {
    run += row_ptr[i + 1];
    row_ptr[i + 1] = static_cast<int32_t>(min(run, static_cast<long long>(INT32_MAX)));
  }
  if (tid == 1023 && part[1023] > capacity) atomicOr(&g_error_word, kErrCapacity);
}

// One warp per (b, h, qb): writes its kb list and full flags.
__global__ void block_fill_kernel(const Geometry g, const uint8_t* __restrict__ kind,
                                  const int32_t* __restrict__ row_ptr, int32_t* __restrict__ col,
                                  uint8_t* __restrict__ full, int64_t capacity) {
  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t n = static_cast<int64_t>(g.BH) * g.nqb;
  if (wid >= n) return;
  const int bh = static_cast<int>(wid / g.nqb), qb = static_cast<int>(wid % g.nqb);
  const TileRanges t = tile_ranges(g, kind[bh], qb);
  const int na = t.a1 - t.a0, cnt = na + (t.b1 - t.b0);
  const int64_t start = row_ptr[wid];
  for (int e = lane; e < cnt; e += 32) {
    const int64_t pos = start + e;
    if (pos >= capacity) break;
    const int kb = (e < na) ? t.a0 + e : t.b0 + (e - na);
    col[pos] = kb;
    full[pos] = tile_full(g, t, kb);
  }
}

}  // namespace svg
