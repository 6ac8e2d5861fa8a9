// rowmap.cuh — one bandwidth-bound row kernel for three stages of the step:
//   * QK-Norm + 3D RoPE ("Sparse VideoGen" WeChat article, "其他优化方法";
//     ICML 2025 report, "Layout Transformation + Kernel 加速"),
//   * the frame-major -> token-major layout transform of temporal heads
//     (article, "硬件高效的 Layout Transformation"),
//   * its inverse on the attention output.
// Grid: a persistent set of blocks (the resident capacity) strides over work
// units of (tensor, head, a run of destination rows); every index is 32-bit.
// Every destination row is produced by LPR = d/8 lanes, each moving one
// 16-byte vector; a warp covers 32/LPR consecutive
// destination rows per step and keeps U steps of loads in flight before
// computing.  QK-Norm + RoPE is the shared routine of norm_rope.cuh, with the
// (cos, sin) table staged in shared memory.  Divisions by F, S and Ws use
// multiply-shift reciprocals.
#pragma once

#include "norm_rope.cuh"
#include "svg_common.cuh"

namespace svg {

enum : int { kRowmapInverse = 4 };

#ifndef SVG_ROWMAP_STEPS
#define SVG_ROWMAP_STEPS 4
#endif
constexpr int kRowmapSteps = SVG_ROWMAP_STEPS;            // row steps each warp keeps in flight
constexpr int kRowmapUnitSteps = 4;                       // block iterations per work unit
constexpr int kRowmapBlocksPerSM = 4;                     // resident blocks of 256 threads per SM

constexpr int kRopeSmemFloats = 24576;  // 96 KB: tables up to this size are staged in shared memory

struct RowmapArgs {
  Geometry g;
  int flags;                 // SVG_LAYOUT | kRowmapInverse: rows move (temporal heads)
  int ntensor;               // tensors processed by this launch (<= 3)
  int norm_tensors;          // the first `norm_tensors` tensors get QK-Norm + RoPE
  const uint16_t* src[3];
  uint16_t* dst[3];
  const float* gamma[3];     // gains of the normalised tensors
  const uint8_t* kind;       // [B*H], needed when rows move
  int rope_floats;           // table size in floats
  RopeArgs rope;             // table in global memory
  FastDiv divF;
};

// STAGED: the RoPE table is copied into shared memory (dynamic, rope_floats * 4
// bytes); otherwise it is read through the read-only data cache.
template <int D, bool STAGED>
__global__ void __launch_bounds__(256, kRowmapBlocksPerSM) rowmap_kernel(const RowmapArgs a) {
  constexpr int LPR = D / 8;       // lanes per row
  constexpr int RPW = 32 / LPR;    // rows per warp step
  constexpr int U = kRowmapSteps;  // warp steps in flight
  constexpr int NW = 8;            // warps per block
  constexpr int UNIT = NW * RPW * U * kRowmapUnitSteps;   // rows per work unit
  extern __shared__ float2 rope_s[];   // a.rope_floats / 2 entries when the table is staged
  const Geometry& g = a.g;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane / LPR, c = lane % LPR;
  const bool inverse = (a.flags & kRowmapInverse) != 0;
  const bool moves = (a.flags & (SVG_LAYOUT | kRowmapInverse)) != 0;

  // RoPE set-up: the table in shared memory (when staged) and this lane's 4 pairs
  const float2* table = STAGED ? rope_s : a.rope.table;
  RopeLane rl{};
  if (a.norm_tensors > 0) {
    if constexpr (STAGED) {
      for (int i = threadIdx.x; i < a.rope_floats / 2; i += blockDim.x) rope_s[i] = __ldg(a.rope.table + i);
    }
    rl = rope_lane<D>(c, a.rope);
  }
  __syncthreads();

  // Work units: (tensor, head, UNIT consecutive destination rows), strided over the grid.
  const int nchunk = (g.L + UNIT - 1) / UNIT;
  const int nunits = a.ntensor * g.BH * nchunk;
  for (int unit = blockIdx.x; unit < nunits; unit += gridDim.x) {
    const int th = unit / nchunk, ch = unit - th * nchunk;
    const int t = th / g.BH, bh = th - t * g.BH;
    const bool norm = t < a.norm_tensors;
    const bool temporal = moves && a.kind[bh] == SVG_HEAD_TEMPORAL;
    uint64_t gam[4] = {0ull, 0ull, 0ull, 0ull};
    if (norm) load_gain(a.gamma[t], c, gam);
    const int64_t hbase = static_cast<int64_t>(bh) * g.L;
    const uint16_t* src = a.src[t] + hbase * D;
    uint16_t* dst = a.dst[t] + hbase * D;
    const int row_end = min(g.L, (ch + 1) * UNIT);
    for (int base = ch * UNIT + warp * RPW * U; base < row_end; base += NW * RPW * U) {
      uint4 x[U];
      int tok[U];
      bool valid[U];
#pragma unroll
      for (int u = 0; u < U; u++) {
        const int p = base + u * RPW + sub;   // destination row in this head
        valid[u] = p < row_end;
        int src_p = p;
        if (temporal && p < g.Lv) {
          if (inverse) {                      // destination frame-major f*S+s <- s*F+f
            const int f = fdiv(p, a.rope.divS), s = p - f * g.S;
            src_p = s * g.F + f;
          } else {                            // destination token-major s*F+f <- f*S+s
            const int s = fdiv(p, a.divF), f = p - s * g.F;
            src_p = f * g.S + s;
          }
        }
        tok[u] = src_p;                       // frame-major token index for RoPE
        x[u] = valid[u] ? __ldg(reinterpret_cast<const uint4*>(src + static_cast<int64_t>(src_p) * D) + c)
                        : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < U; u++) {
        const uint4 y = norm ? norm_rope_vec<D, STAGED>(x[u], tok[u], g, gam, rl, a.rope, table) : x[u];
        const int p = base + u * RPW + sub;
        if (valid[u]) reinterpret_cast<uint4*>(dst + static_cast<int64_t>(p) * D)[c] = y;
      }
    }
  }
}

}  // namespace svg
