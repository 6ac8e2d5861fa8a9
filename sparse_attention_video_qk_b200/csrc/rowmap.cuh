// rowmap.cuh — one bandwidth-bound row kernel for three stages of the step:
//   * QK-Norm + 3D RoPE ("Sparse VideoGen" WeChat article, "其他优化方法";
//     ICML 2025 report, "Layout Transformation + Kernel 加速"),
//   * the frame-major -> token-major layout transform of temporal heads
//     (article, "硬件高效的 Layout Transformation"),
//   * its inverse on the attention output.
// Grid: a persistent set of blocks (the resident capacity) strides over work
// units of (tensor, head, a run of destination rows); every index is 32-bit.  Every destination row is produced by LPR = d/8
// lanes, each moving one 16-byte vector; a warp covers 32/LPR consecutive
// destination rows per step and keeps U steps of loads in flight before
// computing.  The RMSNorm sum of squares is a shuffle reduction over the row's
// lanes.  RoPE: a lane's 4 pairs have fixed sections (computed once); angles
// come from a host-built fp32 (cos, sin) table staged in shared memory, so no
// transcendental runs on the device.  Divisions by F, S and Ws use
// multiply-shift reciprocals.
#pragma once

#include "svg_common.cuh"

namespace svg {

enum : int { kRowmapInverse = 4 };

// n / d for 0 <= n < 2^31 as (umulhi(n, m) + n) >> l, with l = ceil(log2 d)
// and m = floor(2^32 (2^l - d) / d) + 1 (Granlund & Montgomery, "Division by
// invariant integers using multiplication", PLDI 1994).
struct FastDiv {
  uint32_t m;
  int l;
  int d;
};

inline FastDiv make_fastdiv(int d) {
  FastDiv f;
  f.d = d;
  f.l = 0;
  while ((1ll << f.l) < d) f.l++;
  f.m = static_cast<uint32_t>(((1ull << 32) * ((1ull << f.l) - static_cast<uint64_t>(d))) / static_cast<uint64_t>(d) + 1);
  return f;
}

__device__ __forceinline__ int fdiv(int n, const FastDiv& f) {
  const uint32_t hi = __umulhi(static_cast<uint32_t>(n), f.m);
  return static_cast<int>((hi + static_cast<uint32_t>(n)) >> f.l);
}

// packed fp32 pairs (Blackwell f32x2 ALU ops)
__device__ __forceinline__ uint64_t pack_f2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void unpack_f2(uint64_t r, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ uint64_t mul_f2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t fma_f2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

#ifndef SVG_ROWMAP_STEPS
#define SVG_ROWMAP_STEPS 4
#endif
constexpr int kRowmapSteps = SVG_ROWMAP_STEPS;            // row steps each warp keeps in flight
constexpr int kRowmapUnitSteps = 4;                       // block iterations per work unit
constexpr int kRowmapBlocksPerSM = 4;                     // resident blocks of 256 threads per SM

constexpr int kRopeSmemFloats = 24576;  // 96 KB: tables up to this size are staged in shared memory

struct RowmapArgs {
  Geometry g;
  int flags;                 // SVG_NORM_ROPE | SVG_LAYOUT | kRowmapInverse
  int ntensor;               // tensors processed by this launch (<= 3)
  int norm_tensors;          // the first `norm_tensors` tensors get QK-Norm + RoPE
  const uint16_t* src[3];
  uint16_t* dst[3];
  const float* gamma[2];
  const float2* rope;        // (cos, sin) table: section t, then h, then w
  int rope_floats;           // table size in floats
  const uint8_t* kind;       // [B*H], needed when rows move
  float eps;
  int split0, split1;        // widths of the t and h sections (w = d - split0 - split1)
  int rope_off1, rope_off2;  // table offsets (in float2) of the h and w sections
  int rope_vec;              // 1: every section is a multiple of 8 wide, so a lane's 4 pairs share a
                             //    section and sit next to each other in the table
  FastDiv divF, divS, divWs;
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
  int sec[4], tab[4], stride[4];
  if (a.norm_tensors > 0) {
    if constexpr (STAGED) {
      for (int i = threadIdx.x; i < a.rope_floats / 2; i += blockDim.x) rope_s[i] = __ldg(a.rope + i);
    }
    const int n2 = D - a.split0 - a.split1;
#pragma unroll
    for (int i = 0; i < 4; i++) {
      const int e = c * 8 + 2 * i;  // first element of pair i
      if (e < a.split0) {
        sec[i] = 0; tab[i] = e >> 1; stride[i] = a.split0 >> 1;
      } else if (e < a.split0 + a.split1) {
        sec[i] = 1; tab[i] = a.rope_off1 + ((e - a.split0) >> 1); stride[i] = a.split1 >> 1;
      } else {
        sec[i] = 2; tab[i] = a.rope_off2 + ((e - a.split0 - a.split1) >> 1); stride[i] = n2 >> 1;
      }
    }
  }
  __syncthreads();

  // Work units: (tensor, head, UNIT consecutive destination rows), strided over the grid.
  const int nchunk = (g.L + UNIT - 1) / UNIT;
  const int nunits = a.ntensor * g.BH * nchunk;
  for (int unit = blockIdx.x; unit < nunits; unit += gridDim.x) {
    const int th = unit / nchunk, ch = unit - th * nchunk;
    const int t = th / g.BH, bh = th - t * g.BH;
    const bool norm = (a.flags & SVG_NORM_ROPE) && t < a.norm_tensors;
    const bool temporal = moves && a.kind[bh] == SVG_HEAD_TEMPORAL;
    uint64_t gam[4] = {0ull, 0ull, 0ull, 0ull};
    if (norm) {
      const float4* gm = reinterpret_cast<const float4*>(a.gamma[t] + c * 8);
      const float4 g0 = __ldg(gm), g1 = __ldg(gm + 1);
      gam[0] = pack_f2(g0.x, g0.y);
      gam[1] = pack_f2(g0.z, g0.w);
      gam[2] = pack_f2(g1.x, g1.y);
      gam[3] = pack_f2(g1.z, g1.w);
    }
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
            const int f = fdiv(p, a.divS), s = p - f * g.S;
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
        uint4 y = x[u];
        if (norm) {
          // packed fp32 pairs: element pairs (2i, 2i+1) are exactly the RoPE pairs
          uint64_t v2[4];
          const uint32_t w[4] = {x[u].x, x[u].y, x[u].z, x[u].w};
#pragma unroll
          for (int i = 0; i < 4; i++) v2[i] = pack_f2(bf16_lo(w[i]), bf16_hi(w[i]));
          uint64_t ss2 = mul_f2(v2[0], v2[0]);
#pragma unroll
          for (int i = 1; i < 4; i++) ss2 = fma_f2(v2[i], v2[i], ss2);
          float s0, s1;
          unpack_f2(ss2, s0, s1);
          float ss = s0 + s1;
#pragma unroll
          for (int o = LPR / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
          const float inv = rsqrtf(ss * (1.0f / D) + a.eps);
          const uint64_t inv2 = pack_f2(inv, inv);
#pragma unroll
          for (int i = 0; i < 4; i++) v2[i] = mul_f2(mul_f2(v2[i], inv2), gam[i]);
          if (tok[u] < g.Lv) {
            const int f = fdiv(tok[u], a.divS), s = tok[u] - f * g.S;
            const int yy = fdiv(s, a.divWs), xx = s - yy * g.Ws;
            float2 cs[4];
            if (STAGED && a.rope_vec) {
              // the lane's 4 (cos, sin) pairs in two 16-byte shared-memory loads
              const int pos = sec[0] == 0 ? f : (sec[0] == 1 ? yy : xx);
              const float4* t4 = reinterpret_cast<const float4*>(rope_s + tab[0] + pos * stride[0]);
              const float4 c01 = t4[0], c23 = t4[1];
              cs[0] = make_float2(c01.x, c01.y);
              cs[1] = make_float2(c01.z, c01.w);
              cs[2] = make_float2(c23.x, c23.y);
              cs[3] = make_float2(c23.z, c23.w);
            } else {
#pragma unroll
              for (int i = 0; i < 4; i++) {
                const int pos = sec[i] == 0 ? f : (sec[i] == 1 ? yy : xx);
                cs[i] = STAGED ? rope_s[tab[i] + pos * stride[i]] : __ldg(a.rope + tab[i] + pos * stride[i]);
              }
            }
#pragma unroll
            for (int i = 0; i < 4; i++) {
              // (u, v) -> (u c - v s, u s + v c) = (u, u) * (c, s) + (-v, v) * (s, c)
              float u0, u1;
              unpack_f2(v2[i], u0, u1);
              v2[i] = fma_f2(pack_f2(-u1, u1), pack_f2(cs[i].y, cs[i].x),
                             mul_f2(pack_f2(u0, u0), pack_f2(cs[i].x, cs[i].y)));
            }
          }
          float r[8];
#pragma unroll
          for (int i = 0; i < 4; i++) unpack_f2(v2[i], r[2 * i], r[2 * i + 1]);
          y.x = pack_bf16x2(r[0], r[1]);
          y.y = pack_bf16x2(r[2], r[3]);
          y.z = pack_bf16x2(r[4], r[5]);
          y.w = pack_bf16x2(r[6], r[7]);
        }
        const int p = base + u * RPW + sub;
        if (valid[u]) reinterpret_cast<uint4*>(dst + static_cast<int64_t>(p) * D)[c] = y;
      }
    }
  }
}

}  // namespace svg
