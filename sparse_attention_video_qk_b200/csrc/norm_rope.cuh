// norm_rope.cuh — QK-Norm (RMSNorm with a per-channel gain) and 3D RoPE of one
// row, as a device routine that both the row kernel and the profiling kernel
// call, so the two produce the same bf16 bits ("Sparse VideoGen" WeChat
// article, "其他优化方法"; ICML 2025 report, "Layout Transformation + Kernel
// 加速").
//
// A row of d elements is handled by LPR = d/8 consecutive lanes of a warp, lane
// c holding elements [8c, 8c+8) as one 16-byte vector.  The sum of squares is
// four packed fp32 FMAs per lane followed by a butterfly over the row's lanes
// (every lane ends with the same value).  RoPE rotates the pairs (2j, 2j+1)
// inside the t, h, w sections by angles read from a host-built fp32 (cos, sin)
// table, so no transcendental runs on the device.
#pragma once

#include "svg_common.cuh"

namespace svg {

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

// What the routine needs besides the row: the RoPE table and its layout.
struct RopeArgs {
  const float2* table;       // (cos, sin) entries: section t, then h, then w
  float eps;
  int split0, split1;        // widths of the t and h sections (w = d - split0 - split1)
  int off1, off2;            // table offsets (in entries) of the h and w sections
  int vec;                   // 1: every section is a multiple of 8 wide, so a lane's 4 pairs share
                             //    a section and sit next to each other in the table
  FastDiv divS, divWs;       // division by S = Hs*Ws and by Ws
};

// Lane c's four pairs: their section and their table column / row stride.
struct RopeLane {
  int sec[4], tab[4], stride[4];
};

template <int D>
__device__ __forceinline__ RopeLane rope_lane(int c, const RopeArgs& ra) {
  RopeLane rl;
  const int n2 = D - ra.split0 - ra.split1;
#pragma unroll
  for (int i = 0; i < 4; i++) {
    const int e = c * 8 + 2 * i;  // first element of pair i
    if (e < ra.split0) {
      rl.sec[i] = 0; rl.tab[i] = e >> 1; rl.stride[i] = ra.split0 >> 1;
    } else if (e < ra.split0 + ra.split1) {
      rl.sec[i] = 1; rl.tab[i] = ra.off1 + ((e - ra.split0) >> 1); rl.stride[i] = ra.split1 >> 1;
    } else {
      rl.sec[i] = 2; rl.tab[i] = ra.off2 + ((e - ra.split0 - ra.split1) >> 1); rl.stride[i] = n2 >> 1;
    }
  }
  return rl;
}

// Lane c's gains gamma[8c .. 8c+8) as packed pairs.
__device__ __forceinline__ void load_gain(const float* gamma, int c, uint64_t gam[4]) {
  const float4* gm = reinterpret_cast<const float4*>(gamma + c * 8);
  const float4 g0 = __ldg(gm), g1 = __ldg(gm + 1);
  gam[0] = pack_f2(g0.x, g0.y);
  gam[1] = pack_f2(g0.z, g0.w);
  gam[2] = pack_f2(g1.x, g1.y);
  gam[3] = pack_f2(g1.z, g1.w);
}

// QK-Norm, then RoPE for video tokens (tok < Lv, frame-major index), of lane
// c's vector x of one row.  All D/8 lanes of the row call it together (full
// warp).  `table` is ra.table or a copy of it; SMEM_TABLE: the copy is in
// shared memory (16-byte aligned), so the vector loads may be used.
template <int D, bool SMEM_TABLE>
__device__ __forceinline__ uint4 norm_rope_vec(uint4 x, int tok, const Geometry& g, const uint64_t gam[4],
                                              const RopeLane& rl, const RopeArgs& ra, const float2* table) {
  constexpr int LPR = D / 8;
  // packed fp32 pairs: element pairs (2i, 2i+1) are exactly the RoPE pairs
  uint64_t v2[4];
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
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
  const float inv = rsqrtf(ss * (1.0f / D) + ra.eps);
  const uint64_t inv2 = pack_f2(inv, inv);
#pragma unroll
  for (int i = 0; i < 4; i++) v2[i] = mul_f2(mul_f2(v2[i], inv2), gam[i]);
  if (tok < g.Lv) {
    const int f = fdiv(tok, ra.divS), s = tok - f * g.S;
    const int yy = fdiv(s, ra.divWs), xx = s - yy * g.Ws;
    float2 cs[4];
    if (SMEM_TABLE && ra.vec) {
      // the lane's 4 (cos, sin) pairs in two 16-byte shared-memory loads
      const int pos = rl.sec[0] == 0 ? f : (rl.sec[0] == 1 ? yy : xx);
      const float4* t4 = reinterpret_cast<const float4*>(table + rl.tab[0] + pos * rl.stride[0]);
      const float4 c01 = t4[0], c23 = t4[1];
      cs[0] = make_float2(c01.x, c01.y);
      cs[1] = make_float2(c01.z, c01.w);
      cs[2] = make_float2(c23.x, c23.y);
      cs[3] = make_float2(c23.z, c23.w);
    } else {
#pragma unroll
      for (int i = 0; i < 4; i++) {
        const int pos = rl.sec[i] == 0 ? f : (rl.sec[i] == 1 ? yy : xx);
        cs[i] = SMEM_TABLE ? table[rl.tab[i] + pos * rl.stride[i]] : __ldg(table + rl.tab[i] + pos * rl.stride[i]);
      }
    }
#pragma unroll
    for (int i = 0; i < 4; i++) {
      // (u, v) -> (u c - v s, u s + v c) = (u, u) * (c, s) + (-v, v) * (s, c)
      float u0, u1;
      unpack_f2(v2[i], u0, u1);
      v2[i] = fma_f2(pack_f2(-u1, u1), pack_f2(cs[i].y, cs[i].x), mul_f2(pack_f2(u0, u0), pack_f2(cs[i].x, cs[i].y)));
    }
  }
  float r[8];
#pragma unroll
  for (int i = 0; i < 4; i++) unpack_f2(v2[i], r[2 * i], r[2 * i + 1]);
  uint4 y;
  y.x = pack_bf16x2(r[0], r[1]);
  y.y = pack_bf16x2(r[2], r[3]);
  y.z = pack_bf16x2(r[4], r[5]);
  y.w = pack_bf16x2(r[6], r[7]);
  return y;
}

}  // namespace svg
