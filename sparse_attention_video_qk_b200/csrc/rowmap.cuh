// rowmap.cuh — one bandwidth-bound row kernel for three stages of the step:
//   * QK-Norm + 3D RoPE ("Sparse VideoGen" WeChat article, "其他优化方法";
//     ICML 2025 report, "Layout Transformation + Kernel 加速"),
//   * the frame-major -> token-major layout transform of temporal heads
//     (article, "硬件高效的 Layout Transformation"),
//   * its inverse on the attention output.
// Every destination row is produced by LPR = d/8 lanes, each moving one
// 16-byte vector; a warp covers 32/LPR consecutive destination rows per step
// and keeps U steps of loads in flight before computing.  The RMSNorm sum of
// squares is a shuffle reduction over the row's lanes.  RoPE angles come from
// a host-built fp32 (cos, sin) table, so no transcendental runs on the device.
#pragma once

#include "svg_common.cuh"

namespace svg {

enum : int { kRowmapInverse = 4 };

struct RowmapArgs {
  Geometry g;
  int flags;                 // SVG_NORM_ROPE | SVG_LAYOUT | kRowmapInverse
  int ntensor;               // tensors processed by this launch (<= 3)
  int norm_tensors;          // the first `norm_tensors` tensors get QK-Norm + RoPE
  const uint16_t* src[3];
  uint16_t* dst[3];
  const float* gamma[2];
  const float2* rope;        // (cos, sin) table: section t, then h, then w
  const uint8_t* kind;       // [B*H], needed when rows move
  float eps;
  int split0, split1;        // widths of the t and h sections (w = d - split0 - split1)
  int rope_off1, rope_off2;  // table offsets (in float2) of the h and w sections
};

template <int D>
__global__ void __launch_bounds__(256) rowmap_kernel(const RowmapArgs a) {
  constexpr int LPR = D / 8;       // lanes per row
  constexpr int RPW = 32 / LPR;    // rows per warp step
  constexpr int U = 4;             // warp steps in flight
  const Geometry& g = a.g;
  const int lane = threadIdx.x & 31;
  const int sub = lane / LPR, c = lane % LPR;
  const int64_t rows_per_tensor = static_cast<int64_t>(g.BH) * g.L;
  const int64_t total = rows_per_tensor * a.ntensor;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarp = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const bool moves = (a.flags & (SVG_LAYOUT | kRowmapInverse)) != 0;

  for (int64_t base = warp * (RPW * U); base < total; base += nwarp * (RPW * U)) {
    uint4 x[U];
    int64_t dst_row[U];
    int tok[U], tensor[U];
    bool valid[U];
#pragma unroll
    for (int u = 0; u < U; u++) {
      const int64_t gr = base + u * RPW + sub;  // destination row over all tensors
      valid[u] = gr < total;
      tok[u] = 0;
      tensor[u] = 0;
      dst_row[u] = 0;
      x[u] = make_uint4(0, 0, 0, 0);
      if (!valid[u]) continue;
      const int t = static_cast<int>(gr / rows_per_tensor);
      const int64_t rem = gr - t * rows_per_tensor;
      const int bh = static_cast<int>(rem / g.L);
      const int p = static_cast<int>(rem - static_cast<int64_t>(bh) * g.L);
      int src_p = p;
      if (moves && p < g.Lv && a.kind[bh] == SVG_HEAD_TEMPORAL) {
        if (a.flags & kRowmapInverse) {   // destination is frame-major f*S+s <- s*F+f
          const int f = p / g.S, s = p - f * g.S;
          src_p = s * g.F + f;
        } else {                          // destination is token-major s*F+f <- f*S+s
          const int s = p / g.F, f = p - s * g.F;
          src_p = f * g.S + s;
        }
      }
      tok[u] = src_p;                     // frame-major token index for RoPE
      tensor[u] = t;
      const int64_t hrow = static_cast<int64_t>(bh) * g.L;
      x[u] = __ldg(reinterpret_cast<const uint4*>(a.src[t] + (hrow + src_p) * D) + c);
      dst_row[u] = hrow + p;
    }
#pragma unroll
    for (int u = 0; u < U; u++) {
      float v[8];
      const uint32_t w[4] = {x[u].x, x[u].y, x[u].z, x[u].w};
#pragma unroll
      for (int i = 0; i < 4; i++) {
        v[2 * i] = bf16_lo(w[i]);
        v[2 * i + 1] = bf16_hi(w[i]);
      }
      float ss = 0.f;
#pragma unroll
      for (int i = 0; i < 8; i++) ss = fmaf(v[i], v[i], ss);
#pragma unroll
      for (int o = LPR / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (!valid[u]) continue;
      uint4 y = x[u];
      if ((a.flags & SVG_NORM_ROPE) && tensor[u] < a.norm_tensors) {
        const float inv = rsqrtf(ss * (1.0f / D) + a.eps);
        const float4* gm = reinterpret_cast<const float4*>(a.gamma[tensor[u]] + c * 8);
        const float4 g0 = __ldg(gm), g1 = __ldg(gm + 1);
        const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
        for (int i = 0; i < 8; i++) v[i] = v[i] * inv * gg[i];
        if (tok[u] < g.Lv) {
          const int f = tok[u] / g.S, s = tok[u] - f * g.S;
          const int yy = s / g.Ws, xx = s - yy * g.Ws;
#pragma unroll
          for (int i = 0; i < 4; i++) {
            const int e = c * 8 + 2 * i;  // first element of the pair
            int idx;
            if (e < a.split0) {
              idx = f * (a.split0 >> 1) + (e >> 1);
            } else if (e < a.split0 + a.split1) {
              idx = a.rope_off1 + yy * (a.split1 >> 1) + ((e - a.split0) >> 1);
            } else {
              const int n2 = D - a.split0 - a.split1;
              idx = a.rope_off2 + xx * (n2 >> 1) + ((e - a.split0 - a.split1) >> 1);
            }
            const float2 cs = __ldg(a.rope + idx);
            const float u0 = v[2 * i], u1 = v[2 * i + 1];
            v[2 * i] = u0 * cs.x - u1 * cs.y;
            v[2 * i + 1] = u0 * cs.y + u1 * cs.x;
          }
        }
        y.x = pack_bf16x2(v[0], v[1]);
        y.y = pack_bf16x2(v[2], v[3]);
        y.z = pack_bf16x2(v[4], v[5]);
        y.w = pack_bf16x2(v[6], v[7]);
      }
      reinterpret_cast<uint4*>(a.dst[tensor[u]] + dst_row[u] * D)[c] = y;
    }
  }
}

}  // namespace svg
