// profile.cuh — online profiling ("Sparse VideoGen" WeChat article, "Online
// Profiling Strategy"; ICML 2025 report, "动态自适应的稀疏策略" steps 1-3).
//
// For each head, n <= 64 sampled query rows are attended three ways at once:
// densely, with the spatial mask and with the temporal mask.  The three
// softmaxes share one running maximum (softmax is shift invariant), so one
// pass over the keys feeds three accumulators O_dense, O_spatial, O_temporal
// and three row sums.  The keys of a head are split into chunks handled by
// separate CTAs (split-KV); a second kernel merges the chunks, forms
//   MSE_m = mean over rows and columns of (O_m - O_dense)^2
// with a fixed reduction order, and picks SPATIAL iff MSE_s <= MSE_t.
//
// Products run on the tensor cores with mma.sync m16n8k16 (bf16 in, fp32
// accumulate): 8 warps, warp w owns query rows 16*(w%4)..+15 and output
// columns (w/4)*d/2..+d/2 of all three accumulators.  K/V tiles of 64 keys are
// staged through padded shared memory by cp.async, double buffered.
#pragma once

#include "svg_common.cuh"

namespace svg {

constexpr int kProfRows = 64;      // sampled rows per head (padded)
constexpr int kProfKeys = 64;      // keys per tile
constexpr int kProfThreads = 256;
constexpr int kNoKey = -2, kTextKey = -1;

__host__ __device__ constexpr int prof_rec_floats(int D) { return 4 + 3 * D; }

// Number of key chunks per head: enough CTAs for ~3 waves on 148 SMs, at
// least two tiles per chunk.
__host__ __device__ inline int prof_chunks(int BH, int L) {
  const int ntiles = (L + kProfKeys - 1) / kProfKeys;
  int c = (3 * 148 + BH - 1) / BH;
  const int cap = (ntiles + 1) / 2;
  if (c > cap) c = cap;
  if (c < 1) c = 1;
  return c;
}

struct ProfArgs {
  Geometry g;
  float scale_log2;
  const uint16_t* q;
  const uint16_t* k;
  const uint16_t* v;
  const int32_t* sample;
  int n;
  int nchunk;
  int tiles_per_chunk;
  float* ws;           // [BH][nchunk][64][rec]
  float* mse_out;      // [BH][2] or null
  uint8_t* kind_out;   // [BH]
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16_16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <int D>
struct ProfSmem {
  static constexpr int LDS = D + 8;                  // padded row (elements): conflict-free ldmatrix
  static constexpr int TILE = kProfKeys * LDS;       // elements per K or V tile
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = kProfRows * LDS;      // 2 stages
  static constexpr int V_OFF = K_OFF + 2 * TILE;     // 2 stages
  static constexpr int ELEMS = V_OFF + 2 * TILE;
  static constexpr int BYTES = ELEMS * 2 + 2 * kProfKeys * 8;  // + key meta (frame, location) per stage
};

template <int D>
__global__ void __launch_bounds__(kProfThreads, 1) profile_partial_kernel(const ProfArgs a) {
  using SM = ProfSmem<D>;
  constexpr int LDS = SM::LDS;
  constexpr int NK = D / 16;        // k-steps of Q.K^T
  constexpr int NO = D / 16;        // n8 output tiles per warp (d/2 columns)
  extern __shared__ __align__(16) uint16_t psm[];
  int2* meta = reinterpret_cast<int2*>(psm + SM::ELEMS);   // [2][64] (frame, location)
  const Geometry& g = a.g;
  const int bh = blockIdx.y, chunk = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rg = warp & 3, dh = warp >> 2;
  const int gq = lane >> 2, tq = lane & 3;
  const int64_t hoff = static_cast<int64_t>(bh) * g.L * D;
  const uint16_t* Kh = a.k + hoff;
  const uint16_t* Vh = a.v + hoff;
  const int ntiles_all = (g.L + kProfKeys - 1) / kProfKeys;
  const int t_begin = chunk * a.tiles_per_chunk;
  const int t_end = min(ntiles_all, t_begin + a.tiles_per_chunk);
  const int key_end = min(g.L, t_end * kProfKeys);

  // ---- gather the sampled query rows
  for (int i = tid; i < kProfRows * (D / 8); i += kProfThreads) {
    const int r = i / (D / 8), c = i % (D / 8);
    int tok = 0, bytes = 0;
    if (r < a.n) {
      tok = a.sample[r];
      if (tok < 0 || tok >= g.L) {
        atomicOr(&g_error_word, kErrBadIndex);
        tok = 0;
      }
      bytes = 16;
    }
    cp_async16(smem_addr(psm + SM::Q_OFF + r * LDS + c * 8), a.q + hoff + static_cast<int64_t>(tok) * D + c * 8, bytes);
  }
  auto load_tile = [&](int t, int stage) {
    const int k0 = t * kProfKeys;
    for (int i = tid; i < kProfKeys * (D / 8); i += kProfThreads) {
      const int r = i / (D / 8), c = i % (D / 8);
      const int key = k0 + r;
      const bool ok = key < key_end;
      const int64_t off = static_cast<int64_t>(ok ? key : 0) * D + c * 8;
      cp_async16(smem_addr(psm + SM::K_OFF + stage * SM::TILE + r * LDS + c * 8), Kh + off, ok ? 16 : 0);
      cp_async16(smem_addr(psm + SM::V_OFF + stage * SM::TILE + r * LDS + c * 8), Vh + off, ok ? 16 : 0);
    }
    if (tid < kProfKeys) {
      const int key = k0 + tid;
      int2 m;
      if (key >= key_end) m = make_int2(kNoKey, 0);
      else if (key >= g.Lv) m = make_int2(kTextKey, 0);
      else m = make_int2(key / g.S, key % g.S);
      meta[stage * kProfKeys + tid] = m;
    }
  };
  load_tile(t_begin, 0);
  cp_async_commit();

  // ---- per-row state (rows gq and gq+8 of this warp's 16)
  int fq[2], sq[2];
  bool textq[2];
#pragma unroll
  for (int h = 0; h < 2; h++) {
    const int r = rg * 16 + gq + 8 * h;
    int tok = (r < a.n) ? a.sample[r] : 0;
    if (tok < 0 || tok >= g.L) tok = 0;
    textq[h] = tok >= g.Lv;
    fq[h] = tok / g.S;
    sq[h] = tok % g.S;
  }
  float m_run[2] = {-INFINITY, -INFINITY};
  float l_d[2] = {0.f, 0.f}, l_s[2] = {0.f, 0.f}, l_t[2] = {0.f, 0.f};
  float od[NO][4], os[NO][4], ot[NO][4];
#pragma unroll
  for (int j = 0; j < NO; j++)
#pragma unroll
    for (int e = 0; e < 4; e++) od[j][e] = os[j][e] = ot[j][e] = 0.f;

  uint32_t qf[NK][4];
  bool have_q = false;

  for (int t = t_begin; t < t_end; t++) {
    const int stage = (t - t_begin) & 1;
    if (t + 1 < t_end) load_tile(t + 1, stage ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (!have_q) {
#pragma unroll
      for (int kk = 0; kk < NK; kk++) {
        const int mi = lane >> 3;
        const int row = rg * 16 + (mi & 1) * 8 + (lane & 7);
        const int col = kk * 16 + (mi >> 1) * 8;
        ldsm_x4(smem_addr(psm + SM::Q_OFF + row * LDS + col), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
      }
      have_q = true;
    }
    const uint16_t* sK = psm + SM::K_OFF + stage * SM::TILE;
    const uint16_t* sV = psm + SM::V_OFF + stage * SM::TILE;
    const int2* mt = meta + stage * kProfKeys;

    // S = Q K^T for 16 rows x 64 keys
    float sc[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; nt++)
#pragma unroll
      for (int e = 0; e < 4; e++) sc[nt][e] = 0.f;
#pragma unroll
    for (int nt = 0; nt < 8; nt++) {
#pragma unroll
      for (int kk = 0; kk < NK; kk += 2) {
        const int mi = lane >> 3;
        const int row = nt * 8 + (lane & 7);
        const int col = kk * 16 + mi * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4(smem_addr(sK + row * LDS + col), b0, b1, b2, b3);
        mma_bf16_16816(sc[nt], qf[kk], b0, b1);
        mma_bf16_16816(sc[nt], qf[kk + 1], b2, b3);
      }
    }
    // masks, running max, probabilities
    uint32_t msk_s[2] = {0u, 0u}, msk_t[2] = {0u, 0u}, msk_v = 0u;   // bit (nt*2+e) per row half
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 8; nt++) {
#pragma unroll
      for (int e = 0; e < 2; e++) {
        const int kc = nt * 8 + 2 * tq + e;
        const int2 km = mt[kc];
        const int bit = nt * 2 + e;
        if (km.x != kNoKey) msk_v |= 1u << bit;
#pragma unroll
        for (int h = 0; h < 2; h++) {
          const bool text = textq[h] || km.x == kTextKey;
          if (text || abs(fq[h] - km.x) <= g.w) msk_s[h] |= 1u << bit;
          if (text || abs(sq[h] - km.y) <= g.r) msk_t[h] |= 1u << bit;
          const float x = sc[nt][2 * h + e] * a.scale_log2;
          sc[nt][2 * h + e] = x;
          if (km.x != kNoKey) mx[h] = fmaxf(mx[h], x);
        }
      }
    }
    float alpha[2];
#pragma unroll
    for (int h = 0; h < 2; h++) {
      mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
      mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
      const float mn = fmaxf(m_run[h], mx[h]);
      alpha[h] = (m_run[h] == -INFINITY) ? 0.f : exp2f(m_run[h] - mn);
      m_run[h] = mn;
      l_d[h] *= alpha[h];
      l_s[h] *= alpha[h];
      l_t[h] *= alpha[h];
    }
#pragma unroll
    for (int j = 0; j < NO; j++) {
#pragma unroll
      for (int e = 0; e < 4; e++) {
        const float al = alpha[e >> 1];
        od[j][e] *= al;
        os[j][e] *= al;
        ot[j][e] *= al;
      }
    }
    // Per 16-key step: P fragments (bf16; row sums use the rounded values so
    // the weights stay consistent), then O_x += P_x V over this warp's d/2
    // output columns.
#pragma unroll
    for (int ks = 0; ks < 4; ks++) {
      uint32_t pd[4], ps[4], pt[4];
#pragma unroll
      for (int half = 0; half < 2; half++) {     // n8 tile 2ks + half
        const int nt = 2 * ks + half;
#pragma unroll
        for (int h = 0; h < 2; h++) {
          float p[2];
#pragma unroll
          for (int e = 0; e < 2; e++) {
            const int bit = nt * 2 + e;
            const bool ok = (msk_v >> bit) & 1u;
            const float pe = ok ? exp2f(sc[nt][2 * h + e] - m_run[h]) : 0.f;
            p[e] = __bfloat162float(__float2bfloat16_rn(pe));
          }
          const uint32_t bs0 = (msk_s[h] >> (nt * 2)) & 1u, bs1 = (msk_s[h] >> (nt * 2 + 1)) & 1u;
          const uint32_t bt0 = (msk_t[h] >> (nt * 2)) & 1u, bt1 = (msk_t[h] >> (nt * 2 + 1)) & 1u;
          const float ps0 = bs0 ? p[0] : 0.f, ps1 = bs1 ? p[1] : 0.f;
          const float pt0 = bt0 ? p[0] : 0.f, pt1 = bt1 ? p[1] : 0.f;
          l_d[h] += p[0] + p[1];
          l_s[h] += ps0 + ps1;
          l_t[h] += pt0 + pt1;
          const int reg = half * 2 + h;          // a0: (g, lo), a1: (g+8, lo), a2: (g, hi), a3: (g+8, hi)
          pd[reg] = pack_bf16x2(p[0], p[1]);
          ps[reg] = pack_bf16x2(ps0, ps1);
          pt[reg] = pack_bf16x2(pt0, pt1);
        }
      }
#pragma unroll
      for (int j = 0; j < NO; j += 2) {
        const int mi = lane >> 3;
        const int row = ks * 16 + (mi & 1) * 8 + (lane & 7);
        const int col = dh * (D / 2) + j * 8 + (mi >> 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(smem_addr(sV + row * LDS + col), b0, b1, b2, b3);
        mma_bf16_16816(od[j], pd, b0, b1);
        mma_bf16_16816(od[j + 1], pd, b2, b3);
        mma_bf16_16816(os[j], ps, b0, b1);
        mma_bf16_16816(os[j + 1], ps, b2, b3);
        mma_bf16_16816(ot[j], pt, b0, b1);
        mma_bf16_16816(ot[j + 1], pt, b2, b3);
      }
    }
    __syncthreads();   // the stage is refilled by the next iteration's prefetch
  }
  cp_async_wait<0>();

  // ---- write the partial record of rows (gq, gq+8)
  constexpr int REC = prof_rec_floats(D);
  float* base = a.ws + (static_cast<int64_t>(bh) * a.nchunk + chunk) * kProfRows * REC;
#pragma unroll
  for (int h = 0; h < 2; h++) {
    float ld = l_d[h], ls = l_s[h], lt = l_t[h];
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
      ld += __shfl_xor_sync(0xffffffffu, ld, o);
      ls += __shfl_xor_sync(0xffffffffu, ls, o);
      lt += __shfl_xor_sync(0xffffffffu, lt, o);
    }
    const int r = rg * 16 + gq + 8 * h;
    float* rec = base + r * REC;
    if (dh == 0 && tq == 0) {
      rec[0] = m_run[h];
      rec[1] = ld;
      rec[2] = ls;
      rec[3] = lt;
    }
#pragma unroll
    for (int j = 0; j < NO; j++) {
      const int c = dh * (D / 2) + j * 8 + 2 * tq;
      *reinterpret_cast<float2*>(rec + 4 + c) = make_float2(od[j][2 * h], od[j][2 * h + 1]);
      *reinterpret_cast<float2*>(rec + 4 + D + c) = make_float2(os[j][2 * h], os[j][2 * h + 1]);
      *reinterpret_cast<float2*>(rec + 4 + 2 * D + c) = make_float2(ot[j][2 * h], ot[j][2 * h + 1]);
    }
  }
}

// Merge the chunks of one head, compute the two MSEs and the choice.
// 256 threads: thread t handles row t/4 and columns t%4, t%4+4, ...
template <int D>
__global__ void __launch_bounds__(256) profile_combine_kernel(const ProfArgs a) {
  constexpr int REC = prof_rec_floats(D);
  const int bh = blockIdx.x, tid = threadIdx.x;
  const int r = tid >> 2, c0 = tid & 3;
  const float* base = a.ws + static_cast<int64_t>(bh) * a.nchunk * kProfRows * REC;
  double es = 0.0, et = 0.0;
  if (r < a.n) {
    float M = -INFINITY;
    for (int ch = 0; ch < a.nchunk; ch++) M = fmaxf(M, base[(ch * kProfRows + r) * REC]);
    float Ld = 0.f, Ls = 0.f, Lt = 0.f;
    for (int ch = 0; ch < a.nchunk; ch++) {
      const float* rec = base + (ch * kProfRows + r) * REC;
      const float wgt = (rec[0] == -INFINITY) ? 0.f : exp2f(rec[0] - M);
      Ld += wgt * rec[1];
      Ls += wgt * rec[2];
      Lt += wgt * rec[3];
    }
    const float iLd = Ld > 0.f ? 1.f / Ld : 0.f;
    const float iLs = Ls > 0.f ? 1.f / Ls : 0.f;
    const float iLt = Lt > 0.f ? 1.f / Lt : 0.f;
    for (int c = c0; c < D; c += 4) {
      float Od = 0.f, Os = 0.f, Ot = 0.f;
      for (int ch = 0; ch < a.nchunk; ch++) {
        const float* rec = base + (ch * kProfRows + r) * REC;
        const float wgt = (rec[0] == -INFINITY) ? 0.f : exp2f(rec[0] - M);
        Od += wgt * rec[4 + c];
        Os += wgt * rec[4 + D + c];
        Ot += wgt * rec[4 + 2 * D + c];
      }
      const double od = static_cast<double>(Od) * iLd;
      const double ds = static_cast<double>(Os) * iLs - od;
      const double dt = static_cast<double>(Ot) * iLt - od;
      es += ds * ds;
      et += dt * dt;
    }
  }
  __shared__ double red[2][8];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    es += __shfl_xor_sync(0xffffffffu, es, o);
    et += __shfl_xor_sync(0xffffffffu, et, o);
  }
  if ((tid & 31) == 0) {
    red[0][tid >> 5] = es;
    red[1][tid >> 5] = et;
  }
  __syncthreads();
  if (tid == 0) {
    double s = 0.0, t = 0.0;
    for (int w = 0; w < 8; w++) {
      s += red[0][w];
      t += red[1][w];
    }
    const double denom = static_cast<double>(a.n) * D;
    const double ms = s / denom, mt = t / denom;
    if (a.mse_out) {
      a.mse_out[2 * bh] = static_cast<float>(ms);
      a.mse_out[2 * bh + 1] = static_cast<float>(mt);
    }
    a.kind_out[bh] = (ms <= mt) ? SVG_HEAD_SPATIAL : SVG_HEAD_TEMPORAL;
  }
}

}  // namespace svg
