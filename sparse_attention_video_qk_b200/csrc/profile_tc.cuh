// profile_tc.cuh — online profiling on the 5th-generation tensor cores
// ("Sparse VideoGen" WeChat article, "Online Profiling Strategy"; ICML 2025
// report, "动态自适应的稀疏策略" steps 1-3).
//
// For each head, the n <= 64 sampled query rows are attended three ways --
// densely, with the spatial mask and with the temporal mask -- in one pass
// over the keys.  The three softmaxes of a row share its running maximum
// (softmax is shift invariant).  The 64 sampled rows are stacked twice into
// one M = 128 operand, so:
//   * S = Q K^T (M=128, N=128 keys, K=d) gives every sampled row twice;
//   * lanes 0-63 form P_dense and the spatial-masked P_s, lanes 64-127 form
//     P_dense and the temporal-masked P_t; P_s / P_t occupy one 128-row A
//     operand, so O_st = [P_s; P_t] V is one MMA, and O_d = [P_d; P_d] V the other.
// TMEM: S double buffered (2 x 128 columns; after the softmax each 32-column
// chunk holds that chunk's P_st and P_d as packed bf16), O_d (d columns),
// O_st (d columns).
// The keys of a head are split into chunks (split-KV, grid = chunks x heads);
// each CTA writes per-lane partial records (max, row sums, O_d, O_st rows),
// and two small kernels merge the chunks in a fixed order, form
//   MSE_m = mean over rows and columns of (O_m - O_dense)^2
// and choose SPATIAL iff MSE_s <= MSE_t.
// Warp roles as in the attention kernel: warp 0 TMA producer (K/V slot ring),
// warp 1 TMEM allocator + MMA issuer, warps 2-5 softmax (thread = TMEM lane).
#pragma once

#include "attention.cuh"
#include "norm_rope.cuh"
#include "svg_common.cuh"

namespace svg {

constexpr int kProfRows = 64;      // sampled rows per head (padded)
constexpr int kProfKeys = 128;     // keys per tile

// Per-lane partial record: m, l_dense, l_masked, O_dense[d], O_masked[d]
// (stored field-major per chunk: [chunk][field][lane]).
__host__ __device__ constexpr int prof_rec_floats(int D) { return 3 + 2 * D; }

// Key chunks per head: as many as fit in 2 full waves of 148 SMs (one CTA per
// SM), so no partial third wave, and at least two tiles each.
__host__ __device__ inline int prof_chunks(int BH, int L) {
  const int ntiles = (L + kProfKeys - 1) / kProfKeys;
  int c = (2 * 148) / BH;
  const int cap = (ntiles + 1) / 2;
  if (c > cap) c = cap;
  if (c < 1) c = 1;
  return c;
}

// Workspace bytes: partial records + per-(head, row) squared-error sums.
__host__ __device__ inline size_t prof_workspace_bytes(int BH, int L, int D, int nchunk) {
  (void)L;
  return static_cast<size_t>(BH) * nchunk * 128 * prof_rec_floats(D) * sizeof(float) +
         static_cast<size_t>(BH) * kProfRows * 2 * sizeof(double);
}

struct ProfArgs {
  Geometry g;
  float scale_log2;
  const uint16_t* q;   // normalised Q, or raw Q when gamma_q is set
  const float* gamma_q;  // non-null: the gathered rows get QK-Norm + RoPE here (norm_rope.cuh)
  RopeArgs rope;
  const int32_t* sample;
  int n;
  int nchunk;
  int tiles_per_chunk;
  float* ws;           // [BH][nchunk][128][rec]
  double* err;         // [BH][64][2] squared-error sums per sampled row
  float* mse_out;      // [BH][2] or null
  uint8_t* kind_out;   // [BH]
};

// Bits [a, b) of a 128-column row that fall in the 32-column word starting at `base`.
__device__ __forceinline__ uint32_t range_mask(int a, int b, int base) {
  const int lo = max(a - base, 0), hi = min(b - base, 32);
  if (hi <= lo) return 0u;
  const uint32_t upto_hi = (hi >= 32) ? 0xFFFFFFFFu : ((1u << hi) - 1u);
  const uint32_t upto_lo = (1u << lo) - 1u;
  return upto_hi & ~upto_lo;
}

template <int D>
struct ProfCfg {
  static constexpr int PANELS = D / 64;
  static constexpr int PANEL = 128 * 128;        // bytes of one 128-row panel (Q or a K/V tile)
  static constexpr int Q_BYTES = 128 * D * 2;
  static constexpr int SLOT_BYTES = kProfKeys * D * 2;
  static constexpr int NSLOT = (D == 128) ? 6 : 12;
  static constexpr int DATA_BYTES = Q_BYTES + NSLOT * SLOT_BYTES;
  static constexpr int BAR_BYTES = 512;
  static constexpr int SMEM_BYTES = DATA_BYTES + BAR_BYTES + 1024;
  static constexpr int THREADS = 192;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t TM_S0 = 0, TM_S1 = 128, TM_OD = 256, TM_OX = 256 + D;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

template <int D>
__global__ void __launch_bounds__(ProfCfg<D>::THREADS, 1)
    profile_tc_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                      const ProfArgs a) {
  using C = ProfCfg<D>;
  constexpr int NSLOT = C::NSLOT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + C::Q_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::DATA_BYTES);
  auto b_full = [&](int s) { return smem_addr(&bars[s]); };
  auto b_empty = [&](int s) { return smem_addr(&bars[NSLOT + s]); };
  auto b_s = [&](int b) { return smem_addr(&bars[2 * NSLOT + b]); };
  auto b_p = [&](int b) { return smem_addr(&bars[2 * NSLOT + 2 + b]); };
  const uint32_t b_o = smem_addr(&bars[2 * NSLOT + 4]);
  const uint32_t b_drain = smem_addr(&bars[2 * NSLOT + 5]);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(&bars[2 * NSLOT + 6]);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(&bars[2 * NSLOT + 7]);

  const Geometry& g = a.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y, chunk = blockIdx.x;
  const int ntiles_all = (g.L + kProfKeys - 1) / kProfKeys;
  const int t_begin = chunk * a.tiles_per_chunk;
  const int t_end = min(ntiles_all, t_begin + a.tiles_per_chunk);
  const int nT = max(0, t_end - t_begin);
  const int key_end = min(g.L, t_end * kProfKeys);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSLOT; s++) {
      mbar_init(b_full(s), 1);
      mbar_init(b_empty(s), 1);
    }
    mbar_init(b_s(0), 1);
    mbar_init(b_s(1), 1);
    mbar_init(b_p(0), 128);
    mbar_init(b_p(1), 128);
    mbar_init(b_o, 1);
    mbar_init(b_drain, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) tmem_alloc(smem_addr(tmem_slot), C::TMEM_COLS);

  // Gather the sampled Q rows into both halves of the 128-row A operand, in
  // the 128-byte-swizzled K-major layout TMA would produce (16-byte chunk c of
  // row r stored at chunk c ^ (r % 8) of that row's 128-byte panel line).
  // Consecutive lanes take consecutive chunks of one row, and every warp is
  // either fully inside the loop or out of it (THREADS and 128*D/8 are
  // multiples of 32), so the norm routine's butterfly sees whole rows.
  {
    static_assert(C::THREADS % 32 == 0 && (128 * (D / 8)) % 32 == 0, "whole warps in the gather");
    const int64_t hoff = static_cast<int64_t>(bh) * g.L * D;
    const bool norm = a.gamma_q != nullptr;
    uint64_t gam[4] = {0ull, 0ull, 0ull, 0ull};
    RopeLane rl{};
    if (norm) {
      load_gain(a.gamma_q, threadIdx.x % (D / 8), gam);
      rl = rope_lane<D>(threadIdx.x % (D / 8), a.rope);
    }
    for (int i = threadIdx.x; i < 128 * (D / 8); i += C::THREADS) {
      const int r = i / (D / 8), c = i % (D / 8);
      const int sr = r & 63;
      uint4 val = make_uint4(0, 0, 0, 0);
      int tok = 0;
      if (sr < a.n) {
        tok = a.sample[sr];
        if (tok < 0 || tok >= g.L) {
          atomicOr(&g_error_word, kErrBadIndex);
          tok = 0;
        }
        val = __ldg(reinterpret_cast<const uint4*>(a.q + hoff + static_cast<int64_t>(tok) * D) + c);
      }
      if (norm) val = norm_rope_vec<D, false>(val, tok, g, gam, rl, a.rope, a.rope.table);
      const int panel = c >> 3, cc = c & 7;
      *reinterpret_cast<uint4*>(sQ + panel * C::PANEL + r * 128 + ((cc ^ (r & 7)) << 4)) = val;
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // generic writes -> tensor-core reads
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer: K0 V0 K1 V1 ...
    if (lane == 0) {
      tma_prefetch_desc(&tmk);
      tma_prefetch_desc(&tmv);
      int issued = 0;
      for (int i = 0; i < 2 * nT; i++) {
        const int st = i % NSLOT;
        if (i >= NSLOT && !mbar_wait(b_empty(st), ((i / NSLOT) - 1) & 1, abort_flag)) break;
        const int k0 = (t_begin + (i >> 1)) * kProfKeys;
        const CUtensorMap* map = (i & 1) ? &tmv : &tmk;
        mbar_expect_tx(b_full(st), C::SLOT_BYTES);
#pragma unroll
        for (int h = 0; h < 2; h++)
#pragma unroll
          for (int p = 0; p < C::PANELS; p++)
            tma_load_3d(smem_addr(sKV + st * C::SLOT_BYTES + p * C::PANEL + h * 64 * 128), map, p * 64,
                        k0 + h * 64, bh, b_full(st));
        issued = i + 1;
      }
      if (*abort_flag) {
        for (int i = max(0, issued - NSLOT); i < issued; i++) mbar_wait_drain(b_full(i % NSLOT), (i / NSLOT) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t idO = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t q_base = smem_addr(sQ), kv_base = smem_addr(sKV);
      bool issued_any = false;
      for (int j = 0; j <= nT; j++) {
        if (j < nT) {
          const int i = 2 * j, st = i % NSLOT;
          if (!mbar_wait(b_full(st), (i / NSLOT) & 1, abort_flag)) break;
          tc_fence_after();
          const uint32_t dS = tmem + ((j & 1) ? C::TM_S1 : C::TM_S0);
#pragma unroll
          for (int kk = 0; kk < D / 16; kk++) {
            const uint32_t off = (kk >> 2) * C::PANEL + (kk & 3) * 32;
            umma_ss(dS, sdesc_sw128(q_base + off, 16, 1024), sdesc_sw128(kv_base + st * C::SLOT_BYTES + off, 16, 1024),
                    idS, kk > 0);
          }
          umma_commit(b_s(j & 1));
          umma_commit(b_empty(st));
          issued_any = true;
        }
        if (j >= 1) {
          const int t = j - 1;
          const int i = 2 * t + 1, st = i % NSLOT;
          if (!mbar_wait(b_p(t & 1), (t >> 1) & 1, abort_flag)) break;
          if (!mbar_wait(b_full(st), (i / NSLOT) & 1, abort_flag)) break;
          tc_fence_after();
          const uint32_t aP = tmem + ((t & 1) ? C::TM_S1 : C::TM_S0);
#pragma unroll
          for (int kk = 0; kk < 8; kk++) {
            // keys 16kk..16kk+15: P_x at column 32*(kk/2) + 8*(kk%2), P_d 16 columns further
            const uint32_t pcol = 32 * (kk >> 1) + 8 * (kk & 1);
            const uint64_t db = sdesc_sw128(kv_base + st * C::SLOT_BYTES + kk * 2048, C::PANEL, 1024);
            umma_ts(tmem + C::TM_OX, aP + pcol, db, idO, (t > 0 || kk > 0) ? 1u : 0u);        // [P_s; P_t] V
            umma_ts(tmem + C::TM_OD, aP + pcol + 16, db, idO, (t > 0 || kk > 0) ? 1u : 0u);   // [P_d; P_d] V
          }
          umma_commit(b_empty(st));
          umma_commit(b_o);
        }
      }
      if (*abort_flag && issued_any) {
        umma_commit(b_drain);
        mbar_wait_drain(b_drain, 0);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;                 // TMEM lane
    const bool temporal = r >= 64;                // lanes 64-127 carry the temporal mask
    const int srow = r & 63;
    int tok = (srow < a.n) ? a.sample[srow] : 0;
    if (tok < 0 || tok >= g.L) tok = 0;
    const bool textq = tok >= g.Lv;
    const int fq = tok / g.S, sq = tok - (tok / g.S) * g.S;
    const uint32_t tl = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const float sl2 = a.scale_log2;
    const uint64_t sl2x2 = f32x2(sl2, sl2);
    float m_use = -INFINITY;
    float l_d = 0.f, l_x = 0.f;
    bool ok = true;
    for (int j = 0; j < nT; j++) {
      const int b = j & 1;
      const int k0 = (t_begin + j) * kProfKeys;
      // This lane's mask over the tile's 128 columns as 4 words: valid keys
      // [0, ncol); text keys [ct, ncol); spatial lanes: video keys of frames
      // fq-w..fq+w (one interval); temporal lanes: video keys whose spatial
      // index lies in [sq-r, sq+r] (one interval per pass of the spatial
      // index through [0, S); S >= 64 gives at most three in 128 keys).
      const int ncol = min(kProfKeys, key_end - k0);
      const int ct = max(0, min(ncol, g.Lv - k0));      // first text column
      uint32_t mw[4];
      {
        const int nv = textq ? 0 : ct;                  // columns whose key is video
        uint32_t w0 = range_mask(ct, ncol, 0), w1 = range_mask(ct, ncol, 32);
        uint32_t w2 = range_mask(ct, ncol, 64), w3 = range_mask(ct, ncol, 96);
        if (textq) {
          w0 = range_mask(0, ncol, 0); w1 = range_mask(0, ncol, 32);
          w2 = range_mask(0, ncol, 64); w3 = range_mask(0, ncol, 96);
        } else if (!temporal) {
          const int lo = max(fq - g.w, 0) * g.S - k0, hi = min(fq + g.w + 1, g.F) * g.S - k0;
          const int a0 = max(lo, 0), a1 = min(hi, nv);
          w0 |= range_mask(a0, a1, 0); w1 |= range_mask(a0, a1, 32);
          w2 |= range_mask(a0, a1, 64); w3 |= range_mask(a0, a1, 96);
        } else if (g.S >= 64) {
          // column c has spatial index s0 + c - m*S in pass m = 0, 1, 2
          const int s0 = k0 % g.S;
#pragma unroll
          for (int m = 0; m < 3; m++) {
            const int base = m * g.S - s0;                 // column of spatial index 0 in pass m
            const int a0 = max(max(base + sq - g.r, base), 0);
            const int a1 = min(min(base + sq + g.r + 1, base + g.S), nv);
            w0 |= range_mask(a0, a1, 0); w1 |= range_mask(a0, a1, 32);
            w2 |= range_mask(a0, a1, 64); w3 |= range_mask(a0, a1, 96);
          }
        } else {
          // small spatial grids: one column at a time
          int s = k0 % g.S;
          for (int c = 0; c < nv; c++) {
            if (static_cast<unsigned>(s - sq + g.r) <= static_cast<unsigned>(2 * g.r)) {
              if (c < 32) w0 |= 1u << c;
              else if (c < 64) w1 |= 1u << (c - 32);
              else if (c < 96) w2 |= 1u << (c - 64);
              else w3 |= 1u << (c - 96);
            }
            s = (s + 1 == g.S) ? 0 : s + 1;
          }
        }
        mw[0] = w0; mw[1] = w1; mw[2] = w2; mw[3] = w3;
      }
      if (!__all_sync(0xffffffffu, mbar_wait(b_s(b), (j >> 1) & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tS = tl + (b ? C::TM_S1 : C::TM_S0);
      // pass 1: row maximum over the valid columns
      const uint32_t vmask[4] = {range_mask(0, ncol, 0), range_mask(0, ncol, 32), range_mask(0, ncol, 64),
                                 range_mask(0, ncol, 96)};
      float m8[8];
#pragma unroll
      for (int i = 0; i < 8; i++) m8[i] = -INFINITY;
      {
        uint32_t sr[64];
#pragma unroll
        for (int h = 0; h < 2; h++) {
          tmem_ld32(tS + h * 64, sr);
          tmem_ld32(tS + h * 64 + 32, sr + 32);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 64; c += 16) {
#pragma unroll
            for (int i = 0; i < 8; i++) {
              const int c0 = h * 64 + c + i, c1 = c0 + 8;
              const float x0 = ((vmask[c0 >> 5] >> (c0 & 31)) & 1u) ? __uint_as_float(sr[c + i]) : -INFINITY;
              const float x1 = ((vmask[c1 >> 5] >> (c1 & 31)) & 1u) ? __uint_as_float(sr[c + 8 + i]) : -INFINITY;
              m8[i] = fmax3(m8[i], x0, x1);
            }
          }
        }
      }
      const float mx = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
      const float mxs = mx * sl2;
      const bool need_rescale = mxs > m_use + 8.0f;
      if (__any_sync(0xffffffffu, need_rescale)) {
        const float m_new = need_rescale ? mxs : m_use;
        const float alpha = need_rescale ? ((m_use == -INFINITY) ? 0.f : fast_exp2(m_use - m_new)) : 1.f;
        l_d *= alpha;
        l_x *= alpha;
        if (j > 0) {
          if (!__all_sync(0xffffffffu, mbar_wait(b_o, (j - 1) & 1, abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
          uint32_t o[32];
#pragma unroll
          for (int c = 0; c < 2 * D / 32; c++) {      // O_d and O_st are adjacent columns
            tmem_ld32(tl + C::TM_OD + c * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; i++) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tl + C::TM_OD + c * 32, o);
          }
          tmem_wait_st();
        }
        m_use = m_new;
      }
      const float msub = (m_use == -INFINITY) ? 0.f : m_use;
      const uint64_t nmsub2 = f32x2(-msub, -msub);
      // pass 2, 32 columns at a time: P_d on valid keys, P_x = P_d on kept keys;
      // keys 32q..32q+31 become P_x in TMEM columns [32q, 32q+16) and P_d in
      // [32q+16, 32q+32) (packed bf16, 2 keys per column)
      uint64_t accd[2] = {0ull, 0ull}, accx[2] = {0ull, 0ull};
#pragma unroll 1
      for (int q = 0; q < 4; q++) {
        uint32_t sr[32], pd[16], px[16];
        tmem_ld32(tS + q * 32, sr);
        const uint32_t vw = q == 0 ? vmask[0] : q == 1 ? vmask[1] : q == 2 ? vmask[2] : vmask[3];
        const uint32_t kw = q == 0 ? mw[0] : q == 1 ? mw[1] : q == 2 ? mw[2] : mw[3];
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 16; c++) {
          const uint64_t xa = ffma2(f32x2(__uint_as_float(sr[2 * c]), __uint_as_float(sr[2 * c + 1])), sl2x2, nmsub2);
          float x0, x1;
          unpack2(xa, x0, x1);
          float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
          p0 = ((vw >> (2 * c)) & 1u) ? p0 : 0.f;
          p1 = ((vw >> (2 * c + 1)) & 1u) ? p1 : 0.f;
          // the row sums add the bf16-rounded P that the P.V products use, so each
          // masked softmax stays a consistent weighted average
          const uint32_t pk = pack_bf16x2(p0, p1);
          const float r0 = bf16_lo(pk), r1 = bf16_hi(pk);
          const float x0m = ((kw >> (2 * c)) & 1u) ? r0 : 0.f;
          const float x1m = ((kw >> (2 * c + 1)) & 1u) ? r1 : 0.f;
          accd[c & 1] = fadd2(accd[c & 1], f32x2(r0, r1));
          accx[c & 1] = fadd2(accx[c & 1], f32x2(x0m, x1m));
          pd[c] = pk;
          px[c] = pack_bf16x2(x0m, x1m);
        }
        // both go into this chunk's own (already read) S columns [32q, 32q+32)
        tmem_st16(tS + q * 32, px);
        tmem_st16(tS + q * 32 + 16, pd);
      }
      float a0, a1, a2, a3;
      unpack2(accd[0], a0, a1);
      unpack2(accd[1], a2, a3);
      l_d += (a0 + a1) + (a2 + a3);
      unpack2(accx[0], a0, a1);
      unpack2(accx[1], a2, a3);
      l_x += (a0 + a1) + (a2 + a3);
      tmem_wait_st();
      // A parity wait on the O barrier tells "phase k done" from "not done"
      // only when phase k-1 is known done.  The commit behind S_j covers every
      // earlier MMA, so once S_j is ready P.V of tiles <= j-2 are done and the
      // rescale wait above (phase j-1) is unambiguous.  The epilogue waits for
      // phase nT-1, so phase nT-2 is confirmed here, on the last tile, before
      // P_{nT-1} lets P.V_{nT-1} start.
      if (j >= 1 && j == nT - 1 && !__all_sync(0xffffffffu, mbar_wait(b_o, (j - 1) & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_before();
      mbar_arrive(b_p(b));
    }
    // ---------------------------------------------------------- partial record of this lane
    // field-major: field f of lane r at rec[f * 128 + r], so a warp's stores coalesce
    constexpr int REC = prof_rec_floats(D);
    float* rec = a.ws + (static_cast<int64_t>(bh) * a.nchunk + chunk) * 128 * REC + r;
    if (ok && nT > 0 && __all_sync(0xffffffffu, mbar_wait(b_o, (nT - 1) & 1, abort_flag))) {
      tc_fence_after();
      rec[0 * 128] = m_use;
      rec[1 * 128] = l_d;
      rec[2 * 128] = l_x;
#pragma unroll 1
      for (int c = 0; c < 2 * D / 32; c++) {
        uint32_t o[32];
        tmem_ld32(tl + C::TM_OD + c * 32, o);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; i++) rec[(3 + c * 32 + i) * 128] = __uint_as_float(o[i]);
      }
    } else if (ok && nT == 0) {
      rec[0] = -INFINITY;
      rec[128] = 0.f;
      rec[256] = 0.f;
      for (int i = 0; i < 2 * D; i++) rec[(3 + i) * 128] = 0.f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// Merge the chunks of one (head, sampled row): one block of d threads, one
// column each; writes the row's two squared-error sums.
template <int D>
__global__ void __launch_bounds__(D) profile_merge_kernel(const ProfArgs a) {
  constexpr int REC = prof_rec_floats(D);
  const int bh = blockIdx.y, i = blockIdx.x, c = threadIdx.x;
  const float* base = a.ws + static_cast<int64_t>(bh) * a.nchunk * 128 * REC;
  // records are field-major per chunk: field f of lane r at [chunk][f][r]
  // lane i: (m, l_d, l_s, O_d, O_s); lane 64+i: (m, l_d, l_t, O_d, O_t)
  float Ms = -INFINITY, Mt = -INFINITY;
  for (int ch = 0; ch < a.nchunk; ch++) {
    Ms = fmaxf(Ms, base[ch * 128 * REC + i]);
    Mt = fmaxf(Mt, base[ch * 128 * REC + 64 + i]);
  }
  float Ld = 0.f, Ls = 0.f, Lt = 0.f, Od = 0.f, Os = 0.f, Ot = 0.f;
  for (int ch = 0; ch < a.nchunk; ch++) {
    const float* rc = base + ch * 128 * REC;
    const float ms = rc[i], mt = rc[64 + i];
    const float ws = (ms == -INFINITY) ? 0.f : exp2f(ms - Ms);
    const float wt = (mt == -INFINITY) ? 0.f : exp2f(mt - Mt);
    Ld += ws * rc[1 * 128 + i];
    Ls += ws * rc[2 * 128 + i];
    Lt += wt * rc[2 * 128 + 64 + i];
    Od += ws * rc[(3 + c) * 128 + i];
    Os += ws * rc[(3 + D + c) * 128 + i];
    Ot += wt * rc[(3 + D + c) * 128 + 64 + i];
  }
  const double od = (Ld > 0.f) ? static_cast<double>(Od) / Ld : 0.0;
  const double ds = ((Ls > 0.f) ? static_cast<double>(Os) / Ls : 0.0) - od;
  const double dt = ((Lt > 0.f) ? static_cast<double>(Ot) / Lt : 0.0) - od;
  double es = ds * ds, et = dt * dt;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    es += __shfl_xor_sync(0xffffffffu, es, o);
    et += __shfl_xor_sync(0xffffffffu, et, o);
  }
  __shared__ double red[2][D / 32];
  if ((c & 31) == 0) {
    red[0][c >> 5] = es;
    red[1][c >> 5] = et;
  }
  __syncthreads();
  if (c == 0) {
    double s = 0.0, t = 0.0;
    for (int w = 0; w < D / 32; w++) {
      s += red[0][w];
      t += red[1][w];
    }
    a.err[(static_cast<int64_t>(bh) * kProfRows + i) * 2 + 0] = s;
    a.err[(static_cast<int64_t>(bh) * kProfRows + i) * 2 + 1] = t;
  }
}

// Per head: sum the rows' errors in order, MSE, choice.
__global__ void profile_choose_kernel(const ProfArgs a, int D) {
  const int bh = blockIdx.x * blockDim.x + threadIdx.x;
  if (bh >= a.g.BH) return;
  double s = 0.0, t = 0.0;
  for (int i = 0; i < a.n; i++) {
    s += a.err[(static_cast<int64_t>(bh) * kProfRows + i) * 2 + 0];
    t += a.err[(static_cast<int64_t>(bh) * kProfRows + i) * 2 + 1];
  }
  const double denom = static_cast<double>(a.n) * D;
  const double ms = s / denom, mt = t / denom;
  if (a.mse_out) {
    a.mse_out[2 * bh] = static_cast<float>(ms);
    a.mse_out[2 * bh + 1] = static_cast<float>(mt);
  }
  a.kind_out[bh] = (ms <= mt) ? SVG_HEAD_SPATIAL : SVG_HEAD_TEMPORAL;
}

}  // namespace svg
