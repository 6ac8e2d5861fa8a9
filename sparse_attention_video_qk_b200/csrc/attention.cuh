// attention.cuh — block-sparse attention on the 5th-generation tensor cores.
//
// The pages ("Sparse VideoGen" WeChat article, "其他优化方法" and
// "硬件高效的 Layout Transformation"; ICML 2025 report, "Layout Transformation +
// Kernel 加速") describe a custom sparse attention kernel that, after the
// layout transform, reaches close to the 1/density speedup.  This is a
// B200-native design of that kernel:
//
//   * one CTA per (b, h, query tile of 128 rows), text-row tiles first, then
//     head by head for L2 reuse of each head's K and V; 6 warps:
//       warp 0  TMA producer: Q once, then the K and V tiles of the listed
//               key blocks into one ring of shared-memory slots (128-byte
//               swizzle), K released after Q.K^T and V after P.V;
//       warp 1  TMEM allocator and the single MMA-issuing thread;
//       warps 2-5  softmax: thread = query row = TMEM lane.
//   * two listed 64-key blocks (consecutive entries of the CSR list, not
//     necessarily adjacent in memory) form one N = 128 tile: TMA drops them
//     into the two halves of one stage, so S = Q K^T is a single
//     M=128 x N=128 x K=d tcgen05.mma chain into TMEM (N = 64 for an odd tail);
//   * S (fp32, 128 TMEM columns) is double buffered; the softmax writes
//     P = exp2(S * scale*log2e - m) as bf16 into the same columns, and
//     O += P V runs with A = P read from TMEM and B = V (MN-major) from SMEM;
//   * online softmax in fp32 with lazy rescaling: the running maximum moves
//     only when a row's tile maximum exceeds it by more than 8 (log2 units);
//     then l and the TMEM accumulator O are rescaled after the previous P.V
//     has completed;
//   * the token-level mask (the head's kept-key interval plus text keys) is
//     evaluated only in tiles whose `full` flag is 0 and in the ragged last
//     key block.
// Every mbarrier wait is bounded; on time-out the kernel records
// kErrTimeout, drains its outstanding copies and MMAs (bounded again), frees
// TMEM and returns.
#pragma once

#include "svg_common.cuh"

namespace svg {

template <int D>
struct AttnCfg {
  static constexpr int BM = 128;                 // query rows per CTA (MMA M)
  static constexpr int BN = 128;                 // keys per iteration (two 64-key blocks)
  static constexpr int PANELS = D / 64;          // 128-byte swizzle panels per row
  static constexpr int PANEL_Q = BM * 128;       // bytes of one Q panel
  static constexpr int PANEL_KV = BN * 128;      // bytes of one K / V panel
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int SLOT_BYTES = BN * D * 2;  // one K or one V tile
  // K and V tiles share one ring of slots, filled in the order K0 V0 K1 V1 ...
  static constexpr int NSLOT = (D == 128) ? 6 : 12;
  static constexpr int DATA_BYTES = Q_BYTES + NSLOT * SLOT_BYTES;
  static constexpr int BAR_BYTES = 512;
  static constexpr int SMEM_BYTES = DATA_BYTES + BAR_BYTES + 1024;  // + alignment slack
  static constexpr int THREADS = 192;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t TM_S0 = 0, TM_S1 = 128, TM_O = 256;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(1 + 2 * NSLOT + 6 + 2 <= BAR_BYTES / 8, "barrier area");
};

struct AttnArgs {
  Geometry g;
  float scale_log2;              // softmax scale * log2(e)
  const uint8_t* kind;           // [BH]
  const int32_t* row_ptr;        // [BH*nqb + 1]
  const int32_t* col;            // [nnz]
  const uint8_t* full;           // [nnz]
  uint16_t* out;                 // [BH, L, D] bf16, head's layout (or model order, see below)
  float* lse;                    // [BH, L] or null
  int model_order;               // 1: rows of temporal heads are stored back in frame-major order
  // Semantic-permutation mask (all null otherwise): rows and keys are sorted
  // by cluster; a video query of cluster i keeps the video keys of the key
  // clusters in sel[bh*Cq + i] and every text key; text queries keep all.
  const uint64_t* sel;           // [BH][Cq]
  const int32_t* qoff;           // [BH][Cq+1] first position of each query cluster
  const int32_t* koff;           // [BH][Ck+1]
  int Cq, Ck;
  const int32_t* out_perm;       // [BH][Lv] or null: output row of sorted video position p
};

// Row of `out` / `lse` that receives query row `row` (given in the head's
// layout): the row itself, or, with model_order, its frame-major position --
// the inverse layout transform (temporal heads: s*F+f -> f*S+s; text rows
// stay) -- or, with out_perm, the video row the cluster sort put there.
template <bool CLUSTER>
__device__ __forceinline__ int out_row(const AttnArgs& a, int kind, int bh, int row) {
  const Geometry& g = a.g;
  if (row >= g.Lv) return row;
  if constexpr (CLUSTER) {
    // a caller's permutation: an entry outside [0, Lv) is reported and its row not written
    const int p = __ldg(a.out_perm + static_cast<int64_t>(bh) * g.Lv + row);
    if (static_cast<unsigned>(p) >= static_cast<unsigned>(g.Lv)) {
      atomicOr(&g_error_word, kErrBadIndex);
      return -1;
    }
    return p;
  }
  if (!a.model_order || kind != SVG_HEAD_TEMPORAL) return row;
  const int s = row / g.F, f = row - s * g.F;
  return f * g.S + s;
}

// 2^x with the MUFU.EX2 unit (PTX ex2.approx.ftz.f32); 2^-inf = 0.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Packed fp32 pairs (Blackwell f32x2 ALU ops): one instruction for two lanes of work.
__device__ __forceinline__ uint64_t f32x2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void unpack2(uint64_t r, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ bool mbar_wait_drain(uint32_t bar, uint32_t parity) {
  long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitCycles) return false;
  }
  return true;
}

template <int D>
__global__ void __launch_bounds__(AttnCfg<D>::THREADS, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                const __grid_constant__ CUtensorMap tmv, const AttnArgs a) {
  using C = AttnCfg<D>;
  constexpr int NSLOT = C::NSLOT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + C::Q_BYTES;              // NSLOT slots of SLOT_BYTES
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::DATA_BYTES);
  // barrier slots
  const uint32_t b_q = smem_addr(&bars[0]);
  auto b_full = [&](int s) { return smem_addr(&bars[1 + s]); };
  auto b_empty = [&](int s) { return smem_addr(&bars[1 + NSLOT + s]); };
  auto b_s = [&](int b) { return smem_addr(&bars[1 + 2 * NSLOT + b]); };
  auto b_p = [&](int b) { return smem_addr(&bars[3 + 2 * NSLOT + b]); };
  const uint32_t b_o = smem_addr(&bars[5 + 2 * NSLOT]);
  const uint32_t b_drain = smem_addr(&bars[6 + 2 * NSLOT]);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(&bars[7 + 2 * NSLOT]);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(&bars[8 + 2 * NSLOT]);

  const Geometry& g = a.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Work order: first the query tiles that contain text rows (they attend to
  // every key: the longest lists), then the rest head by head, so the CTAs
  // resident at one time read the same head's keys and values out of L2.
  int bh, qb;
  {
    const int qb_text = (g.T > 0) ? g.Lv / g.bq : g.nqb;   // first tile holding a text row
    const int n_heavy = g.nqb - qb_text;
    const int x = blockIdx.x;
    if (x < g.BH * n_heavy) {
      bh = x / n_heavy;
      qb = qb_text + x % n_heavy;
    } else {
      const int y = x - g.BH * n_heavy;
      bh = y / qb_text;
      qb = y % qb_text;
    }
  }
  const int q_row0 = qb * g.bq;

  if (threadIdx.x == 0) {
    mbar_init(b_q, 1);
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int rp0 = a.row_ptr[bh * g.nqb + qb];
  const int rp1 = a.row_ptr[bh * g.nqb + qb + 1];
  const int nblk = rp1 - rp0;
  const int nT = (nblk + 1) >> 1;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Slot sequence i = 0, 1, 2, ...: K of tile i/2 for even i, V for odd i.
    if (lane == 0) {
      tma_prefetch_desc(&tmq);
      tma_prefetch_desc(&tmk);
      tma_prefetch_desc(&tmv);
      mbar_expect_tx(b_q, C::Q_BYTES);
#pragma unroll
      for (int p = 0; p < C::PANELS; p++) tma_load_3d(smem_addr(sQ + p * C::PANEL_Q), &tmq, p * 64, q_row0, bh, b_q);
      int issued = 0;
      for (int i = 0; i < 2 * nT; i++) {
        const int st = i % NSLOT;
        if (i >= NSLOT && !mbar_wait(b_empty(st), ((i / NSLOT) - 1) & 1, abort_flag)) break;
        const int e0 = rp0 + 2 * (i >> 1);
        const int nb = min(2, rp1 - e0);
        const CUtensorMap* map = (i & 1) ? &tmv : &tmk;
        mbar_expect_tx(b_full(st), nb * 64 * D * 2);
        for (int h = 0; h < nb; h++) {
          const int kb = a.col[e0 + h];
#pragma unroll
          for (int p = 0; p < C::PANELS; p++) {
            const uint32_t off = st * C::SLOT_BYTES + p * C::PANEL_KV + h * 64 * 128;
            tma_load_3d(smem_addr(sKV + off), map, p * 64, kb * 64, bh, b_full(st));
          }
        }
        issued = i + 1;
      }
      if (*abort_flag) {
        // let every issued copy land before the CTA exits
        mbar_wait_drain(b_q, 0);
        for (int i = max(0, issued - NSLOT); i < issued; i++)
          mbar_wait_drain(b_full(i % NSLOT), (i / NSLOT) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS128 = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t idS64 = idesc_bf16_f32(128, 64, 0, 0);
      constexpr uint32_t idO = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t q_base = smem_addr(sQ), kv_base = smem_addr(sKV);
      bool ok = mbar_wait(b_q, 0, abort_flag);
      bool issued_any = false;
      for (int j = 0; ok && j <= nT; j++) {
        if (j < nT) {
          // S_j = Q K_j^T; the K slot is released as soon as these MMAs finish
          const int i = 2 * j, st = i % NSLOT;
          if (!mbar_wait(b_full(st), (i / NSLOT) & 1, abort_flag)) break;
          tc_fence_after();
          const int nb = min(2, rp1 - (rp0 + 2 * j));
          const uint32_t dS = tmem + ((j & 1) ? C::TM_S1 : C::TM_S0);
#pragma unroll
          for (int kk = 0; kk < D / 16; kk++) {
            const uint32_t koff = (kk >> 2) * C::PANEL_KV + (kk & 3) * 32;
            const uint32_t qoff = (kk >> 2) * C::PANEL_Q + (kk & 3) * 32;
            const uint64_t da = sdesc_sw128(q_base + qoff, 16, 1024);
            const uint64_t db = sdesc_sw128(kv_base + st * C::SLOT_BYTES + koff, 16, 1024);
            umma_ss(dS, da, db, nb == 2 ? idS128 : idS64, kk > 0);
          }
          umma_commit(b_s(j & 1));
          umma_commit(b_empty(st));
          issued_any = true;
        }
        if (j >= 1) {
          // O += P_{j-1} V_{j-1}
          const int t = j - 1;
          const int i = 2 * t + 1, st = i % NSLOT;
          if (!mbar_wait(b_p(t & 1), (t >> 1) & 1, abort_flag)) break;
          if (!mbar_wait(b_full(st), (i / NSLOT) & 1, abort_flag)) break;
          tc_fence_after();
          const int nb = min(2, rp1 - (rp0 + 2 * t));
          const uint32_t aP = tmem + ((t & 1) ? C::TM_S1 : C::TM_S0);
          for (int kk = 0; kk < nb * 4; kk++) {
            const uint64_t db = sdesc_sw128(kv_base + st * C::SLOT_BYTES + kk * 2048, C::PANEL_KV, 1024);
            umma_ts(tmem + C::TM_O, aP + kk * 8, db, idO, (t > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(b_empty(st));
          umma_commit(b_o);
        }
      }
      if (*abort_flag && issued_any) {
        umma_commit(b_drain);          // arrives when every MMA issued above has finished
        mbar_wait_drain(b_drain, 0);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int q4 = warp & 3;                       // TMEM lane quarter of this warp
    const int r = q4 * 32 + lane;                  // row within the tile
    const int row = q_row0 + r;
    const int kind = a.kind[bh];
    int lo, hi;
    row_interval(g, kind, row, lo, hi);             // rows >= L keep everything (never stored)
    const uint32_t tl = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const float sl2 = a.scale_log2;
    float m_use = -INFINITY;   // running max, log2 units
    float l = 0.f;
    bool ok = true;
    uint32_t sr[128];
    // tile metadata (the listed k-blocks and their full flags), fetched one tile ahead
    int nxt_kb0 = 0, nxt_kb1 = -1, nxt_f0 = 1, nxt_f1 = 1;
    auto fetch_meta = [&](int j) {
      const int e0 = rp0 + 2 * j;
      nxt_kb0 = a.col[e0];
      nxt_f0 = a.full[e0];
      if (e0 + 1 < rp1) {
        nxt_kb1 = a.col[e0 + 1];
        nxt_f1 = a.full[e0 + 1];
      } else {
        nxt_kb1 = -1;
        nxt_f1 = 1;
      }
    };
    if (nT > 0) fetch_meta(0);
    const uint64_t sl2x2 = f32x2(sl2, sl2);
    for (int j = 0; j < nT; j++) {
      const int b = j & 1;
      const int kbs[2] = {nxt_kb0, nxt_kb1};
      const int fls[2] = {nxt_f0, nxt_f1};
      if (j + 1 < nT) fetch_meta(j + 1);
      // waits are made warp-uniform so that the warp-collective tcgen05 ops stay converged
      if (!__all_sync(0xffffffffu, mbar_wait(b_s(b), (j >> 1) & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tS = tl + (b ? C::TM_S1 : C::TM_S0);
#pragma unroll
      for (int c = 0; c < 4; c++) tmem_ld32(tS + c * 32, sr + c * 32);
      tmem_wait_ld();
      // token-level mask on partial tiles, the ragged last key block and an absent second block
#pragma unroll
      for (int h = 0; h < 2; h++) {
        if (kbs[h] < 0) {
#pragma unroll
          for (int c = 0; c < 64; c++) sr[h * 64 + c] = __float_as_uint(-INFINITY);
        } else {
          const int k0 = kbs[h] * 64;
          if (fls[h] == 0 || k0 + 64 > g.L) {
#pragma unroll
            for (int c = 0; c < 64; c++) {
              const int kk = k0 + c;
              const bool keep = (static_cast<unsigned>(kk - lo) < static_cast<unsigned>(hi - lo)) ||
                                (static_cast<unsigned>(kk - g.Lv) < static_cast<unsigned>(g.T));
              if (!keep) sr[h * 64 + c] = __float_as_uint(-INFINITY);
            }
          }
        }
      }
      // row maximum: 8 independent chains of 3-input max, then a small tree
      float m8[8];
#pragma unroll
      for (int i = 0; i < 8; i++) m8[i] = __uint_as_float(sr[i]);
#pragma unroll
      for (int c = 8; c < 128; c += 16) {
#pragma unroll
        for (int i = 0; i < 8; i++) m8[i] = fmax3(m8[i], __uint_as_float(sr[c + i]), __uint_as_float(sr[c + 8 + i]));
      }
      const float mx = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
      const float mxs = mx * sl2;
      const bool need_rescale = mxs > m_use + 8.0f;
      if (__any_sync(0xffffffffu, need_rescale)) {
        const float m_new = need_rescale ? mxs : m_use;
        const float alpha = need_rescale ? ((m_use == -INFINITY) ? 0.f : fast_exp2(m_use - m_new)) : 1.f;
        l *= alpha;
        if (j > 0) {
          // O holds P.V of tiles 0..j-1 once the (j-1)-th P.V has completed
          if (!__all_sync(0xffffffffu, mbar_wait(b_o, (j - 1) & 1, abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
          uint32_t o[32];
#pragma unroll
          for (int c = 0; c < D / 32; c++) {
            tmem_ld32(tl + C::TM_O + c * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; i++) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tl + C::TM_O + c * 32, o);
          }
          tmem_wait_st();
        }
        m_use = m_new;
      }
      const float msub = (m_use == -INFINITY) ? 0.f : m_use;
      const uint64_t nmsub2 = f32x2(-msub, -msub);
      // P = 2^(S*scale*log2e - m): the argument as packed fp32 pairs, 2^x on the
      // MUFU unit; row sum over 8 independent packed chains
      uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int c = 0; c < 64; c++) {
        const uint64_t xa = ffma2(f32x2(__uint_as_float(sr[2 * c]), __uint_as_float(sr[2 * c + 1])), sl2x2, nmsub2);
        float x0, x1;
        unpack2(xa, x0, x1);
        const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
        acc[c & 3] = fadd2(acc[c & 3], f32x2(p0, p1));
        sr[c] = pack_bf16x2(p0, p1);
      }
      float s0, s1, s2, s3, s4, s5, s6, s7;
      unpack2(acc[0], s0, s1);
      unpack2(acc[1], s2, s3);
      unpack2(acc[2], s4, s5);
      unpack2(acc[3], s6, s7);
      l += ((s0 + s1) + (s2 + s3)) + ((s4 + s5) + (s6 + s7));
      tmem_st32(tS, sr);
      tmem_st32(tS + 32, sr + 32);
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
    // ---------------------------------------------------------- epilogue
    const bool row_ok = r < g.bq && row < g.L;
    if (ok && nT > 0 && __all_sync(0xffffffffu, mbar_wait(b_o, (nT - 1) & 1, abort_flag))) {
      tc_fence_after();
      const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
      const int64_t orow_i = static_cast<int64_t>(bh) * g.L + out_row<false>(a, kind, bh, row);
      uint16_t* orow = a.out + orow_i * D;
#pragma unroll
      for (int c = 0; c < D / 32; c++) {
        uint32_t o[32];
        tmem_ld32(tl + C::TM_O + c * 32, o);
        tmem_wait_ld();
        if (row_ok) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int v = 0; v < 4; v++) {
            uint4 pkt;
            pkt.x = pack_bf16x2(__uint_as_float(o[8 * v + 0]) * inv_l, __uint_as_float(o[8 * v + 1]) * inv_l);
            pkt.y = pack_bf16x2(__uint_as_float(o[8 * v + 2]) * inv_l, __uint_as_float(o[8 * v + 3]) * inv_l);
            pkt.z = pack_bf16x2(__uint_as_float(o[8 * v + 4]) * inv_l, __uint_as_float(o[8 * v + 5]) * inv_l);
            pkt.w = pack_bf16x2(__uint_as_float(o[8 * v + 6]) * inv_l, __uint_as_float(o[8 * v + 7]) * inv_l);
            dst[v] = pkt;
          }
        }
      }
      if (row_ok && a.lse) a.lse[orow_i] = (l > 0.f) ? (m_use * 0.69314718055994531f + logf(l)) : -INFINITY;
    } else if (ok && nT == 0 && row_ok) {
      const int64_t orow_i = static_cast<int64_t>(bh) * g.L + out_row<false>(a, kind, bh, row);
      uint4* dst = reinterpret_cast<uint4*>(a.out + orow_i * D);
      for (int v = 0; v < D / 8; v++) dst[v] = make_uint4(0, 0, 0, 0);
      if (a.lse) a.lse[orow_i] = -INFINITY;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace svg
