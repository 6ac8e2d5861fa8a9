// attention.cuh — block-sparse attention on the 5th-generation tensor cores.
//
// The pages ("Sparse VideoGen" WeChat article, "其他优化方法" and
// "硬件高效的 Layout Transformation"; ICML 2025 report, "Layout Transformation +
// Kernel 加速") describe a custom sparse attention kernel that, after the
// layout transform, reaches close to the 1/density speedup.  This is a
// B200-native design of that kernel:
//
//   * one CTA per (b, h, query tile of 128 rows); 6 warps:
//       warp 0  TMA producer: Q once, then K and V tiles of the listed key
//               blocks into an NS-stage shared-memory ring (128-byte swizzle);
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
  static constexpr int KV_BYTES = BN * D * 2;    // one K (or V) stage
  static constexpr int NS = (D == 128) ? 2 : 4;  // pipeline stages
  static constexpr int DATA_BYTES = Q_BYTES + 2 * NS * KV_BYTES;
  static constexpr int SMEM_BYTES = DATA_BYTES + 256 + 1024;  // barriers + alignment slack
  static constexpr int THREADS = 192;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t TM_S0 = 0, TM_S1 = 128, TM_O = 256;
};

struct AttnArgs {
  Geometry g;
  float scale_log2;              // softmax scale * log2(e)
  const uint8_t* kind;           // [BH]
  const int32_t* row_ptr;        // [BH*nqb + 1]
  const int32_t* col;            // [nnz]
  const uint8_t* full;           // [nnz]
  uint16_t* out;                 // [BH, L, D] bf16, head's layout
  float* lse;                    // [BH, L] or null
};

// 2^x with the MUFU.EX2 unit (PTX ex2.approx.ftz.f32); 2^-inf = 0.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
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
  constexpr int NS = C::NS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = smem + C::Q_BYTES;
  uint8_t* sV = sK + NS * C::KV_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::DATA_BYTES);
  // barrier slots
  const uint32_t b_q = smem_addr(&bars[0]);
  auto b_full = [&](int s) { return smem_addr(&bars[1 + s]); };
  auto b_empty = [&](int s) { return smem_addr(&bars[1 + NS + s]); };
  auto b_s = [&](int b) { return smem_addr(&bars[1 + 2 * NS + b]); };
  auto b_p = [&](int b) { return smem_addr(&bars[3 + 2 * NS + b]); };
  const uint32_t b_o = smem_addr(&bars[5 + 2 * NS]);
  const uint32_t b_drain = smem_addr(&bars[6 + 2 * NS]);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(&bars[16]);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(&bars[17]);

  const Geometry& g = a.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x % g.BH;
  const int qb = g.nqb - 1 - static_cast<int>(blockIdx.x / g.BH);   // text-heavy tiles first
  const int q_row0 = qb * g.bq;

  if (threadIdx.x == 0) {
    mbar_init(b_q, 1);
    for (int s = 0; s < NS; s++) {
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
    if (lane == 0) {
      tma_prefetch_desc(&tmq);
      tma_prefetch_desc(&tmk);
      tma_prefetch_desc(&tmv);
      mbar_expect_tx(b_q, C::Q_BYTES);
#pragma unroll
      for (int p = 0; p < C::PANELS; p++) tma_load_3d(smem_addr(sQ + p * C::PANEL_Q), &tmq, p * 64, q_row0, bh, b_q);
      int issued[NS];
#pragma unroll
      for (int s = 0; s < NS; s++) issued[s] = 0;
      for (int j = 0; j < nT; j++) {
        const int st = j % NS;
        if (j >= NS && !mbar_wait(b_empty(st), ((j / NS) - 1) & 1, abort_flag)) break;
        const int e0 = rp0 + 2 * j;
        const int nb = min(2, rp1 - e0);
        mbar_expect_tx(b_full(st), nb * 64 * D * 2 * 2);
        for (int h = 0; h < nb; h++) {
          const int kb = a.col[e0 + h];
#pragma unroll
          for (int p = 0; p < C::PANELS; p++) {
            const uint32_t off = st * C::KV_BYTES + p * C::PANEL_KV + h * 64 * 128;
            tma_load_3d(smem_addr(sK + off), &tmk, p * 64, kb * 64, bh, b_full(st));
            tma_load_3d(smem_addr(sV + off), &tmv, p * 64, kb * 64, bh, b_full(st));
          }
        }
        issued[st]++;
      }
      if (*abort_flag) {
        // let every issued copy land before the CTA exits
        mbar_wait_drain(b_q, 0);
        for (int s = 0; s < NS; s++)
          if (issued[s] > 0) mbar_wait_drain(b_full(s), (issued[s] - 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS128 = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t idS64 = idesc_bf16_f32(128, 64, 0, 0);
      constexpr uint32_t idO = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t q_base = smem_addr(sQ), k_base = smem_addr(sK), v_base = smem_addr(sV);
      bool ok = mbar_wait(b_q, 0, abort_flag);
      bool issued_any = false;
      for (int j = 0; ok && j <= nT; j++) {
        if (j < nT) {
          const int st = j % NS;
          if (!mbar_wait(b_full(st), (j / NS) & 1, abort_flag)) break;
          tc_fence_after();
          const int nb = min(2, rp1 - (rp0 + 2 * j));
          const uint32_t dS = tmem + ((j & 1) ? C::TM_S1 : C::TM_S0);
#pragma unroll
          for (int kk = 0; kk < D / 16; kk++) {
            const uint32_t koff = (kk >> 2) * C::PANEL_KV + (kk & 3) * 32;
            const uint32_t qoff = (kk >> 2) * C::PANEL_Q + (kk & 3) * 32;
            const uint64_t da = sdesc_sw128(q_base + qoff, 16, 1024);
            const uint64_t db = sdesc_sw128(k_base + st * C::KV_BYTES + koff, 16, 1024);
            umma_ss(dS, da, db, nb == 2 ? idS128 : idS64, kk > 0);
          }
          umma_commit(b_s(j & 1));
          issued_any = true;
        }
        if (j >= 1) {
          const int i = j - 1;
          const int st = i % NS;
          if (!mbar_wait(b_p(i & 1), (i >> 1) & 1, abort_flag)) break;
          tc_fence_after();
          const int nb = min(2, rp1 - (rp0 + 2 * i));
          const uint32_t aP = tmem + ((i & 1) ? C::TM_S1 : C::TM_S0);
          for (int kk = 0; kk < nb * 4; kk++) {
            const uint64_t db = sdesc_sw128(v_base + st * C::KV_BYTES + kk * 2048, C::PANEL_KV, 1024);
            umma_ts(tmem + C::TM_O, aP + kk * 8, db, idO, (i > 0 || kk > 0) ? 1u : 0u);
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
    for (int j = 0; j < nT; j++) {
      const int b = j & 1;
      const int e0 = rp0 + 2 * j;
      const int nb = min(2, rp1 - e0);
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
      float mx = -INFINITY;
#pragma unroll
      for (int h = 0; h < 2; h++) {
        if (h < nb) {
          const int kb = a.col[e0 + h];
          const int k0 = kb * 64;
          const bool need = (a.full[e0 + h] == 0) || (k0 + 64 > g.L);
          if (need) {
#pragma unroll
            for (int c = 0; c < 64; c++) {
              const int kk = k0 + c;
              const bool keep = (static_cast<unsigned>(kk - lo) < static_cast<unsigned>(hi - lo)) ||
                                (kk >= g.Lv && kk < g.L);
              if (!keep) sr[h * 64 + c] = __float_as_uint(-INFINITY);
            }
          }
        } else {
#pragma unroll
          for (int c = 0; c < 64; c++) sr[h * 64 + c] = __float_as_uint(-INFINITY);
        }
      }
#pragma unroll
      for (int c = 0; c < 128; c++) mx = fmaxf(mx, __uint_as_float(sr[c]));
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
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < 64; c++) {
        const float p0 = fast_exp2(fmaf(__uint_as_float(sr[2 * c]), sl2, -msub));
        const float p1 = fast_exp2(fmaf(__uint_as_float(sr[2 * c + 1]), sl2, -msub));
        const uint32_t pk = pack_bf16x2(p0, p1);
        rs += bf16_lo(pk) + bf16_hi(pk);
        sr[c] = pk;
      }
      l += rs;
      tmem_st32(tS, sr);
      tmem_st32(tS + 32, sr + 32);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(b_p(b));
    }
    // ---------------------------------------------------------- epilogue
    const bool row_ok = r < g.bq && row < g.L;
    if (ok && nT > 0 && __all_sync(0xffffffffu, mbar_wait(b_o, (nT - 1) & 1, abort_flag))) {
      tc_fence_after();
      const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
      uint16_t* orow = a.out + (static_cast<int64_t>(bh) * g.L + row) * D;
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
      if (row_ok && a.lse) {
        a.lse[static_cast<int64_t>(bh) * g.L + row] =
            (l > 0.f) ? (m_use * 0.69314718055994531f + logf(l)) : -INFINITY;
      }
    } else if (ok && nT == 0 && row_ok) {
      uint4* dst = reinterpret_cast<uint4*>(a.out + (static_cast<int64_t>(bh) * g.L + row) * D);
      for (int v = 0; v < D / 8; v++) dst[v] = make_uint4(0, 0, 0, 0);
      if (a.lse) a.lse[static_cast<int64_t>(bh) * g.L + row] = -INFINITY;
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
