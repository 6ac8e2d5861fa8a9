// attention2.cuh — block-sparse attention with two query tiles per CTA.
//
// Same computation as attn_kernel (see attention.cuh; the pages: "Sparse
// VideoGen" WeChat article, "其他优化方法" and "硬件高效的 Layout
// Transformation"; ICML 2025 report, "Layout Transformation + Kernel 加速"),
// organised so that each K/V tile feeds two 128-row query tiles:
//   * one CTA per (b, h, pair of 128-row query tiles 2p, 2p+1); it walks the
//     sorted union of the two tiles' CSR lists.  A block listed for only one
//     query tile is fully masked for the other (token-level mask), so the
//     result is exactly each tile's own list;
//   * 10 warps: warp 0 TMA producer (K/V slot ring, K0 V0 K1 V1 ...), warp 1
//     TMEM allocator + MMA issuer, warps 2-5 softmax of query tile 0,
//     warps 6-9 softmax of query tile 1 (thread = query row = TMEM lane);
//   * TMEM: S0, S1 (128 columns each; P written back into them as bf16),
//     O0, O1 (d columns each);
//   * MMA order per key tile j: P.V0(j-1), S0(j), P.V1(j-1), S1(j).  While one
//     softmax group works on its tile, the tensor core runs the other group's
//     P.V and S.  The commit behind S_w(j) covers P.V_w(j-1), so a query tile's
//     O accumulator is idle whenever its softmax holds S: rescales need no wait;
//   * the softmax reads S once per tile in 32-column chunks: it exponentiates
//     against the running maximum without tracking the tile's own, keeps the
//     packed P row (64 registers) and stores it once every row sum of the tile
//     is known to stay below 2^64 (then nothing can overflow, however far the
//     running maximum lags).  Otherwise, on the first tile and while a row has
//     no running maximum yet, it takes the tile's maximum, rescales O and
//     computes P from S, still in TMEM.  It fetches the next tile's list
//     entries one tile ahead.
// Every mbarrier wait is bounded; on time-out the kernel records
// kErrTimeout, drains its outstanding copies and MMAs, frees TMEM and returns.
#pragma once

#include "attention.cuh"
#include "svg_common.cuh"

namespace svg {

template <int D>
struct Attn2Cfg {
  static constexpr int BM = 128;
  static constexpr int BN = 128;
  static constexpr int PANELS = D / 64;
  static constexpr int PANEL = 128 * 128;          // bytes of one 128-row panel
  static constexpr int Q_BYTES = BM * D * 2;       // one query tile
  static constexpr int SLOT_BYTES = BN * D * 2;    // one K or V tile
  static constexpr int NSLOT = (D == 128) ? 5 : 12;
  static constexpr int DATA_BYTES = 2 * Q_BYTES + NSLOT * SLOT_BYTES;
  static constexpr int BAR_BYTES = 512;
  static constexpr int SMEM_BYTES = DATA_BYTES + BAR_BYTES + 1024;
  static constexpr int THREADS = 320;
  static constexpr uint32_t TMEM_COLS = 512;
  // TMEM columns: S of query tile w at 128*w, O of query tile w at 256 + d*w
  static __device__ __forceinline__ uint32_t tm_s(int w) { return 128u * w; }
  static __device__ __forceinline__ uint32_t tm_o(int w) { return 256u + static_cast<uint32_t>(D) * w; }
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(2 * NSLOT + 12 <= BAR_BYTES / 8, "barrier area");
  static_assert(NSLOT >= 2, "a K and a V tile in flight");
};

// Walks the sorted union of two ascending CSR lists.  flags per list:
// bit 0 = listed, bit 1 = full (no token-level predicate needed).
struct UnionCursor {
  const int32_t* col;
  const uint8_t* full;
  int ia, ea, ib, eb;
  __device__ __forceinline__ bool next(int& kb, int& fa, int& fb) {
    const int ka = (ia < ea) ? __ldg(col + ia) : INT_MAX;
    const int kc = (ib < eb) ? __ldg(col + ib) : INT_MAX;
    if (ka == INT_MAX && kc == INT_MAX) return false;
    kb = min(ka, kc);
    fa = 0;
    fb = 0;
    if (ka == kb) {
      fa = 1 | (__ldg(full + ia) ? 2 : 0);
      ia++;
    }
    if (kc == kb) {
      fb = 1 | (__ldg(full + ib) ? 2 : 0);
      ib++;
    }
    return true;
  }
};

// CLUSTER: the semantic-permutation mask (a.sel, a.qoff, a.koff, a.out_perm)
// instead of the head kinds' windows; a separate instantiation, so the window
// path carries none of its code.
template <int D, bool CLUSTER>
__global__ void __launch_bounds__(Attn2Cfg<D>::THREADS, 1)
    attn2_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                 const __grid_constant__ CUtensorMap tmv, const AttnArgs a) {
  using C = Attn2Cfg<D>;
  constexpr int NSLOT = C::NSLOT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                              // two query tiles
  uint8_t* sKV = smem + 2 * C::Q_BYTES;            // NSLOT slots
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::DATA_BYTES);
  const uint32_t b_q = smem_addr(&bars[0]);
  auto b_full = [&](int s) { return smem_addr(&bars[1 + s]); };
  auto b_empty = [&](int s) { return smem_addr(&bars[1 + NSLOT + s]); };
  auto b_s = [&](int w) { return smem_addr(&bars[1 + 2 * NSLOT + w]); };
  auto b_p = [&](int w) { return smem_addr(&bars[3 + 2 * NSLOT + w]); };
  auto b_o = [&](int w) { return smem_addr(&bars[5 + 2 * NSLOT + w]); };
  const uint32_t b_drain = smem_addr(&bars[7 + 2 * NSLOT]);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(&bars[8 + 2 * NSLOT]);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(&bars[9 + 2 * NSLOT]);

  const Geometry& g = a.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // work order: pairs holding a text-row tile first, then head by head
  const int npair = (g.nqb + 1) >> 1;
  int bh, pr;
  {
    const int qb_text = (g.T > 0) ? g.Lv / g.bq : g.nqb;
    const int p_text = min(qb_text >> 1, npair);
    const int n_heavy = npair - p_text;
    const int x = blockIdx.x;
    if (x < g.BH * n_heavy) {
      bh = x / n_heavy;
      pr = p_text + x % n_heavy;
    } else {
      const int y = x - g.BH * n_heavy;
      bh = y / p_text;
      pr = y % p_text;
    }
  }
  const int qb0 = 2 * pr, qb1 = 2 * pr + 1;          // qb1 may be past the last tile (empty list)
  const int ra0 = a.row_ptr[bh * g.nqb + qb0], ra1 = a.row_ptr[bh * g.nqb + qb0 + 1];
  const int rb0 = ra1, rb1 = (qb1 < g.nqb) ? a.row_ptr[bh * g.nqb + qb1 + 1] : ra1;

  if (threadIdx.x == 0) {
    mbar_init(b_q, 1);
    for (int s = 0; s < NSLOT; s++) {
      mbar_init(b_full(s), 1);
      mbar_init(b_empty(s), 1);
    }
    for (int w = 0; w < 2; w++) {
      mbar_init(b_s(w), 1);
      mbar_init(b_p(w), 128);
      mbar_init(b_o(w), 1);
    }
    mbar_init(b_drain, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) tmem_alloc(smem_addr(tmem_slot), C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmq);
      tma_prefetch_desc(&tmk);
      tma_prefetch_desc(&tmv);
      mbar_expect_tx(b_q, 2 * C::Q_BYTES);
#pragma unroll
      for (int w = 0; w < 2; w++)
#pragma unroll
        for (int p = 0; p < C::PANELS; p++)
          tma_load_3d(smem_addr(sQ + w * C::Q_BYTES + p * C::PANEL), &tmq, p * 64, (qb0 + w) * g.bq, bh, b_q);
      UnionCursor cur{a.col, a.full, ra0, ra1, rb0, rb1};
      int issued = 0;
      for (int j = 0;; j++) {
        int kb[2], fa, fb;
        int nb = 0;
        if (cur.next(kb[0], fa, fb)) nb = 1;
        if (nb == 1 && cur.next(kb[1], fa, fb)) nb = 2;
        if (nb == 0) break;
        bool ok = true;
        for (int half = 0; half < 2 && ok; half++) {       // K then V of this tile
          const int i = 2 * j + half, st = i % NSLOT;
          if (i >= NSLOT && !mbar_wait(b_empty(st), ((i / NSLOT) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          const CUtensorMap* map = half ? &tmv : &tmk;
          mbar_expect_tx(b_full(st), nb * 64 * D * 2);
          for (int h = 0; h < nb; h++)
#pragma unroll
            for (int p = 0; p < C::PANELS; p++)
              tma_load_3d(smem_addr(sKV + st * C::SLOT_BYTES + p * C::PANEL + h * 64 * 128), map, p * 64,
                          kb[h] * 64, bh, b_full(st));
          issued = i + 1;
        }
        if (!ok) break;
      }
      if (*abort_flag) {
        mbar_wait_drain(b_q, 0);
        for (int i = max(0, issued - NSLOT); i < issued; i++) mbar_wait_drain(b_full(i % NSLOT), (i / NSLOT) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop (converged, so the descriptors stay in
    // uniform registers); one elected lane issues each MMA and commit.
    {
      constexpr uint32_t idS128 = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t idS64 = idesc_bf16_f32(128, 64, 0, 0);
      constexpr uint32_t idO = idesc_bf16_f32(128, D, 0, 1);
      // Descriptors of the operand bases.  An operand at byte offset o from a
      // base has the base's descriptor plus o / 16: the start-address field holds
      // address / 16 in 14 bits and every operand lies inside shared memory
      // (< 256 KB), so the field never carries into the next one.
      const uint64_t dq = sdesc_sw128(smem_addr(sQ), 16, 1024);
      const uint64_t dk = sdesc_sw128(smem_addr(sKV), 16, 1024);
      const uint64_t dv = sdesc_sw128(smem_addr(sKV), C::PANEL, 1024);
      UnionCursor cur{a.col, a.full, ra0, ra1, rb0, rb1};
      auto tile_blocks = [&]() {
        int kb, fa, fb, nb = 0;
        if (cur.next(kb, fa, fb)) nb = 1;
        if (nb == 1 && cur.next(kb, fa, fb)) nb = 2;
        return nb;
      };
      // S_w = Q_w K^T: K = d in steps of 16 (32 bytes of a 128-byte swizzled row; 64 per panel)
      auto issue_s = [&](int w, int st, int nb) {
        const uint64_t a0 = dq + static_cast<uint32_t>((w * C::Q_BYTES) >> 4);
        const uint64_t b0 = dk + static_cast<uint32_t>((st * C::SLOT_BYTES) >> 4);
        const uint32_t id = nb == 2 ? idS128 : idS64;
#pragma unroll
        for (int kk = 0; kk < D / 16; kk++) {
          const uint32_t o16 = static_cast<uint32_t>(((kk >> 2) * C::PANEL + (kk & 3) * 32) >> 4);
          umma_ss_elect(tmem + C::tm_s(w), a0 + o16, b0 + o16, id, kk > 0);
        }
        umma_commit_elect(b_s(w));
      };
      // O_w += P_w V: K = keys in steps of 16 (2048 bytes of the MN-major V tile)
      auto issue_pv = [&](int w, int st, int nb, bool first) {
        const uint64_t b0 = dv + static_cast<uint32_t>((st * C::SLOT_BYTES) >> 4);
        const uint32_t tp = tmem + C::tm_s(w), to = tmem + C::tm_o(w);
        if (nb == 2) {
#pragma unroll
          for (int kk = 0; kk < 8; kk++) umma_ts_elect(to, tp + kk * 8, b0 + kk * (2048 >> 4), idO, (!first || kk > 0) ? 1u : 0u);
        } else {
#pragma unroll
          for (int kk = 0; kk < 4; kk++) umma_ts_elect(to, tp + kk * 8, b0 + kk * (2048 >> 4), idO, (!first || kk > 0) ? 1u : 0u);
        }
        umma_commit_elect(b_o(w));
      };
      // slot and phase of the ring entries: K of tile j is entry 2j, V entry 2j+1
      int sk = 0, pk = 0;              // K of the current tile
      auto advance = [&](int& st, int& ph) {
        st += 2;
        if (st >= NSLOT) {
          st -= NSLOT;
          ph ^= 1;
        }
      };
      int sv = 1, pv = 0;              // V of the previous tile (entry 2j-1 at iteration j)
      // every wait is made warp-uniform, so the warp stays converged for elect.sync
      auto wait_all = [&](uint32_t bar, uint32_t par) { return __all_sync(0xffffffffu, mbar_wait(bar, par, abort_flag)); };
      bool issued_any = false;
      bool ok = wait_all(b_q, 0);
      int nb_prev = 0;
      int nb = ok ? tile_blocks() : 0;
      if (ok && nb > 0) {
        // tile 0: S0, S1
        if (!wait_all(b_full(sk), pk)) ok = false;
        if (ok) {
          tc_fence_after();
          issue_s(0, sk, nb);
          issue_s(1, sk, nb);
          umma_commit_elect(b_empty(sk));
          issued_any = true;
        }
      }
      for (int j = 1; ok && nb > 0; j++) {
        nb_prev = nb;
        nb = tile_blocks();                       // blocks of tile j (0: no tile j)
        const int sv_prev = sv, pv_prev = pv;     // V of tile j-1
        advance(sk, pk);                          // K of tile j
        // P.V0(j-1)
        if (!wait_all(b_p(0), (j - 1) & 1)) break;
        if (!wait_all(b_full(sv_prev), pv_prev)) break;
        tc_fence_after();
        issue_pv(0, sv_prev, nb_prev, j == 1);
        // S0(j)
        if (nb > 0) {
          if (!wait_all(b_full(sk), pk)) break;
          tc_fence_after();
          issue_s(0, sk, nb);
        }
        // P.V1(j-1)
        if (!wait_all(b_p(1), (j - 1) & 1)) break;
        tc_fence_after();
        issue_pv(1, sv_prev, nb_prev, j == 1);
        umma_commit_elect(b_empty(sv_prev));
        // S1(j)
        if (nb > 0) {
          issue_s(1, sk, nb);
          umma_commit_elect(b_empty(sk));
        }
        advance(sv, pv);                          // V of tile j
      }
      if (*abort_flag && issued_any) {
        umma_commit_elect(b_drain);
        mbar_wait_drain(b_drain, 0);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax (two groups)
    const int w = (warp - 2) >> 2;                 // query tile of this group
    const int q4 = warp & 3;                       // TMEM lane quarter
    const int r = q4 * 32 + lane;
    const int row = (qb0 + w) * g.bq + r;
    const int kind = CLUSTER ? static_cast<int>(SVG_HEAD_DENSE) : a.kind[bh];
    int lo, hi;
    row_interval(g, kind, row, lo, hi);
    // semantic-permutation mask: this row's key-cluster set (text rows: all)
    uint64_t rmask = ~0ull;
    const int32_t* ko = nullptr;
    if constexpr (CLUSTER) {
      ko = a.koff + static_cast<int64_t>(bh) * (a.Ck + 1);
      if (row < g.Lv)
        rmask = a.sel[static_cast<int64_t>(bh) * a.Cq + cluster_of(a.qoff + static_cast<int64_t>(bh) * (a.Cq + 1),
                                                                    a.Cq, row)];
    }
    const uint32_t tl = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const uint32_t tS = tl + C::tm_s(w), tO = tl + C::tm_o(w);
    const float sl2 = a.scale_log2;
    const uint64_t sl2x2 = f32x2(sl2, sl2);
    float m_use = -INFINITY, l = 0.f;
    bool ok = true;
    int nT = 0;
    UnionCursor cur{a.col, a.full, ra0, ra1, rb0, rb1};
    // the next tile's blocks and this group's flags, fetched one tile ahead
    int nkb0 = -1, nkb1 = -1, nfl0 = 0, nfl1 = 0;
    auto fetch = [&]() {
      int fa, fb;
      nkb1 = -1;
      nfl1 = 0;
      if (!cur.next(nkb0, fa, fb)) {
        nkb0 = -1;
        return;
      }
      nfl0 = w ? fb : fa;
      if (cur.next(nkb1, fa, fb)) nfl1 = w ? fb : fa;
      else nkb1 = -1;
    };
    fetch();
    for (int j = 0; nkb0 >= 0; j++) {
      const int kbs[2] = {nkb0, nkb1}, fl[2] = {nfl0, nfl1};
      fetch();
      nT = j + 1;
      // per 64-key half: 0 = keep all, 1 = token-level mask, 2 = nothing kept
      // (block absent or not listed for this query tile)
      int mode[2];
#pragma unroll
      for (int h = 0; h < 2; h++) {
        if (kbs[h] < 0 || !(fl[h] & 1)) mode[h] = 2;
        else if (!(fl[h] & 2) || kbs[h] * 64 + 64 > g.L) mode[h] = 1;
        else mode[h] = 0;
      }
      auto apply_mask = [&](uint32_t* v, int q) {
        const int h = q >> 1;
        if (mode[h] == 2) {
#pragma unroll
          for (int c = 0; c < 32; c++) v[c] = __float_as_uint(-INFINITY);
        } else if (mode[h] == 1) {
          const int k0 = kbs[h] * 64 + (q & 1) * 32;
          if constexpr (CLUSTER) {
            // Key clusters are contiguous, so the 32 columns are a few runs of one
            // cluster each; the runs are the same for the whole warp.  A run is
            // kept iff its cluster is in this row's set; text columns always,
            // columns past L never.
            uint32_t keep = 0;
            const int vend = min(k0 + 32, g.Lv);
            if (k0 < vend) {
              int jc = cluster_of(ko, a.Ck, k0);          // ko[jc] <= s0 < ko[Ck] = Lv
              for (int s0 = k0; s0 < vend && jc < a.Ck; jc++) {
                const int e = max(s0, min(__ldg(ko + jc + 1), vend));   // max: a malformed table cannot move back
                if ((rmask >> jc) & 1ull) keep |= span_bits(s0 - k0, e - k0);
                s0 = e;
              }
            }
            const int t0 = max(k0, g.Lv), t1 = min(k0 + 32, g.L);
            if (t0 < t1) keep |= span_bits(t0 - k0, t1 - k0);
#pragma unroll
            for (int c = 0; c < 32; c++)
              if (!((keep >> c) & 1u)) v[c] = __float_as_uint(-INFINITY);
          } else {
            // kept columns: the row's window [lo, hi) and the text keys [Lv, Lv + T),
            // as one 32-bit word (a few instructions instead of two compares per column)
            const int a0 = min(max(lo - k0, 0), 32), a1 = min(max(hi - k0, 0), 32);
            const int t0 = min(max(g.Lv - k0, 0), 32), t1 = min(max(g.Lv + g.T - k0, 0), 32);
            const uint32_t keep = (a0 < a1 ? span_bits(a0, a1) : 0u) | (t0 < t1 ? span_bits(t0, t1) : 0u);
#pragma unroll
            for (int c = 0; c < 32; c++)
              if (!((keep >> c) & 1u)) v[c] = __float_as_uint(-INFINITY);
          }
        }
      };
      if (!__all_sync(0xffffffffu, mbar_wait(b_s(w), j & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // chunk q (32 columns) of S with the mask applied
      auto load_chunk = [&](int q, uint32_t* v) {
        tmem_ld32(tS + q * 32, v);
        tmem_wait_ld();
        apply_mask(v, q);
      };
      auto chunk_max = [&](const uint32_t* v, float* m8) {
#pragma unroll
        for (int c = 0; c < 32; c += 16)
#pragma unroll
          for (int i = 0; i < 8; i++) m8[i] = fmax3(m8[i], __uint_as_float(v[c + i]), __uint_as_float(v[c + 8 + i]));
      };
      // P = 2^(S*scale*log2e - m) of one chunk as 16 packed bf16 pairs, row sums in acc
      auto chunk_exp = [&](const uint32_t* v, uint32_t* pk, uint64_t* acc, uint64_t nm2) {
#pragma unroll
        for (int c = 0; c < 16; c++) {
          const uint64_t xa = ffma2(f32x2(__uint_as_float(v[2 * c]), __uint_as_float(v[2 * c + 1])), sl2x2, nm2);
          float x0, x1;
          unpack2(xa, x0, x1);
          const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
          acc[c & 1] = fadd2(acc[c & 1], f32x2(p0, p1));
          pk[c] = pack_bf16x2(p0, p1);
        }
      };
      uint32_t pk[64];
      uint64_t acc[2] = {0ull, 0ull};
      float m8[8];
#pragma unroll
      for (int i = 0; i < 8; i++) m8[i] = -INFINITY;
      // A pass over the kept chunks of S; `body` sees each chunk with its mask applied.
      auto pass = [&](auto&& body) {
#pragma unroll
        for (int q = 0; q < 4; q++) {
          if (mode[q >> 1] == 2) {
#pragma unroll
            for (int c = 0; c < 16; c++) pk[16 * q + c] = 0u;
            continue;
          }
          uint32_t v[32];
          load_chunk(q, v);
          body(v, q);
        }
      };
      bool rescale;
      if (j > 0 && __all_sync(0xffffffffu, m_use != -INFINITY)) {
        // Every row has a running maximum: exponentiate against it without tracking
        // the tile's maximum.  The result stands while the tile's row sum of
        // 2^(x - m) stays below 2^64: then no P exceeds 2^64, so P (bf16), l and O
        // (fp32) stay far inside their range and keep their relative precision,
        // however far m lags the true maximum.  Otherwise the tile's maximum is
        // taken and the running one moves.
        const uint64_t nm2 = f32x2(-m_use, -m_use);
        pass([&](const uint32_t* v, int q) { chunk_exp(v, pk + 16 * q, acc, nm2); });
        float s0, s1, s2, s3;
        unpack2(acc[0], s0, s1);
        unpack2(acc[1], s2, s3);
        rescale = __any_sync(0xffffffffu, !(((s0 + s1) + (s2 + s3)) < 0x1p64f));
        if (rescale) pass([&](const uint32_t* v, int q) { chunk_max(v, m8); });
      } else {
        // First tile, or a row of the warp has seen no kept key yet: the tile's
        // maximum first, then P against it.  (A combined max-and-exponentiate pass
        // for the second case was measured slower: the kernel's code grew by a
        // third, and sparse lists, which meet this case often, ran up to 18%
        // slower.)
        pass([&](const uint32_t* v, int q) { chunk_max(v, m8); });
        rescale = true;
      }
      if (rescale) {
        const float mx = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
        const float mxs = mx * sl2;
        const bool need_rescale = mxs > m_use + 8.0f;
        const float m_new = need_rescale ? mxs : m_use;
        const float alpha = need_rescale ? ((m_use == -INFINITY) ? 0.f : fast_exp2(m_use - m_new)) : 1.f;
        l *= alpha;
        if (j > 0) {
          // P.V_w(j-1) finished before S_w(j) (same commit), so O_w is idle here
          uint32_t o[32];
#pragma unroll 1
          for (int c = 0; c < D / 32; c++) {
            tmem_ld32(tO + c * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; i++) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tO + c * 32, o);
          }
          tmem_wait_st();
        }
        m_use = m_new;
        // P again from S, which is still in TMEM
        const float msub = (m_use == -INFINITY) ? 0.f : m_use;
        const uint64_t nm2 = f32x2(-msub, -msub);
        acc[0] = 0ull;
        acc[1] = 0ull;
        pass([&](const uint32_t* v, int q) { chunk_exp(v, pk + 16 * q, acc, nm2); });
      }
      // packed P over S columns [0, 64)
      tmem_st32(tS, pk);
      tmem_st32(tS + 32, pk + 32);
      float s0, s1, s2, s3;
      unpack2(acc[0], s0, s1);
      unpack2(acc[1], s2, s3);
      l += (s0 + s1) + (s2 + s3);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(b_p(w));
    }
    // ---------------------------------------------------------- epilogue
    const bool row_ok = (qb0 + w) < g.nqb && r < g.bq && row < g.L;
    if (ok && nT > 0 && __all_sync(0xffffffffu, mbar_wait(b_o(w), (nT - 1) & 1, abort_flag))) {
      tc_fence_after();
      const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
      const int orow_t = row_ok ? out_row<CLUSTER>(a, kind, bh, row) : 0;
      const bool write = row_ok && orow_t >= 0;
      const int64_t orow_i = static_cast<int64_t>(bh) * g.L + orow_t;
      uint16_t* orow = a.out + orow_i * D;
#pragma unroll 1
      for (int c = 0; c < D / 32; c++) {
        uint32_t o[32];
        tmem_ld32(tO + c * 32, o);
        tmem_wait_ld();
        if (write) {
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
      if (write && a.lse) a.lse[orow_i] = (l > 0.f) ? (m_use * 0.69314718055994531f + logf(l)) : -INFINITY;
    } else if (ok && nT == 0 && row_ok) {
      const int orow_t = out_row<CLUSTER>(a, kind, bh, row);
      if (orow_t >= 0) {
        const int64_t orow_i = static_cast<int64_t>(bh) * g.L + orow_t;
        uint4* dst = reinterpret_cast<uint4*>(a.out + orow_i * D);
        for (int v = 0; v < D / 8; v++) dst[v] = make_uint4(0, 0, 0, 0);
        if (a.lse) a.lse[orow_i] = -INFINITY;
      }
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
