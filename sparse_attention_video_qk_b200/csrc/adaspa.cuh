// adaspa.cuh — AdaSpa's blockified search with a cached LSE ("AdaSpa"
// abstract: a blockified sparse pattern; "Fused LSE-Cached Search with
// Head-adaptive Hierarchical Block Sparse Attention"; the pattern and the LSE
// stay the same across denoising steps).
//
// 1. mass_kernel: the exact attention mass of every (query tile, key tile)
//    block, given each row's log-sum-exp from an earlier step:
//        M[qb][kb] = sum_{q in qb, k in kb} 2^(s_qk * scale * log2 e - lse_q * log2 e)
//    in one pass over Q K^T (no normalisation pass: the LSE is known).  One
//    CTA per (b, h, set of NG 128-row query tiles): warp 0 streams K through a
//    TMA slot ring, warp 1 issues S = Q K^T as M=128, N=128 tcgen05 MMAs into
//    TMEM, and each following group of 4 warps exponentiates and sums one query
//    tile's S (thread = row).  With NG = 4 (the default) each group's S is one
//    128-column TMEM buffer and the other groups' MMAs run while a group
//    exponentiates; with NG = 2 it is double-buffered.  The per-row sums of each
//    64-key block are reduced over the tile's 128 rows by shuffles and a fixed
//    4-warp order, so the result does not depend on scheduling.
// 2. select_kernel: per (head, query tile), the video key tiles sorted by
//    mass (descending, lower index first) and the shortest prefix whose
//    running sum reaches p times their total, in 32-bit fixed point; text key
//    tiles always, and query tiles holding text rows keep every key tile.
//    One block per query tile: bitonic sort in shared memory, a block scan of
//    the fixed-point masses, then the kept tiles in increasing order.
//
// Every mbarrier wait is bounded; on time-out the kernel records
// kErrTimeout, drains its outstanding copies and MMAs, frees TMEM and returns.
#pragma once

#include "attention.cuh"
#include "svg_common.cuh"

namespace svg {

// NG query tiles per CTA (one softmax group of 4 warps each).  With NG = 2 each
// group's S is double-buffered in TMEM; with NG = 4 single-buffered, and the
// other groups' MMAs fill the tensor pipe while one group exponentiates.
template <int D, int NG>
struct MassCfg {
  static constexpr int PANELS = D / 64;
  static constexpr int PANEL = 128 * 128;          // bytes of one 128-row panel
  static constexpr int Q_BYTES = 128 * D * 2;      // one query tile
  static constexpr int SLOT_BYTES = 128 * D * 2;   // one 128-key K tile
  static constexpr int NBUF = (NG == 2) ? 2 : 1;   // S buffers per group
  static constexpr int NSLOT = (NG == 2) ? ((D == 128) ? 4 : 8) : ((D == 128) ? 3 : 8);
  static constexpr int DATA_BYTES = NG * Q_BYTES + NSLOT * SLOT_BYTES;
  static constexpr int BAR_BYTES = 1024;
  static constexpr int SMEM_BYTES = DATA_BYTES + BAR_BYTES + 1024;
  static constexpr int THREADS = 64 + 128 * NG;
  static constexpr uint32_t TMEM_COLS = 512;
  static __device__ __forceinline__ uint32_t tm_s(int w, int b) { return 128u * (NBUF * w + b); }
  // barrier slots (8 bytes each): q, full[NSLOT], empty[NSLOT], s[NG][NBUF], free[NG][NBUF],
  // part[NG][2], pfree[NG][2], drain, the TMEM slot, the abort flag, then the partial sums
  static constexpr int BAR_S = 1 + 2 * NSLOT;
  static constexpr int BAR_FREE = BAR_S + NG * NBUF;
  static constexpr int BAR_PART = BAR_FREE + NG * NBUF;
  static constexpr int BAR_PFREE = BAR_PART + 2 * NG;
  static constexpr int BAR_DRAIN = BAR_PFREE + 2 * NG;
  static constexpr int SLOT_TMEM = BAR_DRAIN + 1;
  static constexpr int SLOT_ABORT = SLOT_TMEM + 1;
  static constexpr int SLOT_PART = SLOT_ABORT + 1;  // NG * 2 bufs * 4 warps * 2 floats
  static_assert(NBUF * NG * 128 <= 512, "TMEM columns");
  static_assert(SLOT_PART + NG * 8 <= BAR_BYTES / 8, "barrier area");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// query tiles per CTA of the block-mass launch
#ifndef SVG_MASS_GROUPS
#define SVG_MASS_GROUPS 4
#endif
constexpr int kMassGroups = SVG_MASS_GROUPS;

struct MassArgs {
  Geometry g;
  float scale_log2;        // softmax scale * log2(e)
  const float* lse;        // [BH][L], natural log, cached from an earlier step
  float* mass;             // [BH][nqb][nkb]
};

template <int D, int NG>
__global__ void __launch_bounds__(MassCfg<D, NG>::THREADS, 1)
    mass_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                const MassArgs a) {
  using C = MassCfg<D, NG>;
  constexpr int NSLOT = C::NSLOT, NBUF = C::NBUF;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = smem + NG * C::Q_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::DATA_BYTES);
  const uint32_t b_q = smem_addr(&bars[0]);
  auto b_full = [&](int s) { return smem_addr(&bars[1 + s]); };
  auto b_empty = [&](int s) { return smem_addr(&bars[1 + NSLOT + s]); };
  auto b_s = [&](int w, int b) { return smem_addr(&bars[C::BAR_S + NBUF * w + b]); };
  auto b_free = [&](int w, int b) { return smem_addr(&bars[C::BAR_FREE + NBUF * w + b]); };
  auto b_part = [&](int w, int b) { return smem_addr(&bars[C::BAR_PART + 2 * w + b]); };
  auto b_pfree = [&](int w, int b) { return smem_addr(&bars[C::BAR_PFREE + 2 * w + b]); };
  const uint32_t b_drain = smem_addr(&bars[C::BAR_DRAIN]);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(&bars[C::SLOT_TMEM]);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(&bars[C::SLOT_ABORT]);
  float* part = reinterpret_cast<float*>(&bars[C::SLOT_PART]);   // [NG groups][2 bufs][4 warps][2]

  const Geometry& g = a.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nset = (g.nqb + NG - 1) / NG;             // sets of NG query tiles per head
  const int bh = blockIdx.x / nset, qb0 = NG * (blockIdx.x % nset);
  const int ntile = (g.nkb + 1) >> 1;                  // 128-key tiles: blocks 2j, 2j+1

  if (threadIdx.x == 0) {
    mbar_init(b_q, 1);
    for (int s = 0; s < NSLOT; s++) {
      mbar_init(b_full(s), 1);
      mbar_init(b_empty(s), 1);
    }
    for (int w = 0; w < NG; w++) {
      for (int b = 0; b < NBUF; b++) {
        mbar_init(b_s(w, b), 1);
        mbar_init(b_free(w, b), 128);
      }
      for (int b = 0; b < 2; b++) {
        mbar_init(b_part(w, b), 4);
        mbar_init(b_pfree(w, b), 1);
      }
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
      mbar_expect_tx(b_q, NG * C::Q_BYTES);
#pragma unroll
      for (int w = 0; w < NG; w++)
#pragma unroll
        for (int p = 0; p < C::PANELS; p++)
          tma_load_3d(smem_addr(sQ + w * C::Q_BYTES + p * C::PANEL), &tmq, p * 64, (qb0 + w) * 128, bh, b_q);
      int issued = 0;
      for (int j = 0; j < ntile; j++) {
        const int st = j % NSLOT;
        if (j >= NSLOT && !mbar_wait(b_empty(st), ((j / NSLOT) - 1) & 1, abort_flag)) break;
        const int nb = (2 * j + 1 < g.nkb) ? 2 : 1;
        mbar_expect_tx(b_full(st), nb * 64 * D * 2);
        for (int h = 0; h < nb; h++)
#pragma unroll
          for (int p = 0; p < C::PANELS; p++)
            tma_load_3d(smem_addr(sK + st * C::SLOT_BYTES + p * C::PANEL + h * 64 * 128), &tmk, p * 64,
                        (2 * j + h) * 64, bh, b_full(st));
        issued = j + 1;
      }
      if (*abort_flag) {
        mbar_wait_drain(b_q, 0);
        for (int i = max(0, issued - NSLOT); i < issued; i++) mbar_wait_drain(b_full(i % NSLOT), (i / NSLOT) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS128 = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t idS64 = idesc_bf16_f32(128, 64, 0, 0);
      const uint32_t q_base = smem_addr(sQ), k_base = smem_addr(sK);
      bool issued_any = false;
      bool ok = mbar_wait(b_q, 0, abort_flag);
      for (int j = 0; ok && j < ntile; j++) {
        const int st = j % NSLOT, b = j % NBUF;
        const int nb = (2 * j + 1 < g.nkb) ? 2 : 1;
        if (!mbar_wait(b_full(st), (j / NSLOT) & 1, abort_flag)) break;
        for (int w = 0; w < NG && ok; w++) {
          // S_w buffer b was last read by the softmax at tile j - NBUF
          if (j >= NBUF && !mbar_wait(b_free(w, b), ((j / NBUF) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; kk++) {
            const uint32_t off = (kk >> 2) * C::PANEL + (kk & 3) * 32;
            umma_ss(tmem + C::tm_s(w, b), sdesc_sw128(q_base + w * C::Q_BYTES + off, 16, 1024),
                    sdesc_sw128(k_base + st * C::SLOT_BYTES + off, 16, 1024), nb == 2 ? idS128 : idS64, kk > 0);
          }
          umma_commit(b_s(w, b));
          issued_any = true;
        }
        if (!ok) break;
        umma_commit(b_empty(st));
      }
      if (*abort_flag && issued_any) {
        umma_commit(b_drain);
        mbar_wait_drain(b_drain, 0);
      }
    }
  } else {
    // ------------------------------------------------------------ exponentials (NG groups)
    const int w = (warp - 2) >> 2;                 // query tile of this group
    const int q4 = warp & 3;                       // TMEM lane quarter
    const int wg = (warp - 2) & 3;                 // warp index inside the group
    const int r = q4 * 32 + lane;
    const int row = (qb0 + w) * 128 + r;
    const bool tile_ok = (qb0 + w) < g.nqb;
    // rows past L contribute nothing: 2^(s - inf) = 0
    const float l2 = (row < g.L) ? __ldg(a.lse + static_cast<int64_t>(bh) * g.L + row) * 1.4426950408889634f
                                 : INFINITY;
    const uint64_t sl2x2 = f32x2(a.scale_log2, a.scale_log2);
    const uint64_t nl2x2 = f32x2(-l2, -l2);
    const uint32_t tl = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    float* mrow = a.mass + (static_cast<int64_t>(bh) * g.nqb + qb0 + w) * g.nkb;
    for (int j = 0; j < ntile; j++) {
      const int b = j % NBUF;
      if (!__all_sync(0xffffffffu, mbar_wait(b_s(w, b), (j / NBUF) & 1, abort_flag))) break;
      tc_fence_after();
      const uint32_t tS = tl + C::tm_s(w, b);
      float h[2];
#pragma unroll
      for (int half = 0; half < 2; half++) {
        const int kb = 2 * j + half;
        uint64_t acc[2] = {0ull, 0ull};
        if (kb < g.nkb) {                          // warp-uniform
#pragma unroll
          for (int q = 0; q < 2; q++) {
            uint32_t v[32];
            tmem_ld32(tS + half * 64 + q * 32, v);
            tmem_wait_ld();
            const int k0 = kb * 64 + q * 32;
            if (k0 + 32 > g.L) {                   // the ragged last block: keys past L hold zero rows
#pragma unroll
              for (int c = 0; c < 32; c++)
                if (k0 + c >= g.L) v[c] = __float_as_uint(-INFINITY);
            }
#pragma unroll
            for (int c = 0; c < 16; c++) {
              const uint64_t x = ffma2(f32x2(__uint_as_float(v[2 * c]), __uint_as_float(v[2 * c + 1])), sl2x2, nl2x2);
              float x0, x1;
              unpack2(x, x0, x1);
              acc[c & 1] = fadd2(acc[c & 1], f32x2(fast_exp2(x0), fast_exp2(x1)));
            }
          }
        }
        float s0, s1, s2, s3;
        unpack2(acc[0], s0, s1);
        unpack2(acc[1], s2, s3);
        h[half] = (s0 + s1) + (s2 + s3);
      }
      tc_fence_before();
      mbar_arrive(b_free(w, b));
      // the block sums of this tile over the group's 128 rows: shuffles inside a
      // warp, then the group's first warp adds the four warps in a fixed order.
      // The hand-off goes through mbarriers (bounded waits), double-buffered
      // like S: part(w, b) completes when the four warps have written, pfree(w, b)
      // when the first warp has read them.
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        h[0] += __shfl_xor_sync(0xffffffffu, h[0], o);
        h[1] += __shfl_xor_sync(0xffffffffu, h[1], o);
      }
      const int hb = j & 1;                        // hand-off buffer
      float* pb = part + ((w * 2 + hb) * 4) * 2;
      int okp = 1;
      if (lane == 0) {
        if (j >= 2) okp = mbar_wait(b_pfree(w, hb), ((j >> 1) - 1) & 1, abort_flag);
        if (okp) {
          pb[wg * 2] = h[0];
          pb[wg * 2 + 1] = h[1];
          mbar_arrive(b_part(w, hb));
        }
      }
      if (!__shfl_sync(0xffffffffu, okp, 0)) break;
      if (wg == 0) {
        int okr = 1;
        if (lane == 0) {
          okr = mbar_wait(b_part(w, hb), (j >> 1) & 1, abort_flag);
          if (okr) {
            const float m0 = ((pb[0] + pb[2]) + pb[4]) + pb[6];
            const float m1 = ((pb[1] + pb[3]) + pb[5]) + pb[7];
            mbar_arrive(b_pfree(w, hb));
            if (tile_ok) {
              mrow[2 * j] = m0;
              if (2 * j + 1 < g.nkb) mrow[2 * j + 1] = m1;
            }
          }
        }
        if (!__shfl_sync(0xffffffffu, okr, 0)) break;
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

// ------------------------------------------------------------------ selection

struct SelArgs {
  Geometry g;
  double p;
  const float* mass;       // [BH][nqb][nkb]
};

constexpr int kSelThreads = 1024;
constexpr int kSelMaxTiles = 4096;         // key tiles per query tile (L <= 262,144 at bk = 64)

__device__ __forceinline__ bool sel_before(float ma, int ia, float mb, int ib) {
  return (ma > mb) || (ma == mb && ia < ib);
}

// Block-wide inclusive scan of one int64 per thread (kSelThreads threads).
__device__ __forceinline__ long long sel_block_scan(long long v, long long* warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  if (lane == 31) warp_tot[warp] = v;
  __syncthreads();
  if (warp == 0) {
    long long t = warp_tot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long u = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += u;
    }
    warp_tot[lane] = t;
  }
  __syncthreads();
  const long long base = warp ? warp_tot[warp - 1] : 0;
  __syncthreads();
  return v + base;
}

// FILL = false: row_ptr[t + 1] = number of kept tiles, and with `stash` the
// kept flags at stash[t * nkb + kb]; FILL = true: the kept tiles in increasing
// order at col[row_ptr[t] ...] and full = 1, or with `stash` the flags read
// back from it (no second sort) and col alone written (stash aliases full,
// which the caller then sets to 1).
template <bool FILL>
__global__ void __launch_bounds__(kSelThreads) select_kernel(const SelArgs a, int32_t* __restrict__ row_ptr,
                                                            int32_t* __restrict__ col, uint8_t* full,
                                                            int64_t capacity, int P2, uint8_t* stash) {
  extern __shared__ uint8_t sel_smem[];
  float* sm = reinterpret_cast<float*>(sel_smem);              // [P2] masses, sorted in place
  int* si = reinterpret_cast<int*>(sm + P2);                    // [P2] tile indices
  uint8_t* keep = reinterpret_cast<uint8_t*>(si + P2);          // [P2] kept flags by tile index
  __shared__ long long warp_tot[32];
  __shared__ int s_cut;
  const Geometry& g = a.g;
  const int64_t t = blockIdx.x;                                 // bh * nqb + qb
  const int qb = static_cast<int>(t % g.nqb);
  const int tid = threadIdx.x;
  const float* m = a.mass + t * g.nkb;
  const bool text_q = min(g.L, (qb + 1) * g.bq) > g.Lv;
  // video key tiles: no key in [Lv, L) (without text, every tile)
  const int nv = (g.L == g.Lv) ? g.nkb : min(g.nkb, g.Lv / g.bk);
  const bool reuse = FILL && stash;
  for (int i = tid; i < P2; i += kSelThreads) {
    const bool vid = i < nv;
    if (reuse) {
      keep[i] = (i < g.nkb) ? stash[t * g.nkb + i] : 0;
      continue;
    }
    sm[i] = vid ? __ldg(m + i) : -INFINITY;
    si[i] = i;
    keep[i] = (i < g.nkb && (text_q || !vid)) ? 1 : 0;
  }
  __syncthreads();
  if (!reuse && !text_q && nv > 0) {
    // bitonic sort of (mass, index): heavier first, the lower index first on ties.
    // Exchanges 64 or more positions apart go through shared memory; the rest run
    // in registers inside 64-position segments (lane and lane + 32 of a warp),
    // by shuffles.
    const int lane = tid & 31, warp = tid >> 5;
    for (int k = 2; k <= P2; k <<= 1) {
      int jj = k >> 1;
      for (; jj >= 64; jj >>= 1) {
        for (int i = tid; i < P2; i += kSelThreads) {
          const int l = i ^ jj;
          if (l > i) {
            const bool up = (i & k) == 0;
            const float ma = sm[i], mb = sm[l];
            const int ia = si[i], ib = si[l];
            const bool swap = up ? sel_before(mb, ib, ma, ia) : sel_before(ma, ia, mb, ib);
            if (swap) {
              sm[i] = mb;
              sm[l] = ma;
              si[i] = ib;
              si[l] = ia;
            }
          }
        }
        __syncthreads();
      }
      for (int seg = warp; seg < P2 / 64; seg += kSelThreads / 32) {
        const int pa = seg * 64 + lane, pb = pa + 32;
        float ma = sm[pa], mb = sm[pb];
        int ia = si[pa], ib = si[pb];
        if (jj == 32) {                                 // partners in the same thread
          const bool up = (pa & k) == 0;
          if (up ? sel_before(mb, ib, ma, ia) : sel_before(ma, ia, mb, ib)) {
            const float tm = ma;
            const int ti = ia;
            ma = mb;
            ia = ib;
            mb = tm;
            ib = ti;
          }
        }
        for (int j = min(jj, 16); j > 0; j >>= 1) {
#pragma unroll
          for (int e = 0; e < 2; e++) {
            float& m = e ? mb : ma;
            int& ix = e ? ib : ia;
            const int pos = e ? pb : pa;
            const float om = __shfl_xor_sync(0xffffffffu, m, j);
            const int oi = __shfl_xor_sync(0xffffffffu, ix, j);
            // the lower position of the pair takes the element that comes first in
            // an ascending run, the other one in a descending run
            const bool want_first = ((pos & j) == 0) == ((pos & k) == 0);
            if (want_first != sel_before(m, ix, om, oi)) {
              m = om;
              ix = oi;
            }
          }
        }
        sm[pa] = ma;
        sm[pb] = mb;
        si[pa] = ia;
        si[pb] = ib;
      }
      __syncthreads();
    }
    // fixed-point masses in sorted order: each thread owns P2 / kSelThreads consecutive positions
    const int per = P2 / kSelThreads > 0 ? P2 / kSelThreads : 1;
    const int p0 = tid * per;
    long long own = 0;
    for (int u = 0; u < per; u++) {
      const int pos = p0 + u;
      if (pos < nv) own += static_cast<long long>(static_cast<double>(sm[pos]) * 4294967296.0);
    }
    const long long incl = sel_block_scan(own, warp_tot);
    const long long total = warp_tot[31];
    const double goal = __dmul_rn(a.p, static_cast<double>(total));
    // positions whose inclusive running sum is still below the goal
    long long run = incl - own;
    int below = 0;
    for (int u = 0; u < per; u++) {
      const int pos = p0 + u;
      if (pos < nv) {
        run += static_cast<long long>(static_cast<double>(sm[pos]) * 4294967296.0);
        below += (static_cast<double>(run) < goal) ? 1 : 0;
      }
    }
    if (tid == 0) s_cut = 0;
    __syncthreads();
    if (below) atomicAdd(&s_cut, below);
    __syncthreads();
    const int cut = s_cut;                                      // positions 0..cut are kept
    for (int pos = tid; pos <= cut && pos < nv; pos += kSelThreads) keep[si[pos]] = 1;
    __syncthreads();
  }
  // the kept tiles in increasing order
  const int per = (g.nkb + kSelThreads - 1) / kSelThreads;
  const int i0 = tid * per;
  int cnt = 0;
  for (int u = 0; u < per; u++)
    if (i0 + u < g.nkb) cnt += keep[i0 + u];
  const long long incl = sel_block_scan(cnt, warp_tot);
  if (!FILL) {
    if (tid == kSelThreads - 1) row_ptr[t + 1] = static_cast<int32_t>(incl);
    if (t == 0 && tid == 0) row_ptr[0] = 0;
    if (stash)
      for (int i = tid; i < g.nkb; i += kSelThreads) stash[t * g.nkb + i] = keep[i];
    return;
  }
  int64_t e = row_ptr[t] + (incl - cnt);
  for (int u = 0; u < per; u++) {
    const int kb = i0 + u;
    if (kb < g.nkb && keep[kb]) {
      if (e < capacity) {
        col[e] = kb;
        if (!stash) full[e] = 1;
      }
      e++;
    }
  }
}

}  // namespace svg
