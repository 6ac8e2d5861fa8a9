// svg_lib.cu — the C ABI declared in include/svg.h: host-side argument
// checks, launch geometry, TMA tensor maps, and the host helpers.  All
// kernels are in the included .cuh files (one translation unit).
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "attention.cuh"
#include "attention2.cuh"
#include "block_index.cuh"
#include "profile_tc.cuh"
#include "rowmap.cuh"
#include "svg2.cuh"
#include "adaspa.cuh"
#include "svg_common.cuh"

using namespace svg;

namespace {

constexpr int kNumSMs = 148;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

svg_status check_shape(const svg_shape* s) {
  if (!s) return SVG_ERR_INVALID_ARG;
  if (s->B <= 0 || s->H <= 0 || s->F <= 0 || s->Hs <= 0 || s->Ws <= 0 || s->text_len < 0) return SVG_ERR_SHAPE;
  const long long Lv = static_cast<long long>(s->F) * s->Hs * s->Ws;
  if (Lv + s->text_len != s->L) return SVG_ERR_SHAPE;
  if (s->L >= (1 << 30)) return SVG_ERR_UNSUPPORTED;
  if (s->d != 64 && s->d != 128) return SVG_ERR_UNSUPPORTED;
  if (static_cast<long long>(s->B) * s->H > (1 << 24)) return SVG_ERR_UNSUPPORTED;
  return SVG_OK;
}

svg_status check_params(const svg_shape* s, const svg_params* p, bool need_tiles) {
  if (!p) return SVG_ERR_INVALID_ARG;
  if (p->spatial_frames < 0 || p->temporal_radius < 0) return SVG_ERR_INVALID_ARG;
  if (need_tiles) {
    if (p->block_k != 64) return SVG_ERR_UNSUPPORTED;
    if (p->block_q != 64 && p->block_q != 128) return SVG_ERR_UNSUPPORTED;
  }
  if (!(p->eps >= 0.f) || !(p->softmax_scale >= 0.f)) return SVG_ERR_INVALID_ARG;
  (void)s;
  return SVG_OK;
}

svg_status check_rope(const svg_shape* s, const svg_params* p) {
  const int* sp = p->rope_split;
  if (sp[0] < 0 || sp[1] < 0 || sp[2] < 0) return SVG_ERR_INVALID_ARG;
  if ((sp[0] | sp[1] | sp[2]) & 1) return SVG_ERR_UNSUPPORTED;
  if (sp[0] + sp[1] + sp[2] != s->d) return SVG_ERR_SHAPE;
  if (!(p->rope_base > 0.f)) return SVG_ERR_INVALID_ARG;
  return SVG_OK;
}

Geometry make_geometry(const svg_shape* s, const svg_params* p) {
  Geometry g{};
  g.B = s->B;
  g.H = s->H;
  g.L = s->L;
  g.d = s->d;
  g.F = s->F;
  g.Hs = s->Hs;
  g.Ws = s->Ws;
  g.T = s->text_len;
  g.S = s->Hs * s->Ws;
  g.Lv = g.F * g.S;
  g.BH = s->B * s->H;
  if (p) {
    g.w = p->spatial_frames;
    g.r = p->temporal_radius;
    g.bq = p->block_q > 0 ? p->block_q : 128;
    g.bk = p->block_k > 0 ? p->block_k : 64;
  } else {
    g.bq = 128;
    g.bk = 64;
  }
  g.nqb = (g.L + g.bq - 1) / g.bq;
  g.nkb = (g.L + g.bk - 1) / g.bk;
  return g;
}

float scale_of(const svg_shape* s, const svg_params* p) {
  return (p->softmax_scale > 0.f) ? p->softmax_scale : 1.0f / std::sqrt(static_cast<float>(s->d));
}

svg_status launch_status() {
  return (cudaGetLastError() == cudaSuccess) ? SVG_OK : SVG_ERR_CUDA;
}

// ----------------------------------------------------------- tensor maps --

PFN_cuTensorMapEncodeTiled_v12000 get_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, []() {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 3-D map over a [BH, L, D] bf16 tensor: dims (D, L, BH), box (64, rows, 1),
// 128-byte swizzle; rows past L read as zero.
bool make_map(CUtensorMap* m, const void* base, int D, int L, int BH, int rows) {
  auto enc = get_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(L) * D * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(rows), 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <typename K>
bool set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess;
}

// ------------------------------------------------------------- rowmap ----

// RoPE table layout and constants of the norm routine (norm_rope.cuh).
RopeArgs make_rope_args(const svg_shape* s, const svg_params* p, const float* rope_table) {
  RopeArgs r{};
  r.table = reinterpret_cast<const float2*>(rope_table);
  r.eps = p ? p->eps : 0.f;
  if (p) {
    r.split0 = p->rope_split[0];
    r.split1 = p->rope_split[1];
    r.off1 = s->F * (p->rope_split[0] / 2);
    r.off2 = r.off1 + s->Hs * (p->rope_split[1] / 2);
    r.vec = (p->rope_split[0] % 8 == 0 && p->rope_split[1] % 8 == 0 && p->rope_split[2] % 8 == 0) ? 1 : 0;
  }
  r.divS = make_fastdiv(s->Hs * s->Ws);
  r.divWs = make_fastdiv(s->Ws);
  return r;
}

svg_status launch_rowmap(RowmapArgs a, int D, cudaStream_t st) {
  a.divF = make_fastdiv(a.g.F);
  const int unit_rows = 8 * (32 / (D / 8)) * kRowmapSteps * kRowmapUnitSteps;
  const int64_t nunits = static_cast<int64_t>(a.ntensor) * a.g.BH * ((a.g.L + unit_rows - 1) / unit_rows);
  if (nunits > INT32_MAX) return SVG_ERR_UNSUPPORTED;
  int64_t blocks = static_cast<int64_t>(kNumSMs) * kRowmapBlocksPerSM;   // the resident capacity
  if (blocks > nunits) blocks = nunits;
  const dim3 grid(static_cast<unsigned>(blocks));
  const bool staged = a.norm_tensors > 0 && a.rope_floats <= kRopeSmemFloats;
  const int smem = staged ? a.rope_floats * 4 : 0;
  if (D == 128) {
    if (staged) {
      if (!set_smem(rowmap_kernel<128, true>, smem)) return SVG_ERR_CUDA;
      rowmap_kernel<128, true><<<grid, 256, smem, st>>>(a);
    } else {
      rowmap_kernel<128, false><<<grid, 256, 0, st>>>(a);
    }
  } else {
    if (staged) {
      if (!set_smem(rowmap_kernel<64, true>, smem)) return SVG_ERR_CUDA;
      rowmap_kernel<64, true><<<grid, 256, smem, st>>>(a);
    } else {
      rowmap_kernel<64, false><<<grid, 256, 0, st>>>(a);
    }
  }
  return launch_status();
}

// Profiling: the tensor-core partial kernel over key chunks, the per-row
// merge and the per-head choice.  `workspace` holds
// prof_workspace_bytes(BH, L, d, max_chunks) bytes.
// qn holds normalised Q, or raw Q when gamma_q is given (the sampled rows are
// then normalised in the kernel with rope_table).
svg_status launch_profile(const svg_shape* s, const svg_params* p, const uint16_t* qn, const uint16_t* kn,
                          const uint16_t* v, const int32_t* sample_idx, int n, void* workspace, int max_chunks,
                          float* mse_out, uint8_t* head_kind_out, cudaStream_t cs, const float* gamma_q = nullptr,
                          const float* rope_table = nullptr) {
  ProfArgs a{};
  a.g = make_geometry(s, p);
  a.scale_log2 = scale_of(s, p) * 1.4426950408889634f;
  a.q = qn;
  a.gamma_q = gamma_q;
  a.rope = make_rope_args(s, p, rope_table);
  a.sample = sample_idx;
  a.n = n;
  const int ntiles = (a.g.L + kProfKeys - 1) / kProfKeys;
  const int nchunk = max(1, min(max_chunks, ntiles));
  a.tiles_per_chunk = (ntiles + nchunk - 1) / nchunk;
  a.nchunk = (ntiles + a.tiles_per_chunk - 1) / a.tiles_per_chunk;   // every chunk non-empty
  a.ws = static_cast<float*>(workspace);
  a.err = reinterpret_cast<double*>(static_cast<char*>(workspace) +
                                    static_cast<size_t>(a.g.BH) * a.nchunk * 128 * prof_rec_floats(s->d) * sizeof(float));
  a.mse_out = mse_out;
  a.kind_out = head_kind_out;
  CUtensorMap mk, mv;
  if (!make_map(&mk, kn, s->d, s->L, a.g.BH, 64) || !make_map(&mv, v, s->d, s->L, a.g.BH, 64)) return SVG_ERR_CUDA;
  const dim3 grid(a.nchunk, a.g.BH), mgrid(n, a.g.BH);
  if (s->d == 128) {
    if (!set_smem(profile_tc_kernel<128>, ProfCfg<128>::SMEM_BYTES)) return SVG_ERR_CUDA;
    profile_tc_kernel<128><<<grid, ProfCfg<128>::THREADS, ProfCfg<128>::SMEM_BYTES, cs>>>(mk, mv, a);
    if (launch_status() != SVG_OK) return SVG_ERR_CUDA;
    profile_merge_kernel<128><<<mgrid, 128, 0, cs>>>(a);
  } else {
    if (!set_smem(profile_tc_kernel<64>, ProfCfg<64>::SMEM_BYTES)) return SVG_ERR_CUDA;
    profile_tc_kernel<64><<<grid, ProfCfg<64>::THREADS, ProfCfg<64>::SMEM_BYTES, cs>>>(mk, mv, a);
    if (launch_status() != SVG_OK) return SVG_ERR_CUDA;
    profile_merge_kernel<64><<<mgrid, 64, 0, cs>>>(a);
  }
  if (launch_status() != SVG_OK) return SVG_ERR_CUDA;
  profile_choose_kernel<<<(a.g.BH + 127) / 128, 128, 0, cs>>>(a, s->d);
  return launch_status();
}

// Self-test of the bounded wait: one warp waits on an mbarrier that nothing
// completes.  After the wait limit (about a second) mbar_wait records
// kErrTimeout in the error word and returns false; the kernel then returns.
__global__ void selftest_wait_kernel() {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_addr(&bar), 1);
    abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) (void)mbar_wait(smem_addr(&bar), 0, &abort_flag);
}

}  // namespace

// ===================================================================== ABI

extern "C" {

const char* svg_version(void) { return "svg-b200 0.1 (sm_100a)"; }

const char* svg_status_string(svg_status s) {
  switch (s) {
    case SVG_OK: return "ok";
    case SVG_ERR_INVALID_ARG: return "invalid argument";
    case SVG_ERR_SHAPE: return "inconsistent shape";
    case SVG_ERR_UNSUPPORTED: return "unsupported configuration";
    case SVG_ERR_ALIGNMENT: return "device pointer not 16-byte aligned";
    case SVG_ERR_CAPACITY: return "buffer too small";
    case SVG_ERR_CUDA: return "CUDA error";
    case SVG_ERR_TIMEOUT: return "kernel wait timed out";
  }
  return "unknown status";
}

svg_status svg_step_policy(int step, int total_steps, float dense_fraction, int reprofile_every, int* mode_out) {
  if (!mode_out || total_steps < 1 || step < 0 || step >= total_steps || !(dense_fraction >= 0.f) ||
      !(dense_fraction <= 1.f) || reprofile_every < 1)
    return SVG_ERR_INVALID_ARG;
  // dense iff step / total_steps < dense_fraction, decided in double
  const double cut = static_cast<double>(dense_fraction) * total_steps;
  if (static_cast<double>(step) < cut) {
    *mode_out = SVG_STEP_DENSE;
    return SVG_OK;
  }
  const int first_sparse = static_cast<int>(std::ceil(cut));
  *mode_out = ((step - first_sparse) % reprofile_every == 0) ? SVG_STEP_PROFILE : SVG_STEP_REUSE;
  return SVG_OK;
}

svg_status svg_sample_queries(uint64_t seed, int64_t Lv, int n, int32_t* host_out) {
  if (!host_out || n <= 0 || Lv <= 0 || n > Lv || Lv > INT32_MAX) return SVG_ERR_INVALID_ARG;
  // partial Fisher-Yates over 0..Lv-1; only the touched slots are remembered
  struct Slot { int64_t key, val; };
  const int cap = 4 * n + 8;
  Slot* tab = new Slot[cap];
  int used = 0;
  auto get = [&](int64_t key) -> int64_t {
    for (int i = 0; i < used; i++)
      if (tab[i].key == key) return tab[i].val;
    return key;
  };
  auto put = [&](int64_t key, int64_t val) {
    for (int i = 0; i < used; i++)
      if (tab[i].key == key) {
        tab[i].val = val;
        return;
      }
    tab[used].key = key;
    tab[used].val = val;
    used++;
  };
  uint64_t state = seed;
  for (int i = 0; i < n; i++) {
    state += 0x9E3779B97F4A7C15ull;            // SplitMix64 (Steele, Lea, Flood 2014)
    uint64_t z = state;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    z ^= z >> 31;
    const int64_t j = i + static_cast<int64_t>(z % static_cast<uint64_t>(Lv - i));
    const int64_t vi = get(i), vj = get(j);
    put(i, vj);
    put(j, vi);
    host_out[i] = static_cast<int32_t>(vj);
  }
  delete[] tab;
  return SVG_OK;
}

size_t svg_rope_table_size(const svg_shape* s, const svg_params* p) {
  if (!s || !p) return 0;
  return 2 * (static_cast<size_t>(s->F) * (p->rope_split[0] / 2) + static_cast<size_t>(s->Hs) * (p->rope_split[1] / 2) +
              static_cast<size_t>(s->Ws) * (p->rope_split[2] / 2));
}

svg_status svg_rope_table_fill(const svg_shape* s, const svg_params* p, float* host_out) {
  svg_status st = check_shape(s);
  if (st != SVG_OK) return st;
  if (!p || !host_out) return SVG_ERR_INVALID_ARG;
  if ((st = check_rope(s, p)) != SVG_OK) return st;
  const int npos[3] = {s->F, s->Hs, s->Ws};
  size_t o = 0;
  for (int a = 0; a < 3; a++) {
    const int n = p->rope_split[a];
    for (int pos = 0; pos < npos[a]; pos++) {
      for (int j = 0; j < n / 2; j++) {
        const double th = static_cast<double>(pos) * std::pow(static_cast<double>(p->rope_base), -2.0 * j / n);
        host_out[o++] = static_cast<float>(std::cos(th));
        host_out[o++] = static_cast<float>(std::sin(th));
      }
    }
  }
  return SVG_OK;
}

int64_t svg_block_index_capacity(const svg_shape* s, const svg_params* p) {
  if (check_shape(s) != SVG_OK || !p || p->block_q <= 0 || p->block_k <= 0) return -1;
  const int64_t nqb = (s->L + p->block_q - 1) / p->block_q, nkb = (s->L + p->block_k - 1) / p->block_k;
  return static_cast<int64_t>(s->B) * s->H * nqb * nkb;
}

size_t svg_profile_workspace_size(const svg_shape* s, int n) {
  if (check_shape(s) != SVG_OK || n <= 0) return 0;
  const int BH = s->B * s->H;
  return prof_workspace_bytes(BH, s->L, s->d, prof_chunks(BH, s->L));
}

size_t svg_workspace_size(const svg_shape* s, const svg_params* p) {
  if (check_shape(s) != SVG_OK || check_params(s, p, true) != SVG_OK) return 0;
  return svg_profile_workspace_size(s, kProfRows);
}

svg_status svg_selftest_wait_timeout(void* stream) {
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>();
  return launch_status();
}

svg_status svg_sync_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return SVG_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_error_word, sizeof(int)) != cudaSuccess) return SVG_ERR_CUDA;
  const int zero = 0;
  if (v && cudaMemcpyToSymbol(g_error_word, &zero, sizeof(int)) != cudaSuccess) return SVG_ERR_CUDA;
  if (v & kErrTimeout) return SVG_ERR_TIMEOUT;
  if (v & kErrCapacity) return SVG_ERR_CAPACITY;
  if (v & kErrBadIndex) return SVG_ERR_INVALID_ARG;
  return SVG_OK;
}

svg_status svg_qknorm_rope_layout(const svg_shape* s, const svg_params* p, int flags, const uint16_t* q,
                                  const uint16_t* k, const uint16_t* v, const float* gamma_q, const float* gamma_k,
                                  const float* rope_table, const uint8_t* head_kind, uint16_t* q_out,
                                  uint16_t* k_out, uint16_t* v_out, void* stream) {
  svg::NvtxRange nvtx_range_("svg_qknorm_rope_layout");
  svg_status st = check_shape(s);
  if (st != SVG_OK) return st;
  if (!p) return SVG_ERR_INVALID_ARG;
  if ((st = check_params(s, p, false)) != SVG_OK) return st;
  if (flags == 0 || (flags & ~(SVG_NORM_ROPE | SVG_LAYOUT))) return SVG_ERR_INVALID_ARG;
  const bool norm = (flags & SVG_NORM_ROPE) != 0, layout = (flags & SVG_LAYOUT) != 0;
  // each tensor is given with its output or not at all
  if (!q != !q_out || !k != !k_out || !v != !v_out || (!q && !k)) return SVG_ERR_INVALID_ARG;
  const bool norm_q = norm && q && gamma_q, norm_k = norm && k && gamma_k;
  if (norm) {
    if (!(norm_q || norm_k) || !rope_table) return SVG_ERR_INVALID_ARG;
    if ((st = check_rope(s, p)) != SVG_OK) return st;
  }
  if (layout) {
    if (!v || !head_kind) return SVG_ERR_INVALID_ARG;
  } else if (v || (q && !norm_q) || (k && !norm_k)) {
    return SVG_ERR_INVALID_ARG;       // without LAYOUT, every given tensor is normalised
  }
  const void* ptrs[] = {q, k, v, q_out, k_out, v_out, gamma_q, gamma_k, rope_table};
  for (const void* ptr : ptrs)
    if (ptr && !aligned16(ptr)) return SVG_ERR_ALIGNMENT;
  if ((q && q == q_out) || (k && k == k_out) || (v && v == v_out)) return SVG_ERR_INVALID_ARG;
  RowmapArgs a{};
  a.g = make_geometry(s, p);
  a.flags = flags & SVG_LAYOUT;
  // normalised tensors first, then the ones that only move
  auto add = [&](const uint16_t* src, uint16_t* dst, const float* gamma) {
    a.src[a.ntensor] = src;
    a.dst[a.ntensor] = dst;
    a.gamma[a.ntensor] = gamma;
    a.ntensor++;
  };
  if (norm_q) add(q, q_out, gamma_q);
  if (norm_k) add(k, k_out, gamma_k);
  a.norm_tensors = a.ntensor;
  if (q && !norm_q) add(q, q_out, nullptr);
  if (k && !norm_k) add(k, k_out, nullptr);
  if (v) add(v, v_out, nullptr);
  a.kind = head_kind;
  a.rope_floats = norm ? static_cast<int>(svg_rope_table_size(s, p)) : 0;
  a.rope = make_rope_args(s, p, norm ? rope_table : nullptr);
  return launch_rowmap(a, s->d, static_cast<cudaStream_t>(stream));
}

svg_status svg_inverse_layout(const svg_shape* s, const uint8_t* head_kind, const uint16_t* src, uint16_t* dst,
                              void* stream) {
  svg::NvtxRange nvtx_range_("svg_inverse_layout");
  svg_status st = check_shape(s);
  if (st != SVG_OK) return st;
  if (!head_kind || !src || !dst || src == dst) return SVG_ERR_INVALID_ARG;
  if (!aligned16(src) || !aligned16(dst)) return SVG_ERR_ALIGNMENT;
  RowmapArgs a{};
  a.g = make_geometry(s, nullptr);
  a.flags = kRowmapInverse;
  a.ntensor = 1;
  a.norm_tensors = 0;
  a.src[0] = src;
  a.dst[0] = dst;
  a.kind = head_kind;
  a.rope = make_rope_args(s, nullptr, nullptr);
  return launch_rowmap(a, s->d, static_cast<cudaStream_t>(stream));
}

svg_status svg_profile_heads(const svg_shape* s, const svg_params* p, const uint16_t* qn, const uint16_t* kn,
                             const uint16_t* v, const int32_t* sample_idx, int n, void* workspace,
                             size_t workspace_bytes, float* mse_out, uint8_t* head_kind_out, void* stream) {
  svg::NvtxRange nvtx_range_("svg_profile_heads");
  svg_status st = check_shape(s);
  if (st != SVG_OK) return st;
  if ((st = check_params(s, p, false)) != SVG_OK) return st;
  if (!qn || !kn || !v || !sample_idx || !workspace || !head_kind_out) return SVG_ERR_INVALID_ARG;
  if (n < 1 || n > kProfRows) return SVG_ERR_INVALID_ARG;
  const void* ptrs[] = {qn, kn, v, workspace, mse_out};
  for (const void* ptr : ptrs)
    if (ptr && !aligned16(ptr)) return SVG_ERR_ALIGNMENT;
  if (workspace_bytes < svg_profile_workspace_size(s, n)) return SVG_ERR_CAPACITY;
  return launch_profile(s, p, qn, kn, v, sample_idx, n, workspace, prof_chunks(s->B * s->H, s->L), mse_out,
                        head_kind_out, static_cast<cudaStream_t>(stream));
}

svg_status svg_profile_heads_raw_q(const svg_shape* s, const svg_params* p, const uint16_t* q, const float* gamma_q,
                                   const float* rope_table, const uint16_t* kn, const uint16_t* v,
                                   const int32_t* sample_idx, int n, void* workspace, size_t workspace_bytes,
                                   float* mse_out, uint8_t* head_kind_out, void* stream) {
  svg::NvtxRange nvtx_range_("svg_profile_heads_raw_q");
  svg_status st = check_shape(s);
  if (st != SVG_OK) return st;
  if ((st = check_params(s, p, false)) != SVG_OK) return st;
  if ((st = check_rope(s, p)) != SVG_OK) return st;
  if (!q || !gamma_q || !rope_table || !kn || !v || !sample_idx || !workspace || !head_kind_out)
    return SVG_ERR_INVALID_ARG;
  if (n < 1 || n > kProfRows) return SVG_ERR_INVALID_ARG;
  const void* ptrs[] = {q, gamma_q, rope_table, kn, v, workspace, mse_out};
  for (const void* ptr : ptrs)
    if (ptr && !aligned16(ptr)) return SVG_ERR_ALIGNMENT;
  if (workspace_bytes < svg_profile_workspace_size(s, n)) return SVG_ERR_CAPACITY;
  return launch_profile(s, p, q, kn, v, sample_idx, n, workspace, prof_chunks(s->B * s->H, s->L), mse_out,
                        head_kind_out, static_cast<cudaStream_t>(stream), gamma_q, rope_table);
}

svg_status svg_build_block_index(const svg_shape* s, const svg_params* p, const uint8_t* head_kind,
                                 int32_t* row_ptr, int32_t* col, uint8_t* full, int64_t capacity, void* stream) {
  svg::NvtxRange nvtx_range_("svg_build_block_index");
  svg_status st = check_shape(s);
  if (st != SVG_OK) return st;
  if ((st = check_params(s, p, true)) != SVG_OK) return st;
  if (!head_kind || !row_ptr || !col || !full || capacity < 0) return SVG_ERR_INVALID_ARG;
  const Geometry g = make_geometry(s, p);
  const int64_t n = static_cast<int64_t>(g.BH) * g.nqb;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  block_count_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, cs>>>(g, head_kind, row_ptr);
  if ((st = launch_status()) != SVG_OK) return st;
  block_scan_kernel<<<1, 1024, 0, cs>>>(row_ptr, n, capacity);
  if ((st = launch_status()) != SVG_OK) return st;
  block_fill_kernel<<<static_cast<unsigned>((n * 32 + 255) / 256), 256, 0, cs>>>(g, head_kind, row_ptr, col, full,
                                                                                capacity);
  return launch_status();
}

// Block-sparse attention; model_order = 1 also applies the inverse layout
// (temporal heads' rows are stored back in frame-major order).
// `cluster` (or null) carries the semantic-permutation mask fields (sel, qoff,
// koff, Cq, Ck, out_perm); head_kind is then unused.
static svg_status attention_launch(const svg_shape* s, const svg_params* p, const uint16_t* q, const uint16_t* k,
                                   const uint16_t* v, const uint8_t* head_kind, const int32_t* row_ptr,
                                   const int32_t* col, const uint8_t* full, uint16_t* out, float* lse_out,
                                   int model_order, void* stream, const AttnArgs* cluster = nullptr) {
  svg_status st = check_shape(s);
  if (st != SVG_OK) return st;
  if ((st = check_params(s, p, true)) != SVG_OK) return st;
  if (!q || !k || !v || (!head_kind && !cluster) || !row_ptr || !col || !full || !out) return SVG_ERR_INVALID_ARG;
  if (cluster && p->block_q != 128) return SVG_ERR_UNSUPPORTED;
  const void* ptrs[] = {q, k, v, out};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return SVG_ERR_ALIGNMENT;
  if (out == q || out == k || out == v) return SVG_ERR_INVALID_ARG;
  AttnArgs a{};
  a.g = make_geometry(s, p);
  a.scale_log2 = scale_of(s, p) * 1.4426950408889634f;
  a.kind = head_kind;
  a.row_ptr = row_ptr;
  a.col = col;
  a.full = full;
  a.out = out;
  a.lse = lse_out;
  a.model_order = model_order;
  if (cluster) {
    a.sel = cluster->sel;
    a.qoff = cluster->qoff;
    a.koff = cluster->koff;
    a.Cq = cluster->Cq;
    a.Ck = cluster->Ck;
    a.out_perm = cluster->out_perm;
  }
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, s->d, s->L, a.g.BH, 128) || !make_map(&mk, k, s->d, s->L, a.g.BH, 64) ||
      !make_map(&mv, v, s->d, s->L, a.g.BH, 64))
    return SVG_ERR_CUDA;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (a.g.bq == 128) {
    // two 128-row query tiles per CTA share every K/V tile
    const unsigned grid = static_cast<unsigned>(a.g.BH) * static_cast<unsigned>((a.g.nqb + 1) / 2);
    auto run = [&](auto kern, int threads, int smem) -> svg_status {
      if (!set_smem(kern, smem)) return SVG_ERR_CUDA;
      kern<<<grid, threads, smem, cs>>>(mq, mk, mv, a);
      return launch_status();
    };
    if (s->d == 128) {
      using C = Attn2Cfg<128>;
      return cluster ? run(attn2_kernel<128, true>, C::THREADS, C::SMEM_BYTES)
                     : run(attn2_kernel<128, false>, C::THREADS, C::SMEM_BYTES);
    }
    using C = Attn2Cfg<64>;
    return cluster ? run(attn2_kernel<64, true>, C::THREADS, C::SMEM_BYTES)
                   : run(attn2_kernel<64, false>, C::THREADS, C::SMEM_BYTES);
  }
  const unsigned grid = static_cast<unsigned>(a.g.BH) * static_cast<unsigned>(a.g.nqb);
  if (s->d == 128) {
    if (!set_smem(attn_kernel<128>, AttnCfg<128>::SMEM_BYTES)) return SVG_ERR_CUDA;
    attn_kernel<128><<<grid, AttnCfg<128>::THREADS, AttnCfg<128>::SMEM_BYTES, cs>>>(mq, mk, mv, a);
  } else {
    if (!set_smem(attn_kernel<64>, AttnCfg<64>::SMEM_BYTES)) return SVG_ERR_CUDA;
    attn_kernel<64><<<grid, AttnCfg<64>::THREADS, AttnCfg<64>::SMEM_BYTES, cs>>>(mq, mk, mv, a);
  }
  return launch_status();
}

svg_status svg_block_sparse_attn(const svg_shape* s, const svg_params* p, const uint16_t* q, const uint16_t* k,
                                 const uint16_t* v, const uint8_t* head_kind, const int32_t* row_ptr,
                                 const int32_t* col, const uint8_t* full, uint16_t* out, float* lse_out,
                                 void* stream) {
  svg::NvtxRange nvtx_range_("svg_block_sparse_attn");
  return attention_launch(s, p, q, k, v, head_kind, row_ptr, col, full, out, lse_out, 0, stream);
}

svg_status svg_block_sparse_attn_model_order(const svg_shape* s, const svg_params* p, const uint16_t* q,
                                             const uint16_t* k, const uint16_t* v, const uint8_t* head_kind,
                                             const int32_t* row_ptr, const int32_t* col, const uint8_t* full,
                                             uint16_t* out, float* lse_out, void* stream) {
  svg::NvtxRange nvtx_range_("svg_block_sparse_attn_model_order");
  return attention_launch(s, p, q, k, v, head_kind, row_ptr, col, full, out, lse_out, 1, stream);
}

svg_status svg_attention_step(const svg_shape* s, const svg_params* p, const uint16_t* q, const uint16_t* k,
                              const uint16_t* v, const float* gamma_q, const float* gamma_k, const float* rope_table,
                              const int32_t* sample_idx, int n, const uint8_t* head_kind_in, uint16_t* kn,
                              uint16_t* qp, uint16_t* kp, uint16_t* vp, uint16_t* op, uint16_t* out,
                              uint8_t* head_kind_out, float* mse_out, int32_t* row_ptr, int32_t* col, uint8_t* full,
                              int64_t capacity, void* workspace, size_t workspace_bytes, void* stream) {
  svg::NvtxRange nvtx_range_("svg_attention_step");
  svg_status st;
  if (!head_kind_out) return SVG_ERR_INVALID_ARG;
  // 1. QK-Norm + RoPE of K (profiling reads every normalised key)
  if ((st = svg_qknorm_rope_layout(s, p, SVG_NORM_ROPE, nullptr, k, nullptr, nullptr, gamma_k, rope_table, nullptr,
                                   nullptr, kn, nullptr, stream)) != SVG_OK)
    return st;
  // 2. profiling; the sampled Q rows are normalised inside the kernel, with the same routine
  const uint8_t* kinds = head_kind_in;
  if (!kinds) {
    if ((st = svg_profile_heads_raw_q(s, p, q, gamma_q, rope_table, kn, v, sample_idx, n, workspace, workspace_bytes,
                                      mse_out, head_kind_out, stream)) != SVG_OK)
      return st;
    kinds = head_kind_out;
  }
  // 3. block index
  if ((st = svg_build_block_index(s, p, kinds, row_ptr, col, full, capacity, stream)) != SVG_OK) return st;
  // 4. one pass: QK-Norm + RoPE of Q, and all three tensors into the heads' layouts
  if ((st = svg_qknorm_rope_layout(s, p, SVG_NORM_ROPE | SVG_LAYOUT, q, kn, v, gamma_q, nullptr, rope_table, kinds,
                                   qp, kp, vp, stream)) != SVG_OK)
    return st;
  // 5. attention, with the inverse layout in its epilogue unless the head-layout output is wanted
  if (!op)
    return svg_block_sparse_attn_model_order(s, p, qp, kp, vp, kinds, row_ptr, col, full, out, nullptr, stream);
  if ((st = svg_block_sparse_attn(s, p, qp, kp, vp, kinds, row_ptr, col, full, op, nullptr, stream)) != SVG_OK)
    return st;
  return svg_inverse_layout(s, kinds, op, out, stream);
}

// ------------------------------------------- semantic-aware permutation (SVG2)

size_t svg2_kmeans_workspace_size(const svg_shape* s, int C) {
  if (!s || C < 1) return 0;
  return static_cast<size_t>(s->B) * s->H * C * s->d * sizeof(unsigned long long);
}

svg_status svg2_kmeans(const svg_shape* s, const uint16_t* x, int C, int iters, int init, float* cent,
                       uint8_t* assign, int32_t* counts, void* workspace, size_t workspace_bytes, void* stream) {
  svg::NvtxRange nvtx_range_("svg2_kmeans");
  svg_status st = check_shape(s);
  if (st != SVG_OK) return st;
  const int Lv = s->F * s->Hs * s->Ws;
  if (!x || !cent || !assign || !counts || !workspace) return SVG_ERR_INVALID_ARG;
  if (C < 1 || C > kMaxClusters || C > Lv || iters < 0) return SVG_ERR_INVALID_ARG;
  const void* ptrs[] = {x, cent, workspace};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return SVG_ERR_ALIGNMENT;
  if (workspace_bytes < svg2_kmeans_workspace_size(s, C)) return SVG_ERR_CAPACITY;
  KmArgs a{};
  a.BH = s->B * s->H;
  a.L = s->L;
  a.Lv = Lv;
  a.C = C;
  a.x = x;
  a.cent = cent;
  a.assign = assign;
  a.counts = counts;
  a.sum = static_cast<unsigned long long*>(workspace);
  a.xmax = km_value_bound(Lv);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * a.BH * C, cs) != cudaSuccess) return SVG_ERR_CUDA;
  if (cudaMemsetAsync(workspace, 0, svg2_kmeans_workspace_size(s, C), cs) != cudaSuccess) return SVG_ERR_CUDA;
  const dim3 cgrid(C, a.BH), agrid((Lv + kKmAssignRows - 1) / kKmAssignRows, a.BH), sgrid((Lv + kKmUpdateRows - 1) / kKmUpdateRows, a.BH);
  const int asmem = km_assign_smem(C, s->d), ssmem = 3 * C * s->d * 4;
  auto run = [&](auto D_) -> svg_status {
    constexpr int D = decltype(D_)::value;
    if (!set_smem(km_assign_kernel<D>, asmem) || !set_smem(km_sum_kernel<D>, ssmem)) return SVG_ERR_CUDA;
    if (init) km_init_kernel<D><<<cgrid, D, 0, cs>>>(a);
    for (int t = 0; t < iters; t++) {
      km_assign_kernel<D><<<agrid, kKmAssignThreads, asmem, cs>>>(a);
      km_sum_kernel<D><<<sgrid, 256, ssmem, cs>>>(a);
      km_mean_kernel<D><<<cgrid, D, 0, cs>>>(a);
    }
    km_assign_kernel<D><<<agrid, kKmAssignThreads, asmem, cs>>>(a);
    return launch_status();
  };
  return s->d == 128 ? run(std::integral_constant<int, 128>{}) : run(std::integral_constant<int, 64>{});
}

svg_status svg2_permutation(const svg_shape* s, const uint8_t* assign, int C, int32_t* perm, int32_t* off,
                            void* stream) {
  svg::NvtxRange nvtx_range_("svg2_permutation");
  svg_status st = check_shape(s);
  if (st != SVG_OK) return st;
  if (!assign || !perm || !off || C < 1 || C > kMaxClusters) return SVG_ERR_INVALID_ARG;
  const int Lv = s->F * s->Hs * s->Ws;
  km_perm_kernel<<<s->B * s->H, 1024, 0, static_cast<cudaStream_t>(stream)>>>(assign, Lv, C, perm, off);
  return launch_status();
}

svg_status svg2_select(const svg_shape* s, const svg_params* p, const float* cq, const float* ck,
                       const int32_t* counts_k, int Cq, int Ck, double top_p, uint64_t* sel, void* stream) {
  svg::NvtxRange nvtx_range_("svg2_select");
  svg_status st = check_shape(s);
  if (st != SVG_OK) return st;
  if ((st = check_params(s, p, false)) != SVG_OK) return st;
  if (!cq || !ck || !counts_k || !sel) return SVG_ERR_INVALID_ARG;
  if (Cq < 1 || Cq > kMaxClusters || Ck < 1 || Ck > kMaxClusters) return SVG_ERR_INVALID_ARG;
  if (!(top_p > 0.0) || !(top_p <= 1.0)) return SVG_ERR_INVALID_ARG;
  const double scale = p->softmax_scale > 0.f ? static_cast<double>(p->softmax_scale) : 1.0 / std::sqrt(static_cast<double>(s->d));
  km_select_kernel<<<dim3(Cq, s->B * s->H), 64, 0, static_cast<cudaStream_t>(stream)>>>(cq, ck, counts_k, Cq, Ck,
                                                                                        s->d, scale, top_p, sel);
  return launch_status();
}

svg_status svg2_permute(const svg_shape* s, const int32_t* perm_q, const int32_t* perm_k, const uint16_t* q,
                        const uint16_t* k, const uint16_t* v, uint16_t* q_out, uint16_t* k_out, uint16_t* v_out,
                        void* stream) {
  svg::NvtxRange nvtx_range_("svg2_permute");
  svg_status st = check_shape(s);
  if (st != SVG_OK) return st;
  if (!perm_q || !perm_k || !q || !k || !v || !q_out || !k_out || !v_out) return SVG_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, q_out, k_out, v_out};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return SVG_ERR_ALIGNMENT;
  if (q == q_out || k == k_out || v == v_out) return SVG_ERR_INVALID_ARG;
  KmGatherArgs a{};
  a.BH = s->B * s->H;
  a.L = s->L;
  a.Lv = s->F * s->Hs * s->Ws;
  a.divL = make_fastdiv(s->L);
  const uint16_t* src[3] = {q, k, v};
  uint16_t* dst[3] = {q_out, k_out, v_out};
  const int32_t* pi[3] = {perm_q, perm_k, perm_k};
  for (int t = 0; t < 3; t++) {
    a.src[t] = src[t];
    a.dst[t] = dst[t];
    a.perm[t] = pi[t];
  }
  const int64_t units = static_cast<int64_t>(a.BH) * a.L * (s->d / 8);
  const int64_t per_block = 256LL * kKmGatherU;
  const unsigned blocks = static_cast<unsigned>(std::min<int64_t>((units + per_block - 1) / per_block, 148LL * 8));
  const dim3 grid(blocks, 3);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (s->d == 128) km_gather_kernel<128><<<grid, 256, 0, cs>>>(a);
  else km_gather_kernel<64><<<grid, 256, 0, cs>>>(a);
  return launch_status();
}

svg_status svg2_build_block_index(const svg_shape* s, const svg_params* p, int Cq, int Ck, const int32_t* qoff,
                                  const int32_t* koff, const uint64_t* sel, int32_t* row_ptr, int32_t* col,
                                  uint8_t* full, int64_t capacity, void* stream) {
  svg::NvtxRange nvtx_range_("svg2_build_block_index");
  svg_status st = check_shape(s);
  if (st != SVG_OK) return st;
  if ((st = check_params(s, p, true)) != SVG_OK) return st;
  if (!qoff || !koff || !sel || !row_ptr || !col || !full || capacity < 0) return SVG_ERR_INVALID_ARG;
  if (Cq < 1 || Cq > kMaxClusters || Ck < 1 || Ck > kMaxClusters) return SVG_ERR_INVALID_ARG;
  const Geometry g0 = make_geometry(s, p);
  Km2Geom g{};
  g.BH = g0.BH;
  g.L = g0.L;
  g.Lv = g0.Lv;
  g.bq = g0.bq;
  g.bk = g0.bk;
  g.nqb = g0.nqb;
  g.nkb = g0.nkb;
  g.Cq = Cq;
  g.Ck = Ck;
  g.qoff = qoff;
  g.koff = koff;
  g.sel = sel;
  const int64_t n = static_cast<int64_t>(g.BH) * g.nqb;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const unsigned blocks = static_cast<unsigned>((n * 32 + 255) / 256);   // one warp per query tile
  km2_list_kernel<false><<<blocks, 256, 0, cs>>>(g, row_ptr, col, full, capacity);
  if ((st = launch_status()) != SVG_OK) return st;
  block_scan_kernel<<<1, 1024, 0, cs>>>(row_ptr, n, capacity);
  if ((st = launch_status()) != SVG_OK) return st;
  km2_list_kernel<true><<<blocks, 256, 0, cs>>>(g, row_ptr, col, full, capacity);
  return launch_status();
}

svg_status svg2_attention(const svg_shape* s, const svg_params* p, const uint16_t* q, const uint16_t* k,
                          const uint16_t* v, int Cq, int Ck, const int32_t* qoff, const int32_t* koff,
                          const uint64_t* sel, const int32_t* perm_q, const int32_t* row_ptr, const int32_t* col,
                          const uint8_t* full, uint16_t* out, float* lse_out, void* stream) {
  svg::NvtxRange nvtx_range_("svg2_attention");
  if (!qoff || !koff || !sel || !perm_q) return SVG_ERR_INVALID_ARG;
  if (Cq < 1 || Cq > kMaxClusters || Ck < 1 || Ck > kMaxClusters) return SVG_ERR_INVALID_ARG;
  AttnArgs c{};
  c.sel = sel;
  c.qoff = qoff;
  c.koff = koff;
  c.Cq = Cq;
  c.Ck = Ck;
  c.out_perm = perm_q;
  return attention_launch(s, p, q, k, v, nullptr, row_ptr, col, full, out, lse_out, 0, stream, &c);
}

// ------------------------------------------------ AdaSpa blockified search

svg_status svg_adaspa_block_mass(const svg_shape* s, const svg_params* p, const uint16_t* q, const uint16_t* k,
                                 const float* lse, float* mass, void* stream) {
  svg::NvtxRange nvtx_range_("svg_adaspa_block_mass");
  svg_status st = check_shape(s);
  if (st != SVG_OK) return st;
  if ((st = check_params(s, p, true)) != SVG_OK) return st;
  if (!q || !k || !lse || !mass) return SVG_ERR_INVALID_ARG;
  if (p->block_q != 128 || p->block_k != 64) return SVG_ERR_UNSUPPORTED;
  const void* ptrs[] = {q, k};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return SVG_ERR_ALIGNMENT;
  MassArgs a{};
  a.g = make_geometry(s, p);
  a.scale_log2 = scale_of(s, p) * 1.4426950408889634f;
  a.lse = lse;
  a.mass = mass;
  CUtensorMap mq, mk;
  if (!make_map(&mq, q, s->d, s->L, a.g.BH, 128) || !make_map(&mk, k, s->d, s->L, a.g.BH, 64)) return SVG_ERR_CUDA;
  constexpr int NG = kMassGroups;
  const unsigned grid = static_cast<unsigned>(a.g.BH) * static_cast<unsigned>((a.g.nqb + NG - 1) / NG);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  auto run = [&](auto kern, int threads, int smem) -> svg_status {
    if (!set_smem(kern, smem)) return SVG_ERR_CUDA;
    kern<<<grid, threads, smem, cs>>>(mq, mk, a);
    return launch_status();
  };
  if (s->d == 128) return run(mass_kernel<128, NG>, MassCfg<128, NG>::THREADS, MassCfg<128, NG>::SMEM_BYTES);
  return run(mass_kernel<64, NG>, MassCfg<64, NG>::THREADS, MassCfg<64, NG>::SMEM_BYTES);
}

svg_status svg_adaspa_select(const svg_shape* s, const svg_params* p, const float* mass, double top_p,
                             int32_t* row_ptr, int32_t* col, uint8_t* full, int64_t capacity, void* stream) {
  svg::NvtxRange nvtx_range_("svg_adaspa_select");
  svg_status st = check_shape(s);
  if (st != SVG_OK) return st;
  if ((st = check_params(s, p, true)) != SVG_OK) return st;
  if (!mass || !row_ptr || !col || !full || capacity < 0) return SVG_ERR_INVALID_ARG;
  if (!(top_p > 0.0) || !(top_p <= 1.0)) return SVG_ERR_INVALID_ARG;
  SelArgs a{};
  a.g = make_geometry(s, p);
  a.p = top_p;
  a.mass = mass;
  if (a.g.nkb > kSelMaxTiles) return SVG_ERR_UNSUPPORTED;
  int P2 = 64;                                   // the sort works on 64-position segments
  while (P2 < a.g.nkb) P2 <<= 1;
  const int smem = P2 * 9;
  const int64_t n = static_cast<int64_t>(a.g.BH) * a.g.nqb;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  // with room for every tile's flags, `full` keeps them between the passes (no second sort)
  const bool room = capacity >= n * a.g.nkb;
  uint8_t* stash = room ? full : nullptr;
  select_kernel<false><<<static_cast<unsigned>(n), kSelThreads, smem, cs>>>(a, row_ptr, col, full, capacity, P2,
                                                                            stash);
  if ((st = launch_status()) != SVG_OK) return st;
  block_scan_kernel<<<1, 1024, 0, cs>>>(row_ptr, n, capacity);
  if ((st = launch_status()) != SVG_OK) return st;
  select_kernel<true><<<static_cast<unsigned>(n), kSelThreads, smem, cs>>>(a, row_ptr, col, full, capacity, P2,
                                                                           stash);
  if ((st = launch_status()) != SVG_OK) return st;
  if (room && cudaMemsetAsync(full, 1, static_cast<size_t>(capacity), cs) != cudaSuccess) return SVG_ERR_CUDA;
  return SVG_OK;
}

}  // extern "C"

// Profiling with library-owned scratch (svg_profile_heads_noalloc).
#include "profile_noalloc.cuh"
// The step on host buffers, copies overlapped with the passes (svg_attention_step_host).
#include "host_step.cuh"
