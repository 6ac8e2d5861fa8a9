// profile_noalloc.cuh — svg_profile_heads_noalloc: the profiling stage with
// its scratch in a fixed device array owned by the library, for callers that
// can hand over only input and output buffers.  Included at the end of
// svg_lib.cu (same translation unit as the kernels it launches).
#pragma once

#include <mutex>

#include "profile_tc.cuh"
#include "svg_common.cuh"

namespace svg {

// Size of the fixed scratch.  Every GPU that loads the library holds this
// array until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;   // 16 MiB

// The scratch itself.  In host code this name is only a host-side stand-in,
// never a device address: the device address comes from
// cudaGetSymbolAddress (see noalloc_scratch below).
static __device__ __align__(256) float g_profile_scratch[kNoAllocScratchBytes / sizeof(float)];

// Device address of g_profile_scratch on the current device, looked up once
// per device (with that device current) and cached.
inline svg_status noalloc_scratch(float** out) {
  static std::mutex mu;
  static float* cache[256] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256) return SVG_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_profile_scratch) != cudaSuccess || !p) return SVG_ERR_CUDA;
    cache[dev] = static_cast<float*>(p);
  }
  *out = cache[dev];
  return SVG_OK;
}

}  // namespace svg

extern "C" svg_status svg_profile_heads_noalloc(const svg_shape* s, const svg_params* p, const uint16_t* qn,
                                                const uint16_t* kn, const uint16_t* v, const int32_t* sample_idx,
                                                int n, float* mse_out, uint8_t* head_kind_out, void* stream) {
  svg::NvtxRange nvtx_range_("svg_profile_heads_noalloc");
  using namespace svg;
  svg_status st = check_shape(s);
  if (st != SVG_OK) return st;
  if ((st = check_params(s, p, false)) != SVG_OK) return st;
  if (!qn || !kn || !v || !sample_idx || !head_kind_out) return SVG_ERR_INVALID_ARG;
  if (n < 1 || n > kProfRows) return SVG_ERR_INVALID_ARG;
  const void* ptrs[] = {qn, kn, v, mse_out};
  for (const void* ptr : ptrs)
    if (ptr && !aligned16(ptr)) return SVG_ERR_ALIGNMENT;
  const int BH = s->B * s->H;
  // bytes of one key chunk of partial records for every head, plus the per-row error sums
  const size_t per_chunk = static_cast<size_t>(BH) * 128 * prof_rec_floats(s->d) * sizeof(float);
  const size_t fixed = static_cast<size_t>(BH) * kProfRows * 2 * sizeof(double);
  if (fixed + per_chunk > kNoAllocScratchBytes) return SVG_ERR_CAPACITY;   // launches nothing
  const size_t fit = (kNoAllocScratchBytes - fixed) / per_chunk;
  float* scratch = nullptr;
  if ((st = noalloc_scratch(&scratch)) != SVG_OK) return st;
  const int nchunk = static_cast<int>(fit < static_cast<size_t>(prof_chunks(BH, s->L)) ? fit : prof_chunks(BH, s->L));
  return launch_profile(s, p, qn, kn, v, sample_idx, n, scratch, nchunk, mse_out, head_kind_out,
                        static_cast<cudaStream_t>(stream));
}
