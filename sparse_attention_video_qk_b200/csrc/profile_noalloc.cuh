// profile_noalloc.cuh — svg_profile_heads_noalloc: the profiling stage with
// its scratch in a fixed device array owned by the library, for callers that
// can hand over only input and output buffers.  Included at the end of
// svg_lib.cu (same translation unit as the kernels it launches).
#pragma once

#include <mutex>

#include "profile.cuh"
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
  // bytes of one key chunk of partial records for every head
  const size_t per_chunk = static_cast<size_t>(BH) * kProfRows * prof_rec_floats(s->d) * sizeof(float);
  const size_t fit = kNoAllocScratchBytes / per_chunk;
  if (fit < 1) return SVG_ERR_CAPACITY;   // B*H*64*(4+3d)*4 bytes exceed the fixed scratch
  float* scratch = nullptr;
  if ((st = noalloc_scratch(&scratch)) != SVG_OK) return st;

  ProfArgs a{};
  a.g = make_geometry(s, p);
  a.scale_log2 = scale_of(s, p) * 1.4426950408889634f;
  a.q = qn;
  a.k = kn;
  a.v = v;
  a.sample = sample_idx;
  a.n = n;
  const int ntiles = (a.g.L + kProfKeys - 1) / kProfKeys;
  int nchunk = prof_chunks(BH, a.g.L);
  if (static_cast<size_t>(nchunk) > fit) nchunk = static_cast<int>(fit);
  a.tiles_per_chunk = (ntiles + nchunk - 1) / nchunk;
  a.nchunk = (ntiles + a.tiles_per_chunk - 1) / a.tiles_per_chunk;   // every chunk non-empty
  a.ws = scratch;
  a.mse_out = mse_out;
  a.kind_out = head_kind_out;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  dim3 grid(a.nchunk, BH);
  if (s->d == 128) {
    if (!set_smem(profile_partial_kernel<128>, ProfSmem<128>::BYTES)) return SVG_ERR_CUDA;
    profile_partial_kernel<128><<<grid, kProfThreads, ProfSmem<128>::BYTES, cs>>>(a);
    if ((st = launch_status()) != SVG_OK) return st;
    profile_combine_kernel<128><<<BH, 256, 0, cs>>>(a);
  } else {
    if (!set_smem(profile_partial_kernel<64>, ProfSmem<64>::BYTES)) return SVG_ERR_CUDA;
    profile_partial_kernel<64><<<grid, kProfThreads, ProfSmem<64>::BYTES, cs>>>(a);
    if ((st = launch_status()) != SVG_OK) return st;
    profile_combine_kernel<64><<<BH, 256, 0, cs>>>(a);
  }
  return launch_status();
}
