// host_step.cuh — svg_attention_step_host: the whole attention step on host
// buffers, with the host->device copies of the inputs and the device->host
// copy of the output overlapped with the passes.  The B*H heads are split into
// head groups: group g+1 is copied in (one stream) while group g runs the five
// passes of svg_attention_step (a second stream), and each group's output is
// copied out (a third stream) while the next group runs.  Every stage is per
// head, so the result is that of the one-shot step.  The three streams and
// their events belong to the library (one set per device, created on first
// use); the device buffers are the caller's workspace.  Included at the end of
// svg_lib.cu.
#pragma once

#include <mutex>
#include <vector>

#include "svg_common.cuh"

namespace svg {
namespace hoststep {

inline size_t up256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Head group g of `groups` over BH heads: sizes differ by at most one, the
// larger groups first.
inline int group_size(int BH, int groups, int g) { return BH / groups + (g < BH % groups ? 1 : 0); }
inline int group_start(int BH, int groups, int g) { return g * (BH / groups) + (g < BH % groups ? g : BH % groups); }

// Byte offsets of the workspace's buffers.
struct Layout {
  size_t q, k, v, out, kinds, gamma_q, gamma_k, sample, table;  // whole problem
  size_t kn, qp, kp, vp, row_ptr, col, full, prof;                    // one head group (the largest)
  size_t total;
  int64_t capacity;
  size_t prof_bytes, table_floats;
};

inline svg_shape group_shape(const svg_shape* s, int heads) {
  svg_shape g = *s;
  g.B = 1;
  g.H = heads;
  return g;
}

inline bool layout_of(const svg_shape* s, const svg_params* p, int n, int groups, Layout* L) {
  const int BH = s->B * s->H;
  const int gmax = group_size(BH, groups, 0);
  const size_t head_bytes = static_cast<size_t>(s->L) * s->d * 2;
  const svg_shape gs = group_shape(s, gmax);
  L->capacity = svg_block_index_capacity(&gs, p);
  if (L->capacity <= 0) return false;
  // the profiling scratch depends on the head count (key chunks per head):
  // the larger of the two group sizes' needs
  const svg_shape gsmall = group_shape(s, BH / groups);
  L->prof_bytes = std::max(svg_profile_workspace_size(&gs, n), svg_profile_workspace_size(&gsmall, n));
  L->table_floats = svg_rope_table_size(s, p);
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o += up256(bytes);
    return at;
  };
  L->q = take(BH * head_bytes);
  L->k = take(BH * head_bytes);
  L->v = take(BH * head_bytes);
  L->out = take(BH * head_bytes);
  L->kinds = take(static_cast<size_t>(BH));
  L->gamma_q = take(static_cast<size_t>(s->d) * sizeof(float));
  L->gamma_k = take(static_cast<size_t>(s->d) * sizeof(float));
  L->sample = take(static_cast<size_t>(n) * sizeof(int32_t));
  L->table = take(L->table_floats * sizeof(float));
  L->kn = take(gmax * head_bytes);
  L->qp = take(gmax * head_bytes);
  L->kp = take(gmax * head_bytes);
  L->vp = take(gmax * head_bytes);
  L->row_ptr = take((static_cast<size_t>(gmax) * ((s->L + p->block_q - 1) / p->block_q) + 1) * sizeof(int32_t));
  L->col = take(static_cast<size_t>(L->capacity) * sizeof(int32_t));
  L->full = take(static_cast<size_t>(L->capacity));
  L->prof = take(std::max<size_t>(L->prof_bytes, 16));
  L->total = o;
  return true;
}

// The library's streams and events of one device.
struct DeviceStreams {
  std::mutex mu;
  bool ready = false;
  cudaStream_t in = nullptr, comp = nullptr, out = nullptr;
  std::vector<cudaEvent_t> events;
  float* table_stage = nullptr;      // pinned host staging of the RoPE table
  size_t table_stage_floats = 0;
  cudaEvent_t table_copied = nullptr;
  bool table_pending = false;
};

constexpr int kMaxDevices = 64;

inline DeviceStreams* device_streams(int dev) {
  static DeviceStreams all[kMaxDevices];
  return (dev >= 0 && dev < kMaxDevices) ? &all[dev] : nullptr;
}

// Streams and events exist once per device; `need` events are available
// afterwards.  Called with ds->mu held.
inline bool ensure(DeviceStreams* ds, size_t need) {
  if (!ds->ready) {
    if (cudaStreamCreateWithFlags(&ds->in, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&ds->comp, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&ds->out, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&ds->table_copied, cudaEventDisableTiming) != cudaSuccess)
      return false;
    ds->ready = true;
  }
  while (ds->events.size() < need) {
    cudaEvent_t e;
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return false;
    ds->events.push_back(e);
  }
  return true;
}

// Waits for one device's library streams, then frees its streams, events and
// pinned staging.  Called with ds->mu held.
inline bool release(DeviceStreams* ds, int dev) {
  if (!ds->ready && ds->events.empty() && ds->table_stage == nullptr) return true;
  bool good = cudaSetDevice(dev) == cudaSuccess;
  for (cudaStream_t st : {ds->in, ds->comp, ds->out})
    if (st) good &= cudaStreamSynchronize(st) == cudaSuccess;
  for (cudaEvent_t e : ds->events) good &= cudaEventDestroy(e) == cudaSuccess;
  ds->events.clear();
  if (ds->table_copied) good &= cudaEventDestroy(ds->table_copied) == cudaSuccess;
  for (cudaStream_t st : {ds->in, ds->comp, ds->out})
    if (st) good &= cudaStreamDestroy(st) == cudaSuccess;
  if (ds->table_stage) good &= cudaFreeHost(ds->table_stage) == cudaSuccess;
  ds->in = ds->comp = ds->out = nullptr;
  ds->table_copied = nullptr;
  ds->table_stage = nullptr;
  ds->table_stage_floats = 0;
  ds->table_pending = false;
  ds->ready = false;
  return good;
}

}  // namespace hoststep
}  // namespace svg

extern "C" svg_status svg_release(void) {
  using namespace svg;
  int prev = -1;
  bool touched = false, good = true;
  for (int dev = 0; dev < hoststep::kMaxDevices; dev++) {
    hoststep::DeviceStreams* ds = hoststep::device_streams(dev);
    std::lock_guard<std::mutex> lock(ds->mu);
    if (!ds->ready && ds->events.empty() && ds->table_stage == nullptr) continue;
    if (!touched) {
      touched = true;
      good &= cudaGetDevice(&prev) == cudaSuccess;
    }
    good &= hoststep::release(ds, dev);
  }
  if (touched && prev >= 0) good &= cudaSetDevice(prev) == cudaSuccess;
  return good ? SVG_OK : SVG_ERR_CUDA;
}

extern "C" size_t svg_attention_step_host_workspace_size(const svg_shape* s, const svg_params* p, int n,
                                                          int groups) {
  using namespace svg;
  if (check_shape(s) != SVG_OK || check_params(s, p, true) != SVG_OK || n < 1 || groups < 1 ||
      groups > s->B * s->H)
    return 0;
  hoststep::Layout L;
  if (!hoststep::layout_of(s, p, n, groups, &L)) return 0;
  return L.total;
}

extern "C" svg_status svg_attention_step_host(const svg_shape* s, const svg_params* p, const uint16_t* q_host,
                                              const uint16_t* k_host, const uint16_t* v_host,
                                              const float* gamma_q_host, const float* gamma_k_host,
                                              const int32_t* sample_idx_host, int n, uint16_t* out_host,
                                              uint8_t* head_kind_out_host, int groups, void* workspace,
                                              size_t workspace_bytes, void* stream) {
  svg::NvtxRange nvtx_range_("svg_attention_step_host");
  using namespace svg;
  svg_status st = check_shape(s);
  if (st != SVG_OK) return st;
  if ((st = check_params(s, p, true)) != SVG_OK) return st;
  if ((st = check_rope(s, p)) != SVG_OK) return st;
  if (!q_host || !k_host || !v_host || !gamma_q_host || !gamma_k_host || !sample_idx_host || !out_host || !workspace)
    return SVG_ERR_INVALID_ARG;
  const int BH = s->B * s->H;
  if (n < 1 || n > kProfRows || groups < 1 || groups > BH) return SVG_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return SVG_ERR_ALIGNMENT;
  hoststep::Layout L;
  if (!hoststep::layout_of(s, p, n, groups, &L)) return SVG_ERR_INVALID_ARG;
  if (workspace_bytes < L.total) return SVG_ERR_CAPACITY;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SVG_ERR_CUDA;
  hoststep::DeviceStreams* ds = hoststep::device_streams(dev);
  if (!ds) return SVG_ERR_UNSUPPORTED;

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  auto at = [&](size_t off) { return ws + off; };
  uint16_t* q = reinterpret_cast<uint16_t*>(at(L.q));
  uint16_t* k = reinterpret_cast<uint16_t*>(at(L.k));
  uint16_t* v = reinterpret_cast<uint16_t*>(at(L.v));
  uint16_t* out = reinterpret_cast<uint16_t*>(at(L.out));
  uint8_t* kinds = at(L.kinds);
  float* gq = reinterpret_cast<float*>(at(L.gamma_q));
  float* gk = reinterpret_cast<float*>(at(L.gamma_k));
  int32_t* sample = reinterpret_cast<int32_t*>(at(L.sample));
  float* table = reinterpret_cast<float*>(at(L.table));
  const size_t head_elems = static_cast<size_t>(s->L) * s->d;
  cudaStream_t caller = static_cast<cudaStream_t>(stream);

  std::lock_guard<std::mutex> lock(ds->mu);
  const size_t nev = 2 + 2 * static_cast<size_t>(groups);
  if (!hoststep::ensure(ds, nev)) return SVG_ERR_CUDA;
  cudaEvent_t ev_start = ds->events[0], ev_end = ds->events[1];
  auto ev_in = [&](int g) { return ds->events[2 + 2 * g]; };
  auto ev_done = [&](int g) { return ds->events[3 + 2 * g]; };
  auto ok = [](cudaError_t e) { return e == cudaSuccess; };

  // The RoPE table is built on the host into a pinned staging buffer; the
  // previous call's copy out of it must have run before it is rewritten.
  if (ds->table_pending && !ok(cudaEventSynchronize(ds->table_copied))) return SVG_ERR_CUDA;
  ds->table_pending = false;
  if (ds->table_stage_floats < L.table_floats) {
    if (ds->table_stage && !ok(cudaFreeHost(ds->table_stage))) return SVG_ERR_CUDA;
    ds->table_stage = nullptr;
    ds->table_stage_floats = 0;
    if (!ok(cudaMallocHost(reinterpret_cast<void**>(&ds->table_stage), L.table_floats * sizeof(float))))
      return SVG_ERR_CUDA;
    ds->table_stage_floats = L.table_floats;
  }
  if ((st = svg_rope_table_fill(s, p, ds->table_stage)) != SVG_OK) return st;

  // everything starts after the caller's earlier work on its stream
  if (!ok(cudaEventRecord(ev_start, caller)) || !ok(cudaStreamWaitEvent(ds->in, ev_start, 0)) ||
      !ok(cudaStreamWaitEvent(ds->comp, ev_start, 0)) || !ok(cudaStreamWaitEvent(ds->out, ev_start, 0)))
    return SVG_ERR_CUDA;
  const size_t dsz = static_cast<size_t>(s->d) * sizeof(float);
  if (!ok(cudaMemcpyAsync(gq, gamma_q_host, dsz, cudaMemcpyHostToDevice, ds->in)) ||
      !ok(cudaMemcpyAsync(gk, gamma_k_host, dsz, cudaMemcpyHostToDevice, ds->in)) ||
      !ok(cudaMemcpyAsync(sample, sample_idx_host, static_cast<size_t>(n) * sizeof(int32_t), cudaMemcpyHostToDevice,
                          ds->in)) ||
      !ok(cudaMemcpyAsync(table, ds->table_stage, L.table_floats * sizeof(float), cudaMemcpyHostToDevice, ds->in)) ||
      !ok(cudaEventRecord(ds->table_copied, ds->in)))
    return SVG_ERR_CUDA;
  ds->table_pending = true;
  // inputs, group by group
  for (int g = 0; g < groups; g++) {
    const size_t h0 = hoststep::group_start(BH, groups, g), nh = hoststep::group_size(BH, groups, g);
    const size_t off = h0 * head_elems, bytes = nh * head_elems * 2;
    if (!ok(cudaMemcpyAsync(q + off, q_host + off, bytes, cudaMemcpyHostToDevice, ds->in)) ||
        !ok(cudaMemcpyAsync(k + off, k_host + off, bytes, cudaMemcpyHostToDevice, ds->in)) ||
        !ok(cudaMemcpyAsync(v + off, v_host + off, bytes, cudaMemcpyHostToDevice, ds->in)) ||
        !ok(cudaEventRecord(ev_in(g), ds->in)))
      return SVG_ERR_CUDA;
  }
  // the five passes per group, each group's output copied out behind it
  for (int g = 0; g < groups; g++) {
    const int h0 = hoststep::group_start(BH, groups, g), nh = hoststep::group_size(BH, groups, g);
    const size_t off = static_cast<size_t>(h0) * head_elems;
    const svg_shape gs = hoststep::group_shape(s, nh);
    if (!ok(cudaStreamWaitEvent(ds->comp, ev_in(g), 0))) return SVG_ERR_CUDA;
    st = svg_attention_step(&gs, p, q + off, k + off, v + off, gq, gk, table, sample, n, nullptr,
                            reinterpret_cast<uint16_t*>(at(L.kn)), reinterpret_cast<uint16_t*>(at(L.qp)),
                            reinterpret_cast<uint16_t*>(at(L.kp)), reinterpret_cast<uint16_t*>(at(L.vp)), nullptr,
                            out + off, kinds + h0, nullptr,
                            reinterpret_cast<int32_t*>(at(L.row_ptr)), reinterpret_cast<int32_t*>(at(L.col)),
                            at(L.full), L.capacity, at(L.prof), L.prof_bytes, ds->comp);
    if (st != SVG_OK) return st;
    if (!ok(cudaEventRecord(ev_done(g), ds->comp)) || !ok(cudaStreamWaitEvent(ds->out, ev_done(g), 0)) ||
        !ok(cudaMemcpyAsync(out_host + off, out + off, static_cast<size_t>(nh) * head_elems * 2,
                            cudaMemcpyDeviceToHost, ds->out)))
      return SVG_ERR_CUDA;
  }
  if (head_kind_out_host &&
      !ok(cudaMemcpyAsync(head_kind_out_host, kinds, static_cast<size_t>(BH), cudaMemcpyDeviceToHost, ds->out)))
    return SVG_ERR_CUDA;
  // the caller's stream resumes once the last copy is done
  if (!ok(cudaEventRecord(ev_end, ds->out)) || !ok(cudaStreamWaitEvent(caller, ev_end, 0))) return SVG_ERR_CUDA;
  return SVG_OK;
}
