// C ABI of libmla.so (declared in include/mla.h): argument checks, per-device
// state (workspace, error word, SM count), and the launch sequence of each call.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "mla.h"
#include "mla_internal.h"

namespace {

using namespace mla;

// One error word per device: a file-scope device variable, so it exists as soon
// as the library is loaded on a device and needs no allocation.
__device__ int g_device_error;

constexpr int kMaxDevices = 64;

struct DeviceState {
  bool init = false;
  int sm_count = 0;
  int* err = nullptr;           // device address of g_device_error
  void* ws = nullptr;           // workspace base
  size_t ws_bytes = 0;
  bool ws_external = false;     // set by mla_set_workspace
  // timing
  std::vector<cudaEvent_t> events;  // 4 per recorded call
  int timed_calls = 0;
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];
std::atomic<int> g_knobs[8];
std::atomic<int> g_timing{0};
thread_local char g_msg[512] = "";

mla_status_t fail(mla_status_t s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof g_msg, fmt, ap);
  va_end(ap);
  return s;
}

mla_status_t cuda_fail(cudaError_t e, const char* what) {
  return fail(MLA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Current device's state, initialised on first use (must hold g_mu).
mla_status_t device_state(DeviceState** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(MLA_ERR_UNSUPPORTED, "device ordinal %d", dev);
  DeviceState& d = g_dev[dev];
  if (!d.init) {
    e = cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    e = cudaGetSymbolAddress(reinterpret_cast<void**>(&d.err), g_device_error);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(error word)");
    d.init = true;
  }
  *out = &d;
  return MLA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Decode kernel choice: the knob (2 = dim-split pair, 3 = head-split pair), else the
// head-split pair kernel.  Both handle 1..128 rows per launch.
int pick_kernel(int heads) {
  if (heads < 1 || heads > MLA_MAX_HEADS) return -1;
  const int k = g_knobs[MLA_KNOB_DECODE_KERNEL].load();
  if (k == 0) return 3;
  return (k == 2 || k == 3) ? k : -1;
}

int num_workers_for(const DeviceState& d, int kernel, int heads) {
  (void)heads;
  const int forced = g_knobs[MLA_KNOB_NUM_WORKERS].load();
  if (forced > 0) return forced;
  const int occ = kernel == 2 ? decode_tc_max_workers(d.sm_count) : decode_pair_max_workers(d.sm_count);
  return std::max(1, std::min(d.sm_count / 2, occ));  // CTA pairs
}

mla_status_t ensure_workspace(DeviceState& d, size_t need, cudaStream_t stream) {
  if (need <= d.ws_bytes) return MLA_OK;
  if (d.ws_external)
    return fail(MLA_ERR_WORKSPACE, "workspace of %zu bytes is smaller than the %zu bytes needed", d.ws_bytes, need);
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(stream, &cs);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamIsCapturing");
  if (cs != cudaStreamCaptureStatusNone)
    return fail(MLA_ERR_WORKSPACE, "workspace must grow to %zu bytes but the stream is capturing", need);
  if (d.ws) {
    e = cudaFree(d.ws);  // waits for work that may still use it
    d.ws = nullptr;
    d.ws_bytes = 0;
    if (e != cudaSuccess) return cuda_fail(e, "cudaFree(workspace)");
  }
  e = cudaMalloc(&d.ws, need);
  if (e != cudaSuccess) {
    d.ws = nullptr;
    return cuda_fail(e, "cudaMalloc(workspace)");
  }
  d.ws_bytes = need;
  return MLA_OK;
}

void record_event(DeviceState& d, int idx, cudaStream_t stream) {
  if (!g_timing.load()) return;
  const size_t i = (size_t)d.timed_calls * 4 + idx;
  while (d.events.size() <= i) {
    cudaEvent_t ev;
    if (cudaEventCreate(&ev) != cudaSuccess) return;
    d.events.push_back(ev);
  }
  cudaEventRecord(d.events[i], stream);
}

}  // namespace

namespace mla {
// The per-device facts mla_decode uses (decode kernel, worker count, error word),
// for the allocation-free entry point in noalloc.cu.
mla_status_t decode_plan(int heads, int* kernel, int* num_workers, int** err_word) {
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState* d = nullptr;
  mla_status_t s = device_state(&d);
  if (s != MLA_OK) return s;
  *kernel = pick_kernel(heads);
  if (*kernel < 0) return fail(MLA_ERR_UNSUPPORTED, "requested decode kernel does not handle heads = %d", heads);
  *num_workers = num_workers_for(*d, *kernel, heads);
  *err_word = d->err;
  return MLA_OK;
}

mla_status_t record_error(mla_status_t s, const char* msg) { return fail(s, "%s", msg); }

cudaError_t launch_decode(int kernel, const DecodeArgs& a, cudaStream_t stream) {
  return kernel == 2 ? launch_decode_tc(a, stream) : launch_decode_pair(a, stream);
}

int decode_granule(int kernel) { return kernel == 3 ? 4 : 1; }

int schedule_whole_slack() {
  if (g_knobs[MLA_KNOB_NUM_WORKERS].load() > 0) return -1;
  const int v = g_knobs[MLA_KNOB_SPLIT_POLICY].load();
  return v == 0 ? 16 : v == 1 ? -1 : 1 << 30;
}

int schedule_piece_cost() {
  const int v = g_knobs[MLA_KNOB_PIECE_COST].load();
  return v > 0 ? std::min(v - 1, kMaxPieceCost) : 8;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

cudaError_t allow_dynamic_smem(const void* kernel, int bytes, bool (&done)[64]) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool tracked = dev >= 0 && dev < 64;
  if (tracked && done[dev]) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && tracked) done[dev] = true;
  return e;
}

int knob_value(int knob) { return (knob >= 0 && knob < 8) ? g_knobs[knob].load() : 0; }
}  // namespace mla

extern "C" {

const char* mla_status_string(mla_status_t s) {
  switch (s) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED";
    case MLA_ERR_WORKSPACE: return "MLA_ERR_WORKSPACE";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA";
    case MLA_ERR_DEVICE_BAD_PAGE: return "MLA_ERR_DEVICE_BAD_PAGE";
    case MLA_ERR_DEVICE_TIMEOUT: return "MLA_ERR_DEVICE_TIMEOUT";
  }
  return "MLA_ERR_UNKNOWN";
}

const char* mla_last_error_message(void) { return g_msg; }

mla_status_t mla_set_knob(mla_knob_t knob, int value) {
  if ((int)knob < 0 || (int)knob >= 8) return fail(MLA_ERR_INVALID_ARG, "unknown knob %d", (int)knob);
  if (value < 0) return fail(MLA_ERR_INVALID_ARG, "knob value %d < 0", value);
  g_knobs[knob].store(value);
  return MLA_OK;
}

int mla_get_knob(mla_knob_t knob) {
  if ((int)knob < 0 || (int)knob >= 8) return -1;
  return g_knobs[knob].load();
}

int mla_selected_decode_kernel(int heads) {
  if (heads < 1 || heads > MLA_MAX_HEADS) return -1;
  return pick_kernel(heads);
}

size_t mla_workspace_size(int batch, int heads, int max_blocks) {
  (void)max_blocks;
  if (batch <= 0 || heads <= 0) return 0;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState* d = nullptr;
  if (device_state(&d) != MLA_OK) return 0;
  const int group = std::min(heads, (int)MLA_MAX_HEADS);  // rows per decode launch
  const int kernel = pick_kernel(group);
  const int P = num_workers_for(*d, kernel < 0 ? 1 : kernel, group);
  return carve_schedule(nullptr, batch, group, P, nullptr);
}

mla_status_t mla_set_workspace(void* dev_ptr, size_t bytes) {
  if (dev_ptr && (reinterpret_cast<uintptr_t>(dev_ptr) & 255u))
    return fail(MLA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState* d = nullptr;
  mla_status_t s = device_state(&d);
  if (s != MLA_OK) return s;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  if (d->ws && !d->ws_external) {
    e = cudaFree(d->ws);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFree(workspace)");
  }
  d->ws = dev_ptr;
  d->ws_bytes = dev_ptr ? bytes : 0;
  d->ws_external = dev_ptr != nullptr;
  return MLA_OK;
}

mla_status_t mla_get_device_error(mla_stream_t stream) {
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState* d = nullptr;
  mla_status_t s = device_state(&d);
  if (s != MLA_OK) return s;
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int v = 0;
  e = cudaMemcpy(&v, d->err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "read error word");
  const int zero = 0;
  e = cudaMemcpy(d->err, &zero, sizeof(int), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cuda_fail(e, "clear error word");
  if (v == 0) return MLA_OK;
  return v == MLA_ERR_DEVICE_TIMEOUT ? MLA_ERR_DEVICE_TIMEOUT : MLA_ERR_DEVICE_BAD_PAGE;
}

}  // extern "C"

namespace mla {
namespace {

// mla_decode and mla_decode_multi: `heads` rows per sequence, made of s_q query
// tokens of heads / s_q heads each.  More than 128 rows (s_q > 1 only) run as groups of
// at most 128 rows, each a decode and a combine over the same schedule: every group
// reads the cache once more.
constexpr int kMaxRows = 16 * MLA_MAX_HEADS;  // query rows per sequence for mla_decode_multi

mla_status_t decode_call(const void* q, const void* kv_cache, const int32_t* block_table, const int32_t* cache_seqlens,
                         float* out, float* lse, int batch, int s_q, int heads, int num_pages, int max_blocks,
                         float softmax_scale, mla_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (batch < 0 || heads < 0 || max_blocks < 0 || num_pages < 0)
    return fail(MLA_ERR_INVALID_ARG, "negative size (batch %d, heads %d, max_blocks %d, num_pages %d)", batch, heads,
                max_blocks, num_pages);
  if (batch == 0) return MLA_OK;
  if (!q || !kv_cache || !cache_seqlens || !out || !lse)
    return fail(MLA_ERR_INVALID_ARG, "null pointer argument");
  if (heads < 1 || heads > (s_q > 1 ? kMaxRows : MLA_MAX_HEADS))
    return fail(MLA_ERR_UNSUPPORTED, "%d rows per sequence outside [1, %d]", heads, s_q > 1 ? kMaxRows : MLA_MAX_HEADS);
  if (max_blocks < 1) return fail(MLA_ERR_INVALID_ARG, "max_blocks must be >= 1");
  if (block_table && num_pages < 1) return fail(MLA_ERR_INVALID_ARG, "paged cache with num_pages < 1");
  if ((long long)batch * max_blocks > (1LL << 31) - 1 || (long long)max_blocks * MLA_PAGE_TOKENS > (1LL << 30))
    return fail(MLA_ERR_UNSUPPORTED, "cache too large for 32-bit page indexing");
  if ((long long)batch * ((long long)max_blocks + kMaxPieceCost) > (1LL << 31) - 1)
    return fail(MLA_ERR_UNSUPPORTED, "batch too large for the 32-bit split schedule");
  if (!aligned16(q) || !aligned16(kv_cache) || !aligned16(out))
    return fail(MLA_ERR_INVALID_ARG, "q, kv_cache and out must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(block_table) & 3u) || (reinterpret_cast<uintptr_t>(cache_seqlens) & 3u) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return fail(MLA_ERR_INVALID_ARG, "int32/fp32 arrays must be 4-byte aligned");
  if (!std::isfinite(softmax_scale)) return fail(MLA_ERR_INVALID_ARG, "softmax_scale is not finite");

  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState* d = nullptr;
  mla_status_t s = device_state(&d);
  if (s != MLA_OK) return s;
  const int group = std::min(heads, (int)MLA_MAX_HEADS);  // rows per launch
  const int kernel = pick_kernel(group);
  if (kernel < 0) return fail(MLA_ERR_UNSUPPORTED, "requested decode kernel does not handle heads = %d", heads);
  const int P = num_workers_for(*d, kernel, group);
  const size_t need = carve_schedule(nullptr, batch, group, P, nullptr);
  s = ensure_workspace(*d, need, stream);
  if (s != MLA_OK) return s;

  DecodeArgs a{};
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.kv = static_cast<const __nv_bfloat16*>(kv_cache);
  a.block_table = block_table;
  a.seqlens = cache_seqlens;
  a.out = out;
  a.lse = lse;
  a.batch = batch;
  a.heads = group;
  a.num_pages = num_pages;
  a.max_blocks = max_blocks;
  a.scale = softmax_scale;
  a.err = d->err;
  carve_schedule(d->ws, batch, group, P, &a.sched);
  a.wait_limit = g_knobs[MLA_KNOB_WAIT_LIMIT].load() > 0 ? g_knobs[MLA_KNOB_WAIT_LIMIT].load() : 2000;  // ms
  a.withhold_arrive = g_knobs[MLA_KNOB_WITHHOLD_ARRIVE].load();
  a.s_q = s_q;
  a.hq = heads / s_q;
  a.row_stride = heads;
  a.row0 = 0;
  a.min_pages = g_knobs[MLA_KNOB_MIN_PAGES].load() > 0 ? g_knobs[MLA_KNOB_MIN_PAGES].load() : 4;
  a.granule = decode_granule(kernel);
  a.whole_slack = schedule_whole_slack();
  a.piece_cost = schedule_piece_cost();

  // The decode CTAs derive the split schedule themselves: the timing slot of the
  // schedule (events 0 -> 1) stays empty.
  record_event(*d, 0, stream);
  record_event(*d, 1, stream);
  cudaError_t e = cudaSuccess;
  for (int r0 = 0; r0 < heads; r0 += group) {
    a.row0 = r0;
    a.heads = std::min(group, heads - r0);
    e = launch_decode(kernel, a, stream);
    if (e != cudaSuccess) return cuda_fail(e, "decode launch");
    if (r0 + group >= heads) record_event(*d, 2, stream);
    e = launch_combine(a, stream);
    if (e != cudaSuccess) return cuda_fail(e, "combine launch");
  }
  record_event(*d, 3, stream);
  if (g_timing.load()) d->timed_calls++;
  return MLA_OK;
}

}  // namespace
}  // namespace mla

extern "C" {

mla_status_t mla_decode(const void* q, const void* kv_cache, const int32_t* block_table,
                        const int32_t* cache_seqlens, float* out, float* lse, int batch, int heads,
                        int num_pages, int max_blocks, float softmax_scale, mla_stream_t stream) {
  return decode_call(q, kv_cache, block_table, cache_seqlens, out, lse, batch, 1, heads, num_pages, max_blocks,
                     softmax_scale, stream);
}

mla_status_t mla_decode_multi(const void* q, const void* kv_cache, const int32_t* block_table,
                              const int32_t* cache_seqlens, float* out, float* lse, int batch, int s_q, int heads,
                              int num_pages, int max_blocks, float softmax_scale, mla_stream_t stream) {
  if (s_q < 1 || heads < 0) return fail(MLA_ERR_INVALID_ARG, "s_q = %d, heads = %d", s_q, heads);
  if (heads > MLA_MAX_HEADS) return fail(MLA_ERR_UNSUPPORTED, "heads = %d > 128", heads);
  if ((long long)s_q * heads > kMaxRows)
    return fail(MLA_ERR_UNSUPPORTED, "s_q x heads = %lld rows > %d", (long long)s_q * heads, kMaxRows);
  return decode_call(q, kv_cache, block_table, cache_seqlens, out, lse, batch, s_q, s_q * heads, num_pages,
                     max_blocks, softmax_scale, stream);
}

mla_status_t mla_absorb_q(const void* q_nope, const void* q_rope, const void* w_uk, void* q_out, int batch,
                          int heads, mla_stream_t stream) {
  if (batch < 0 || heads < 0) return fail(MLA_ERR_INVALID_ARG, "negative size");
  if (batch == 0) return MLA_OK;
  if (!q_nope || !q_rope || !w_uk || !q_out) return fail(MLA_ERR_INVALID_ARG, "null pointer argument");
  if (heads < 1 || heads > MLA_MAX_HEADS) return fail(MLA_ERR_UNSUPPORTED, "heads = %d outside [1, 128]", heads);
  if (!aligned16(q_nope) || !aligned16(q_rope) || !aligned16(w_uk) || !aligned16(q_out))
    return fail(MLA_ERR_INVALID_ARG, "absorb_q operands must be 16-byte aligned");
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState* d = nullptr;
  mla_status_t s = device_state(&d);
  if (s != MLA_OK) return s;
  cudaError_t e = launch_absorb_q(static_cast<const __nv_bfloat16*>(q_nope), static_cast<const __nv_bfloat16*>(q_rope),
                                  static_cast<const __nv_bfloat16*>(w_uk), static_cast<__nv_bfloat16*>(q_out), batch,
                                  heads, d->err, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MLA_OK : cuda_fail(e, "absorb_q launch");
}

mla_status_t mla_absorb_o(const float* out_latent, const void* w_uv, float* out, int batch, int heads,
                          mla_stream_t stream) {
  if (batch < 0 || heads < 0) return fail(MLA_ERR_INVALID_ARG, "negative size");
  if (batch == 0) return MLA_OK;
  if (!out_latent || !w_uv || !out) return fail(MLA_ERR_INVALID_ARG, "null pointer argument");
  if (heads < 1 || heads > MLA_MAX_HEADS) return fail(MLA_ERR_UNSUPPORTED, "heads = %d outside [1, 128]", heads);
  if (!aligned16(out_latent) || !aligned16(w_uv) || !aligned16(out))
    return fail(MLA_ERR_INVALID_ARG, "absorb_o operands must be 16-byte aligned");
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState* d = nullptr;
  mla_status_t s = device_state(&d);
  if (s != MLA_OK) return s;
  cudaError_t e = launch_absorb_o(out_latent, static_cast<const __nv_bfloat16*>(w_uv), out, batch, heads, d->err,
                                  reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MLA_OK : cuda_fail(e, "absorb_o launch");
}

mla_status_t mla_timing_enable(int enable) {
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState* d = nullptr;
  mla_status_t s = device_state(&d);
  if (s != MLA_OK) return s;
  d->timed_calls = 0;
  g_timing.store(enable ? 1 : 0);
  return MLA_OK;
}

mla_status_t mla_timing_read(float ms[3], int* calls) {
  if (!ms || !calls) return fail(MLA_ERR_INVALID_ARG, "null pointer argument");
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState* d = nullptr;
  mla_status_t s = device_state(&d);
  if (s != MLA_OK) return s;
  ms[0] = ms[1] = ms[2] = 0.f;
  *calls = d->timed_calls;
  if (d->timed_calls > 0) {
    cudaError_t e = cudaEventSynchronize(d->events[(size_t)d->timed_calls * 4 - 1]);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventSynchronize");
    for (int c = 0; c < d->timed_calls; ++c) {
      for (int k = 0; k < 3; ++k) {
        float t = 0.f;
        e = cudaEventElapsedTime(&t, d->events[(size_t)c * 4 + k], d->events[(size_t)c * 4 + k + 1]);
        if (e != cudaSuccess) return cuda_fail(e, "cudaEventElapsedTime");
        ms[k] += t;
      }
    }
  }
  d->timed_calls = 0;
  return MLA_OK;
}

}  // extern "C"
