// mla_decode_noalloc: the same decode as mla_decode, for callers that must not
// allocate device memory.
//
// mla_decode keeps its split partials and per-sequence records in a workspace that
// it grows with cudaMalloc on first need (or that the caller hands over).  Some
// callers can do neither: a serving runtime that has already reserved all device
// memory for its own pool, or latency-critical paths where cudaMalloc's implicit
// device synchronisation is not acceptable.  This variant takes its
// scratch from one file-scope __device__ array instead: kNoAllocScratchBytes
// (32 MiB) that every GPU which loads the library holds until the process exits.
//
// Contract:
//  - Sizes whose records and partials do not fit the array are rejected with
//    MLA_ERR_UNSUPPORTED before anything is launched.  To fit, the call may use
//    fewer split workers than mla_decode (at 128 heads at most 63 CTA pairs), so
//    its results agree with mla_decode's within rounding, not bit for bit.
//  - The first call on a device looks up the array's device address
//    (cudaGetSymbolAddress, with that device current).
//  - Every call on a device shares the one array, and the array keeps the last
//    call's contents.  Nothing in it has to start at zero: the decode grid of each call
//    rewrites the per-sequence records and every partial slot before the combine
//    reads them.  Calls that overlap on the GPU (other streams, other host
//    threads) race on the array and must be serialised by the caller.
//  - No cudaMalloc, cudaFree or allocating library call is made.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <mutex>

#include "mla.h"
#include "mla_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

std::mutex g_setup_mu;
void* g_scratch_addr[kMaxDevices] = {};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

mla_status_t reject(mla_status_t s, const char* msg) { return mla::record_error(s, msg); }

}  // namespace

extern "C" mla_status_t mla_decode_noalloc(const void* q, const void* kv_cache, const int32_t* block_table,
                                           const int32_t* cache_seqlens, float* out, float* lse, int batch,
                                           int heads, int num_pages, int max_blocks, float softmax_scale,
                                           mla_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (batch < 0 || heads < 0 || max_blocks < 0 || num_pages < 0) return reject(MLA_ERR_INVALID_ARG, "negative size");
  if (batch == 0) return MLA_OK;
  if (!q || !kv_cache || !cache_seqlens || !out || !lse) return reject(MLA_ERR_INVALID_ARG, "null pointer argument");
  if (heads < 1 || heads > MLA_MAX_HEADS) return reject(MLA_ERR_UNSUPPORTED, "heads outside [1, 128]");
  if (max_blocks < 1) return reject(MLA_ERR_INVALID_ARG, "max_blocks must be >= 1");
  if (block_table && num_pages < 1) return reject(MLA_ERR_INVALID_ARG, "paged cache with num_pages < 1");
  if ((long long)batch * max_blocks > (1LL << 31) - 1 || (long long)max_blocks * MLA_PAGE_TOKENS > (1LL << 30))
    return reject(MLA_ERR_UNSUPPORTED, "cache too large for 32-bit page indexing");
  if ((long long)batch * ((long long)max_blocks + mla::kMaxPieceCost) > (1LL << 31) - 1)
    return reject(MLA_ERR_UNSUPPORTED, "batch too large for the 32-bit split schedule");
  if (!aligned16(q) || !aligned16(kv_cache) || !aligned16(out))
    return reject(MLA_ERR_INVALID_ARG, "q, kv_cache and out must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(block_table) & 3u) || (reinterpret_cast<uintptr_t>(cache_seqlens) & 3u) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return reject(MLA_ERR_INVALID_ARG, "int32/fp32 arrays must be 4-byte aligned");
  if (!std::isfinite(softmax_scale)) return reject(MLA_ERR_INVALID_ARG, "softmax_scale is not finite");

  // Fewer workers shrink the partial storage; reject what does not fit even with one.
  if (mla::carve_schedule(nullptr, batch, heads, 1, nullptr) > kNoAllocScratchBytes) {
    char msg[160];
    snprintf(msg, sizeof msg, "batch %d x heads %d needs more than the %zu-byte static scratch of mla_decode_noalloc",
             batch, heads, kNoAllocScratchBytes);
    return reject(MLA_ERR_UNSUPPORTED, msg);
  }
  int kernel = 0, workers = 0;
  int* err = nullptr;
  mla_status_t s = mla::decode_plan(heads, &kernel, &workers, &err);
  if (s != MLA_OK) return s;
  while (workers > 1 && mla::carve_schedule(nullptr, batch, heads, workers, nullptr) > kNoAllocScratchBytes) --workers;

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) return reject(MLA_ERR_CUDA, "cudaGetDevice failed");
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_setup_mu);
    if (!g_scratch_addr[dev]) {
      // Host code only knows the array's host-side shadow; the kernels need its device address.
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_decode_scratch);
      if (e != cudaSuccess || !p) return reject(MLA_ERR_CUDA, "cudaGetSymbolAddress(static decode scratch) failed");
      g_scratch_addr[dev] = p;
    }
    scratch = g_scratch_addr[dev];
  }

  mla::DecodeArgs a{};
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.kv = static_cast<const __nv_bfloat16*>(kv_cache);
  a.block_table = block_table;
  a.seqlens = cache_seqlens;
  a.out = out;
  a.lse = lse;
  a.batch = batch;
  a.heads = heads;
  a.num_pages = num_pages;
  a.max_blocks = max_blocks;
  a.scale = softmax_scale;
  a.err = err;
  mla::carve_schedule(scratch, batch, heads, workers, &a.sched);
  const int wl = mla::knob_value(MLA_KNOB_WAIT_LIMIT);
  a.wait_limit = wl > 0 ? wl : 2000;
  a.withhold_arrive = 0;
  a.s_q = 1;
  a.hq = heads;
  a.row_stride = heads;
  a.row0 = 0;
  const int mp = mla::knob_value(MLA_KNOB_MIN_PAGES);
  a.min_pages = mp > 0 ? mp : 4;
  a.granule = mla::decode_granule(kernel);
  a.whole_slack = mla::schedule_whole_slack();
  a.piece_cost = mla::schedule_piece_cost();

  e = mla::launch_decode(kernel, a, stream);
  if (e != cudaSuccess) return reject(MLA_ERR_CUDA, "decode launch failed");
  e = mla::launch_combine(a, stream);
  if (e != cudaSuccess) return reject(MLA_ERR_CUDA, "combine launch failed");
  return MLA_OK;
}
