// Split schedule: turns the device-resident sequence lengths into worker page
// ranges without a host round trip (see the Schedule comment in mla_internal.h).
#include "mla_device.cuh"
#include "mla_internal.h"

namespace mla {

namespace {

constexpr int kSchedThreads = 1024;

// Largest b in [0, B) with start[b] <= g (start is non-decreasing, start[0] = 0).
__device__ int seq_of_page(const int* start, int B, int g) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (start[mid] <= g) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__global__ void __launch_bounds__(kSchedThreads) schedule_kernel(const int32_t* __restrict__ seqlens, int B,
                                                                 int max_blocks, int min_pages, Schedule s,
                                                                 int* err) {
  __shared__ int warp_sums[kSchedThreads / 32];
  __shared__ int carry;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  grid_dep_launch_dependents();  // the decode grid may start its prologue now; it waits for this grid's writes
  if (tid == 0) carry = 0;
  __syncthreads();

  // 1. Exclusive prefix sum of pages per sequence, 1024 sequences per pass.
  for (int base = 0; base < B; base += kSchedThreads) {
    const int b = base + tid;
    int n = 0;
    if (b < B) {
      int T = seqlens[b];
      if (T < 0 || T > max_blocks * kPage) {
        set_device_error(err, MLA_ERR_DEVICE_BAD_PAGE);
        T = 0;  // the sequence is reported as invalid below; no page of it is read
      }
      n = (T + kPage - 1) / kPage;
    }
    int x = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int w = warp_sums[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      warp_sums[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    const int incl = x + (warp ? warp_sums[warp - 1] : 0) + carry;
    if (b < B) s.seq_start[b] = incl - n;
    __syncthreads();
    if (tid == kSchedThreads - 1) carry = incl;
    __syncthreads();
  }
  if (tid == 0) s.seq_start[B] = carry;
  __threadfence_block();
  __syncthreads();

  const int N = carry;
  const int P = s.num_workers;
  int q = (N + P - 1) / P;
  if (q < min_pages) q = min_pages;
  if (q < 1) q = 1;
  if (tid == 0) *s.quota = q;

  // 2. Worker ranges.
  for (int w = tid; w < P; w += kSchedThreads) {
    WorkerRange r{-1, 0, -1, 0};
    const long long g0 = (long long)w * q;
    if (g0 < N) {
      const int g1 = (int)(g0 + q < (long long)N ? g0 + q : (long long)N);
      r.b0 = seq_of_page(s.seq_start, B, (int)g0);
      r.p0 = (int)g0 - s.seq_start[r.b0];
      r.b1 = seq_of_page(s.seq_start, B, g1 - 1);
      r.p1 = g1 - s.seq_start[r.b1];
    }
    s.ranges[w] = r;
  }

  // 3. Per-sequence piece counts.
  for (int b = tid; b < B; b += kSchedThreads) {
    const int st = s.seq_start[b];
    const int n = s.seq_start[b + 1] - st;
    const int T = seqlens[b];
    SeqInfo si;
    si.first_worker = st / q;
    si.num_pieces = n > 0 ? (st + n - 1) / q - st / q + 1 : 0;
    if (T < 0 || T > max_blocks * kPage) si.num_pieces = -1;
    s.seq[b] = si;
  }
}

}  // namespace

size_t carve_schedule(void* base, int batch, int heads, int num_workers, Schedule* s) {
  auto align = [](size_t x) { return (x + 255) & ~size_t(255); };
  size_t off = 0;
  char* p = static_cast<char*>(base);
  auto take = [&](size_t bytes) {
    void* r = p ? p + off : nullptr;
    off = align(off + bytes);
    return r;
  };
  Schedule t;
  t.num_workers = num_workers;
  t.ranges = static_cast<WorkerRange*>(take(sizeof(WorkerRange) * num_workers));
  t.seq_start = static_cast<int*>(take(sizeof(int) * (batch + 1)));
  t.seq = static_cast<SeqInfo*>(take(sizeof(SeqInfo) * batch));
  t.quota = static_cast<int*>(take(sizeof(int)));
  t.part_lse = static_cast<float*>(take(sizeof(float) * 2 * (size_t)num_workers * heads));
  t.part_o = static_cast<float*>(take(sizeof(float) * 2 * (size_t)num_workers * heads * kDLatent));
  if (s) *s = t;
  return off;
}

cudaError_t launch_schedule(const int32_t* seqlens, int batch, int max_blocks, int min_pages,
                            const Schedule& s, int* err, cudaStream_t stream) {
  schedule_kernel<<<1, kSchedThreads, 0, stream>>>(seqlens, batch, max_blocks, min_pages, s, err);
  return cudaGetLastError();
}

}  // namespace mla
