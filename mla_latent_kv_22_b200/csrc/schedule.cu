// Split schedule: turns the device-resident sequence lengths into worker page
// ranges without a host round trip (see the Schedule comment in mla_internal.h).
#include "mla_device.cuh"
#include "mla_internal.h"

namespace mla {

namespace {

constexpr int kSchedThreads = 1024;

__global__ void __launch_bounds__(kSchedThreads) schedule_kernel(const int32_t* __restrict__ seqlens, int B,
                                                                 int max_blocks, int min_pages, int granule,
                                                                 int whole_slack, Schedule s, int* err) {
  __shared__ int warp_sums[kSchedThreads / 32];
  __shared__ int carry;
  __shared__ int max_pages;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  grid_dep_launch_dependents();  // the decode grid may start its prologue now; it waits for this grid's writes
  // Launched as a programmatic dependent of whatever ran before on the stream (which may
  // have written the lengths, or still read this workspace): only the launch overlaps it.
  grid_dep_wait();
  if (tid == 0) {
    carry = 0;
    max_pages = 0;
  }
  __syncthreads();

  // 1. Exclusive prefix sum of pages per sequence, 1024 sequences per pass.  With a
  // single pass, each thread keeps its sequence's start, page count and validity.
  int my_start = 0, my_n = 0;
  bool my_bad = false;
  for (int base = 0; base < B; base += kSchedThreads) {
    const int b = base + tid;
    int n = 0;
    bool bad = false;
    if (b < B) {
      int T = seqlens[b];
      if (T < 0 || T > max_blocks * kPage) {
        set_device_error(err, MLA_ERR_DEVICE_BAD_PAGE);
        T = 0;  // the sequence is reported as invalid below; no page of it is read
        bad = true;
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
    if (n > 0) atomicMax(&max_pages, n);
    my_start = incl - n;
    my_n = n;
    my_bad = bad;
    __syncthreads();
    if (tid == kSchedThreads - 1) carry = incl;
    __syncthreads();
  }
  if (tid == 0) s.seq_start[B] = carry;
  if (B > kSchedThreads) __syncthreads();  // step 3 reloads seq_start[b + 1]

  const int N = carry;
  const int P = s.num_workers;
  int q = (N + P - 1) / P;
  if (q < min_pages) q = min_pages;
  if (q < 1) q = 1;
  q = (q + granule - 1) / granule * granule;
  if (tid == 0) *s.quota = q;

  // Whole sequences, one per worker, when there are no more sequences than workers and
  // the longest costs at most whole_slack pages more than the split quota: a split
  // sequence pays for a piece boundary in its workers and for the combine, so nearly
  // uniform lengths run faster unsplit (whole_slack < 0: always split).
  if (whole_slack >= 0 && B <= P && max_pages <= q + whole_slack) {
    for (int w = tid; w < P; w += kSchedThreads) {
      int n = 0;
      if (w < B) {
        const int T = seqlens[w];
        n = (T < 0 || T > max_blocks * kPage) ? 0 : (T + kPage - 1) / kPage;
      }
      s.ranges[w] = n > 0 ? WorkerRange{w, 0, w, n} : WorkerRange{-1, 0, -1, 0};
    }
    for (int b = tid; b < B; b += kSchedThreads) {
      const int T = seqlens[b];
      const bool bad = T < 0 || T > max_blocks * kPage;
      SeqInfo si;
      si.first_worker = b;
      si.num_pieces = bad ? -1 : (T > 0 ? 1 : 0);
      si.first_slot = b;
      s.seq[b] = si;
    }
    return;
  }

  // 2. Workers past the last page have no work.
  for (int w = tid; w < P; w += kSchedThreads)
    if ((long long)w * q >= N) s.ranges[w] = WorkerRange{-1, 0, -1, 0};

  // 3. Per sequence: its piece count, and the range ends of the workers that overlap
  // it.  Worker w covers pages [w q, min((w+1) q, N)); its first page lies in exactly
  // one non-empty sequence, which writes (b0, p0), and so does its last page, which
  // writes (b1, p1), so every field is written once and no search is needed.
  for (int b = tid; b < B; b += kSchedThreads) {
    int st = my_start, n = my_n;
    bool bad = my_bad;
    if (B > kSchedThreads) {  // several passes: reload what this thread's pass computed
      st = s.seq_start[b];
      n = s.seq_start[b + 1] - st;
      const int T = seqlens[b];
      bad = T < 0 || T > max_blocks * kPage;
    }
    SeqInfo si;
    si.first_worker = st / q;
    si.num_pieces = n > 0 ? (st + n - 1) / q - st / q + 1 : 0;
    // The first piece is the worker's first sequence iff the worker's range starts at
    // the sequence's first page; every later piece starts its worker's range.
    si.first_slot = st % q == 0 ? si.first_worker : P + si.first_worker;
    if (bad) si.num_pieces = -1;
    s.seq[b] = si;
    if (n > 0) {
      for (int w = st / q; w <= (st + n - 1) / q; ++w) {
        const int g0 = w * q;
        const int g1 = min(g0 + q, N);
        if (g0 >= st) {
          s.ranges[w].b0 = b;
          s.ranges[w].p0 = g0 - st;
        }
        if (g1 <= st + n) {
          s.ranges[w].b1 = b;
          s.ranges[w].p1 = g1 - st;
        }
      }
    }
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

cudaError_t launch_schedule(const int32_t* seqlens, int batch, int max_blocks, int min_pages, int granule,
                            int whole_slack, const Schedule& s, int* err, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1, 1, 1);
  cfg.blockDim = dim3(kSchedThreads, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, schedule_kernel, seqlens, batch, max_blocks, min_pages, granule < 1 ? 1 : granule,
                            whole_slack, s, err);
}

}  // namespace mla
