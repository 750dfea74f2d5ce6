// The split schedule, derived inside the decode grid: every CTA computes its worker's
// page range from the sequence lengths (the same arithmetic in every CTA), so no
// separate grid has to run, and be waited for, before the first page load.
//
// The pages of all sequences are laid end to end (sequence-major); with N pages in all
// and P workers, worker w takes [w q, min((w+1) q, N)), q = max(ceil(N / P), min_pages)
// rounded up to the kernel's page granule.  When there are no more sequences than
// workers and the longest is at most whole_slack pages above q, every sequence instead
// runs whole on worker b (nearly uniform lengths run faster unsplit: a split sequence
// pays for a piece boundary in its workers and for the combine).  CTA c also writes the
// sequence records (SeqInfo) of the sequences b = c, c + gridDim.x, ... that the
// combine grid reads, and reports their invalid lengths.
#pragma once

#include "mla_device.cuh"
#include "mla_internal.h"

namespace mla {

// Pages of sequence b; an invalid length (negative, or beyond the block table) has none.
__device__ __forceinline__ int seq_pages(const int32_t* seqlens, int max_blocks, int b) {
  const int T = seqlens[b];
  return (T < 0 || T > max_blocks * kPage) ? 0 : (T + kPage - 1) / kPage;
}

struct RangeScratch {
  int red_sum[32], red_max[32];  // per-warp partials
  int carry;                     // pages before the current pass of the scan
  int total, maxp;
  WorkerRange rg;
};

// Called by every thread of the CTA (block-uniform control flow, blockDim.x a multiple
// of 32) with the call's lengths, batch size B, block-table width, worker count P and
// schedule knobs; writes this CTA's share of the records `seq`, and on return rs.rg
// holds worker w's range (b0 < 0: no work).  Not inlined: it runs once per CTA and
// keeps its registers out of the kernel's main loops.
static __device__ __noinline__ void derive_worker_range(const int32_t* seqlens, int B, int max_blocks, int P,
                                                       int min_pages, int granule, int whole_slack, SeqInfo* seq,
                                                       int* err, int w, RangeScratch& rs) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  auto owns = [&](int b) { return b % (int)gridDim.x == (int)blockIdx.x; };

  // 1. Total pages and the longest sequence.
  int sum = 0, mx = 0;
  for (int b = tid; b < B; b += blockDim.x) {
    const int n = seq_pages(seqlens, max_blocks, b);
    sum += n;
    mx = max(mx, n);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sum += __shfl_xor_sync(0xffffffffu, sum, o);
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  if (lane == 0) {
    rs.red_sum[warp] = sum;
    rs.red_max[warp] = mx;
  }
  if (tid == 0) {
    rs.carry = 0;
    rs.rg = WorkerRange{-1, 0, -1, 0};
  }
  __syncthreads();
  if (tid == 0) {
    int s = 0, m = 0;
    for (int i = 0; i < nw; ++i) {
      s += rs.red_sum[i];
      m = max(m, rs.red_max[i]);
    }
    rs.total = s;
    rs.maxp = m;
  }
  __syncthreads();
  const int N = rs.total;
  int q = (N + P - 1) / P;
  if (q < min_pages) q = min_pages;
  if (q < 1) q = 1;
  q = (q + granule - 1) / granule * granule;

  if (whole_slack >= 0 && B <= P && rs.maxp <= q + whole_slack) {
    // 2a. One whole sequence per worker.
    if (tid == 0 && w < B) {
      const int n = seq_pages(seqlens, max_blocks, w);
      if (n > 0) rs.rg = WorkerRange{w, 0, w, n};
    }
    for (int b = tid; b < B; b += blockDim.x) {
      if (!owns(b)) continue;
      const int T = seqlens[b];
      const bool bad = T < 0 || T > max_blocks * kPage;
      if (bad) set_device_error(err, MLA_ERR_DEVICE_BAD_PAGE);
      seq[b] = SeqInfo{b, bad ? -1 : (T > 0 ? 1 : 0), b};
    }
    __syncthreads();
    return;
  }

  // 2b. Exclusive prefix sum of pages, blockDim.x sequences per pass.  Worker w's first
  // page lies in exactly one non-empty sequence, which writes (b0, p0), and so does its
  // last page, which writes (b1, p1).
  const long long g0 = (long long)w * q, g1 = min(g0 + q, (long long)N);
  for (int base = 0; base < B; base += blockDim.x) {
    const int b = base + tid;
    const int n = b < B ? seq_pages(seqlens, max_blocks, b) : 0;
    int x = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) rs.red_sum[warp] = x;
    __syncthreads();
    int before = rs.carry;
    for (int i = 0; i < warp; ++i) before += rs.red_sum[i];
    const int st = before + x - n;  // first page of sequence b in the list
    if (b < B) {
      if (n > 0 && g0 < N) {
        if (g0 >= st && g0 < st + n) {
          rs.rg.b0 = b;
          rs.rg.p0 = (int)(g0 - st);
        }
        if (g1 > st && g1 <= st + n) {
          rs.rg.b1 = b;
          rs.rg.p1 = (int)(g1 - st);
        }
      }
      if (owns(b)) {
        const int T = seqlens[b];
        const bool bad = T < 0 || T > max_blocks * kPage;
        if (bad) set_device_error(err, MLA_ERR_DEVICE_BAD_PAGE);
        SeqInfo si;
        si.first_worker = st / q;
        si.num_pieces = bad ? -1 : (n > 0 ? (st + n - 1) / q - st / q + 1 : 0);
        // The first piece is the worker's first sequence iff the worker's range starts at
        // the sequence's first page; every later piece starts its worker's range.
        si.first_slot = st % q == 0 ? si.first_worker : P + si.first_worker;
        seq[b] = si;
      }
    }
    __syncthreads();
    if (tid == blockDim.x - 1) rs.carry = st + n;
    __syncthreads();
  }
}

}  // namespace mla
