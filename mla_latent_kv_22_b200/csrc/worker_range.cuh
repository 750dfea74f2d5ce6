// The split schedule, derived inside the decode grid: every CTA computes its worker's
// page range from the sequence lengths (the same arithmetic in every CTA), so no
// separate grid has to run, and be waited for, before the first page load.
//
// The sequences are laid end to end, each as `piece_cost` units of fixed cost followed by
// its pages (an empty sequence takes no units); with W units in all and P workers, worker
// w takes the pages inside units [w q, min((w+1) q, W)), q = max(ceil(W / P), min_pages)
// rounded up to the kernel's page granule.  A piece costs its worker a q' staging, a
// pipeline fill and an epilogue besides its pages, so charging each sequence for one
// evens out workers that hold several short pieces against workers that hold one long
// one (a worker's range also pays at most once for continuing a sequence, the same for
// every worker).  piece_cost = 0 is a split by pages alone.  When there are no more
// sequences than workers and the longest is at most whole_slack pages above the pages-only
// share ceil(pages / P), every sequence instead runs whole on worker b (nearly uniform
// lengths run faster unsplit: a split sequence pays for a piece boundary in its workers
// and for the combine).  CTA c also writes the sequence records (SeqInfo) of the
// sequences b = c, c + gridDim.x, ... that the combine grid reads, and reports their
// invalid lengths.
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
  int red_sum[32], red_units[32], red_max[32];  // per-warp partials
  int carry;                                    // units before the current pass of the scan
  int total, total_units, maxp;
  WorkerRange rg;
};

// Called by every thread of the CTA (block-uniform control flow, blockDim.x a multiple
// of 32) with the call's lengths, batch size B, block-table width, worker count P and
// schedule knobs; writes this CTA's share of the records `seq`, and on return rs.rg
// holds worker w's range (b0 < 0: no work).  Not inlined: it runs once per CTA and
// keeps its registers out of the kernel's main loops.
static __device__ __noinline__ void derive_worker_range(const int32_t* seqlens, int B, int max_blocks, int P,
                                                       int min_pages, int granule, int whole_slack, int piece_cost,
                                                       SeqInfo* seq, int* err, int w, RangeScratch& rs) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  auto owns = [&](int b) { return b % (int)gridDim.x == (int)blockIdx.x; };
  auto units = [&](int n) { return n > 0 ? n + piece_cost : 0; };  // a sequence's share of the layout

  // 1. Total pages, total units and the longest sequence.
  long long sum = 0, wsum = 0;
  int mx = 0;
  for (int b = tid; b < B; b += blockDim.x) {
    const int n = seq_pages(seqlens, max_blocks, b);
    sum += n;
    wsum += units(n);
    mx = max(mx, n);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sum += __shfl_xor_sync(0xffffffffu, sum, o);
    wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  if (lane == 0) {
    rs.red_sum[warp] = (int)sum;
    rs.red_units[warp] = (int)wsum;
    rs.red_max[warp] = mx;
  }
  if (tid == 0) {
    rs.carry = 0;
    rs.rg = WorkerRange{-1, 0, -1, 0};
  }
  __syncthreads();
  if (tid == 0) {
    int s = 0, u = 0, m = 0;
    for (int i = 0; i < nw; ++i) {
      s += rs.red_sum[i];
      u += rs.red_units[i];
      m = max(m, rs.red_max[i]);
    }
    rs.total = s;
    rs.total_units = u;
    rs.maxp = m;
  }
  __syncthreads();
  auto share = [&](int total) {
    int q = (total + P - 1) / P;
    if (q < min_pages) q = min_pages;
    if (q < 1) q = 1;
    return (q + granule - 1) / granule * granule;
  };

  if (whole_slack >= 0 && B <= P && rs.maxp <= share(rs.total) + whole_slack) {
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

  // 2b. Exclusive prefix sum of units, blockDim.x sequences per pass.  Sequence b occupies
  // units [st, st + units(n)); its pages sit at [pos, pos + n), pos = st + piece_cost, and
  // the next non-empty sequence's pages start at st + units(n) + piece_cost.  Worker w's
  // first piece is the sequence whose pages meet [g0, g1) with st <= g0 (no earlier pages
  // in the range), and its last piece the one whose pages meet it with g1 <= the next
  // sequence's first page: each is written by exactly one thread.
  const int W = rs.total_units;
  const int q = share(W);
  const long long g0 = (long long)w * q, g1 = min(g0 + q, (long long)W);
  for (int base = 0; base < B; base += blockDim.x) {
    const int b = base + tid;
    const int n = b < B ? seq_pages(seqlens, max_blocks, b) : 0;
    const int u = units(n);
    int x = u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) rs.red_sum[warp] = x;
    __syncthreads();
    int before = rs.carry;
    for (int i = 0; i < warp; ++i) before += rs.red_sum[i];
    const int st = before + x - u;  // first unit of sequence b
    if (b < B) {
      const int pos = st + (n > 0 ? piece_cost : 0);  // its first page in the layout
      if (n > 0 && g0 < W && max(g0, (long long)pos) < min(g1, (long long)pos + n)) {
        if (g0 >= st) {
          rs.rg.b0 = b;
          rs.rg.p0 = (int)(max(g0, (long long)pos) - pos);
        }
        if (g1 <= (long long)pos + n + piece_cost) {
          rs.rg.b1 = b;
          rs.rg.p1 = (int)(min(g1, (long long)pos + n) - pos);
        }
      }
      if (owns(b)) {
        const int T = seqlens[b];
        const bool bad = T < 0 || T > max_blocks * kPage;
        if (bad) set_device_error(err, MLA_ERR_DEVICE_BAD_PAGE);
        SeqInfo si;
        si.first_worker = pos / q;
        si.num_pieces = bad ? -1 : (n > 0 ? (pos + n - 1) / q - pos / q + 1 : 0);
        // The first piece is its worker's first piece iff no earlier pages fall in that
        // worker's units (its range starts at or after st); every later piece starts its
        // worker's range.
        si.first_slot = si.first_worker * q >= st ? si.first_worker : P + si.first_worker;
        seq[b] = si;
      }
    }
    __syncthreads();
    if (tid == blockDim.x - 1) rs.carry = st + u;
    __syncthreads();
  }
}

}  // namespace mla
