// Split-KV absorbed-MLA decode on the 5th-generation tensor cores (tcgen05/TMEM/TMA).
//
// Work split.  One worker = one CTA pair (a 2-CTA cluster) walking a page range of
// the split schedule.  All 128 heads of a sequence share each cached row, so per
// 64-token page the work is two dense contractions with the heads on M = 128:
//     S[128 x 64]  = q'[128 x 576] . K^T      (scores over all 576 dims)
//     O[128 x 512] += P[128 x 64]  . V         (V = the first 512 dims of the rows)
// O in fp32 is 128 x 512 x 4 B = all of one SM's tensor memory, so the pair splits
// it: CTA r keeps O[:, 256r : 256r+256) and contracts the scores over its own dims
// (latent [256r, 256r+256) plus rope [512+32r, 512+32r+32)).  Each CTA therefore
// loads only its part of every row (HBM and L2 traffic 1x), computes a partial S,
// and the two partials are exchanged through distributed shared memory by bulk
// copies and added.  Each exchanged score is the top 3 bytes of its fp32 pattern
// (sign, exponent, 15 mantissa bits); on arrival its lowest byte holds a byte of
// another value (relative error < 2^-15), 4 values in 12 bytes: 24 KB per page each
// way.  Each CTA adds its own exact partial to the peer's, so the two softmaxes agree
// to that rounding; each CTA normalises its half of O by its own row sums, and rank
// 0 writes the lse.
//
// Pipeline.  The exchange has a long latency, so the softmax threads are software
// pipelined: in each iteration they first send page j+1's partial (stage A) and
// then finish page j (stage B), whose partial was sent one iteration earlier.  A
// receive buffer is handed back to the peer as soon as it has been read.  S is
// freed as soon as the softmax has loaded it (stage A), so the score MMA of the
// next page runs while the softmax finishes this one; P (bf16) goes to TMEM and
// is the A operand of the PV MMA.
//
// Roles (384 threads): warp 0 issues TMA loads (and L2 prefetches a few pages
// ahead), warp 1 allocates TMEM and issues MMAs (whichever of the next score MMA
// and the next PV is ready first), warp 2 zeroes value rows past the sequence end
// before PV reads them and hands read receive buffers back to the peer, warp 3
// copies each page's packed partial scores to the peer, and warps 4..11 are the
// softmax warps: each owns 16 head rows (TMEM lanes) and all 64 columns of every
// page, both halves of a row in one warp (16x32bx2 TMEM access), and stages q',
// exchanges partial scores, runs the online softmax (log2 domain, lazy rescale by
// at most 2^8), writes P, rescales O when needed, and writes the epilogue.
//
// TMEM (512 columns): O [0,256) fp32; q' (this CTA's 256 latent + 32 rope dims)
// [256,400) as bf16 pairs, the A operand of QK^T; S [400,464) fp32; P [464,496) as
// bf16 pairs, the A operand of PV.
// Shared memory: 4 stages x (4 latent boxes [64 tokens x 64 dims], 128B swizzle:
// K-major B of QK^T and MN-major B of PV; 1 rope box [64 tokens x 32 dims], 64B
// swizzle); a 24 KB send buffer and two 24 KB receive buffers.
//
// Several query tokens per sequence (decode_tc_kernel<true>): the rows are s_q query
// tokens of hq heads each, read from and written to a per-sequence row stride with a row
// offset (a launch handles at most 128 rows), and each row's valid columns end at its
// query's causal window; a row (or a piece) that sees no token gets out 0, lse -inf.
//
// Every mbarrier wait is bounded by a time limit; on expiry the kernel records
// MLA_ERR_DEVICE_TIMEOUT, tells the peer CTA to stop, drains its own TMA, bulk-copy
// and MMA work, frees TMEM and returns.  No trap.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "mla_device.cuh"
#include "mla_internal.h"
#include "sm100_ptx.cuh"
#include "worker_range.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int kThreads = 384;
constexpr int kStages = 4;
constexpr int kLatBox = 64 * 128;                 // [64 rows x 64 bf16], 128B swizzle
constexpr int kRopeBox = 64 * 64;                 // [64 rows x 32 bf16], 64B swizzle
constexpr int kStageBytes = 4 * kLatBox + kRopeBox;  // 36864
constexpr int kXRow = 64 * 3;                     // one head row of partial scores, 24 bits per value
constexpr int kXBytes = 128 * kXRow;              // 24576: [128 heads x 64 tokens] partial scores
constexpr int kSmemTx = kStages * kStageBytes;                // 147456: send buffer
constexpr int kSmemRx = kSmemTx + kXBytes;                    // 172032: 2 receive buffers
constexpr int kSmemBytes = kSmemRx + 2 * kXBytes;             // 221184
constexpr int kSmemAlloc = kSmemBytes + 1024;                 // + alignment slack
// Every region lies inside the allocation, and the allocation, with the kernel's static
// shared memory (under 4 KB), inside the 227 KB a CTA may have.
static_assert(kStages * kStageBytes <= kSmemTx && kSmemTx + kXBytes <= kSmemRx && kSmemRx + 2 * kXBytes <= kSmemBytes,
              "shared-memory regions overlap or leave the allocation");
static_assert(kSmemAlloc + 4096 <= 232448, "dynamic + static shared memory above the per-CTA limit");
static_assert(kStageBytes % 1024 == 0, "swizzled stage tiles must start on 1024-byte boundaries");

constexpr uint32_t kTmemCols = 512;
// O fp32 [0,256); q' (latent 256 dims, then this CTA's 32 rope dims) as bf16 pairs
// [256,400); S fp32 [400,464); P bf16 pairs [464,496).
constexpr uint32_t kColO = 0, kColQ = 256, kColS = 400, kColP = 464;
static_assert(kColO + 256 <= kColQ && kColQ + 144 <= kColS && kColS + 64 <= kColP && kColP + 32 <= kTmemCols,
              "tensor-memory regions overlap or leave the allocation");

constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 64, 0, 0);   // A (q', TMEM), B K-major
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 256, 0, 1);  // A (P, TMEM), B MN-major

constexpr float kRescaleThreshold = 8.0f;  // log2 units: P may reach 2^8 before O is rescaled
constexpr int kPrefetch = 4;               // pages pulled into L2 ahead of the stage loads

enum Bar {
  kKvFull = 0,
  kKvEmpty = kKvFull + kStages,
  kVReady = kKvEmpty + kStages,
  kSFull = kVReady + kStages,
  kSFree = kSFull + 1,
  kPFull = kSFree + 1,
  kRxFull = kPFull + 1,     // [buffer]
  kPeerFree = kRxFull + 2,  // [buffer]
  kTxWritable = kPeerFree + 2,
  kTxReady = kTxWritable + 1,
  kRxRead = kTxReady + 1,  // [page parity] every softmax warp has read receive buffer u
  kODone = kRxRead + 2,    // PV(g) complete: O holds page g, P may be rewritten
  kOFull = kODone + 1,
  kQReady = kOFull + 1,
  kDrain = kQReady + 1,
  kNumBars = kDrain + 1
};

struct Piece {
  int b, pa, pe;
};

// Iterates the sequence pieces of a worker's range in schedule order.
struct PieceIter {
  WorkerRange rg;
  int b;
  __device__ explicit PieceIter(const WorkerRange& r) : rg(r), b(r.b0) {}
  // The lengths are passed at each call, so the iterator holds no copy of them.
  __device__ bool next(Piece& pc, const int32_t* seqlens, int max_blocks) {
    if (rg.b0 < 0) return false;
    while (b <= rg.b1) {
      const int cur = b++;
      const int n = seq_pages(seqlens, max_blocks, cur);
      const int pa = (cur == rg.b0) ? rg.p0 : 0;
      const int pe = (cur == rg.b1) ? rg.p1 : n;
      if (pa < pe) {
        pc = {cur, pa, pe};
        return true;
      }
    }
    return false;
  }
};

__device__ __forceinline__ uint64_t now_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

struct Ctl {
  int* err;
  volatile int* abort;     // this CTA's abort flag
  uint32_t peer_abort;     // the peer's abort flag (cluster address)
  uint64_t limit_ns;
};

// Records a timed-out wait: the error word, this CTA's abort flag and the peer's.
__device__ __noinline__ void wait_timed_out(int* err, volatile int* abort, uint32_t peer_abort) {
  set_device_error(err, MLA_ERR_DEVICE_TIMEOUT);
  *abort = 1;
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(peer_abort), "r"(1) : "memory");
}

// Bounded wait on a local mbarrier phase; on timeout or abort returns false.  Inline
// and small: try_wait suspends the thread until the phase completes or a hardware
// time limit passes; only every 64th probe reads the abort flag and the global timer
// (the start time is taken at the first such check), and the timeout itself is a call.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, const Ctl& c) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = 0;
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63) == 0) {
      if (*c.abort) return false;
      const uint64_t t = now_ns();
      if (t0 == 0) {
        t0 = t;
      } else if (t - t0 > c.limit_ns) {
        wait_timed_out(c.err, c.abort, c.peer_abort);
        return false;
      }
    }
  }
}

// Spin (bounded by time, ignoring the abort flag) until a phase completes: used only
// while draining work that is already in flight.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = now_ns();
  while (!mbar_try_wait(bar, parity) && now_ns() - t0 < limit_ns) {
  }
}

__device__ __forceinline__ int page_of(const DecodeArgs& a, int b, int p) {
  return a.block_table ? a.block_table[(size_t)b * a.max_blocks + p] : b * a.max_blocks + p;
}

// kCausal: the rows of a sequence are several query tokens (DecodeArgs::s_q > 1),
// each row masked to its query's window.
template <bool kCausal>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap kv_map, const __grid_constant__ CUtensorMap rope_map,
                     const DecodeArgs a, uint64_t limit_ns) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[kNumBars];
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;
  __shared__ RangeScratch range_s;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t s_tx = sbase + kSmemTx, s_rx = sbase + kSmemRx;
  auto bar = [&](int i) { return smem_u32(&bars[i]); };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int w = blockIdx.x >> 1;
  const Schedule& sc = a.sched;
  const int P = sc.num_workers;
  const int np = a.block_table ? a.num_pages : a.batch * a.max_blocks;

  if (tid == 0) {
    abort_s = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(kKvFull + s), 1);
      mbar_init(bar(kKvEmpty + s), 1);
      mbar_init(bar(kVReady + s), 1);
    }
    mbar_init(bar(kSFull), 1);      // MMA commit
    mbar_init(bar(kSFree), 8);      // every softmax warp has loaded its half of S
    mbar_init(bar(kPFull), 8);      // one arrival per softmax warp
    for (int u = 0; u < 2; ++u) {
      mbar_init(bar(kRxFull + u), 1);     // armed (expect_tx) here, bytes from the peer
      mbar_init(bar(kPeerFree + u), 1);   // the peer's receive buffer u is read and re-armed
    }
    mbar_init(bar(kTxWritable), 1);
    mbar_init(bar(kTxReady), 8);
    for (int u = 0; u < 2; ++u) mbar_init(bar(kRxRead + u), 8);
    mbar_init(bar(kODone), 1);
    mbar_init(bar(kOFull), 1);
    mbar_init(bar(kQReady), 8);     // every softmax warp has staged its part of q'
    mbar_init(bar(kDrain), 1);
    // Both receive buffers are armed (pages 0 and 1) before the peer may send.
    mbar_expect_tx(bar(kRxFull + 0), kXBytes);
    mbar_expect_tx(bar(kRxFull + 1), kXBytes);
    fence_mbar_init();
    tma_prefetch_desc(&kv_map);
    tma_prefetch_desc(&rope_map);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_base_s), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // barriers of both CTAs initialised before any remote arrive
  tc_fence_after();
  // Everything above overlaps the previous grid on the stream; from here on its writes
  // (the lengths, q, the block table) are visible.
  grid_dep_wait();
  // Every thread takes part in deriving this worker's page range (and this CTA's share of
  // the sequence records the combine reads).
  derive_worker_range(a.seqlens, a.batch, a.max_blocks, a.sched.num_workers, a.min_pages, a.granule,
                      a.whole_slack, a.piece_cost, a.sched.seq, a.err, w, range_s);
  // Each role reads the range from shared memory where it starts (volatile, so the
  // read is not hoisted and the range is not held in registers across the kernel).
  auto rg_load = [&]() {
    const volatile WorkerRange& v = range_s.rg;
    return WorkerRange{v.b0, v.p0, v.b1, v.p1};
  };
  const uint32_t tmem = tmem_base_s;
  Ctl ctl{a.err, &abort_s, map_to_rank(smem_u32(&abort_s), peer), limit_ns};

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      PieceIter pi(rg_load());
      Piece pc;
      int it = 0;
      bool ok = true;
      // A second walk over the same pages runs kPrefetch pages ahead and pulls this
      // CTA's part of each page into L2, so the loads into the stage ring (whose
      // depth is bounded by shared memory) see L2 rather than HBM latency.
      PieceIter pf(rg_load());
      Piece fc;
      bool fvalid = pf.next(fc, a.seqlens, a.max_blocks);
      int fp = fvalid ? fc.pa : 0;
      auto prefetch_next = [&]() {
        if (!fvalid) return;
        const int pid = page_of(a, fc.b, fp);
        if ((unsigned)pid < (unsigned)np) {
          const int y = pid * kPage;
#pragma unroll
          for (int i = 0; i < 4; ++i) tma_prefetch_l2_2d(&kv_map, 256 * rank + 64 * i, y);
          tma_prefetch_l2_2d(&rope_map, kDLatent + 32 * rank, y);
        }
        if (++fp >= fc.pe) {
          fvalid = pf.next(fc, a.seqlens, a.max_blocks);
          fp = fvalid ? fc.pa : 0;
        }
      };
      for (int i = 0; i < kPrefetch; ++i) prefetch_next();
      while (ok && pi.next(pc, a.seqlens, a.max_blocks)) {
        for (int p = pc.pa; p < pc.pe; ++p, ++it) {
          const int s = it % kStages;
          int pid = page_of(a, pc.b, p);  // table read issued before the wait, off the critical path
          prefetch_next();
          if (!wait_bar(bar(kKvEmpty + s), ((it / kStages) & 1) ^ 1, ctl)) { ok = false; break; }
          if ((unsigned)pid >= (unsigned)np) pid = 0;  // reported by the softmax warps; load something valid
          if (a.withhold_arrive && w == 0 && rank == 0 && it == 1) continue;  // timeout test: never arrives
          const uint32_t dst = sbase + s * kStageBytes;
          mbar_expect_tx(bar(kKvFull + s), kStageBytes);
          const int y = pid * kPage;
#pragma unroll
          for (int i = 0; i < 4; ++i) tma_load_2d(dst + i * kLatBox, &kv_map, 256 * rank + 64 * i, y, bar(kKvFull + s));
          tma_load_2d(dst + 4 * kLatBox, &rope_map, kDLatent + 32 * rank, y, bar(kKvFull + s));
        }
      }
      // Drain: every load issued into a stage lands before the CTA may exit (bounded).
      for (int k = 0; k < kStages && k < it; ++k) {
        const int j = it - 1 - k;
        if (a.withhold_arrive && w == 0 && rank == 0 && j == 1) continue;
        drain_wait(bar(kKvFull + j % kStages), (j / kStages) & 1, limit_ns);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      PieceIter pi(rg_load());
      Piece pc;
      int it = 0, piece = 0;
      bool ok = true;
      auto do_qk = [&](int g) {
        const int s = g % kStages;
        tc_fence_after();
        const uint32_t kbase = sbase + s * kStageBytes;
        const uint32_t d = tmem + kColS;
#pragma unroll
        for (int kc = 0; kc < 16; ++kc)
          mma_ts(d, tmem + kColQ + kc * 8, desc_sw128(kbase + (kc >> 2) * kLatBox + (kc & 3) * 32, 16, 1024),
                 kIdescQK, kc > 0 ? 1u : 0u);
#pragma unroll
        for (int i = 0; i < 2; ++i)
          mma_ts(d, tmem + kColQ + 128 + i * 8, desc_sw64(kbase + 4 * kLatBox + i * 32, 16, 512), kIdescQK, 1u);
        mma_commit(bar(kSFull));
      };
      auto do_pv = [&](int g, bool first) {
        const int s = g % kStages;
        tc_fence_after();
        const uint32_t vbase = sbase + s * kStageBytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ts(tmem + kColO, tmem + kColP + kk * 8, desc_sw128(vbase + kk * 2048, 8192, 1024), kIdescPV,
                 (first && kk == 0) ? 0u : 1u);
        mma_commit(bar(kKvEmpty + s));
        // The next completion of ODone after PV(g) is PV(g+1), which needs P(g+1),
        // which is written only after every softmax warp has seen PV(g) done.
        mma_commit(bar(kODone));
      };
      // Issues whichever is ready first: the next score MMA (its S buffer freed and its
      // page loaded) or the next PV (its P written and its value rows cleaned), so score
      // MMAs run up to two pages ahead and never queue behind a PV that waits for the
      // softmax.  When neither is ready the thread sleeps (a bounded, hinted try_wait)
      // on the barrier of the next event: the next P, or the S buffer or page of the
      // next score MMA, leaving the issue slots to the softmax warps.
      auto qk_ready = [&](int g) {
        return (g < 1 || mbar_test(bar(kSFree), (g - 1) & 1)) &&
               mbar_test(bar(kKvFull + g % kStages), (g / kStages) & 1);
      };
      auto pv_ready = [&](int g) {
        return mbar_test(bar(kPFull), g & 1) &&
               mbar_test(bar(kVReady + g % kStages), (g / kStages) & 1);
      };
      while (ok && pi.next(pc, a.seqlens, a.max_blocks)) {
        if (!wait_bar(bar(kQReady), piece & 1, ctl)) { ok = false; break; }
        const int n = pc.pe - pc.pa, end = it + n;
        int gq = it, gp = it;
        uint64_t idle_since = 0;
        uint32_t idle = 0;
        while (gp < end) {
          // PV first: it frees a stage (stage residency bounds the page rate) and the
          // tensor pipe runs MMAs in issue order.
          bool prog = false;
          if (gp < gq && pv_ready(gp)) {
            do_pv(gp, gp == it);
            ++gp;
            prog = true;
          }
          if (gq < end && qk_ready(gq)) {
            do_qk(gq++);
            prog = true;
          }
          if (prog) {
            idle_since = 0;
            idle = 0;
            continue;
          }
          if (gp < gq) {
            mbar_try_wait_hint(bar(kPFull), gp & 1, 100);
          } else if (gq >= 1 && !mbar_test(bar(kSFree), (gq - 1) & 1)) {  // next: QK(gq)
            mbar_try_wait_hint(bar(kSFree), (gq - 1) & 1, 100);
          } else {
            mbar_try_wait_hint(bar(kKvFull + gq % kStages), (gq / kStages) & 1, 100);
          }
          if ((++idle & 15) != 0) continue;
          if (abort_s) { ok = false; break; }
          const uint64_t t = now_ns();
          if (idle_since == 0) {
            idle_since = t;
          } else if (t - idle_since > limit_ns) {
            set_device_error(a.err, MLA_ERR_DEVICE_TIMEOUT);
            abort_s = 1;
            asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(ctl.peer_abort), "r"(1) : "memory");
            ok = false;
            break;
          }
        }
        if (!ok) break;
        mma_commit(bar(kOFull));
        it += n;
        ++piece;
      }
      // Drain every MMA this thread issued before TMEM is released.
      mma_commit(bar(kDrain));
      drain_wait(bar(kDrain), 0, limit_ns);
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------------------ tail rows of V,
    // and receive buffers handed back to the peer
    const uint32_t peer_free = map_to_rank(bar(kPeerFree), peer);
    PieceIter pi(rg_load());
    Piece pc;
    int it = 0;
    bool ok = true;
    while (ok && pi.next(pc, a.seqlens, a.max_blocks)) {
      const int T = a.seqlens[pc.b];
      for (int p = pc.pa; p < pc.pe; ++p, ++it) {
        const int s = it % kStages;
        if (!__all_sync(0xffffffffu, wait_bar(bar(kKvFull + s), (it / kStages) & 1, ctl))) { ok = false; break; }
        const int valid = min(kPage, T - p * kPage);
        if (valid < kPage) {
          // Rows >= valid may hold anything (NaN included); P is 0 there but 0 * NaN is
          // NaN, so zero them in the four value boxes before PV reads the stage.
          uint8_t* st = smem + s * kStageBytes;
          const int nrow = kPage - valid;
          for (int idx = lane; idx < nrow * 4 * 8; idx += 32) {
            const int box = idx / (nrow * 8), rem = idx % (nrow * 8);
            const int row = valid + rem / 8, chunk = rem % 8;
            *reinterpret_cast<uint4*>(st + box * kLatBox + row * 128 + chunk * 16) = make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kVReady + s));
        // Every softmax warp has read receive buffer u: re-arm it for page it+2 and let
        // the peer send.  RxRead is per page parity, so its next completion on this
        // parity needs page it+2, which the peer can only send after this: the wait
        // cannot fall behind.
        const int u = it & 1;
        if (!__all_sync(0xffffffffu, wait_bar(bar(kRxRead + u), (it >> 1) & 1, ctl))) { ok = false; break; }
        if (lane == 0) {
          mbar_expect_tx(bar(kRxFull + u), kXBytes);
          mbar_arrive_cluster(peer_free + u * 8);
        }
      }
    }
  } else if (warp == 3) {
    // ------------------------------------------------------------ score sender:
    // copies each page's packed partial scores into the peer's receive buffer
    if (lane == 0) {
      const uint32_t rx_peer = map_to_rank(s_rx, peer);
      const uint32_t peer_rx_full = map_to_rank(bar(kRxFull), peer);
      mbar_arrive(bar(kTxWritable));  // the send buffer starts free
      PieceIter pi(rg_load());
      Piece pc;
      int it = 0;
      bool ok = true;
      while (ok && pi.next(pc, a.seqlens, a.max_blocks)) {
        for (int p = pc.pa; p < pc.pe; ++p, ++it) {
          // All 8 softmax warps wrote their rows, and the peer has read page it-2 out of
          // its receive buffer u and re-armed it (both buffers start armed).
          const int u = it & 1, k = it >> 1;
          if (!wait_bar(bar(kTxReady), it & 1, ctl) || !wait_bar(bar(kPeerFree + u), (k & 1) ^ 1, ctl)) {
            ok = false;
            break;
          }
          bulk_copy_to_peer(rx_peer + u * kXBytes, s_tx, kXBytes, peer_rx_full + u * 8);
          bulk_wait_read_all();           // the copy has read the send buffer
          mbar_arrive(bar(kTxWritable));  // the softmax may write the next page into it
        }
      }
      bulk_wait_all();  // our copies into the peer have landed
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax warps
    // Each softmax warp owns 16 head rows (TMEM lanes) of its lane quadrant and all 64
    // score columns of every page.  In the 16x32bx2 access shape thread t holds row
    // (t mod 16) and column half t / 16, so both halves of a row sit in one warp and
    // their maxima and sums meet through one shuffle.
    const int sw = warp - 4;               // softmax warp 0..7
    const int wg = sw >> 2;                // which 16 lanes of the quadrant (and which half of q')
    const int q = warp & 3;                // lane quadrant of this warp
    const int ch = lane >> 4;              // column half of the row held by this thread
    const int row = 32 * q + 16 * wg + (lane & 15);                 // head row = TMEM lane
    const uint32_t lane_off = (uint32_t)(32 * q + 16 * wg) << 16;  // first of this warp's 16 lanes
    const uint32_t t_o = tmem + lane_off + kColO;  // O rows: this thread's 128 columns start 128 ch on
    const uint32_t t_p = tmem + lane_off + kColP;  // P rows: this thread's 16 columns start 16 ch on
    // q' is staged with 32x32b stores (thread = lane of the quadrant); the two warps of
    // a quadrant split its latent columns.
    const int qrow = 32 * q + lane;
    const uint32_t qlane_off = (uint32_t)(32 * q) << 16;
    const uint32_t t_q = tmem + qlane_off + kColQ + 64 * wg;
    // Scores stay unscaled (raw q'.k) until the exponent: a negative scale is moved
    // into q' as an exact sign flip, so max over raw scores is max over scaled ones
    // and each P costs one FFMA and one EX2.
    const float scale2 = fabsf(a.scale) * kLog2e;
    const uint32_t qsign = a.scale < 0.f ? 0x80008000u : 0u;
    const float thr_raw = scale2 > 0.f ? kRescaleThreshold / scale2 : INFINITY;
    uint8_t* txrow = smem + kSmemTx + row * kXRow;
    const int sw2 = (row >> 1) & 3;  // chunk swizzle of 192-byte rows: XOR keeps groups of 4 chunks
    PieceIter pi(rg_load());
    Piece pc;
    int it = 0, piece = 0;
    bool ok = true;
    float cur[32], nxt[32];  // scores of the page being finished / of the next page

    // Stage A of global page g: load this thread's half of the partial scores, free
    // the S buffer, and send them to the peer.
    auto stage_a = [&](int g, float (&own)[32]) -> bool {
      if (!__all_sync(0xffffffffu, wait_bar(bar(kSFull), g & 1, ctl))) return false;
      tc_fence_after();
      uint32_t r0[32];
      tmem_ld16x2_32<32>(tmem + lane_off + kColS, r0);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kSFree));  // one arrival per warp: 32 on one word would serialise
#pragma unroll
      for (int c = 0; c < 32; ++c) own[c] = __uint_as_float(r0[c]);
      // The previous page's copy out of the send buffer has finished reading it.
      if (!__all_sync(0xffffffffu, wait_bar(bar(kTxWritable), g & 1, ctl))) return false;
      // Each value is sent as the top 3 bytes of its fp32 pattern: 4 values a, b, c, d
      // travel as the words (low byte first) [d1 a1 a2 a3] [d2 b1 b2 b3] [d3 c1 c2 c3],
      // i.e. a, b and c with their lowest byte replaced by one byte of d; 32 values
      // are 6 chunks.
      {
        uint32_t wd[24];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          wd[3 * e + 0] = __byte_perm(r0[4 * e + 0], r0[4 * e + 3], 0x3215);
          wd[3 * e + 1] = __byte_perm(r0[4 * e + 1], r0[4 * e + 3], 0x3216);
          wd[3 * e + 2] = __byte_perm(r0[4 * e + 2], r0[4 * e + 3], 0x3217);
        }
#pragma unroll
        for (int c = 0; c < 6; ++c)
          *reinterpret_cast<uint4*>(txrow + (((6 * ch + c) ^ sw2) * 16)) =
              make_uint4(wd[4 * c], wd[4 * c + 1], wd[4 * c + 2], wd[4 * c + 3]);
      }
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kTxReady));
      return true;
    };

    while (ok && pi.next(pc, a.seqlens, a.max_blocks)) {
      const int b = pc.b, n = pc.pe - pc.pa;
      const int T = a.seqlens[b];
      // Tokens this row attends to: all T, or its query token's causal window.
      const int Tq = kCausal && row < a.heads ? T - (a.s_q - 1 - (a.row0 + row) / a.hq) : T;
      // ---- stage q' for this sequence into TMEM: this CTA's latent half (split
      // between the two warps of each lane quadrant) and its 32 rope dims
      {
        uint32_t qv[16];
        const bool live = qrow < a.heads;
        const size_t qbase = kCausal ? (size_t)b * a.row_stride + a.row0 : (size_t)b * a.heads;
        const uint4* src = reinterpret_cast<const uint4*>(a.q + (qbase + (live ? qrow : 0)) * kDQK);
#pragma unroll
        for (int c = 0; c < 4; ++c) {  // 4 x 32 dims of this warp's 128 latent dims
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint4 v = live ? src[32 * rank + 16 * wg + 4 * c + k] : make_uint4(0, 0, 0, 0);
            qv[4 * k + 0] = v.x ^ qsign;
            qv[4 * k + 1] = v.y ^ qsign;
            qv[4 * k + 2] = v.z ^ qsign;
            qv[4 * k + 3] = v.w ^ qsign;
          }
          tmem_st16(t_q + c * 16, qv);
        }
        if (wg == 0) {  // this CTA's 32 rope dims: 16 columns after the latent ones
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint4 v = live ? src[kDLatent / 8 + 4 * rank + k] : make_uint4(0, 0, 0, 0);
            qv[4 * k + 0] = v.x ^ qsign;
            qv[4 * k + 1] = v.y ^ qsign;
            qv[4 * k + 2] = v.z ^ qsign;
            qv[4 * k + 3] = v.w ^ qsign;
          }
          tmem_st16(tmem + qlane_off + kColQ + 128, qv);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kQReady));
      }
      float m = -INFINITY, l = 0.f;  // running max of raw scores, running sum
      bool bad = false;
      int pid_next = page_of(a, b, pc.pa);
      // Stage B of page j of this piece: add the peer's partial, online softmax, write P.
      auto stage_b = [&](int j, float (&x)[32]) -> bool {
        const int g = it + j, u = g & 1, k = g >> 1, p = pc.pa + j;
        if (!__all_sync(0xffffffffu, wait_bar(bar(kRxFull + u), k & 1, ctl))) return false;
        {
          const uint8_t* rxrow = smem + kSmemRx + u * kXBytes + row * kXRow;
          uint32_t wd[24];
#pragma unroll
          for (int c = 0; c < 6; ++c) {
            const uint4 v = *reinterpret_cast<const uint4*>(rxrow + (((6 * ch + c) ^ sw2) * 16));
            wd[4 * c] = v.x;
            wd[4 * c + 1] = v.y;
            wd[4 * c + 2] = v.z;
            wd[4 * c + 3] = v.w;
          }
          // Each word read as an fp32 pattern is its value with the lowest mantissa
          // byte replaced by another value's byte: relative error below 2^-15.  d is
          // rebuilt as [d1 d1 d2 d3] (low byte first), with the same bound.
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const uint32_t w0 = wd[3 * e], w1 = wd[3 * e + 1], w2 = wd[3 * e + 2];
            const uint32_t t = __byte_perm(w0, w1, 0x4000);  // [d1 d1 d1 d2]
            const float d = __uint_as_float(__byte_perm(t, w2, 0x4310));
            const uint64_t s01 = f2_add(f2_pack(x[4 * e], x[4 * e + 1]), f2_pack(__uint_as_float(w0), __uint_as_float(w1)));
            const uint64_t s23 = f2_add(f2_pack(x[4 * e + 2], x[4 * e + 3]), f2_pack(__uint_as_float(w2), d));
            f2_unpack(s01, x[4 * e], x[4 * e + 1]);
            f2_unpack(s23, x[4 * e + 2], x[4 * e + 3]);
          }
        }
        const int pid = pid_next;
        if ((unsigned)pid >= (unsigned)np) {
          bad = true;
          set_device_error(a.err, MLA_ERR_DEVICE_BAD_PAGE);
        }
        const int valid = min(kPage, Tq - p * kPage) - 32 * ch;  // valid columns of this half
        const bool ragged = valid < 32;                          // only a sequence's last page
        if (ragged) {
#pragma unroll
          for (int c = 0; c < 32; ++c) x[c] = c < valid ? x[c] : -INFINITY;
        }
        // max is exact, so a tree of three-input maxima gives the same value as a chain
        float m11[11];
#pragma unroll
        for (int c = 0; c < 10; ++c) m11[c] = fmax3(x[3 * c], x[3 * c + 1], x[3 * c + 2]);
        m11[10] = fmaxf(x[30], x[31]);
        const float hm = fmaxf(fmax3(fmax3(m11[0], m11[1], m11[2]), fmax3(m11[3], m11[4], m11[5]),
                                     fmax3(m11[6], m11[7], m11[8])),
                               fmaxf(m11[9], m11[10]));  // depends on every value read from the receive buffer
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kRxRead + u));
        // The next page's table entry is read here, right after a release (an arrive
        // with release semantics waits for this thread's outstanding loads), so the
        // read overlaps the exponentials and is back before the next release.
        if (j + 1 < n) pid_next = page_of(a, b, p + 1);
        const float tmax = fmaxf(hm, __shfl_xor_sync(0xffffffffu, hm, 16));
        const float m_new = fmaxf(m, tmax);
        const bool need = !(m_new <= m + thr_raw);  // also true while m is -inf
        const float alpha = !need ? 1.f : (m == -INFINITY ? 0.f : fast_exp2((m - m_new) * scale2));
        if (need) m = m_new;
        if (__any_sync(0xffffffffu, need && j > 0)) {
          // O must hold PV(g-1) before it is rescaled (rare path).
          if (!__all_sync(0xffffffffu, wait_bar(bar(kODone), (g - 1) & 1, ctl))) return false;
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            tmem_ld16x2_32<128>(t_o + c * 32, r);
            tmem_wait_ld();
            uint32_t w0[16], w1[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              w0[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
              w1[e] = __float_as_uint(__uint_as_float(r[16 + e]) * alpha);
            }
            tmem_st16x2_16<128>(t_o + c * 32, w0);
            tmem_st16x2_16<128>(t_o + c * 32 + 16, w1);
          }
          tmem_wait_st();
          tc_fence_before();
        }
        l *= alpha;
        const float ms = m * scale2;
        const uint64_t s2 = f2_pack(scale2, scale2), nms = f2_pack(-ms, -ms);
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          float y0, y1;
          f2_unpack(f2_fma(f2_pack(x[c], x[c + 1]), s2, nms), y0, y1);
          x[c] = fast_exp2(y0);
          x[c + 1] = fast_exp2(y1);
        }
        if (ragged) {  // a zero scale turns -inf into NaN above
#pragma unroll
          for (int c = 0; c < 32; ++c) x[c] = c < valid ? x[c] : 0.f;
        }
        uint64_t a01 = f2_pack(0.f, 0.f), a23 = a01;  // four running sums, two per instruction
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          a01 = f2_add(a01, f2_pack(x[c], x[c + 1]));
          a23 = f2_add(a23, f2_pack(x[c + 2], x[c + 3]));
        }
        float rs0, rs1, rs2, rs3;
        f2_unpack(a01, rs0, rs1);
        f2_unpack(a23, rs2, rs3);
        l += (rs0 + rs1) + (rs2 + rs3);
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) pk[c] = pack_bf16x2(x[2 * c], x[2 * c + 1]);
        // P [128 heads x 64 tokens] as bf16 pairs in TMEM (the PV A operand): this
        // thread's 16 columns of its row.  The columns were last read by PV(g-1).
        if (g >= 1 && !__all_sync(0xffffffffu, wait_bar(bar(kODone), (g - 1) & 1, ctl))) return false;
        tc_fence_after();
        tmem_st16x2_16<16>(t_p, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kPFull));
        return true;
      };
      // Step j sends page j's partial (stage A) and finishes page j-1 (stage B); each
      // stage is inlined once and the register arrays rotate.
      for (int j = 0; j <= n && ok; ++j) {
        if (j < n && !(ok = stage_a(it + j, nxt))) break;
        if (j > 0 && !(ok = stage_b(j - 1, cur))) break;
#pragma unroll
        for (int c = 0; c < 32; ++c) cur[c] = nxt[c];
      }
      if (!ok) break;
      // ---- epilogue: O / l (this thread's 128 of the CTA's 256 dims), lse
      if (!__all_sync(0xffffffffu, wait_bar(bar(kOFull), piece & 1, ctl))) { ok = false; break; }
      tc_fence_after();
      const float l_row = l + __shfl_xor_sync(0xffffffffu, l, 16);
      // A causal row can see no token of a piece (or of its sequence): out 0, lse -inf.
      const bool none = kCausal && l_row == 0.f;
      const float inv = bad ? NAN : (none ? 0.f : 1.f / l_row);
      const float lse_v = bad ? NAN : (none ? -INFINITY : (m * scale2 + __log2f(l_row)) * kLn2);
      const bool complete = pc.pa == 0 && pc.pe == seq_pages(a.seqlens, a.max_blocks, b);
      float* obase;
      float* lbase;
      if (complete) {
        const size_t rbase = kCausal ? (size_t)b * a.row_stride + a.row0 : (size_t)b * a.heads;
        obase = a.out + rbase * kDLatent;
        lbase = a.lse + rbase;
      } else {
        const int slot = (b == pi.rg.b0) ? w : P + w;
        obase = sc.part_o + (size_t)slot * a.heads * kDLatent;
        lbase = sc.part_lse + (size_t)slot * a.heads;
      }
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld16x2_32<128>(t_o + c * 32, r);
        tmem_wait_ld();
        if (row < a.heads) {
          float4* dst = reinterpret_cast<float4*>(obase + (size_t)row * kDLatent + 256 * rank + 128 * ch + 32 * c);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(__uint_as_float(r[4 * e]) * inv, __uint_as_float(r[4 * e + 1]) * inv,
                                 __uint_as_float(r[4 * e + 2]) * inv, __uint_as_float(r[4 * e + 3]) * inv);
        }
      }
      if (rank == 0 && ch == 0 && row < a.heads) lbase[row] = lse_v;
      tc_fence_before();
      it += n;
      ++piece;
    }
  }

  // ------------------------------------------------------------ teardown
  if (tid == 0) grid_dep_launch_dependents();  // the combine grid may launch (it waits for this grid's writes)
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer no longer writes into this CTA's shared memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

int decode_tc_max_workers(int sm_count) {
  static int cached_dev[64];
  static bool have[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  if (!have[dev]) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (sm_count / 2), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemAlloc;
    cudaFuncSetAttribute(decode_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc);
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, decode_tc_kernel<false>, &cfg) != cudaSuccess || clusters <= 0)
      clusters = sm_count / 2;
    cached_dev[dev] = clusters;
    have[dev] = true;
  }
  return cached_dev[dev];
}

cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t stream) {
  static bool done1[64] = {}, done2[64] = {};
  cudaError_t e = allow_dynamic_smem(reinterpret_cast<const void*>(decode_tc_kernel<false>), kSmemAlloc, done1);
  if (e == cudaSuccess) e = allow_dynamic_smem(reinterpret_cast<const void*>(decode_tc_kernel<true>), kSmemAlloc, done2);
  if (e != cudaSuccess) return e;
  auto encode = tensor_map_encoder();
  if (!encode) return cudaErrorNotSupported;
  // The cache as a 2-D tensor [rows, 576]: latent boxes of 64 dims (128B swizzle) and
  // rope boxes of 32 dims (64B swizzle), 64 rows (one page) each.
  CUtensorMap kv_map, rope_map;
  const uint64_t rows = (uint64_t)(a.block_table ? a.num_pages : a.batch * a.max_blocks) * kPage;
  cuuint64_t dims[2] = {(cuuint64_t)kDQK, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kDQK * 2};
  cuuint32_t estr[2] = {1, 1};
  cuuint32_t box_lat[2] = {64, 64};
  cuuint32_t box_rope[2] = {32, 64};
  CUresult r = encode(&kv_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<__nv_bfloat16*>(a.kv), dims, strides,
                      box_lat, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  r = encode(&rope_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<__nv_bfloat16*>(a.kv), dims, strides,
             box_rope, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  const uint64_t limit_ns = (uint64_t)(a.wait_limit > 0 ? a.wait_limit : 1000) * 1000000ull;  // wait_limit in ms
  // Launched as a programmatic dependent of whatever precedes it on the stream (the
  // previous call's combine, or the grid that wrote q'): the prologue (barrier set-up,
  // TMEM allocation, descriptor prefetch) overlaps that grid's tail.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * a.sched.num_workers, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemAlloc;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return a.s_q > 1 ? cudaLaunchKernelEx(&cfg, decode_tc_kernel<true>, kv_map, rope_map, a, limit_ns)
                   : cudaLaunchKernelEx(&cfg, decode_tc_kernel<false>, kv_map, rope_map, a, limit_ns);
}

}  // namespace mla
