// Split-KV absorbed-MLA decode with pair-wide (cta_group::2) tcgen05 MMAs.
//
// Work split.  One worker = one CTA pair (a 2-CTA cluster) walking a page range of
// the split schedule, four 64-token pages (256 tokens) per step.  The 128 query rows
// (heads) are split between the pair: CTA r owns rows [64r, 64r+64).  Both
// contractions of a step are pair-wide MMAs issued by CTA 0 with M = 128 rows, 64 in
// each CTA:
//     S[128 x 256] = q'[128 x 576] . K^T      B = the step's 256 cached rows; CTA r
//                                              supplies tokens [128r, 128r+128), two
//                                              whole pages, all 576 dims
//     O[128 x 512] += P[128 x 256] . V        two MMAs of N = 256 dims; CTA r supplies
//                                              dims [256j + 128r, +128) of all 256 tokens
// The tensor cores of the pair exchange each CTA's half of B, so no score crosses the
// pair in software: each CTA holds the scores and the output of its own 64 heads and
// runs their softmax alone.  For the value product each CTA reloads its 128-dim half of
// every row the pair fetched for the scores; that second read hits L2 (the rows were
// fetched a few microseconds earlier), so HBM sees every cached byte once.
//
// Tensor memory (pair-wide M = 128: 64 rows per CTA, the N columns of an accumulator
// split in two halves over TMEM lanes 0-63 and 64-127).  In CTA r, lane l < 64 holds
// head 64r + l and the first half of the columns, lane l >= 64 holds head 64r + l - 64
// and the second:
//   [0, 256)    O: block j = [128j, 128j+128) holds dims [256j, 256j+128) in lanes
//               0-63 and dims [256j+128, 256j+256) in lanes 64-127
//   [256, 384)  S of one step: tokens [0,128) in lanes 0-63, [128,256) in lanes 64-127
//   [384, 512)  q' dims [0, 256) as the A operand of the first score MMAs (the pair-wide
//               A layout: lanes l and l + 64 both hold head 64r + (l & 63))
// Shared memory (per CTA): q' dims [256, 576) of the CTA's 64 heads (5 boxes of [64
// rows x 64 dims], 128B swizzle, 40 KB), P of its heads (4 boxes of [64 rows x 64
// tokens]: the A operand of PV, 32 KB), and a ring of 4 slots of four boxes (32 KB): a
// score slot holds two 64-dim column blocks of the CTA's two pages (two 128-row
// K-major B tiles; the rope slot only one), a value slot the CTA's two 128-dim halves
// of one page (MN-major B tiles).
//
// Roles (384 threads per CTA).  Warp 0: TMA producer (q' per piece, then the ring in
// the order the MMAs consume it: scores of step i, then values of step i-1).  Warp 1: TMEM allocation; in CTA 0 the MMA
// issuer.  Warp 2: zeroes the value rows past a sequence's end (P is 0 there but
// 0 * NaN is NaN) in value slots of a ragged last page, which land on a barrier of
// their own CTA.  Warps 4-11: softmax, two warps per TMEM lane quadrant, each owning 64
// of the 128 columns of its 32 lanes: per step, maxima of the four threads holding a
// head meet through shared memory, the lazy reference maximum moves only when a
// step's maximum exceeds it by more than 2^8 (O is then rescaled, after the previous
// PV), P = 2^(y - ref) in bf16 goes to shared memory, and the epilogue writes out / lse
// (or a normalised partial for the combine kernel).
//
// Every mbarrier wait is bounded by a time limit; on expiry the kernel records
// MLA_ERR_DEVICE_TIMEOUT, tells the peer CTA to stop, drains its work in flight and
// returns.  No trap.
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
constexpr int kBox = 8192;              // [64 rows x 64 bf16], 128B swizzle
constexpr int kSlotBytes = 4 * kBox;    // one ring slot: four boxes
constexpr int kSlots = 4;
constexpr int kStepPages = 4;
constexpr int kQKSlots = 5;             // score slots per step: dim blocks (0,1) .. (6,7), then rope
constexpr int kPVSlots = 4;             // value slots per step: one per page
constexpr int kQTmemBoxes = 4;          // q' dims [0, 256) live in tensor memory ...
constexpr int kQSmemBoxes = 5;          // ... dims [256, 576) in shared memory
constexpr int kOffQ = 0;
constexpr int kOffP = kQSmemBoxes * kBox;
constexpr int kOffRing = kOffP + 4 * kBox;
constexpr int kSmemBytes = kOffRing + kSlots * kSlotBytes;  // 204800
constexpr int kSmemAlloc = kSmemBytes + 1024;               // + alignment slack
// Every region lies inside the allocation, and the allocation, with the kernel's static
// shared memory (under 4 KB), inside the 227 KB a CTA may have.
static_assert(kOffQ + kQSmemBoxes * kBox <= kOffP && kOffP + 4 * kBox <= kOffRing &&
                  kOffRing + kSlots * kSlotBytes <= kSmemBytes,
              "shared-memory regions overlap or leave the allocation");
static_assert(kSmemAlloc + 4096 <= 232448, "dynamic + static shared memory above the per-CTA limit");
static_assert(kOffP % 1024 == 0 && kOffRing % 1024 == 0 && kSlotBytes % 1024 == 0 && kBox % 1024 == 0,
              "128B-swizzled tiles must start on 1024-byte boundaries");

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0, kColS = 256, kColQ = 384;
static_assert(kColO + 256 <= kColS && kColS + 128 <= kColQ && kColQ + 2 * kQTmemBoxes * 16 <= kTmemCols,
              "tensor-memory regions overlap or leave the allocation");
constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 256, 0, 0);  // A q' K-major, B rows K-major
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 256, 0, 1);  // A P K-major, B rows MN-major
constexpr uint16_t kBothCtas = 3;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P may reach 2^8 before O is rescaled

enum Bar {
  kFull = 0,                  // [slot] CTA 0: both CTAs' boxes of the slot landed
  kEmpty = kFull + kSlots,    // [slot] both: the MMAs that read the slot are done
  kTFull = kEmpty + kSlots,   // [slot] both: a value slot of a ragged last page landed here
  kTReady = kTFull + kSlots,  // CTA 0: both CTAs zeroed the rows past the sequence end
  kQFull = kTReady + 1,       // CTA 0: q' of both CTAs landed
  kQEmpty = kQFull + 1,       // both: the piece's last score MMA no longer reads q'
  kQReady = kQEmpty + 1,      // CTA 0: the 16 softmax warps staged q' dims [0, 256) in TMEM
  kSFull = kQReady + 1,       // both: a step's scores are in S
  kSFree = kSFull + 1,        // CTA 0: the 16 softmax warps of the pair read S
  kPFull = kSFree + 1,        // CTA 0: the 16 softmax warps wrote P (and rescaled O)
  kODone = kPFull + 1,        // both: a step's PV is done (P may be rewritten)
  kOFull = kODone + 1,        // both: the piece's last PV is done
  kOFree = kOFull + 1,        // CTA 0: the 16 softmax warps read O in the epilogue
  kGroup = kOFree + 1,        // [2] the 4 softmax warps that share a set of heads met
  kDrain = kGroup + 2,
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
  volatile int* abort;  // this CTA's abort flag
  uint32_t peer_abort;  // the peer's abort flag (cluster address)
  uint64_t limit_ns;
};

// Records a timed-out wait: the error word, this CTA's abort flag and the peer's.
__device__ __noinline__ void wait_timed_out(int* err, volatile int* abort, uint32_t peer_abort) {
  set_device_error(err, MLA_ERR_DEVICE_TIMEOUT);
  *abort = 1;
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(peer_abort), "r"(1) : "memory");
}

// Bounded wait on a local mbarrier phase; false on timeout or abort.  try_wait suspends
// the thread until the phase completes or a hardware time limit passes; every 64th probe
// reads the abort flag and the global timer.
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

// wait_bar for the MMA issuer's ring: CTA-scope acquire (the phase is completed by the
// pair's TMA transactions, and only the tensor cores read the data).
__device__ __forceinline__ bool wait_ring(uint32_t bar, uint32_t parity, const Ctl& c) {
  if (mbar_try_wait_cta(bar, parity)) return true;
  return wait_bar(bar, parity, c);
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

// Arrive on a barrier of CTA 0: a CTA-scope release on CTA 0 itself, a cluster-scope
// release (remote arrive) from CTA 1.
__device__ __forceinline__ void arrive_cta0(uint32_t rank, uint32_t local_bar, uint32_t cluster_bar) {
  if (rank == 0) mbar_arrive(local_bar);
  else mbar_arrive_cluster(cluster_bar);
}

// Facts of a piece shared by every role.
struct PieceInfo {
  int steps;    // ceil(pages / 4)
  int tail_pp;  // page (within the sequence) that is a ragged last page of this piece, or -1
  int tail_valid;  // valid rows of that page
};

__device__ __forceinline__ PieceInfo piece_info(const DecodeArgs& a, const Piece& pc) {
  PieceInfo f;
  f.steps = (pc.pe - pc.pa + kStepPages - 1) / kStepPages;
  const int T = a.seqlens[pc.b];
  const int nseq = seq_pages(a.seqlens, a.max_blocks, pc.b);
  f.tail_valid = T & (kPage - 1);
  f.tail_pp = (pc.pe == nseq && f.tail_valid != 0) ? pc.pe - 1 : -1;
  return f;
}

template <bool kCausal>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    decode_pair_kernel(const __grid_constant__ CUtensorMap kv_map, const __grid_constant__ CUtensorMap q_map,
                       const DecodeArgs a, uint64_t limit_ns) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[kNumBars];
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;
  __shared__ RangeScratch range_s;
  __shared__ float mx_s[2][2][2][64];  // [step parity][token half][column half][head]
  __shared__ float lsum_s[2][2][64];   // [token half][column half][head]

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int w = blockIdx.x >> 1;
  const Schedule& sc = a.sched;
  const int P = sc.num_workers;
  const int np = a.block_table ? a.num_pages : a.batch * a.max_blocks;
  const int oob_row = np * kPage;  // a box starting here reads zeros

  if (tid == 0) {
    abort_s = 0;
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(bar(kFull + s), 1);   // CTA 0's producer arms it with both CTAs' bytes
      mbar_init(bar(kEmpty + s), 1);  // MMA commit
      mbar_init(bar(kTFull + s), 1);  // this CTA's producer arms it
    }
    mbar_init(bar(kTReady), 2);
    mbar_init(bar(kQFull), 1);
    mbar_init(bar(kQEmpty), 1);
    mbar_init(bar(kQReady), 16);
    mbar_init(bar(kSFull), 1);
    mbar_init(bar(kSFree), 16);
    mbar_init(bar(kPFull), 16);
    mbar_init(bar(kODone), 1);
    mbar_init(bar(kOFull), 1);
    mbar_init(bar(kOFree), 16);
    for (int u = 0; u < 2; ++u) mbar_init(bar(kGroup + u), 4);
    mbar_init(bar(kDrain), 1);
    fence_mbar_init();
    tma_prefetch_desc(&kv_map);
    tma_prefetch_desc(&q_map);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(&tmem_base_s), kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // barriers and tensor memory of both CTAs ready before any remote access
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
  // Barriers of CTA 0 as cluster addresses (remote arrivals, completions of the pair's loads).
  auto bar0 = [&](int i) { return map_to_rank(bar(i), 0); };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      PieceIter pi(rg_load());
      Piece pc;
      int k = 0, piece = 0;  // ring fills, pieces
      bool ok = true;
      // One ring fill: nbox boxes (x[i], y[i]) into slot k % kSlots once the MMAs have
      // released it.  A value slot of a ragged last page completes on this CTA's own
      // barrier (the zeroing warp cleans it first); every other fill completes on CTA 0's
      // barrier, armed by CTA 0 with the bytes of both CTAs.
      auto fill = [&](const int (&x)[4], const int (&y)[4], int nbox, bool tail) -> bool {
        const int s = k % kSlots;
        if (!wait_bar(bar(kEmpty + s), ((k / kSlots) & 1) ^ 1, ctl)) return false;
        const uint32_t dst = sbase + kOffRing + s * kSlotBytes;
        if (a.withhold_arrive && w == 0 && rank == 0 && k == 1) {  // timeout test: never completes
          ++k;
          return true;
        }
        if (!tail) {
          if (rank == 0) mbar_expect_tx(bar(kFull + s), 2 * nbox * kBox);
          const uint32_t fb = bar0(kFull + s);
          for (int i = 0; i < nbox; ++i) tma_load_2d_pair(dst + i * kBox, &kv_map, x[i], y[i], fb);
        } else {
          mbar_expect_tx(bar(kTFull + s), nbox * kBox);
          for (int i = 0; i < nbox; ++i) tma_load_2d(dst + i * kBox, &kv_map, x[i], y[i], bar(kTFull + s));
          if (rank == 0) mbar_arrive(bar(kFull + s));  // completes the slot's phase without bytes
        }
        ++k;
        return true;
      };
      while (ok && pi.next(pc, a.seqlens, a.max_blocks)) {
        const PieceInfo f = piece_info(a, pc);
        const int b = pc.b;
        // Row y of the piece's page pp (out-of-range page ids and pages past the piece
        // read zeros).
        auto row_of = [&](int pp) -> int {
          if (pp >= pc.pe) return oob_row;
          const int pid = page_of(a, b, pp);
          if ((unsigned)pid >= (unsigned)np) {
            set_device_error(a.err, MLA_ERR_DEVICE_BAD_PAGE);
            return oob_row;
          }
          return pid * kPage;
        };
        // Rows of the pages of steps i-1 (values), i (scores) and i+1 (read a step early,
        // so the block-table loads are never waited for).
        int y_prev[4], y_cur[4], y_next[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          y_cur[p] = row_of(pc.pa + p);
          y_next[p] = row_of(pc.pa + kStepPages + p);
        }
        // q' of this piece, once the previous piece's score MMAs are done with the tile.
        if (!wait_bar(bar(kQEmpty), (piece & 1) ^ 1, ctl)) { ok = false; break; }
        if (rank == 0) mbar_expect_tx(bar(kQFull), 2 * kQSmemBoxes * kBox);
        {
          const int qy = (kCausal ? b * a.row_stride + a.row0 : b * a.heads) + 64 * (int)rank;
          const uint32_t qb = bar0(kQFull);
#pragma unroll 1
          for (int d = 0; d < kQSmemBoxes; ++d)
            tma_load_2d_pair(sbase + kOffQ + d * kBox, &q_map, 64 * (kQTmemBoxes + d), qy, qb);
        }
        for (int i = 0; i <= f.steps && ok; ++i) {
          if (i < f.steps) {
            // scores of step i: dim blocks (2m, 2m+1) of this CTA's two pages, then the
            // rope block; each block's two pages form one 128-row tile
            const int ya = y_cur[2 * rank], yb = y_cur[2 * rank + 1];
#pragma unroll 1
            for (int m = 0; m < kQKSlots && ok; ++m) {
              const int d0 = 2 * m, d1 = m < 4 ? 2 * m + 1 : 2 * m;
              const int x[4] = {64 * d0, 64 * d0, 64 * d1, 64 * d1}, y[4] = {ya, yb, ya, yb};
              ok = fill(x, y, m < 4 ? 4 : 2, false);
            }
          }
          if (i >= 1 && ok) {
            // values of step i-1: this CTA's 128 dims of both dim blocks of each page
#pragma unroll 1
            for (int p = 0; p < 4 && ok; ++p) {
              const int x0 = 128 * (int)rank, yv = y_prev[p];
              const int x[4] = {x0, x0 + 64, 256 + x0, 256 + x0 + 64}, y[4] = {yv, yv, yv, yv};
              ok = fill(x, y, 4, pc.pa + kStepPages * (i - 1) + p == f.tail_pp);
            }
          }
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            y_prev[p] = y_cur[p];
            y_cur[p] = y_next[p];
            y_next[p] = row_of(pc.pa + kStepPages * (i + 2) + p);
          }
        }
        ++piece;
      }
      // Drain: CTA 0 waits for the last fills of each slot it armed (both CTAs' bytes).
      if (rank == 0) {
        for (int j = 0; j < kSlots && j < k; ++j) {
          const int kk = k - 1 - j;
          if (a.withhold_arrive && w == 0 && kk == 1) continue;
          drain_wait(bar(kFull + kk % kSlots), (kk / kSlots) & 1, limit_ns);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (CTA 0)
    // The whole warp runs the issue loop in uniform control flow and one elected lane
    // issues each MMA and commit, so the issue path stays short.
    if (rank == 0) {
      PieceIter pi(rg_load());
      Piece pc;
      int g = 0, piece = 0, tails = 0;
      bool ok = true;
      // Descriptors are built once per operand tile and stepped along K by constant adds
      // (a K-major step of 16 dims is 32 bytes, an MN-major step of 16 tokens 2048 bytes).
      constexpr uint64_t kKMajor = desc_sw128_const(16, 1024), kMNMajor = desc_sw128_const(8192, 1024);
      const uint64_t dq0 = kKMajor | desc_addr(sbase + kOffQ), dp0 = kKMajor | desc_addr(sbase + kOffP);
      const uint32_t ring4 = desc_addr(sbase + kOffRing);
      // The ring position as a slot index and a phase bit.  The value slot of a ragged
      // last page also waits for both CTAs to have zeroed its rows past the sequence end;
      // kTReady completes once per such page, `tails` counts them.
      int slot = 0;
      uint32_t sphase = 0;
      auto take_slot = [&](bool tail) -> bool {
        if (!__all_sync(0xffffffffu, wait_ring(bar(kFull + slot), sphase, ctl))) return false;
        if (tail) {  // the zeroing warps' stores (generic proxy, fenced to the async proxy)
          if (!__all_sync(0xffffffffu, wait_bar(bar(kTReady), tails & 1, ctl))) return false;
          tc_fence_after();
          ++tails;
        }
        return true;
      };
      auto release_slot = [&]() {
        mma_commit_pair_elect(bar(kEmpty + slot), kBothCtas);
        if (++slot == kSlots) {
          slot = 0;
          sphase ^= 1u;
        }
      };
      // Scores of step gs into the one S buffer, once the softmax of step gs - 1 has read
      // it: q' dims [0, 256) from tensor memory, [256, 576) from shared memory.
      auto do_qk = [&](int gs) -> bool {
        if (gs >= 1 && !__all_sync(0xffffffffu, wait_bar(bar(kSFree), (gs - 1) & 1, ctl))) return false;
        tc_fence_after();
        const uint32_t d = tmem + kColS;
#pragma unroll 1
        for (int m = 0; m < kQKSlots; ++m) {
          if (!take_slot(false)) return false;
          const uint64_t bk = kKMajor | (ring4 + slot * (kSlotBytes >> 4));
          if (m < 2) {  // dim blocks 2m, 2m+1 < 4: q' from tensor memory
            mma_pair_ts_x4_elect<2>(d, tmem + kColQ + 64 * m, bk, kIdescQK, m != 0 ? 1u : 0u);
            mma_pair_ts_x4_elect<2>(d, tmem + kColQ + 64 * m + 32, bk + 2 * (kBox >> 4), kIdescQK, 1u);
          } else if (m < 4) {
            const uint64_t aq = dq0 + (uint64_t)((2 * m - kQTmemBoxes) * (kBox >> 4));
            mma_pair_x4_elect<2, 2>(d, aq, bk, kIdescQK, 1u);
            mma_pair_x4_elect<2, 2>(d, aq + (kBox >> 4), bk + 2 * (kBox >> 4), kIdescQK, 1u);
          } else {  // rope block (dims 512..575)
            mma_pair_x4_elect<2, 2>(d, dq0 + (uint64_t)((8 - kQTmemBoxes) * (kBox >> 4)), bk, kIdescQK, 1u);
          }
          release_slot();
        }
        mma_commit_pair_elect(bar(kSFull), kBothCtas);
        return true;
      };
      auto do_pv = [&](int gs, bool first, int step_pp0, int tail_pp) -> bool {
        if (!__all_sync(0xffffffffu, wait_bar(bar(kPFull), gs & 1, ctl))) return false;
        if (first && piece > 0 && !__all_sync(0xffffffffu, wait_bar(bar(kOFree), (piece - 1) & 1, ctl))) return false;
        tc_fence_after();
#pragma unroll 1
        for (int p = 0; p < 4; ++p) {
          if (!take_slot(step_pp0 + p == tail_pp)) return false;
          const uint64_t ap = dp0 + (uint64_t)(p * (kBox >> 4));
          const uint64_t bv = kMNMajor | (ring4 + slot * (kSlotBytes >> 4));
          const uint32_t acc = (first && p == 0) ? 0u : 1u;
          mma_pair_x4_elect<2, 128>(tmem + kColO, ap, bv, kIdescPV, acc);  // dims block 0
          mma_pair_x4_elect<2, 128>(tmem + kColO + 128, ap, bv + 2 * (kBox >> 4), kIdescPV, acc);  // block 1
          release_slot();
        }
        mma_commit_pair_elect(bar(kODone), kBothCtas);
        return true;
      };
      while (ok && pi.next(pc, a.seqlens, a.max_blocks)) {
        const PieceInfo f = piece_info(a, pc);
        if (!__all_sync(0xffffffffu, wait_bar(bar(kQFull), piece & 1, ctl)) ||
            !__all_sync(0xffffffffu, wait_bar(bar(kQReady), piece & 1, ctl))) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int i = 0; i <= f.steps && ok; ++i) {
          if (i < f.steps) {
            ok = do_qk(g + i);
            if (ok && i == f.steps - 1) mma_commit_pair_elect(bar(kQEmpty), kBothCtas);  // q' may be reloaded
          }
          if (i >= 1 && ok) ok = do_pv(g + i - 1, i == 1, pc.pa + kStepPages * (i - 1), f.tail_pp);
        }
        if (!ok) break;
        mma_commit_pair_elect(bar(kOFull), kBothCtas);
        g += f.steps;
        ++piece;
      }
      // Drain every MMA this warp issued before tensor memory is released.
      mma_commit_pair_elect(bar(kDrain), 1);
      drain_wait(bar(kDrain), 0, limit_ns);
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------------------ value rows past a
    // sequence's end, in the value slots of its ragged last page
    PieceIter pi(rg_load());
    Piece pc;
    int k = 0;
    int tcnt[kSlots];
#pragma unroll
    for (int s = 0; s < kSlots; ++s) tcnt[s] = 0;
    bool ok = true;
    const uint32_t tready0 = bar0(kTReady);
    while (ok && pi.next(pc, a.seqlens, a.max_blocks)) {
      const PieceInfo f = piece_info(a, pc);
      for (int i = 0; i <= f.steps && ok; ++i) {
        if (i < f.steps) k += kQKSlots;
        if (i < 1) continue;
        const int pp0 = pc.pa + kStepPages * (i - 1);
        if (f.tail_pp < pp0 || f.tail_pp >= pp0 + 4) {
          k += kPVSlots;
          continue;
        }
        for (int p = 0; p < 4 && ok; ++p, ++k) {
          if (pp0 + p != f.tail_pp) continue;
          const int s = k % kSlots;
          int par = 0;
#pragma unroll
          for (int z = 0; z < kSlots; ++z)
            if (z == s) par = tcnt[z]++ & 1;
          if (!__all_sync(0xffffffffu, wait_bar(bar(kTFull + s), par, ctl))) { ok = false; break; }
          uint8_t* st = smem + kOffRing + s * kSlotBytes;
          const int nrow = kPage - f.tail_valid;
          for (int idx = lane; idx < 4 * nrow * 8; idx += 32) {  // the four boxes of the slot
            const int box = idx / (nrow * 8), rem = idx % (nrow * 8);
            const int row = f.tail_valid + rem / 8, chunk = rem % 8;
            *reinterpret_cast<uint4*>(st + box * kBox + row * 128 + chunk * 16) = make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async();
          __syncwarp();
          if (lane == 0) arrive_cta0(rank, bar(kTReady), tready0);
        }
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax warps
    const int sw = warp - 4;
    const int q = warp & 3;          // TMEM lane quadrant
    const int c = sw >> 2;           // which 64 of the quadrant's 128 columns (and O block)
    const int L = 32 * q + lane;     // TMEM lane
    const int h = L & 63;            // head within this CTA
    const int hh = L >> 6;           // token half of the step held in this lane
    const int row = 64 * (int)rank + h;  // row of the launch
    const uint32_t lane_addr = (uint32_t)(32 * q) << 16;
    // The 4 warps holding the same heads (quadrants q and q+2, both column halves) meet
    // on a group barrier (bounded wait, unlike a named barrier) once per step and once per
    // epilogue; `meets` counts those meetings.
    const uint32_t grp_bar = bar(kGroup + (q & 1));
    int meets = 0;
    auto meet = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(grp_bar);
      const bool r = __all_sync(0xffffffffu, wait_bar(grp_bar, meets & 1, ctl));
      ++meets;
      return r;
    };
    const float scale2 = a.scale * kLog2e;
    const float thr = kRescaleThreshold;
    const uint32_t sfree0 = bar0(kSFree), pfull0 = bar0(kPFull), ofree0 = bar0(kOFree), qready0 = bar0(kQReady);
    uint8_t* prow = smem + kOffP + (2 * hh + c) * kBox + h * 128;
    // q' dims [0, 256) of sequence b's rows into tensor memory (the A operand of the first
    // four score slots), in the pair-wide layout: lane L holds head L & 63, so lanes h and
    // h + 64 hold the same row; column half c stages dims [128c, 128c + 128).  Rows past
    // the launch's heads are zero.
    auto stage_q = [&](int b) {
      const bool live = row < a.heads;
      const size_t grow = (kCausal ? (size_t)b * a.row_stride + a.row0 : (size_t)b * a.heads) + row;
      const uint4* src = reinterpret_cast<const uint4*>(a.q + grow * kDQK + 128 * c);
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4) {
        uint32_t v[16];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint4 x = live ? src[4 * k4 + e] : make_uint4(0, 0, 0, 0);
          v[4 * e] = x.x;
          v[4 * e + 1] = x.y;
          v[4 * e + 2] = x.z;
          v[4 * e + 3] = x.w;
        }
        tmem_st16(tmem + lane_addr + kColQ + 64 * c + 16 * k4, v);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) arrive_cta0(rank, bar(kQReady), qready0);
    };
    PieceIter pi(rg_load()), pn(rg_load());  // pn runs one piece ahead
    Piece pc, nc;
    bool have_next = pn.next(nc, a.seqlens, a.max_blocks);
    if (have_next) stage_q(nc.b);  // the first piece's q' (tensor memory is unused so far)
    int g = 0, piece = 0;
    bool ok = true;

    while (ok && pi.next(pc, a.seqlens, a.max_blocks)) {
      have_next = pn.next(nc, a.seqlens, a.max_blocks);
      const PieceInfo f = piece_info(a, pc);
      const int b = pc.b;
      const int T = a.seqlens[b];
      // Tokens this row attends to: all T, or its query token's causal window.
      const int Tq = kCausal && row < a.heads ? T - (a.s_q - 1 - (a.row0 + row) / a.hq) : T;
      const int tok_end = min(Tq, pc.pe * kPage);
      float m = -INFINITY, l = 0.f;  // reference maximum (log2 units), running sum
      bool bad = false;
      for (int i = 0; i < f.steps && ok; ++i) {
        const int gs = g + i, u = gs & 1;
        // Out-of-range page ids of this step make the sequence NaN (the producer reads
        // zeros for them and records the error).
        {
          const int pp = pc.pa + kStepPages * i + lane;
          bool badp = false;
          if (lane < 4 && pp < pc.pe) badp = (unsigned)page_of(a, b, pp) >= (unsigned)np;
          bad |= __any_sync(0xffffffffu, badp);
        }
        if (!__all_sync(0xffffffffu, wait_bar(bar(kSFull), gs & 1, ctl))) { ok = false; break; }
        tc_fence_after();
        float y[64];
        {
          uint32_t r0[32], r1[32];
          tmem_ld32(tmem + lane_addr + kColS + 64 * c, r0);
          tmem_ld32(tmem + lane_addr + kColS + 64 * c + 32, r1);
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) arrive_cta0(rank, bar(kSFree), sfree0);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            y[j] = __uint_as_float(r0[j]);
            y[32 + j] = __uint_as_float(r1[j]);
          }
        }
        const int lim = tok_end - ((pc.pa + kStepPages * i) * kPage + 128 * hh + 64 * c);  // valid columns
        const uint64_t s2 = f2_pack(scale2, scale2);
#pragma unroll
        for (int j = 0; j < 64; j += 2) {
          float y0, y1;
          f2_unpack(f2_mul(f2_pack(y[j], y[j + 1]), s2), y0, y1);
          y[j] = j < lim ? y0 : -INFINITY;
          y[j + 1] = j + 1 < lim ? y1 : -INFINITY;
        }
        float m22[22];
#pragma unroll
        for (int j = 0; j < 21; ++j) m22[j] = fmax3(y[3 * j], y[3 * j + 1], y[3 * j + 2]);
        m22[21] = y[63];
        float lm = m22[21];
#pragma unroll
        for (int j = 0; j < 21; j += 3) lm = fmaxf(lm, fmax3(m22[j], m22[j + 1], m22[j + 2]));
        mx_s[u][hh][c][h] = lm;
        if (!meet()) { ok = false; break; }
        const float m_step = fmaxf(fmaxf(mx_s[u][0][0][h], mx_s[u][0][1][h]), fmaxf(mx_s[u][1][0][h], mx_s[u][1][1][h]));
        const float m_new = fmaxf(m, m_step);
        const bool need = !(m_new <= m + thr);  // also true while m is -inf and a token is seen
        const float alpha = !need ? 1.f : (m == -INFINITY ? 0.f : fast_exp2(m - m_new));
        if (need) m = m_new;
        bool waited = false;
        if (__any_sync(0xffffffffu, need && i > 0)) {
          // O must hold PV(gs-1) before it is rescaled (rare path).
          if (!__all_sync(0xffffffffu, wait_bar(bar(kODone), (gs - 1) & 1, ctl))) { ok = false; break; }
          waited = true;
          tc_fence_after();
#pragma unroll 1
          for (int cc = 0; cc < 4; ++cc) {
            uint32_t r[32];
            const uint32_t ta = tmem + lane_addr + kColO + 128 * c + 32 * cc;
            tmem_ld32(ta, r);
            tmem_wait_ld();
            uint32_t w0[16], w1[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              w0[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
              w1[e] = __float_as_uint(__uint_as_float(r[16 + e]) * alpha);
            }
            tmem_st16(ta, w0);
            tmem_st16(ta + 16, w1);
          }
          tmem_wait_st();
        }
        l *= alpha;
        const uint64_t nm = f2_pack(-m, -m);
        uint64_t acc0 = f2_pack(0.f, 0.f), acc1 = acc0;
        uint32_t pk[32];
#pragma unroll
        for (int j = 0; j < 64; j += 4) {
          float a0, a1, a2, a3;
          f2_unpack(f2_add(f2_pack(y[j], y[j + 1]), nm), a0, a1);
          f2_unpack(f2_add(f2_pack(y[j + 2], y[j + 3]), nm), a2, a3);
          // masked columns hold -inf: 2^-inf = 0 (and the -inf reference of an empty
          // row only meets masked columns)
          a0 = j < lim ? fast_exp2(a0) : 0.f;
          a1 = j + 1 < lim ? fast_exp2(a1) : 0.f;
          a2 = j + 2 < lim ? fast_exp2(a2) : 0.f;
          a3 = j + 3 < lim ? fast_exp2(a3) : 0.f;
          acc0 = f2_add(acc0, f2_pack(a0, a1));
          acc1 = f2_add(acc1, f2_pack(a2, a3));
          pk[j / 2] = pack_bf16x2(a0, a1);
          pk[j / 2 + 1] = pack_bf16x2(a2, a3);
        }
        {
          float s0, s1, s2_, s3;
          f2_unpack(acc0, s0, s1);
          f2_unpack(acc1, s2_, s3);
          l += (s0 + s1) + (s2_ + s3);
        }
        // P shares one buffer: PV(gs-1) must be done reading it.
        if (gs >= 1 && !waited && !__all_sync(0xffffffffu, wait_bar(bar(kODone), (gs - 1) & 1, ctl))) {
          ok = false;
          break;
        }
#pragma unroll
        for (int ch = 0; ch < 8; ++ch)
          *reinterpret_cast<uint4*>(prow + ((ch ^ (h & 7)) * 16)) =
              make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
        fence_proxy_async();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) arrive_cta0(rank, bar(kPFull), pfull0);
      }
      if (!ok) break;
      // ---- the next piece's q' into tensor memory, once this piece's last score MMA has
      // read the current one (so the next piece's scores can start during this epilogue)
      if (have_next) {
        if (!__all_sync(0xffffffffu, wait_bar(bar(kQEmpty), piece & 1, ctl))) { ok = false; break; }
        tc_fence_after();
        stage_q(nc.b);
      }
      // ---- epilogue: O / l for this thread's 128 dims, lse
      lsum_s[hh][c][h] = l;
      if (!meet()) { ok = false; break; }
      const float l_row = (lsum_s[0][0][h] + lsum_s[0][1][h]) + (lsum_s[1][0][h] + lsum_s[1][1][h]);
      if (!__all_sync(0xffffffffu, wait_bar(bar(kOFull), piece & 1, ctl))) { ok = false; break; }
      tc_fence_after();
      const bool none = kCausal && l_row == 0.f;  // a causal row that sees no token of the piece
      const float inv = bad ? NAN : (none ? 0.f : 1.f / l_row);
      const float lse_v = bad ? NAN : (none ? -INFINITY : (m + __log2f(l_row)) * kLn2);
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
      // The warp's 32 rows x 128 dims leave through its own 4 KB of the P buffer (free:
      // every value MMA of the piece is done, and this warp writes the next piece's P
      // there only after this loop), 32 dims at a time: each thread stages its row (16-byte
      // chunks XOR-swizzled by row, so neither side conflicts on banks), then 8 lanes store
      // one row's 128 contiguous bytes -- against 32 rows touched by every store when each
      // thread wrote its own row.
      uint8_t* const stage = smem + kOffP + (2 * hh + c) * kBox + 32 * (q & 1) * 128;
      const int sr = lane >> 3, sk = lane & 7;  // staged row within a group of 4, chunk
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_addr + kColO + 128 * c + 32 * cc, r);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 8; ++e)
          *reinterpret_cast<float4*>(stage + lane * 128 + ((e ^ (lane & 7)) * 16)) =
              make_float4(__uint_as_float(r[4 * e]) * inv, __uint_as_float(r[4 * e + 1]) * inv,
                          __uint_as_float(r[4 * e + 2]) * inv, __uint_as_float(r[4 * e + 3]) * inv);
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int rr = 4 * i + sr;                            // staged row = lane rr of this warp
          const int orow = 64 * (int)rank + 32 * (q & 1) + rr;  // its row of the launch
          const float4 v = *reinterpret_cast<const float4*>(stage + rr * 128 + ((sk ^ (rr & 7)) * 16));
          if (orow < a.heads)
            *reinterpret_cast<float4*>(obase + (size_t)orow * kDLatent + 256 * c + 128 * hh + 32 * cc + 4 * sk) = v;
        }
        __syncwarp();  // the staging area is rewritten by the next 32 dims
      }
      if (hh == 0 && c == 0 && row < a.heads) lbase[row] = lse_v;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) arrive_cta0(rank, bar(kOFree), ofree0);
      g += f.steps;
      ++piece;
    }
  }

  // ------------------------------------------------------------ teardown
  if (tid == 0) grid_dep_launch_dependents();  // the combine grid may launch (it waits for this grid's writes)
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer's MMAs, loads and arrivals are done with this CTA
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

}  // namespace

int decode_pair_max_workers(int sm_count) {
  static int cached[64];
  static bool have[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  if (!have[dev]) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (sm_count / 2), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemAlloc;
    cudaFuncSetAttribute(decode_pair_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc);
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, decode_pair_kernel<false>, &cfg) != cudaSuccess || clusters <= 0)
      clusters = sm_count / 2;
    cached[dev] = clusters;
    have[dev] = true;
  }
  return cached[dev];
}

cudaError_t launch_decode_pair(const DecodeArgs& a, cudaStream_t stream) {
  static bool done1[64] = {}, done2[64] = {};
  cudaError_t e = allow_dynamic_smem(reinterpret_cast<const void*>(decode_pair_kernel<false>), kSmemAlloc, done1);
  if (e == cudaSuccess)
    e = allow_dynamic_smem(reinterpret_cast<const void*>(decode_pair_kernel<true>), kSmemAlloc, done2);
  if (e != cudaSuccess) return e;
  auto encode = tensor_map_encoder();
  if (!encode) return cudaErrorNotSupported;
  // The cache as a 2-D tensor [rows, 576] and q' as [rows of all sequences, 576], both
  // read in boxes of 64 rows x 64 dims (128B swizzle); every box starts at an x
  // coordinate that is a multiple of 64 elements (128 bytes).
  CUtensorMap kv_map, q_map;
  cuuint32_t estr[2] = {1, 1};
  cuuint32_t box[2] = {64, 64};
  {
    const uint64_t rows = (uint64_t)(a.block_table ? a.num_pages : a.batch * a.max_blocks) * kPage;
    cuuint64_t dims[2] = {(cuuint64_t)kDQK, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)kDQK * 2};
    if (encode(&kv_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<__nv_bfloat16*>(a.kv), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    const uint64_t rows = (uint64_t)a.batch * (a.s_q > 1 ? a.row_stride : a.heads);
    cuuint64_t dims[2] = {(cuuint64_t)kDQK, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)kDQK * 2};
    if (encode(&q_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<__nv_bfloat16*>(a.q), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const uint64_t limit_ns = (uint64_t)(a.wait_limit > 0 ? a.wait_limit : 1000) * 1000000ull;  // wait_limit in ms
  // Launched as a programmatic dependent of whatever precedes it on the stream (the
  // previous call's combine, or the grid that wrote q'): the prologue (barrier set-up,
  // tensor-memory allocation, descriptor prefetch) overlaps that grid's tail.
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
  return a.s_q > 1 ? cudaLaunchKernelEx(&cfg, decode_pair_kernel<true>, kv_map, q_map, a, limit_ns)
                   : cudaLaunchKernelEx(&cfg, decode_pair_kernel<false>, kv_map, q_map, a, limit_ns);
}

}  // namespace mla
