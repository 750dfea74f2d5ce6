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
// and the two partials are exchanged through distributed shared memory and added in
// the same order on both sides, so both CTAs run an identical softmax.
//
// Roles (256 threads): warp 0 issues TMA loads, warp 1 allocates TMEM and issues
// MMAs, warp 2 zeroes value rows past the sequence end before PV reads them,
// warps 4..7 (one thread per head row = TMEM lane) stage q', exchange partial
// scores, run the online softmax (log2 domain, lazy rescale by at most 2^8), write
// P as bf16 into TMEM, rescale O when needed, and write the epilogue.
//
// TMEM (512 columns): O [0,256) fp32, S double buffer [256,320) [320,384) fp32 with
// P (bf16 pairs) aliased over the first 32 columns of its S buffer, q' latent half
// [384,512) as bf16 pairs (the A operand of QK^T).
// Shared memory: 3 stages x 5 boxes of [64 tokens x 64 dims] bf16 (128B swizzle):
// boxes 0..3 = this CTA's latent dims (K-major B of QK^T and MN-major B of PV),
// box 4 = the 64 rope dims (both CTAs load it; each uses its 32); the rope part of
// q' [128 x 64] (A operand from shared memory); two 32 KB receive buffers for the
// peer's partial scores.
//
// Every mbarrier wait is bounded by a time limit; on expiry the kernel records
// MLA_ERR_DEVICE_TIMEOUT, tells the peer CTA to stop, drains its own TMA and MMA
// work, frees TMEM and returns.  No trap.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "mla_device.cuh"
#include "mla_internal.h"
#include "sm100_ptx.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int kThreads = 256;
constexpr int kStages = 3;
constexpr int kBoxBytes = 64 * 128;              // [64 rows x 64 bf16], 128B swizzle
constexpr int kStageBytes = 5 * kBoxBytes;       // 40960
constexpr int kQRopeBytes = 128 * 128;           // [128 heads x 64 rope dims]
constexpr int kRxBytes = 128 * 64 * 4;           // [128 heads x 64 fp32]
constexpr int kSmemStages = 0;
constexpr int kSmemQRope = kStages * kStageBytes;            // 122880
constexpr int kSmemRx = kSmemQRope + kQRopeBytes;             // 139264
constexpr int kSmemBytes = kSmemRx + 2 * kRxBytes;            // 204800
constexpr int kSmemAlloc = kSmemBytes + 1024;                 // + alignment slack

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0, kColS = 256, kColQ = 384;

constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 64, 0, 0);   // A tmem/smem K-major, B K-major
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 256, 0, 1);  // A tmem K-major, B MN-major

constexpr float kRescaleThreshold = 8.0f;  // log2 units: P may reach 2^8 before O is rescaled

enum Bar {
  kKvFull = 0, kKvEmpty = kKvFull + kStages, kVReady = kKvEmpty + kStages, kSFull = kVReady + kStages,
  kPFull = kSFull + 2, kRxFull = kPFull + 2, kTxFree = kRxFull + 2, kODone = kTxFree + 2, kOFull = kODone + 4,
  kQReady = kOFull + 1, kDrain = kQReady + 1, kNumBars = kDrain + 1
};

struct Piece {
  int b, pa, pe;
};

// Iterates the sequence pieces of worker w in schedule order.
struct PieceIter {
  const Schedule& sc;
  WorkerRange rg;
  int b;
  __device__ PieceIter(const Schedule& s, int w) : sc(s), rg(s.ranges[w]), b(rg.b0) {}
  __device__ bool next(Piece& pc) {
    if (rg.b0 < 0) return false;
    while (b <= rg.b1) {
      const int cur = b++;
      const int n = sc.seq_start[cur + 1] - sc.seq_start[cur];
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

// Bounded wait on a local mbarrier phase; on timeout or abort returns false.
__device__ __noinline__ bool wait_bar(uint32_t bar, uint32_t parity, const Ctl& c) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = now_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63) == 0) {
      if (*c.abort) return false;
      if (now_ns() - t0 > c.limit_ns) {
        set_device_error(c.err, MLA_ERR_DEVICE_TIMEOUT);
        *c.abort = 1;
        asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(c.peer_abort), "r"(1) : "memory");
        return false;
      }
    }
  }
}

__device__ __forceinline__ int page_of(const DecodeArgs& a, int b, int p) {
  return a.block_table ? a.block_table[(size_t)b * a.max_blocks + p] : b * a.max_blocks + p;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap kv_map, const DecodeArgs a, uint64_t limit_ns) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[kNumBars];
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t s_stage0 = sbase + kSmemStages, s_qrope = sbase + kSmemQRope, s_rx = sbase + kSmemRx;
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
    for (int u = 0; u < 2; ++u) {
      mbar_init(bar(kSFull + u), 1);
      mbar_init(bar(kPFull + u), 128);
      mbar_init(bar(kRxFull + u), 128);
      mbar_init(bar(kTxFree + u), 128);
    }
    for (int q = 0; q < 4; ++q) mbar_init(bar(kODone + q), 1);
    mbar_init(bar(kOFull), 1);
    mbar_init(bar(kQReady), 128);
    mbar_init(bar(kDrain), 1);
    fence_mbar_init();
    tma_prefetch_desc(&kv_map);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_base_s), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // barriers of both CTAs initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  Ctl ctl{a.err, &abort_s, map_to_rank(smem_u32(&abort_s), peer), limit_ns};

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      PieceIter pi(sc, w);
      Piece pc;
      int it = 0;
      bool ok = true;
      while (ok && pi.next(pc)) {
        for (int p = pc.pa; p < pc.pe; ++p, ++it) {
          const int s = it % kStages;
          if (!wait_bar(bar(kKvEmpty + s), ((it / kStages) & 1) ^ 1, ctl)) { ok = false; break; }
          int pid = page_of(a, pc.b, p);
          if ((unsigned)pid >= (unsigned)np) pid = 0;  // reported by the softmax warps; load something valid
          if (a.withhold_arrive && w == 0 && rank == 0 && it == 1) continue;  // timeout test: never arrives
          const uint32_t dst = s_stage0 + s * kStageBytes;
          mbar_expect_tx(bar(kKvFull + s), kStageBytes);
          const int y = pid * kPage;
#pragma unroll
          for (int i = 0; i < 4; ++i) tma_load_2d(dst + i * kBoxBytes, &kv_map, 256 * rank + 64 * i, y, bar(kKvFull + s));
          tma_load_2d(dst + 4 * kBoxBytes, &kv_map, kDLatent, y, bar(kKvFull + s));
        }
      }
      // Drain: every load issued into a stage lands before the CTA may exit (bounded).
      for (int k = 0; k < kStages && k < it; ++k) {
        const int j = it - 1 - k;
        if (a.withhold_arrive && w == 0 && rank == 0 && j == 1) continue;
        const int s = j % kStages;
        const uint64_t t0 = now_ns();
        while (!mbar_try_wait(bar(kKvFull + s), (j / kStages) & 1) && now_ns() - t0 < limit_ns) {
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      PieceIter pi(sc, w);
      Piece pc;
      int it = 0, piece = 0;
      bool ok = true;
      auto issue_pv = [&](int itp, bool first) -> bool {
        const int s = itp % kStages, u = itp & 1;
        if (!wait_bar(bar(kPFull + u), (itp >> 1) & 1, ctl)) return false;
        if (!wait_bar(bar(kVReady + s), (itp / kStages) & 1, ctl)) return false;
        tc_fence_after();
        const uint32_t vbase = s_stage0 + s * kStageBytes;
        const uint32_t p_col = tmem + kColS + 64 * u;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ts(tmem + kColO, p_col + kk * 8, desc_sw128(vbase + kk * 2048, 8192, 1024), kIdescPV,
                 (first && kk == 0) ? 0u : 1u);
        mma_commit(bar(kKvEmpty + s));
#pragma unroll
        for (int q = 0; q < 4; ++q) mma_commit(bar(kODone + q));
        return true;
      };
      while (ok && pi.next(pc)) {
        if (!wait_bar(bar(kQReady), piece & 1, ctl)) { ok = false; break; }
        tc_fence_after();
        const int n = pc.pe - pc.pa;
        for (int j = 0; j < n && ok; ++j) {
          const int itj = it + j, s = itj % kStages, u = itj & 1;
          if (!wait_bar(bar(kKvFull + s), (itj / kStages) & 1, ctl)) { ok = false; break; }
          tc_fence_after();
          const uint32_t kbase = s_stage0 + s * kStageBytes;
          const uint32_t d = tmem + kColS + 64 * u;
#pragma unroll
          for (int kc = 0; kc < 16; ++kc)
            mma_ts(d, tmem + kColQ + kc * 8, desc_sw128(kbase + (kc >> 2) * kBoxBytes + (kc & 3) * 32, 16, 1024),
                   kIdescQK, kc > 0 ? 1u : 0u);
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int kr = 2 * (int)rank + i;
            mma_ss(d, desc_sw128(s_qrope + kr * 32, 16, 1024),
                   desc_sw128(kbase + 4 * kBoxBytes + kr * 32, 16, 1024), kIdescQK, 1u);
          }
          mma_commit(bar(kSFull + u));
          if (j > 0 && !issue_pv(itj - 1, j == 1)) { ok = false; break; }
        }
        if (!ok) break;
        if (!issue_pv(it + n - 1, n == 1)) { ok = false; break; }
        mma_commit(bar(kOFull));
        it += n;
        ++piece;
      }
      // Drain every MMA this thread issued before TMEM is released.
      mma_commit(bar(kDrain));
      const uint64_t t0 = now_ns();
      while (!mbar_try_wait(bar(kDrain), 0) && now_ns() - t0 < limit_ns) {
      }
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------------------ tail rows of V
    PieceIter pi(sc, w);
    Piece pc;
    int it = 0;
    bool ok = true;
    while (ok && pi.next(pc)) {
      const int T = a.seqlens[pc.b];
      for (int p = pc.pa; p < pc.pe; ++p, ++it) {
        const int s = it % kStages;
        if (!__all_sync(0xffffffffu, wait_bar(bar(kKvFull + s), (it / kStages) & 1, ctl))) { ok = false; break; }
        const int valid = min(kPage, T - p * kPage);
        if (valid < kPage) {
          // Rows >= valid may hold anything (NaN included); P is 0 there but 0 * NaN is
          // NaN, so zero them in the four value boxes before PV reads the stage.
          uint8_t* st = smem + kSmemStages + s * kStageBytes;
          const int nrow = kPage - valid;
          for (int idx = lane; idx < nrow * 4 * 8; idx += 32) {
            const int box = idx / (nrow * 8), rem = idx % (nrow * 8);
            const int row = valid + rem / 8, chunk = rem % 8;
            *reinterpret_cast<uint4*>(st + box * kBoxBytes + row * 128 + chunk * 16) = make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kVReady + s));
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax warpgroup
    const int row = tid - 128;             // head row = TMEM lane
    const int q = warp & 3;                // lane quadrant of this warp
    const uint32_t lane_off = (uint32_t)(32 * q) << 16;
    const uint32_t t_o = tmem + lane_off + kColO;
    const uint32_t t_q = tmem + lane_off + kColQ;
    const uint32_t rx_peer = map_to_rank(s_rx, peer) + row * 256;
    const uint32_t peer_rx_full = map_to_rank(bar(kRxFull), peer);
    const uint32_t peer_tx_free = map_to_rank(bar(kTxFree), peer);
    const float scale2 = a.scale * kLog2e;
    PieceIter pi(sc, w);
    Piece pc;
    int it = 0, piece = 0, od = 0;  // od: o_done phases known complete
    bool ok = true;
    while (ok && pi.next(pc)) {
      const int b = pc.b, n = pc.pe - pc.pa;
      const int T = a.seqlens[b];
      // ---- stage q' for this sequence: latent half -> TMEM, rope -> smem (128B swizzle)
      {
        uint32_t qv[16];
        const bool live = row < a.heads;
        const uint4* src = reinterpret_cast<const uint4*>(a.q + ((size_t)b * a.heads + (live ? row : 0)) * kDQK);
#pragma unroll
        for (int c = 0; c < 8; ++c) {  // 8 x 32 dims of this CTA's 256 latent dims
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint4 v = live ? src[(256 * rank) / 8 + c * 4 + k] : make_uint4(0, 0, 0, 0);
            qv[4 * k + 0] = v.x;
            qv[4 * k + 1] = v.y;
            qv[4 * k + 2] = v.z;
            qv[4 * k + 3] = v.w;
          }
          tmem_st16(t_q + c * 16, qv);
        }
        uint8_t* qr = smem + kSmemQRope + row * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 v = live ? src[kDLatent / 8 + c] : make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4*>(qr + ((c ^ (row & 7)) * 16)) = v;
        }
        tmem_wait_st();
        fence_proxy_async();
        tc_fence_before();
        mbar_arrive(bar(kQReady));
      }
      float m = -INFINITY, l = 0.f;
      bool bad = false;
      for (int j = 0; j < n; ++j) {
        const int itj = it + j, u = itj & 1, ph = (itj >> 1) & 1, p = pc.pa + j;
        if (!__all_sync(0xffffffffu, wait_bar(bar(kSFull + u), ph, ctl))) { ok = false; break; }
        tc_fence_after();
        // PV(j-2) finished before QK^T(j) did: retire its o_done phase (no stall).
        while (od <= it + j - 2) {
          if (!__all_sync(0xffffffffu, wait_bar(bar(kODone + q), od & 1, ctl))) { ok = false; break; }
          ++od;
        }
        if (!ok) break;
        float x[64];
        {
          uint32_t r0[32], r1[32];
          tmem_ld32(tmem + lane_off + kColS + 64 * u, r0);
          tmem_ld32(tmem + lane_off + kColS + 64 * u + 32, r1);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            x[k] = __uint_as_float(r0[k]);
            x[32 + k] = __uint_as_float(r1[k]);
          }
        }
        // ---- exchange partial scores with the peer CTA
        if (!__all_sync(0xffffffffu, wait_bar(bar(kTxFree + u), ph ^ 1, ctl))) { ok = false; break; }
        const uint32_t dst = rx_peer + u * kRxBytes;
#pragma unroll
        for (int c = 0; c < 16; ++c)
          st_cluster_v4(dst + ((c ^ (row & 7)) * 16), x[4 * c], x[4 * c + 1], x[4 * c + 2], x[4 * c + 3]);
        mbar_arrive_cluster(peer_rx_full + u * 8);
        if (!__all_sync(0xffffffffu, wait_bar(bar(kRxFull + u), ph, ctl))) { ok = false; break; }
        {
          const uint8_t* src = smem + kSmemRx + u * kRxBytes + row * 256;
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const float4 v = *reinterpret_cast<const float4*>(src + ((c ^ (row & 7)) * 16));
            // Both CTAs add (own + peer) for their own first operand; fp32 addition is
            // commutative, so both hold bit-identical scores.
            x[4 * c + 0] += v.x;
            x[4 * c + 1] += v.y;
            x[4 * c + 2] += v.z;
            x[4 * c + 3] += v.w;
          }
        }
        mbar_arrive_cluster(peer_tx_free + u * 8);
        // ---- online softmax, log2 domain
        const int pid = page_of(a, b, p);
        if ((unsigned)pid >= (unsigned)np) {
          bad = true;
          set_device_error(a.err, MLA_ERR_DEVICE_BAD_PAGE);
        }
        const int valid = min(kPage, T - p * kPage);
        float tmax = -INFINITY;
#pragma unroll
        for (int k = 0; k < 64; ++k) {
          x[k] = k < valid ? x[k] * scale2 : -INFINITY;
          tmax = fmaxf(tmax, x[k]);
        }
        const float m_new = fmaxf(m, tmax);
        const bool need = m_new > m + kRescaleThreshold;
        const float alpha = need ? fast_exp2(m - m_new) : 1.f;
        if (need) m = m_new;
        if (__any_sync(0xffffffffu, need && j > 0)) {
          // O must hold PV(j-1) before it is rescaled (rare path).
          while (od <= it + j - 1) {
            if (!__all_sync(0xffffffffu, wait_bar(bar(kODone + q), od & 1, ctl))) { ok = false; break; }
            ++od;
          }
          if (!ok) break;
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < 8; ++c) {
            uint32_t r[32];
            tmem_ld32(t_o + c * 32, r);
            tmem_wait_ld();
            uint32_t w0[16], w1[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              w0[k] = __float_as_uint(__uint_as_float(r[k]) * alpha);
              w1[k] = __float_as_uint(__uint_as_float(r[16 + k]) * alpha);
            }
            tmem_st16(t_o + c * 32, w0);
            tmem_st16(t_o + c * 32 + 16, w1);
          }
          tmem_wait_st();
        }
        l *= alpha;
        uint32_t pk[32];
        float rs = 0.f;
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const float p0 = fast_exp2(x[2 * k] - m);
          const float p1 = fast_exp2(x[2 * k + 1] - m);
          rs += p0 + p1;
          pk[k] = pack_bf16x2(p0, p1);
        }
        l += rs;
        {
          uint32_t h0[16], h1[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            h0[k] = pk[k];
            h1[k] = pk[16 + k];
          }
          tmem_st16(tmem + lane_off + kColS + 64 * u, h0);
          tmem_st16(tmem + lane_off + kColS + 64 * u + 16, h1);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(kPFull + u));
      }
      if (!ok) break;
      // ---- epilogue: O / l (this CTA's 256 dims), lse
      if (!__all_sync(0xffffffffu, wait_bar(bar(kOFull), piece & 1, ctl))) { ok = false; break; }
      tc_fence_after();
      od = it + n;  // every PV of this piece has completed
      const float inv = bad ? NAN : 1.f / l;
      const float lse_v = bad ? NAN : (m + __log2f(l)) * kLn2;
      const bool complete = pc.pa == 0 && pc.pe == sc.seq_start[b + 1] - sc.seq_start[b];
      float* obase;
      float* lbase;
      if (complete) {
        obase = a.out + (size_t)b * a.heads * kDLatent;
        lbase = a.lse + (size_t)b * a.heads;
      } else {
        const int slot = (b == sc.ranges[w].b0) ? w : P + w;
        obase = sc.part_o + (size_t)slot * a.heads * kDLatent;
        lbase = sc.part_lse + (size_t)slot * a.heads;
      }
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t r[32];
        tmem_ld32(t_o + c * 32, r);
        tmem_wait_ld();
        if (row < a.heads) {
          float4* dst = reinterpret_cast<float4*>(obase + (size_t)row * kDLatent + 256 * rank + 32 * c);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            dst[k] = make_float4(__uint_as_float(r[4 * k]) * inv, __uint_as_float(r[4 * k + 1]) * inv,
                                 __uint_as_float(r[4 * k + 2]) * inv, __uint_as_float(r[4 * k + 3]) * inv);
        }
      }
      if (rank == 0 && row < a.heads) lbase[row] = lse_v;
      tc_fence_before();
      it += n;
      ++piece;
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer no longer writes into this CTA's shared memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
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

}  // namespace

bool decode_tc_supported(int heads) { return heads >= 1 && heads <= 128; }

int decode_tc_max_workers(int sm_count) {
  static int cached = -1;
  if (cached < 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (sm_count / 2), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemAlloc;
    cudaFuncSetAttribute(decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc);
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, decode_tc_kernel, &cfg) != cudaSuccess || clusters <= 0)
      clusters = sm_count / 2;
    cached = clusters;
  }
  return cached;
}

cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t stream) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  auto encode = get_encode();
  if (!encode) return cudaErrorNotSupported;
  CUtensorMap map;
  const uint64_t rows = (uint64_t)(a.block_table ? a.num_pages : a.batch * a.max_blocks) * kPage;
  cuuint64_t dims[2] = {(cuuint64_t)kDQK, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kDQK * 2};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<__nv_bfloat16*>(a.kv), dims, strides,
                      box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  const uint64_t limit_ns = (uint64_t)(a.wait_limit > 0 ? a.wait_limit : 1000) * 1000000ull;  // wait_limit in ms
  decode_tc_kernel<<<2 * a.sched.num_workers, kThreads, kSmemAlloc, stream>>>(map, a, limit_ns);
  return cudaGetLastError();
}

}  // namespace mla
