// Key and value absorption on the 5th-generation tensor cores: per call, H small
// GEMMs, each of one head's weights against the whole batch.
//
//   absorb_q:  q'[b,h,0:512] = q_nope[b,h,:] W_UK[h]   ([B x 128] x [128 x 512]),
//              q'[b,h,512:576] = q_rope[b,h,:]
//   absorb_o:  out[b,h,:] = bf16(out_latent[b,h,:]) W_UV[h]   ([B x 512] x [512 x 128])
// (glossary entry, "why absorb in decode": q^C (W^UK)^T and (sum_t p_t c_t) W^UV.)
//
// Both are HBM-bound (about 1 GFLOP against tens of MB at the largest workload), so
// they are written for streaming.  A work item is one head and a tile of up to 128
// batch rows (the MMA's M; rows past the batch are zero-filled by TMA on load and
// clipped by TMA on store); CTAs are persistent over items, one per SM.  Roles:
// warps 0-3 own the 128 TMEM lanes (epilogue, and for absorb_o the fp32 -> bf16
// conversion of A), warp 4 issues TMA loads, warp 5 allocates TMEM and issues the
// MMAs.  The accumulator is double-buffered in TMEM, so one tile's epilogue runs
// under the next tile's MMAs.  Every wait is bounded: on expiry the kernel records
// MLA_ERR_DEVICE_TIMEOUT, lets in-flight copies and MMAs finish, frees TMEM and
// returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "mla_device.cuh"
#include "mla_internal.h"
#include "sm100_ptx.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int kThreads = 192;
constexpr int kRows = 128;                // batch rows per item (MMA M)
constexpr int kBox = kRows * 128;         // one [128 rows x 128 B] 128B-swizzled TMA box: 16 KB

// ---------------------------------------------------------------- helpers
__device__ __forceinline__ uint64_t now_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

struct Guard {
  int* err;
  volatile int* abort;
  uint64_t limit_ns;
};

// Bounded wait on an mbarrier phase; false on timeout (recorded) or abort.
__device__ __forceinline__ bool wait_on(uint32_t bar, uint32_t parity, const Guard& g) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = 0;
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63) == 0) {
      if (*g.abort) return false;
      const uint64_t t = now_ns();
      if (t0 == 0) {
        t0 = t;
      } else if (t - t0 > g.limit_ns) {
        set_device_error(g.err, MLA_ERR_DEVICE_TIMEOUT);
        *g.abort = 1;
        return false;
      }
    }
  }
}
__device__ __forceinline__ void drain_on(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = now_ns();
  while (!mbar_try_wait(bar, parity) && now_ns() - t0 < limit_ns) {
  }
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void* map, int x, int y, int z, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
          dst),
      "l"(map), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}
// Tiled store of one box from shared memory (coordinates are never negative here).
__device__ __forceinline__ void tma_store_3d(const void* map, uint32_t src, int x, int y, int z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(map), "r"(x),
               "r"(y), "r"(z), "r"(src)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// At most one committed bulk group still reading shared memory.
__device__ __forceinline__ void bulk_wait_read_1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void bar_sync_epilogue() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// 32 fp32 -> 16-byte chunks [q4] of bf16 (8 values each).
__device__ __forceinline__ uint4 pack8(const uint32_t* v) {
  return make_uint4(pack_bf16x2(__uint_as_float(v[0]), __uint_as_float(v[1])),
                    pack_bf16x2(__uint_as_float(v[2]), __uint_as_float(v[3])),
                    pack_bf16x2(__uint_as_float(v[4]), __uint_as_float(v[5])),
                    pack_bf16x2(__uint_as_float(v[6]), __uint_as_float(v[7])));
}

// ================================================================ absorb_q
// Item (head h, batch tile mt): A = q_nope[128 rows x 128 k] (two K-major boxes), then
// four n-tiles of 128: B = W_UK[h][128 k x 128 n] (two MN-major boxes), D = 128 x 128
// fp32 in TMEM, written out as bf16 through shared memory by TMA stores.
constexpr int kQA = 2 * kBox, kQB = 2 * kBox, kQO = 2 * kBox;  // 32 KB each
constexpr int kQBStages = 4;             // every n-tile of an item's weights in flight at once
constexpr int kQSmA = 0, kQSmB = kQA, kQSmO = kQSmB + kQBStages * kQB;
constexpr int kQSmem = kQSmO + 2 * kQO;  // 224 KB: A, B[4], out[2]
constexpr int kQNt = kDLatent / 128;     // n-tiles per item
constexpr uint32_t kQIdesc = idesc_bf16_f32(128, 128, 0, 1);

enum QBar { kQAFull = 0, kQAEmpty, kQBFull, kQBEmpty = kQBFull + kQBStages, kQDFull = kQBEmpty + kQBStages, kQDEmpty = kQDFull + 2, kQDone = kQDEmpty + 2, kQNumBars };

__global__ void __launch_bounds__(kThreads, 1)
    absorb_q_tc_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                       const __grid_constant__ CUtensorMap map_o, const __nv_bfloat16* __restrict__ q_rope,
                       __nv_bfloat16* __restrict__ q_out, int B, int H, int* err, uint64_t limit_ns) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[kQNumBars];
  __shared__ uint32_t tmem_s;
  __shared__ int abort_s;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int mtiles = (B + kRows - 1) / kRows;
  const int items = H * mtiles;

  if (tid == 0) {
    abort_s = 0;
    mbar_init(bar(kQAFull), 1);
    mbar_init(bar(kQAEmpty), 1);
    for (int i = 0; i < kQBStages; ++i) {
      mbar_init(bar(kQBFull + i), 1);
      mbar_init(bar(kQBEmpty + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(kQDFull + i), 1);
      mbar_init(bar(kQDEmpty + i), 4);  // one arrival per epilogue warp
    }
    mbar_init(bar(kQDone), 1);
    fence_mbar_init();
    tma_prefetch_desc(&map_a);
    tma_prefetch_desc(&map_b);
    tma_prefetch_desc(&map_o);
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(&tmem_s), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Launched as a programmatic dependent: the set-up above overlaps the previous grid,
  // whose writes (the inputs) are complete and visible after this wait.
  if (tid == 0) grid_dep_launch_dependents();
  grid_dep_wait();
  const uint32_t tmem = tmem_s;
  const Guard gd{err, &abort_s, limit_ns};

  if (warp == 4) {
    // ---------------------------------------------------------------- TMA loads
    if (lane == 0) {
      int it = 0, g = 0, ga = 0, gb = 0;  // items, n-tiles; loads issued into A and B
      bool ok = true;
      for (int item = blockIdx.x; ok && item < items; item += gridDim.x, ++it) {
        const int h = item % H, b0 = (item / H) * kRows;
        if (!wait_on(bar(kQAEmpty), (it & 1) ^ 1, gd)) { ok = false; break; }
        mbar_expect_tx(bar(kQAFull), kQA);
        tma_load_3d(sbase + kQSmA, &map_a, 0, h, b0, bar(kQAFull));
        tma_load_3d(sbase + kQSmA + kBox, &map_a, 64, h, b0, bar(kQAFull));
        ++ga;
        for (int j = 0; j < kQNt; ++j, ++g) {
          const int s = g % kQBStages;
          if (!wait_on(bar(kQBEmpty + s), ((g / kQBStages) & 1) ^ 1, gd)) { ok = false; break; }
          mbar_expect_tx(bar(kQBFull + s), kQB);
          tma_load_3d(sbase + kQSmB + s * kQB, &map_b, 128 * j, 0, h, bar(kQBFull + s));
          tma_load_3d(sbase + kQSmB + s * kQB + kBox, &map_b, 128 * j + 64, 0, h, bar(kQBFull + s));
          ++gb;
        }
      }
      // Every load issued lands before the CTA may exit (bounded).
      if (ga > 0) drain_on(bar(kQAFull), (ga - 1) & 1, limit_ns);
      for (int k = 0; k < kQBStages && k < gb; ++k) {
        const int l = gb - 1 - k;
        drain_on(bar(kQBFull + l % kQBStages), (l / kQBStages) & 1, limit_ns);
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // ---------------------------------------------------------------- MMA issue
    if (lane == 0) {
      int it = 0, g = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < items; item += gridDim.x, ++it) {
        if (!wait_on(bar(kQAFull), it & 1, gd)) { ok = false; break; }
        for (int j = 0; j < kQNt; ++j, ++g) {
          const int s = g % kQBStages, d = g & 1;
          if (!wait_on(bar(kQBFull + s), (g / kQBStages) & 1, gd) ||
              !wait_on(bar(kQDEmpty + d), ((g >> 1) & 1) ^ 1, gd)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t ab = sbase + kQSmA, bb = sbase + kQSmB + s * kQB;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(tmem + d * 128, desc_sw128(ab + (kk >> 2) * kBox + (kk & 3) * 32, 16, 1024),
                   desc_sw128(bb + kk * 2048, kBox, 1024), kQIdesc, kk > 0 ? 1u : 0u);
          mma_commit(bar(kQBEmpty + s));
          mma_commit(bar(kQDFull + d));
        }
        if (!ok) break;
        mma_commit(bar(kQAEmpty));
      }
      mma_commit(bar(kQDone));
      drain_on(bar(kQDone), 0, limit_ns);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue: thread = batch row
    // The four warps meet at named barriers, so none of them leaves the loops early:
    // after a failed wait they keep the same barrier sequence and skip the work.
    const int r = 32 * warp + lane;
    const uint32_t t_row = tmem + ((uint32_t)(32 * warp) << 16);
    int it = 0, g = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < items; item += gridDim.x, ++it) {
      const int h = item % H, b0 = (item / H) * kRows;
      const int b = b0 + r;
      if (ok && b < B) {  // the rope half of q' is a copy
        const uint4* src = reinterpret_cast<const uint4*>(q_rope + ((size_t)b * H + h) * kDRope);
        uint4* dst = reinterpret_cast<uint4*>(q_out + ((size_t)b * H + h) * kDQK + kDLatent);
#pragma unroll
        for (int c = 0; c < 8; ++c) dst[c] = src[c];
      }
      for (int j = 0; j < kQNt; ++j, ++g) {
        const int d = g & 1;
        if (ok) ok = __all_sync(0xffffffffu, wait_on(bar(kQDFull + d), (g >> 1) & 1, gd));
        tc_fence_after();
        // Output buffer d was last stored from two n-tiles ago: that store has read it.
        if (tid == 0) bulk_wait_read_1();
        bar_sync_epilogue();
        if (ok) {
          uint8_t* ob = smem + kQSmO + d * kQO;
#pragma unroll
          for (int c = 0; c < 4; ++c) {  // 32 columns at a time
            uint32_t v[32];
            tmem_ld32(t_row + d * 128 + 32 * c, v);
            tmem_wait_ld();
            uint8_t* row = ob + (c >> 1) * kBox + r * 128;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              const int chunk = (c & 1) * 4 + q4;
              *reinterpret_cast<uint4*>(row + ((chunk ^ (r & 7)) * 16)) = pack8(v + 8 * q4);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(kQDEmpty + d));
          fence_proxy_async();
        }
        // Every epilogue warp agrees on ok here: a warp that failed set the abort flag,
        // and the store below is issued only if all four wrote their rows.
        bar_sync_epilogue();
        if (tid == 0 && !abort_s) {
          tma_store_3d(&map_o, sbase + kQSmO + d * kQO, 128 * j, h, b0);
          tma_store_3d(&map_o, sbase + kQSmO + d * kQO + kBox, 128 * j + 64, h, b0);
          bulk_commit();
        }
      }
    }
    if (tid == 0) bulk_wait_all();  // every store has completed before the CTA exits
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// ================================================================ absorb_o
// Item (head h, batch tile mt): K = 512 in eight chunks of 64.  Per chunk, TMA brings
// the fp32 out_latent rows [128 x 64] (two 128B-swizzled boxes of 32 floats) and the
// weights W_UV[h][64 k x 128 n] (two MN-major boxes); four converter warps round the
// fp32 rows to bf16 (nearest even) into the K-major A operand; the MMA warp adds the
// chunk's four K = 16 steps into D = 128 x 128 fp32 in TMEM.  The epilogue writes D
// through shared memory by TMA stores.  Warps 0-3 epilogue, 4-7 convert, 8 TMA, 9 MMA.
constexpr int kOThreads = 320;
constexpr int kOF = 2 * kBox, kOA = kBox, kOB = kBox, kOO = 4 * kBox;  // 32, 16, 16, 64 KB
constexpr int kOFStages = 2, kOStages = 3;
constexpr int kOSmF = 0, kOSmA = kOFStages * kOF, kOSmB = kOSmA + kOStages * kOA, kOSmO = kOSmB + kOStages * kOB;
constexpr int kOSmem = kOSmO + kOO;  // 224 KB
constexpr int kOChunks = kDLatent / 64;
constexpr uint32_t kOIdesc = idesc_bf16_f32(128, 128, 0, 1);

enum OBar {
  kOFFull = 0,
  kOFEmpty = kOFFull + kOFStages,
  kOBFull = kOFEmpty + kOFStages,
  kOABEmpty = kOBFull + kOStages,  // MMA done with A and B of a stage
  kOAReady = kOABEmpty + kOStages,
  kODFull = kOAReady + kOStages,
  kODEmpty = kODFull + 2,
  kODone = kODEmpty + 2,
  kONumBars
};

__global__ void __launch_bounds__(kOThreads, 1)
    absorb_o_tc_kernel(const __grid_constant__ CUtensorMap map_f, const __grid_constant__ CUtensorMap map_w,
                       const __grid_constant__ CUtensorMap map_o, int B, int H, int* err, uint64_t limit_ns) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[kONumBars];
  __shared__ uint32_t tmem_s;
  __shared__ int abort_s;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int items = H * ((B + kRows - 1) / kRows);

  if (tid == 0) {
    abort_s = 0;
    for (int i = 0; i < kOFStages; ++i) {
      mbar_init(bar(kOFFull + i), 1);
      mbar_init(bar(kOFEmpty + i), 4);  // one arrival per converter warp
    }
    for (int i = 0; i < kOStages; ++i) {
      mbar_init(bar(kOBFull + i), 1);
      mbar_init(bar(kOABEmpty + i), 1);
      mbar_init(bar(kOAReady + i), 4);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(kODFull + i), 1);
      mbar_init(bar(kODEmpty + i), 4);
    }
    mbar_init(bar(kODone), 1);
    fence_mbar_init();
    tma_prefetch_desc(&map_f);
    tma_prefetch_desc(&map_w);
    tma_prefetch_desc(&map_o);
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(&tmem_s), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (tid == 0) grid_dep_launch_dependents();
  grid_dep_wait();  // as in absorb_q: the inputs are complete from here on
  const uint32_t tmem = tmem_s;
  const Guard gd{err, &abort_s, limit_ns};

  if (warp == 8) {
    // ---------------------------------------------------------------- TMA loads
    if (lane == 0) {
      int gf = 0, gb = 0;  // fp32 A and weight chunks issued
      bool ok = true;
      for (int item = blockIdx.x; ok && item < items; item += gridDim.x) {
        const int h = item % H, b0 = (item / H) * kRows;
        for (int c = 0; c < kOChunks; ++c) {
          const int f = gf % kOFStages, s = gb % kOStages;
          if (!wait_on(bar(kOFEmpty + f), ((gf / kOFStages) & 1) ^ 1, gd)) { ok = false; break; }
          mbar_expect_tx(bar(kOFFull + f), kOF);
          tma_load_3d(sbase + kOSmF + f * kOF, &map_f, 64 * c, h, b0, bar(kOFFull + f));
          tma_load_3d(sbase + kOSmF + f * kOF + kBox, &map_f, 64 * c + 32, h, b0, bar(kOFFull + f));
          ++gf;
          if (!wait_on(bar(kOABEmpty + s), ((gb / kOStages) & 1) ^ 1, gd)) { ok = false; break; }
          mbar_expect_tx(bar(kOBFull + s), kOB);
          tma_load_3d(sbase + kOSmB + s * kOB, &map_w, 0, 64 * c, h, bar(kOBFull + s));
          tma_load_3d(sbase + kOSmB + s * kOB + kBox / 2, &map_w, 64, 64 * c, h, bar(kOBFull + s));
          ++gb;
        }
      }
      // Every load issued lands before the CTA may exit (bounded).
      for (int k = 0; k < kOFStages && k < gf; ++k) {
        const int l = gf - 1 - k;
        drain_on(bar(kOFFull + l % kOFStages), (l / kOFStages) & 1, limit_ns);
      }
      for (int k = 0; k < kOStages && k < gb; ++k) {
        const int l = gb - 1 - k;
        drain_on(bar(kOBFull + l % kOStages), (l / kOStages) & 1, limit_ns);
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ---------------------------------------------------------------- MMA issue
    if (lane == 0) {
      int it = 0, g = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < items; item += gridDim.x, ++it) {
        const int d = it & 1;
        if (!wait_on(bar(kODEmpty + d), ((it >> 1) & 1) ^ 1, gd)) { ok = false; break; }
        for (int c = 0; c < kOChunks; ++c, ++g) {
          const int s = g % kOStages;
          if (!wait_on(bar(kOAReady + s), (g / kOStages) & 1, gd) || !wait_on(bar(kOBFull + s), (g / kOStages) & 1, gd)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t ab = sbase + kOSmA + s * kOA, bb = sbase + kOSmB + s * kOB;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(tmem + d * 128, desc_sw128(ab + kk * 32, 16, 1024), desc_sw128(bb + kk * 2048, kBox / 2, 1024),
                   kOIdesc, (c > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bar(kOABEmpty + s));
        }
        if (!ok) break;
        mma_commit(bar(kODFull + d));
      }
      mma_commit(bar(kODone));
      drain_on(bar(kODone), 0, limit_ns);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- fp32 -> bf16 A: thread = batch row
    const int r = tid - 128;
    int g = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < items; item += gridDim.x) {
      for (int c = 0; c < kOChunks; ++c, ++g) {
        const int f = g % kOFStages, s = g % kOStages;
        if (!__all_sync(0xffffffffu, wait_on(bar(kOFFull + f), (g / kOFStages) & 1, gd) &&
                                         wait_on(bar(kOABEmpty + s), ((g / kOStages) & 1) ^ 1, gd))) {
          ok = false;
          break;
        }
        const uint8_t* frow = smem + kOSmF + f * kOF + r * 128;
        uint8_t* arow = smem + kOSmA + s * kOA + r * 128;
#pragma unroll
        for (int q = 0; q < 8; ++q) {  // bf16 chunk q: k 8q..8q+7 = fp32 box q/4, chunks 2(q%4), 2(q%4)+1
          const uint8_t* fb = frow + (q >> 2) * kBox;
          const int c0 = 2 * (q & 3);
          const float4 x = *reinterpret_cast<const float4*>(fb + ((c0 ^ (r & 7)) * 16));
          const float4 y = *reinterpret_cast<const float4*>(fb + (((c0 + 1) ^ (r & 7)) * 16));
          *reinterpret_cast<uint4*>(arow + ((q ^ (r & 7)) * 16)) =
              make_uint4(pack_bf16x2(x.x, x.y), pack_bf16x2(x.z, x.w), pack_bf16x2(y.x, y.y), pack_bf16x2(y.z, y.w));
        }
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bar(kOFEmpty + f));
          mbar_arrive(bar(kOAReady + s));
        }
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue: thread = batch row
    // As in absorb_q, the four warps keep the same named-barrier sequence after a failure.
    const int r = 32 * warp + lane;
    const uint32_t t_row = tmem + ((uint32_t)(32 * warp) << 16);
    int it = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < items; item += gridDim.x, ++it) {
      const int h = item % H, b0 = (item / H) * kRows;
      const int d = it & 1;
      if (ok) ok = __all_sync(0xffffffffu, wait_on(bar(kODFull + d), (it >> 1) & 1, gd));
      tc_fence_after();
      if (tid == 0) bulk_wait_all();  // the previous item's store has finished with the buffer
      bar_sync_epilogue();
      if (ok) {
        uint8_t* row = smem + kOSmO + r * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c) {  // 32 columns = one box
          uint32_t v[32];
          tmem_ld32(t_row + d * 128 + 32 * c, v);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<uint4*>(row + c * kBox + ((q ^ (r & 7)) * 16)) =
                make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kODEmpty + d));
        fence_proxy_async();
      }
      bar_sync_epilogue();
      if (tid == 0 && !abort_s) {
#pragma unroll
        for (int c = 0; c < 4; ++c) tma_store_3d(&map_o, sbase + kOSmO + c * kBox, 32 * c, h, b0);
        bulk_commit();
      }
    }
    if (tid == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
  }();
  return fn;
}

// 3-D tiled map: dims innermost first (elements), strides of dims 1 and 2 in bytes.
bool map3d(CUtensorMap* m, CUtensorMapDataType t, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
           uint64_t s1, uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2, CUtensorMapSwizzle sw) {
  auto enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {s1, s2};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, t, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Launch as a programmatic dependent of the previous grid on the stream.
template <typename... Params, typename... Args>
cudaError_t launch_dependent(void (*kernel)(Params...), int grid, int threads, int smem, cudaStream_t stream,
                             Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

int sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 1;
  }
  return n;
}

}  // namespace

cudaError_t launch_absorb_q(const __nv_bfloat16* q_nope, const __nv_bfloat16* q_rope, const __nv_bfloat16* w_uk,
                            __nv_bfloat16* q_out, int batch, int heads, int* err, cudaStream_t stream) {
  CUtensorMap ma, mb, mo;
  const uint64_t H = heads, Bn = batch;
  const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const auto sw = CU_TENSOR_MAP_SWIZZLE_128B;
  if (!map3d(&ma, bf, q_nope, MLA_D_NOPE, H, Bn, MLA_D_NOPE * 2, H * MLA_D_NOPE * 2, 64, 1, kRows, sw) ||
      !map3d(&mb, bf, w_uk, kDLatent, MLA_D_NOPE, H, kDLatent * 2, (uint64_t)MLA_D_NOPE * kDLatent * 2, 64,
             MLA_D_NOPE, 1, sw) ||
      !map3d(&mo, bf, q_out, kDQK, H, Bn, kDQK * 2, H * kDQK * 2, 64, 1, kRows, sw))
    return cudaErrorInvalidValue;
  const int smem = kQSmem + 1024;
  static bool done[64] = {};
  cudaError_t e = allow_dynamic_smem(reinterpret_cast<const void*>(absorb_q_tc_kernel), smem, done);
  if (e != cudaSuccess) return e;
  const int items = heads * ((batch + kRows - 1) / kRows);
  const int grid = items < sm_count() ? items : sm_count();
  return launch_dependent(absorb_q_tc_kernel, grid, kThreads, smem, stream, ma, mb, mo, q_rope, q_out, batch, heads,
                          err, 2000ull * 1000000ull);
}

cudaError_t launch_absorb_o(const float* out_latent, const __nv_bfloat16* w_uv, float* out, int batch, int heads,
                            int* err, cudaStream_t stream) {
  CUtensorMap mf, mw, mo;
  const uint64_t H = heads, Bn = batch;
  const auto sw = CU_TENSOR_MAP_SWIZZLE_128B;
  if (!map3d(&mf, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, out_latent, kDLatent, H, Bn, kDLatent * 4, H * kDLatent * 4, 32, 1,
             kRows, sw) ||
      !map3d(&mw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w_uv, MLA_D_V, kDLatent, H, MLA_D_V * 2,
             (uint64_t)kDLatent * MLA_D_V * 2, 64, 64, 1, sw) ||
      !map3d(&mo, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, out, MLA_D_V, H, Bn, MLA_D_V * 4, H * MLA_D_V * 4, 32, 1, kRows, sw))
    return cudaErrorInvalidValue;
  const int smem = kOSmem + 1024;
  static bool done[64] = {};
  cudaError_t e = allow_dynamic_smem(reinterpret_cast<const void*>(absorb_o_tc_kernel), smem, done);
  if (e != cudaSuccess) return e;
  const int items = heads * ((batch + kRows - 1) / kRows);
  const int grid = items < sm_count() ? items : sm_count();
  return launch_dependent(absorb_o_tc_kernel, grid, kOThreads, smem, stream, mf, mw, mo, batch, heads, err,
                          2000ull * 1000000ull);
}

}  // namespace mla
