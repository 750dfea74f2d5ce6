// Key and value absorption: H independent small GEMMs (warp-level tensor cores).
//
//   absorb_q:  q'[b,h,0:512] = q_nope[b,h,:] W_UK[h]   ([B x 128] x [128 x 512]),
//              q'[b,h,512:576] = q_rope[b,h,:]
//   absorb_o:  out[b,h,:] = bf16(out_latent[b,h,:]) W_UV[h]   ([B x 512] x [512 x 128])
// (glossary entry, "why absorb in decode": q^C (W^UK)^T and (sum_t p_t c_t) W^UV.)
//
// Both are HBM-bound (about 1 GFLOP against tens of MB at the largest workload),
// so they are written for streaming: absorb_q computes a 64 x 128 output tile of
// one head per CTA, loading its operands in two halves of K so the first half's
// MMAs overlap the second half's loads, and writes the tile through shared memory
// as whole rows; absorb_o computes a 64 x 128 tile of one head per CTA, streaming
// K = 512 through a three-stage cp.async ring (fp32 out_latent is rounded to bf16
// as its fragments are read).  Operands sit in XOR-swizzled shared memory; the
// MMAs are warp-level bf16 tensor-core instructions with fp32 accumulation.
#include "mla_device.cuh"
#include "mla_internal.h"

namespace mla {
namespace {

constexpr int kThreads = 128;
constexpr int kTileM = 64, kTileN = 128, kTileK = 128;
constexpr int kChunks = kTileK * 2 / 16;  // 16 chunks of 16 B per 128-wide bf16 row

__device__ __forceinline__ uint32_t swz16(int r, int c) { return (uint32_t)(r * kChunks + (c ^ (r & 7))) * 16u; }

// acc[16x128] += A[16 x 16 k] * B[16 k x 128] over k-steps [kc0, kc1) of 16, for
// warp rows [16w, 16w+16).
__device__ __forceinline__ void warp_tile_mma(float (&acc)[16][4], uint32_t a_s, uint32_t b_s, int warp, int lane,
                                              int kc0, int kc1) {
  const int a_row = warp * 16 + (lane & 15);
  const int b_row = (lane & 7) + (((lane >> 3) & 1) << 3);
#pragma unroll
  for (int kc = kc0; kc < kc1; ++kc) {
    uint32_t af[4];
    ldmatrix_x4(af, a_s + swz16(a_row, kc * 2 + (lane >> 4)));
#pragma unroll
    for (int nn = 0; nn < kTileN / 16; ++nn) {
      uint32_t bf[4];
      ldmatrix_x4_trans(bf, b_s + swz16(kc * 16 + b_row, nn * 2 + (lane >> 4)));
      mma_bf16_16816(acc[2 * nn], af, bf[0], bf[1]);
      mma_bf16_16816(acc[2 * nn + 1], af, bf[2], bf[3]);
    }
  }
}

// Stage rows [r0, r1) and 16-byte chunks [c0, c1) of a [rows x 128] bf16 block (row
// stride in elements) into swizzled smem; rows >= valid_rows are zero-filled.
__device__ __forceinline__ void stage_bf16(uint32_t dst, const __nv_bfloat16* src, size_t stride, int r0, int r1,
                                           int c0, int c1, int valid_rows, const void* safe) {
  const int nc = c1 - c0;
  for (int i = threadIdx.x; i < (r1 - r0) * nc; i += kThreads) {
    const int r = r0 + i / nc, c = c0 + i % nc;
    const bool ok = r < valid_rows;
    cp_async_16(dst + swz16(r, c), ok ? (const void*)(src + r * stride + c * 8) : safe, ok ? 16 : 0);
  }
}

__global__ void __launch_bounds__(kThreads) absorb_q_kernel(const __nv_bfloat16* __restrict__ q_nope,
                                                            const __nv_bfloat16* __restrict__ q_rope,
                                                            const __nv_bfloat16* __restrict__ w_uk,
                                                            __nv_bfloat16* __restrict__ q_out, int B, int H) {
  __shared__ __align__(128) uint8_t a_tile[kTileM * kTileK * 2];
  __shared__ __align__(128) uint8_t b_tile[kTileK * kTileN * 2];
  const int b0 = blockIdx.x * kTileM, n0 = blockIdx.y * kTileN, h = blockIdx.z;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int rows = min(kTileM, B - b0);
  const __nv_bfloat16* a_src = q_nope + ((size_t)b0 * H + h) * MLA_D_NOPE;
  const __nv_bfloat16* b_src = w_uk + (size_t)h * MLA_D_NOPE * kDLatent + n0;
  // K in two halves: k [0,64) is A chunks [0,8) and B rows [0,64).
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    stage_bf16(smem_u32(a_tile), a_src, (size_t)H * MLA_D_NOPE, 0, kTileM, 8 * half, 8 * half + 8, rows, q_nope);
    stage_bf16(smem_u32(b_tile), b_src, kDLatent, 64 * half, 64 * half + 64, 0, kChunks, kTileK, w_uk);
    cp_async_commit();
  }

  float acc[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
  cp_async_wait<1>();
  __syncthreads();
  warp_tile_mma(acc, smem_u32(a_tile), smem_u32(b_tile), warp, lane, 0, 4);
  cp_async_wait<0>();
  __syncthreads();
  warp_tile_mma(acc, smem_u32(a_tile), smem_u32(b_tile), warp, lane, 4, 8);
  __syncthreads();  // every warp is done with a_tile: it now holds the bf16 output tile

  // Output tile [64 rows x 128 dims] bf16 through shared memory, then whole 256-byte
  // row segments to global memory.
  const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int row = warp * 16 + g + r * 8;
#pragma unroll
    for (int i = 0; i < 16; ++i)  // columns 8i + 2 t4, +1: chunk i, word t4
      *reinterpret_cast<uint32_t*>(a_tile + swz16(row, i) + t4 * 4) = pack_bf16x2(acc[i][2 * r], acc[i][2 * r + 1]);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < rows * kChunks; i += kThreads) {
    const int r = i / kChunks, c = i % kChunks;
    *reinterpret_cast<uint4*>(q_out + ((size_t)(b0 + r) * H + h) * kDQK + n0 + c * 8) =
        *reinterpret_cast<const uint4*>(a_tile + swz16(r, c));
  }
  if (blockIdx.y == 0) {  // rope half of q' is a copy
    for (int i = threadIdx.x; i < rows * 8; i += kThreads) {
      const int r = i >> 3, c = i & 7;
      const uint4 v = *reinterpret_cast<const uint4*>(q_rope + ((size_t)(b0 + r) * H + h) * kDRope + c * 8);
      *reinterpret_cast<uint4*>(q_out + ((size_t)(b0 + r) * H + h) * kDQK + kDLatent + c * 8) = v;
    }
  }
}

constexpr int kOKc = 64;                                  // K per stage
constexpr int kOStages = 3;
constexpr int kOABytes = kTileM * kOKc * 4;               // fp32 A chunk [64 rows x 64 k]
constexpr int kOStageBytes = kOABytes + kOKc * kTileN * 2;  // + bf16 B chunk [64 k x 128 n]
constexpr int kOSmem = kOStages * kOStageBytes;           // 96 KB

__global__ void __launch_bounds__(kThreads) absorb_o_kernel(const float* __restrict__ out_latent,
                                                            const __nv_bfloat16* __restrict__ w_uv,
                                                            float* __restrict__ out, int B, int H) {
  extern __shared__ __align__(1024) uint8_t smem_o[];
  const int b0 = blockIdx.x * kTileM, h = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int rows = min(kTileM, B - b0);
  const uint32_t sb = smem_u32(smem_o);
  // Stage s <- K chunk kc: A rows of 64 fp32 (16 chunks of 16 B, chunk c of row r at
  // c ^ (r & 7)), B rows of 128 bf16 in the same swizzle.
  auto load = [&](int kc, int s) {
    const uint32_t a_s = sb + s * kOStageBytes, b_s = a_s + kOABytes;
    const int k0 = kc * kOKc;
    for (int i = threadIdx.x; i < kTileM * 16; i += kThreads) {
      const int r = i >> 4, c = i & 15;
      const bool ok = r < rows;
      cp_async_16(a_s + r * 256 + ((c ^ (r & 7)) * 16),
                  ok ? (const void*)(out_latent + ((size_t)(b0 + r) * H + h) * kDLatent + k0 + c * 4) : out_latent,
                  ok ? 16 : 0);
    }
    for (int i = threadIdx.x; i < kOKc * 16; i += kThreads) {
      const int r = i >> 4, c = i & 15;
      cp_async_16(b_s + swz16(r, c), w_uv + ((size_t)h * kDLatent + k0 + r) * MLA_D_V + c * 8, 16);
    }
  };
  float acc[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
  constexpr int kNk = kDLatent / kOKc;  // 8 chunks
  load(0, 0);
  cp_async_commit();
  load(1, 1);
  cp_async_commit();
  const int g = lane >> 2, t4 = lane & 3;
  const int b_row = (lane & 7) + (((lane >> 3) & 1) << 3);
#pragma unroll 1
  for (int kc = 0; kc < kNk; ++kc) {
    if (kc + 2 < kNk) load(kc + 2, (kc + 2) % kOStages);
    cp_async_commit();  // possibly empty: keeps one group per chunk
    cp_async_wait<2>();  // chunk kc has landed
    __syncthreads();
    const uint8_t* a_p = smem_o + (kc % kOStages) * kOStageBytes;
    const uint32_t b_s = sb + (kc % kOStages) * kOStageBytes + kOABytes;
#pragma unroll
    for (int ks = 0; ks < kOKc / 16; ++ks) {
      // A fragment of m16n8k16 (rows g, g+8; k 2 t4, 2 t4 + 8), rounded to bf16 here.
      uint32_t af[4];
#pragma unroll
      for (int hk = 0; hk < 2; ++hk) {
        const int k = ks * 16 + 2 * t4 + 8 * hk;
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
          const int r = warp * 16 + g + 8 * hr;
          const float2 v = *reinterpret_cast<const float2*>(a_p + r * 256 + (((k >> 2) ^ (r & 7)) * 16) + (k & 3) * 4);
          af[hr + 2 * hk] = pack_bf16x2(v.x, v.y);
        }
      }
#pragma unroll
      for (int nn = 0; nn < kTileN / 16; ++nn) {
        uint32_t bf[4];
        ldmatrix_x4_trans(bf, b_s + swz16(ks * 16 + b_row, nn * 2 + (lane >> 4)));
        mma_bf16_16816(acc[2 * nn], af, bf[0], bf[1]);
        mma_bf16_16816(acc[2 * nn + 1], af, bf[2], bf[3]);
      }
    }
    __syncthreads();  // the stage is refilled by the next iteration's load
  }

#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int row = warp * 16 + g + r * 8;
    if (row < rows) {
      float* dst = out + ((size_t)(b0 + row) * H + h) * MLA_D_V + t4 * 2;
#pragma unroll
      for (int i = 0; i < 16; ++i) *reinterpret_cast<float2*>(dst + i * 8) = make_float2(acc[i][2 * r], acc[i][2 * r + 1]);
    }
  }
}

}  // namespace

cudaError_t launch_absorb_q(const __nv_bfloat16* q_nope, const __nv_bfloat16* q_rope, const __nv_bfloat16* w_uk,
                            __nv_bfloat16* q_out, int batch, int heads, cudaStream_t stream) {
  dim3 grid((batch + kTileM - 1) / kTileM, kDLatent / kTileN, heads);
  absorb_q_kernel<<<grid, kThreads, 0, stream>>>(q_nope, q_rope, w_uk, q_out, batch, heads);
  return cudaGetLastError();
}

cudaError_t launch_absorb_o(const float* out_latent, const __nv_bfloat16* w_uv, float* out, int batch, int heads,
                            cudaStream_t stream) {
  // 96 KB of dynamic shared memory (set on every call: the attribute is per device).
  const cudaError_t attr = cudaFuncSetAttribute(absorb_o_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kOSmem);
  if (attr != cudaSuccess) return attr;
  dim3 grid((batch + kTileM - 1) / kTileM, heads);
  absorb_o_kernel<<<grid, kThreads, kOSmem, stream>>>(out_latent, w_uv, out, batch, heads);
  return cudaGetLastError();
}

}  // namespace mla
