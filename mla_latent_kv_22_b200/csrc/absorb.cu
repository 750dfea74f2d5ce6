// Key and value absorption: H independent small GEMMs (warp-level tensor cores).
//
//   absorb_q:  q'[b,h,0:512] = q_nope[b,h,:] W_UK[h]   ([B x 128] x [128 x 512]),
//              q'[b,h,512:576] = q_rope[b,h,:]
//   absorb_o:  out[b,h,:] = bf16(out_latent[b,h,:]) W_UV[h]   ([B x 512] x [512 x 128])
// (glossary entry, "why absorb in decode": q^C (W^UK)^T and (sum_t p_t c_t) W^UV.)
//
// Both are HBM-bound (about 1 GFLOP against tens of MB at the largest workload):
// one CTA computes a 64 x 128 output tile of one head with 4 warps, operands
// staged through swizzled shared memory.
#include "mla_device.cuh"
#include "mla_internal.h"

namespace mla {
namespace {

constexpr int kThreads = 128;
constexpr int kTileM = 64, kTileN = 128, kTileK = 128;
constexpr int kChunks = kTileK * 2 / 16;  // 16 chunks of 16 B per 128-wide bf16 row

__device__ __forceinline__ uint32_t swz16(int r, int c) { return (uint32_t)(r * kChunks + (c ^ (r & 7))) * 16u; }

// acc[16x128] += A[16 x 128] * B[128 x 128] for warp rows [16w, 16w+16).
__device__ __forceinline__ void warp_tile_mma(float (&acc)[16][4], uint32_t a_s, uint32_t b_s, int warp, int lane) {
  const int a_row = warp * 16 + (lane & 15);
  const int b_row = (lane & 7) + (((lane >> 3) & 1) << 3);
#pragma unroll
  for (int kc = 0; kc < kTileK / 16; ++kc) {
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

// Stage a [rows x 128] bf16 block (row stride in elements) into swizzled smem.
__device__ __forceinline__ void stage_bf16(uint32_t dst, const __nv_bfloat16* src, size_t stride, int rows,
                                           int valid_rows, const void* safe) {
  for (int i = threadIdx.x; i < rows * kChunks; i += kThreads) {
    const int r = i / kChunks, c = i % kChunks;
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
  stage_bf16(smem_u32(a_tile), q_nope + ((size_t)b0 * H + h) * MLA_D_NOPE, (size_t)H * MLA_D_NOPE, kTileM, rows,
             q_nope);
  stage_bf16(smem_u32(b_tile), w_uk + (size_t)h * MLA_D_NOPE * kDLatent + n0, kDLatent, kTileK, kTileK, w_uk);
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();

  float acc[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
  warp_tile_mma(acc, smem_u32(a_tile), smem_u32(b_tile), warp, lane);

  const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int row = warp * 16 + g + r * 8;
    if (row < rows) {
      __nv_bfloat16* dst = q_out + ((size_t)(b0 + row) * H + h) * kDQK + n0 + t4 * 2;
#pragma unroll
      for (int i = 0; i < 16; ++i)
        *reinterpret_cast<uint32_t*>(dst + i * 8) = pack_bf16x2(acc[i][2 * r], acc[i][2 * r + 1]);
    }
  }
  if (blockIdx.y == 0) {  // rope half of q' is a copy
    for (int i = threadIdx.x; i < rows * 8; i += kThreads) {
      const int r = i >> 3, c = i & 7;
      const uint4 v = *reinterpret_cast<const uint4*>(q_rope + ((size_t)(b0 + r) * H + h) * kDRope + c * 8);
      *reinterpret_cast<uint4*>(q_out + ((size_t)(b0 + r) * H + h) * kDQK + kDLatent + c * 8) = v;
    }
  }
}

__global__ void __launch_bounds__(kThreads) absorb_o_kernel(const float* __restrict__ out_latent,
                                                            const __nv_bfloat16* __restrict__ w_uv,
                                                            float* __restrict__ out, int B, int H) {
  __shared__ __align__(128) uint8_t a_tile[kTileM * kTileK * 2];
  __shared__ __align__(128) uint8_t b_tile[kTileK * kTileN * 2];
  const int b0 = blockIdx.x * kTileM, h = blockIdx.z;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int rows = min(kTileM, B - b0);
  float acc[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;

  for (int k0 = 0; k0 < kDLatent; k0 += kTileK) {
    stage_bf16(smem_u32(b_tile), w_uv + ((size_t)h * kDLatent + k0) * MLA_D_V, MLA_D_V, kTileK, kTileK, w_uv);
    cp_async_commit();
    // A: fp32 -> bf16 (round to nearest even), 8 values (one 16-byte chunk) per step.
    for (int i = threadIdx.x; i < kTileM * kChunks; i += kThreads) {
      const int r = i / kChunks, c = i % kChunks;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (r < rows) {
        const float4* src = reinterpret_cast<const float4*>(out_latent + ((size_t)(b0 + r) * H + h) * kDLatent + k0 + c * 8);
        const float4 x = src[0], y = src[1];
        v = make_uint4(pack_bf16x2(x.x, x.y), pack_bf16x2(x.z, x.w), pack_bf16x2(y.x, y.y), pack_bf16x2(y.z, y.w));
      }
      *reinterpret_cast<uint4*>(a_tile + swz16(r, c)) = v;
    }
    cp_async_wait<0>();
    __syncthreads();
    warp_tile_mma(acc, smem_u32(a_tile), smem_u32(b_tile), warp, lane);
    __syncthreads();
  }

  const int g = lane >> 2, t4 = lane & 3;
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
  dim3 grid((batch + kTileM - 1) / kTileM, 1, heads);
  absorb_o_kernel<<<grid, kThreads, 0, stream>>>(out_latent, w_uv, out, batch, heads);
  return cudaGetLastError();
}

}  // namespace mla
