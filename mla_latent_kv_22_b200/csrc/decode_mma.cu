// Split-KV absorbed-MLA decode on the warp-level tensor-core path (mma.sync).
//
// One CTA = one worker x 64 heads.  The worker walks its page range (see
// Schedule); per sequence piece it stages q' for its 64 heads in shared memory
// once, then streams 64-token pages through a two-stage cp.async ring and runs
// the online softmax of the glossary's paging/online-softmax note:
//   S = q' K^T (all 576 dims), running max m and sum l in the log2 domain,
//   O = O * 2^(m_old - m_new) + P V  with V = the first 512 dims of the same rows.
// Warp w owns heads [16*(w%4), +16) and value dims [256*(w/4), +256); the two
// warps of a head group compute the same S (no exchange needed) and keep their
// halves of O in registers.
//
// Rows at or beyond the sequence length, and pages with an invalid id, are
// zero-filled by the copy itself (src-size 0), so poison in the cache is never
// read; an invalid page id sets the error word and makes the piece NaN.
#include "mla_device.cuh"
#include "mla_internal.h"

namespace mla {
namespace {

constexpr int kHeadsPerCta = 64;
constexpr int kThreads = 256;
constexpr int kRowChunks = kDQK * 2 / 16;                // 72 16-byte chunks per row
constexpr int kTileBytes = 64 * kDQK * 2;                // 73728: 64 rows x 576 bf16
constexpr int kSmemBytes = 3 * kTileBytes;               // q' tile + 2 KV stages

// Byte offset of 16-byte chunk c of row r in a swizzled [64 x 576] bf16 tile.
// XOR-ing the chunk's low 3 bits with the row keeps ldmatrix free of bank conflicts.
__device__ __forceinline__ uint32_t swz(int r, int c) { return (uint32_t)(r * kRowChunks + (c ^ (r & 7))) * 16u; }

// Copy 64 rows of 576 bf16 into a swizzled tile; rows >= valid are zero-filled.
__device__ __forceinline__ void load_tile(uint32_t dst, const __nv_bfloat16* src_rows, int row_stride_elems,
                                          int valid, const void* safe_src) {
  for (int i = threadIdx.x; i < 64 * kRowChunks; i += kThreads) {
    const int r = i / kRowChunks, c = i - r * kRowChunks;
    const bool ok = r < valid;
    const void* src = ok ? (const void*)(src_rows + (size_t)r * row_stride_elems + c * 8) : safe_src;
    cp_async_16(dst + swz(r, c), src, ok ? 16 : 0);
  }
}

__global__ void __launch_bounds__(kThreads, 1) decode_mma_kernel(DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t q_s = smem_u32(smem);
  const uint32_t kv_s0 = q_s + kTileBytes;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int hg = warp & 3;   // 16-head group within the CTA
  const int dh = warp >> 2;  // value-dim half
  const int g = lane >> 2, t4 = lane & 3;
  const int w = blockIdx.x;
  const int h0 = blockIdx.y * kHeadsPerCta;
  const Schedule& sc = a.sched;
  const WorkerRange rg = sc.ranges[w];
  if (rg.b0 < 0) return;
  const int P = sc.num_workers;
  const float scale2 = a.scale * kLog2e;

  for (int b = rg.b0; b <= rg.b1; ++b) {
    const int st = sc.seq_start[b];
    const int n_pages = sc.seq_start[b + 1] - st;
    const int pa = (b == rg.b0) ? rg.p0 : 0;
    const int pe = (b == rg.b1) ? rg.p1 : n_pages;
    if (pa >= pe) continue;
    const int T = a.seqlens[b];
    const bool complete = (pa == 0 && pe == n_pages);

    // Stage q' rows h0..h0+63 of sequence b (rows beyond H are zero).
    load_tile(q_s, a.q + ((size_t)b * a.heads + h0) * kDQK, kDQK, a.heads - h0, a.q);

    auto page_id = [&](int p) -> int {
      return a.block_table ? a.block_table[(size_t)b * a.max_blocks + p] : b * a.max_blocks + p;
    };
    const int np = a.block_table ? a.num_pages : a.batch * a.max_blocks;
    bool bad = false;
    auto issue_page = [&](int p, int stage) {
      const int pid = page_id(p);
      const bool ok = (unsigned)pid < (unsigned)np;
      if (!ok) {
        bad = true;
        if (tid == 0) set_device_error(a.err, MLA_ERR_DEVICE_BAD_PAGE);
      }
      const int valid = ok ? min(kPage, T - p * kPage) : 0;
      load_tile(kv_s0 + stage * kTileBytes, a.kv + (size_t)(ok ? pid : 0) * kPage * kDQK, kDQK, valid, a.kv);
    };

    issue_page(pa, 0);
    cp_async_commit();

    float o[32][4];
#pragma unroll
    for (int i = 0; i < 32; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m_r[2] = {-INFINITY, -INFINITY};
    float l_r[2] = {0.f, 0.f};

    for (int p = pa; p < pe; ++p) {
      const int stage = (p - pa) & 1;
      if (p + 1 < pe) {
        issue_page(p + 1, stage ^ 1);
        cp_async_commit();
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();
      const uint32_t kv_s = kv_s0 + stage * kTileBytes;
      const int valid = min(kPage, T - p * kPage);

      // ---- S[16 x 64] = q'[16 x 576] K[64 x 576]^T ----
      float s[8][4];
#pragma unroll
      for (int j = 0; j < 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
      const int a_row = hg * 16 + (lane & 15);
      const int b_row = (lane & 7) + ((lane >> 4) << 3);
      const int b_csel = (lane >> 3) & 1;
#pragma unroll 4
      for (int kc = 0; kc < kDQK / 16; ++kc) {
        uint32_t af[4];
        ldmatrix_x4(af, q_s + swz(a_row, kc * 2 + (lane >> 4)));
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t bf[4];
          ldmatrix_x4(bf, kv_s + swz(j * 16 + b_row, kc * 2 + b_csel));
          mma_bf16_16816(s[2 * j], af, bf[0], bf[1]);
          mma_bf16_16816(s[2 * j + 1], af, bf[2], bf[3]);
        }
      }

      // ---- online softmax (log2 domain) ----
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int tok = j * 8 + t4 * 2 + (e & 1);
          float v = s[j][e] * scale2;
          v = tok < valid ? v : -INFINITY;
          s[j][e] = v;
          mx[e >> 1] = fmaxf(mx[e >> 1], v);
        }
      }
      float alpha[2];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
        mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
        const float m_new = fmaxf(m_r[r], mx[r]);
        alpha[r] = fast_exp2(m_r[r] - m_new);
        m_r[r] = m_new;
      }
      float rs[2] = {0.f, 0.f};
      uint32_t pf[4][4];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float p0 = fast_exp2(s[j][0] - m_r[0]);
        const float p1 = fast_exp2(s[j][1] - m_r[0]);
        const float p2 = fast_exp2(s[j][2] - m_r[1]);
        const float p3 = fast_exp2(s[j][3] - m_r[1]);
        rs[0] += p0 + p1;
        rs[1] += p2 + p3;
        pf[j >> 1][(j & 1) * 2 + 0] = pack_bf16x2(p0, p1);
        pf[j >> 1][(j & 1) * 2 + 1] = pack_bf16x2(p2, p3);
      }
      l_r[0] = l_r[0] * alpha[0] + rs[0];
      l_r[1] = l_r[1] * alpha[1] + rs[1];
      if (alpha[0] != 1.f || alpha[1] != 1.f) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          o[i][0] *= alpha[0];
          o[i][1] *= alpha[0];
          o[i][2] *= alpha[1];
          o[i][3] *= alpha[1];
        }
      }

      // ---- O[16 x 256] += P[16 x 64] V[64 x 256] ----
      const int v_row = (lane & 7) + (((lane >> 3) & 1) << 3);
      const int v_csel = lane >> 4;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        // A fragment of P for tokens 16kk..16kk+15: tiles 2kk (a0,a1) and 2kk+1 (a2,a3).
        const uint32_t pa_frag[4] = {pf[kk][0], pf[kk][1], pf[kk][2], pf[kk][3]};
#pragma unroll
        for (int dn = 0; dn < 16; ++dn) {
          uint32_t bf[4];
          const int chunk = (dh * 256 + dn * 16) / 8 + v_csel;
          ldmatrix_x4_trans(bf, kv_s + swz(kk * 16 + v_row, chunk));
          mma_bf16_16816(o[2 * dn], pa_frag, bf[0], bf[1]);
          mma_bf16_16816(o[2 * dn + 1], pa_frag, bf[2], bf[3]);
        }
      }
      __syncthreads();  // the stage is refilled by the next iteration's prefetch
    }

    // ---- epilogue: normalise, write out/lse or the partial slot ----
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      l_r[r] += __shfl_xor_sync(0xffffffffu, l_r[r], 1);
      l_r[r] += __shfl_xor_sync(0xffffffffu, l_r[r], 2);
    }
    const bool any_bad = __syncthreads_or(bad);
    const float inv[2] = {any_bad ? NAN : 1.f / l_r[0], any_bad ? NAN : 1.f / l_r[1]};
    const float lse_v[2] = {any_bad ? NAN : (m_r[0] + __log2f(l_r[0])) * kLn2,
                            any_bad ? NAN : (m_r[1] + __log2f(l_r[1])) * kLn2};
    float* obase;
    float* lbase;
    size_t hstride;
    if (complete) {
      obase = a.out + (size_t)b * a.heads * kDLatent;
      lbase = a.lse + (size_t)b * a.heads;
      hstride = kDLatent;
    } else {
      const int slot = (b == rg.b0) ? w : P + w;
      obase = sc.part_o + (size_t)slot * a.heads * kDLatent;
      lbase = sc.part_lse + (size_t)slot * a.heads;
      hstride = kDLatent;
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int h = h0 + hg * 16 + g + r * 8;
      if (h < a.heads) {
        float* orow = obase + (size_t)h * hstride + dh * 256 + t4 * 2;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          float2 v = make_float2(o[i][2 * r] * inv[r], o[i][2 * r + 1] * inv[r]);
          *reinterpret_cast<float2*>(orow + i * 8) = v;
        }
        if (dh == 0 && t4 == 0) lbase[h] = lse_v[r];
      }
    }
    __syncthreads();  // q' tile is reloaded for the next sequence
  }
}

}  // namespace

int decode_mma_heads_per_cta() { return kHeadsPerCta; }

cudaError_t launch_decode_mma(const DecodeArgs& a, cudaStream_t stream) {
  static bool done[64] = {};
  cudaError_t e = allow_dynamic_smem(reinterpret_cast<const void*>(decode_mma_kernel), kSmemBytes, done);
  if (e != cudaSuccess) return e;
  dim3 grid(a.sched.num_workers, (a.heads + kHeadsPerCta - 1) / kHeadsPerCta);
  decode_mma_kernel<<<grid, kThreads, kSmemBytes, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace mla
