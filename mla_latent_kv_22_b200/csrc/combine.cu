// Split combine: merges the pieces of each split sequence by their log-sum-exp.
//
// For pieces s with normalised outputs O_s and lse L_s:
//   L = ln sum_s e^{L_s},  out = sum_s e^{L_s - L} O_s
// -- the rescaling the glossary's online-softmax note applies tile by tile, applied
// once more across workers.  One warp per (sequence, head); each lane owns 16 of
// the 512 dims as four float4 so every warp-wide load is 512 contiguous bytes.  The
// partial slot of each piece comes from the sequence record (SeqInfo), so the loads
// depend on one read only.
// Sequences covered by a single worker were written by the decode kernel already;
// empty sequences get out = 0, lse = -inf; invalid lengths get NaN.
#include "mla_device.cuh"
#include "mla_internal.h"

namespace mla {
namespace {

constexpr int kWarps = 4;

__global__ void __launch_bounds__(kWarps * 32) combine_kernel(DecodeArgs a) {
  grid_dep_launch_dependents();  // the next grid (absorb_o, or the next call's decode) may launch; it waits for this one
  grid_dep_wait();  // the decode grid's partials are complete and visible
  const int b = blockIdx.x;
  const int lane = threadIdx.x & 31;
  const int h = blockIdx.y * kWarps + (threadIdx.x >> 5);
  if (h >= a.heads) return;
  const Schedule& sc = a.sched;
  const SeqInfo si = sc.seq[b];
  const size_t orow = (size_t)b * a.row_stride + a.row0 + h;  // this row in out and lse
  float4* out4 = reinterpret_cast<float4*>(a.out + orow * kDLatent);
  if (si.num_pieces == 1) return;
  if (si.num_pieces <= 0) {
    const float v = si.num_pieces == 0 ? 0.f : NAN;
#pragma unroll
    for (int i = 0; i < 4; ++i) out4[lane + 32 * i] = make_float4(v, v, v, v);
    if (lane == 0) a.lse[orow] = si.num_pieces == 0 ? -INFINITY : NAN;
    return;
  }
  const int np = si.num_pieces;
  auto src_of = [&](int k) {
    const int slot = k == 0 ? si.first_slot : si.first_worker + k;
    return reinterpret_cast<const float4*>(sc.part_o + ((size_t)slot * a.heads + h) * kDLatent);
  };
  auto lse_of = [&](int k) {
    const int slot = k == 0 ? si.first_slot : si.first_worker + k;
    return sc.part_lse[(size_t)slot * a.heads + h];
  };
  // The loads of the first kPre pieces (all that a sequence split in two needs) are
  // issued together, right after the sequence record, so a warp waits for memory
  // twice: lane k holds the lse of piece k and every lane its 16 dims of each piece's
  // output.  Later pieces are loaded one by one.  The sums run in piece order either
  // way.
  constexpr int kPre = 2;
  const float lk = lane < np ? lse_of(lane) : -INFINITY;
  float4 v[kPre][4];
#pragma unroll
  for (int k = 0; k < kPre; ++k) {
    if (k < np) {
      const float4* src = src_of(k);
#pragma unroll
      for (int i = 0; i < 4; ++i) v[k][i] = src[lane + 32 * i];
    }
  }
  float L = lk;
  for (int k = lane + 32; k < np; k += 32) L = fmaxf(L, lse_of(k));
#pragma unroll
  for (int o = 16; o; o >>= 1) L = fmaxf(L, __shfl_xor_sync(0xffffffffu, L, o));
  if (L == -INFINITY) {
    // No piece saw a token: a query row whose causal window is empty (several query
    // tokens per sequence).  A NaN lse (a bad page) still makes the row NaN.
    const bool nan = __any_sync(0xffffffffu, lk != lk);
    const float v = nan ? NAN : 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) out4[lane + 32 * i] = make_float4(v, v, v, v);
    if (lane == 0) a.lse[orow] = nan ? NAN : -INFINITY;
    return;
  }

  float4 acc[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  float wsum = 0.f;
  auto add = [&](float wk, const float4 (&x)[4]) {
    wsum += wk;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[i].x += wk * x[i].x;
      acc[i].y += wk * x[i].y;
      acc[i].z += wk * x[i].z;
      acc[i].w += wk * x[i].w;
    }
  };
#pragma unroll
  for (int k = 0; k < kPre; ++k)
    if (k < np) add(expf(__shfl_sync(0xffffffffu, lk, k) - L), v[k]);
  for (int k = kPre; k < np; ++k) {
    const float4* src = src_of(k);
    float4 x[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = src[lane + 32 * i];
    add(expf((k < 32 ? __shfl_sync(0xffffffffu, lk, k) : lse_of(k)) - L), x);
  }
  const float inv = 1.f / wsum;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    out4[lane + 32 * i] = make_float4(acc[i].x * inv, acc[i].y * inv, acc[i].z * inv, acc[i].w * inv);
  if (lane == 0) a.lse[orow] = L + logf(wsum);
}

}  // namespace

cudaError_t launch_combine(const DecodeArgs& a, cudaStream_t stream) {
  dim3 grid(a.batch, (a.heads + kWarps - 1) / kWarps);
  // Launched as a programmatic dependent of the decode grid: its launch overlaps
  // the decode's tail, and grid_dep_wait() orders it after the decode's writes.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kWarps * 32, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, combine_kernel, a);
}

}  // namespace mla
