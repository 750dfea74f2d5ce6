// Split combine: merges the pieces of each split sequence by their log-sum-exp.
//
// For pieces s with normalised outputs O_s and lse L_s:
//   L = ln sum_s e^{L_s},  out = sum_s e^{L_s - L} O_s
// -- the rescaling the glossary's online-softmax note applies tile by tile, applied
// once more across workers.  One warp per (sequence, head); each lane owns 16 of
// the 512 dims as four float4 so every warp-wide load is 512 contiguous bytes.
// Sequences covered by a single worker were written by the decode kernel already;
// empty sequences get out = 0, lse = -inf; invalid lengths get NaN.
#include "mla_device.cuh"
#include "mla_internal.h"

namespace mla {
namespace {

constexpr int kWarps = 4;

__global__ void __launch_bounds__(kWarps * 32) combine_kernel(DecodeArgs a) {
  grid_dep_wait();  // the decode grid's partials are complete and visible
  const int b = blockIdx.x;
  const int lane = threadIdx.x & 31;
  const int h = blockIdx.y * kWarps + (threadIdx.x >> 5);
  if (h >= a.heads) return;
  const Schedule& sc = a.sched;
  const SeqInfo si = sc.seq[b];
  float4* out4 = reinterpret_cast<float4*>(a.out + ((size_t)b * a.heads + h) * kDLatent);
  if (si.num_pieces == 1) return;
  if (si.num_pieces <= 0) {
    const float v = si.num_pieces == 0 ? 0.f : NAN;
#pragma unroll
    for (int i = 0; i < 4; ++i) out4[lane + 32 * i] = make_float4(v, v, v, v);
    if (lane == 0) a.lse[(size_t)b * a.heads + h] = si.num_pieces == 0 ? -INFINITY : NAN;
    return;
  }
  const int P = sc.num_workers;
  const int q = *sc.quota;
  const int st = sc.seq_start[b];
  auto slot_of = [&](int k) {
    const int w = si.first_worker + k;
    return (w * q >= st) ? w : P + w;  // the piece is the worker's first sequence iff its range starts in b
  };
  float L = -INFINITY;
  for (int k = lane; k < si.num_pieces; k += 32) L = fmaxf(L, sc.part_lse[(size_t)slot_of(k) * a.heads + h]);
#pragma unroll
  for (int o = 16; o; o >>= 1) L = fmaxf(L, __shfl_xor_sync(0xffffffffu, L, o));

  float4 acc[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  float wsum = 0.f;
  for (int k = 0; k < si.num_pieces; ++k) {
    const int slot = slot_of(k);
    const float wk = expf(sc.part_lse[(size_t)slot * a.heads + h] - L);
    wsum += wk;
    const float4* src = reinterpret_cast<const float4*>(sc.part_o + ((size_t)slot * a.heads + h) * kDLatent);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 v = src[lane + 32 * i];
      acc[i].x += wk * v.x;
      acc[i].y += wk * v.y;
      acc[i].z += wk * v.z;
      acc[i].w += wk * v.w;
    }
  }
  const float inv = 1.f / wsum;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    out4[lane + 32 * i] = make_float4(acc[i].x * inv, acc[i].y * inv, acc[i].z * inv, acc[i].w * inv);
  if (lane == 0) a.lse[(size_t)b * a.heads + h] = L + logf(wsum);
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
