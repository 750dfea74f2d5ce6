// Host-side interface between the C-ABI layer (api.cu) and the kernel files.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <cudaTypedefs.h>

#include "mla.h"

namespace mla {

// Split schedule, derived on the device by every decode CTA (worker_range.cuh).
//
// The pages of all sequences are laid end to end (sequence-major); worker w takes
// the contiguous range [w*q, min((w+1)*q, N)) of that list, q = max(ceil(N/P),
// min_pages) rounded up to the kernel's page granule.  A worker's range covers a tail
// of its first sequence, whole middle sequences and a head of its last one.  A
// sequence that one worker covers entirely is written straight to out/lse; otherwise
// every worker writes its piece (normalised partial output and its lse) to a partial
// slot -- slot w when the sequence is the worker's first, slot P + w otherwise -- and
// the combine kernel merges the pieces by their lse.  Everything depends only on the
// sequence lengths, the batch size and P.
struct WorkerRange {
  int b0, p0;  // first sequence and its first page
  int b1, p1;  // last sequence and one past its last page (b0 < 0: no work)
};

struct SeqInfo {
  int first_worker;  // worker holding the sequence's first page
  int num_pieces;    // workers covering it; 0 = empty sequence; -1 = invalid length
  int first_slot;    // partial slot of the first piece (piece k > 0 is in slot first_worker + k)
};

struct Schedule {
  SeqInfo* seq;         // [B], written by the decode grid, read by the combine grid
  float* part_lse;      // [2P, H]  (natural-log lse of each piece)
  float* part_o;        // [2P, H, 512] normalised partial outputs
  int num_workers;      // P
};

// Workspace carve-up; `base` may be null to just compute the size.
size_t carve_schedule(void* base, int batch, int heads, int num_workers, Schedule* s);

struct DecodeArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* kv;
  const int32_t* block_table;  // null = contiguous cache
  const int32_t* seqlens;
  float* out;
  float* lse;
  int batch, heads, num_pages, max_blocks;
  float scale;
  int* err;
  Schedule sched;
  int wait_limit;       // bounded-wait time limit in milliseconds (tcgen05 kernel)
  int withhold_arrive;  // test hook (tcgen05 kernel)
  // Several query tokens per sequence (tcgen05 kernel only): a sequence has
  // row_stride = s_q x hq query rows in q, out and lse (row r = query r / hq; query i
  // sees the first T - s_q + 1 + i cached tokens), of which one launch handles the
  // `heads` rows starting at row0.  s_q = 1, hq = row_stride = heads, row0 = 0 otherwise.
  int s_q, hq, row_stride, row0;
  // Split schedule, derived by every decode CTA (worker_range.cuh): the least pages per
  // worker, the page granule of the kernel's steps, the whole-sequence slack (< 0:
  // always split), and the pages a piece is charged for its fixed cost.
  int min_pages, granule, whole_slack, piece_cost;
};

// The whole-sequence slack for the current knobs (a forced worker count always splits).
int schedule_whole_slack();
// The pages a split charges each sequence for its fixed cost, for the current knobs (at
// most kMaxPieceCost, so that batch x (max_blocks + cost) units fit the device's 32-bit
// schedule arithmetic whenever the host's size check passes).
constexpr int kMaxPieceCost = 256;
int schedule_piece_cost();
cudaError_t launch_combine(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_absorb_q(const __nv_bfloat16* q_nope, const __nv_bfloat16* q_rope,
                            const __nv_bfloat16* w_uk, __nv_bfloat16* q_out, int batch, int heads, int* err,
                            cudaStream_t stream);
cudaError_t launch_absorb_o(const float* out_latent, const __nv_bfloat16* w_uv, float* out, int batch,
                            int heads, int* err, cudaStream_t stream);

// Raises `kernel`'s dynamic shared memory limit to `bytes` on the current device, once
// per device (the attribute belongs to the device's context); `done` is the caller's
// per-device record.  Defined in api.cu.
cudaError_t allow_dynamic_smem(const void* kernel, int bytes, bool (&done)[64]);

// Defined in api.cu: the per-device decode plan, the thread's last-error text,
// and raw knob values.
mla_status_t decode_plan(int heads, int* kernel, int* num_workers, int** err_word);
mla_status_t record_error(mla_status_t s, const char* msg);
int knob_value(int knob);

// Decode kernels (mla_selected_decode_kernel's numbering): 2 = the CTA pair split by
// dims with partial scores exchanged through distributed shared memory
// (decode_tc.cu), 3 = the CTA pair split by heads with pair-wide MMAs (decode_pair.cu).
cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t stream);
int decode_tc_max_workers(int sm_count);
cudaError_t launch_decode_pair(const DecodeArgs& a, cudaStream_t stream);
int decode_pair_max_workers(int sm_count);
// The launch of kernel `kernel` and its page granule of the schedule.
cudaError_t launch_decode(int kernel, const DecodeArgs& a, cudaStream_t stream);
int decode_granule(int kernel);

// cuTensorMapEncodeTiled from the driver (resolved once; null if unavailable).  Defined in api.cu.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

}  // namespace mla
