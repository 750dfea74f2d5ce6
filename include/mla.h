/*
 * mla.h -- C ABI of libmla.so: absorbed Multi-head Latent Attention decode on
 * NVIDIA B200 (sm_100a).
 *
 * What is computed (one new query token per sequence, s_q = 1):
 *
 *   Each cached token t of sequence b is one 576-wide bf16 row
 *       row_t = [ c_t (512 latent dims) | k_rope_t (64 rope dims) ],
 *   shared by every query head ("Multi-head Latent Attention" glossary entry,
 *   teaching abstraction: the cache holds the latent c^KV plus one decoupled
 *   rope key shared across heads).
 *
 *   The absorbed query of head h is q'_h = [ q_nope_h W_UK[h] (512) | q_rope_h (64) ]
 *   (glossary, "why absorb in decode": q^C (W^UK)^T; FlashMLA issue #16
 *   "up matrix is not involved?": q goes from [bs, H, 128] to [bs, H, 512]
 *   concatenated with q_rope [bs, H, 64], and the attention output is
 *   [bs, H, 512]).
 *
 *   mla_decode computes, for every (b, h), with T = cache_seqlens[b]:
 *       s_t  = softmax_scale * <q'_h, row_t>          (all 576 dims: content + rope score)
 *       lse  = ln sum_t exp(s_t)                      (natural log, scale included)
 *       out  = sum_t exp(s_t - lse) * row_t[0:512]    (values = the latent itself)
 *   and mla_absorb_o lifts out to per-head values: out_h W_UV[h]
 *   (glossary: sum_t p_t (c_t W^UV) = (sum_t p_t c_t) W^UV).
 *
 * Conventions shared by every entry point
 *   - Pointers marked "device" must be device memory of the current CUDA device;
 *     "host" pointers are host memory.  Every tensor is dense, row-major, with the
 *     layout given; base addresses must be 16-byte aligned.
 *   - The caller owns every tensor; the library never frees or retains them past
 *     the call.  The library owns only its workspace and a per-device error word.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream).  No entry point below synchronises the host except
 *     mla_get_device_error and mla_set_workspace.
 *   - Errors found on the host (null pointer, unsupported size, misalignment)
 *     return a status before anything is launched.  Errors found on the device
 *     (a page id outside [0, num_pages), a bounded wait that ran out) set the
 *     per-device error word, read by mla_get_device_error; the affected
 *     sequences' outputs are NaN.  No kernel traps.
 *   - Fixed widths: latent 512, rope 64 (row 576), page 64 tokens, and for the
 *     absorption GEMMs 128 no-rope query dims and 128 value dims.  Heads 1..128.
 */
#ifndef MLA_H_
#define MLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* mla_stream_t; /* same handle as cudaStream_t */

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1,     /* null pointer, negative size, misaligned address      */
  MLA_ERR_UNSUPPORTED = 2,     /* a size outside what the kernels handle (e.g. H > 128) */
  MLA_ERR_WORKSPACE = 3,       /* workspace too small and cannot grow (external, or capture) */
  MLA_ERR_CUDA = 4,            /* a CUDA runtime call failed; see mla_last_error_message */
  MLA_ERR_DEVICE_BAD_PAGE = 5, /* device: a block-table entry outside [0, num_pages)   */
  MLA_ERR_DEVICE_TIMEOUT = 6   /* device: a bounded wait gave up                        */
} mla_status_t;

enum {
  MLA_D_LATENT = 512,
  MLA_D_ROPE = 64,
  MLA_D_QK = 576,
  MLA_PAGE_TOKENS = 64,
  MLA_D_NOPE = 128,
  MLA_D_V = 128,
  MLA_MAX_HEADS = 128
};

/*
 * mla_decode -- split-KV absorbed decode against the (paged) latent cache.
 *
 * q             device bf16 [batch, heads, 576]: q'_h = [q_nope W_UK | q_rope].
 * kv_cache      device bf16.  Paged (block_table != NULL): [num_pages, 64, 576],
 *               token t of sequence b is row t % 64 of page block_table[b][t / 64]
 *               (glossary, capacity section: the latent cache can still be paged
 *               into blocks).  Contiguous (block_table == NULL):
 *               [batch, max_blocks * 64, 576]; num_pages is ignored.
 * block_table   device int32 [batch, max_blocks], or NULL.  Entries at or beyond
 *               ceil(T_b / 64) are never read.
 * cache_seqlens device int32 [batch], 0 <= T_b <= max_blocks * 64 (read on the
 *               device only; never copied to the host).
 * out           device fp32 [batch, heads, 512], fully overwritten.
 * lse           device fp32 [batch, heads], natural-log sum of exp(scaled score),
 *               fully overwritten.  T_b = 0 gives out = 0, lse = -inf.
 * softmax_scale multiplies the whole 576-dim dot product (1/sqrt(192) for
 *               128 no-rope + 64 rope query dims, as the glossary's runnable check
 *               scales by 1/sqrt(d_k + d_r)).
 * Rows of a last page beyond T_b, and unused block-table entries, may hold
 * anything (NaN included); they do not affect the result.
 * Uses the library workspace (split partials and per-sequence records): see
 * mla_workspace_size / mla_set_workspace.  The split of each sequence depends
 * only on (batch, heads, cache_seqlens, the device's SM count), never on page
 * ids, so a paged and a contiguous cache holding the same rows give
 * bit-identical results.
 */
mla_status_t mla_decode(const void* q, const void* kv_cache, const int32_t* block_table,
                        const int32_t* cache_seqlens, float* out, float* lse,
                        int batch, int heads, int num_pages, int max_blocks,
                        float softmax_scale, mla_stream_t stream);

/*
 * mla_decode_multi -- mla_decode with s_q query tokens per sequence (multi-token
 * prediction, speculative verification): the s_q new tokens are the last s_q
 * cached rows of each sequence, and each attends causally.
 *
 * q       device bf16 [batch, s_q, heads, 576]
 * out     device fp32 [batch, s_q, heads, 512], fully overwritten
 * lse     device fp32 [batch, s_q, heads], fully overwritten
 * Query i (0 <= i < s_q) of sequence b sits at position T_b - s_q + i and attends
 * to the cached tokens t <= T_b - s_q + i, i.e. the first T_b - s_q + 1 + i rows;
 * a query whose window is empty (T_b < s_q - i) gets out = 0, lse = -inf.  The
 * pages describe single-token decode only; this is the causal reading of several
 * new tokens appended to the cache before the call.  Each query row is computed as
 * in mla_decode (s_q = 1 gives exactly mla_decode), with the s_q x heads rows of a
 * sequence sharing every load of its cached rows.
 * s_q >= 1, heads <= 128 and s_q * heads <= 2048, else MLA_ERR_UNSUPPORTED.
 * Up to 128 rows share one pass over the cache; more rows run as groups of 128,
 * each group reading the cache again.  Every other
 * argument, the workspace, determinism and error behaviour are those of
 * mla_decode (mla_workspace_size takes s_q * heads as its heads).
 */
mla_status_t mla_decode_multi(const void* q, const void* kv_cache, const int32_t* block_table,
                              const int32_t* cache_seqlens, float* out, float* lse,
                              int batch, int s_q, int heads, int num_pages, int max_blocks,
                              float softmax_scale, mla_stream_t stream);

/*
 * mla_absorb_q -- key absorption, H independent GEMMs [batch x 128] x [128 x 512].
 *
 * q_nope  device bf16 [batch, heads, 128]
 * q_rope  device bf16 [batch, heads, 64]
 * w_uk    device bf16 [heads, 128, 512]; row i of head h holds the latent weights of
 *         key dim i (the glossary's W^UK_h transposed), so
 * q_out   device bf16 [batch, heads, 576] receives
 *         q_out[b,h,0:512]   = q_nope[b,h,:] W_UK[h]   (fp32 accumulate, bf16 round-to-nearest-even)
 *         q_out[b,h,512:576] = q_rope[b,h,:]           (copied)
 * (glossary, "why absorb in decode", first identity; FlashMLA issue #16.)
 */
mla_status_t mla_absorb_q(const void* q_nope, const void* q_rope, const void* w_uk, void* q_out,
                          int batch, int heads, mla_stream_t stream);

/*
 * mla_absorb_o -- value absorption, H independent GEMMs [batch x 512] x [512 x 128].
 *
 * out_latent device fp32 [batch, heads, 512] (mla_decode's out); rounded to bf16
 *            (nearest-even) on load, fp32 accumulate.
 * w_uv       device bf16 [heads, 512, 128]
 * out        device fp32 [batch, heads, 128] = out_latent[b,h,:] W_UV[h]
 * (glossary, "why absorb in decode", second identity; FlashMLA issue #16: the
 * [bs, H, 512] output is projected independently of the attention kernel.)
 */
mla_status_t mla_absorb_o(const float* out_latent, const void* w_uv, float* out,
                          int batch, int heads, mla_stream_t stream);

/*
 * mla_decode_noalloc -- mla_decode for callers that cannot allocate device memory.
 *
 * The pages have no counterpart of this call; it exists for callers such as a
 * serving runtime that has already reserved all device memory for its own pool,
 * or latency-critical paths that cannot absorb cudaMalloc's implicit device
 * synchronisation.  Arguments, layouts, results and errors are those of
 * mla_decode.  Instead of the workspace, it uses one 32 MiB static device array
 * that each GPU loading the library holds until exit; it never calls cudaMalloc or
 * cudaFree.  Sizes whose split partials and per-sequence records do not fit are
 * rejected with MLA_ERR_UNSUPPORTED before any launch; to fit, it may split over fewer workers
 * than mla_decode, so results match mla_decode within rounding, not bit for bit.
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress).  All calls on a device share the array (it keeps the last
 * call's contents; nothing in it must start at zero): calls that overlap on the GPU
 * race and must be serialised by the caller.
 */
mla_status_t mla_decode_noalloc(const void* q, const void* kv_cache, const int32_t* block_table,
                                const int32_t* cache_seqlens, float* out, float* lse,
                                int batch, int heads, int num_pages, int max_blocks,
                                float softmax_scale, mla_stream_t stream);

/* Bytes of workspace mla_decode needs on the current device for these sizes. */
size_t mla_workspace_size(int batch, int heads, int max_blocks);

/*
 * Give the library a caller-owned device buffer (>= 256-byte aligned) as the
 * current device's workspace; NULL returns to library-owned, grow-only storage
 * (allocated with cudaMalloc on first need, refused while `stream` is capturing a
 * graph).  The buffer must stay valid while calls that use it may run.  Blocks
 * until the device is idle before switching.
 */
mla_status_t mla_set_workspace(void* dev_ptr, size_t bytes);

/*
 * Synchronise `stream`, then read and clear the current device's error word.
 * Returns MLA_OK, MLA_ERR_DEVICE_BAD_PAGE or MLA_ERR_DEVICE_TIMEOUT (or
 * MLA_ERR_CUDA if the synchronisation itself failed).
 */
mla_status_t mla_get_device_error(mla_stream_t stream);

/* Static text for a status code. */
const char* mla_status_string(mla_status_t status);

/* Detail of the last host-side error on this thread (static storage, never NULL). */
const char* mla_last_error_message(void);

/* ---------------------------------------------------------------------------
 * Testing and measurement hooks.  They change how work is split or which decode
 * kernel runs, never what is computed.
 * ------------------------------------------------------------------------- */
typedef enum {
  MLA_KNOB_NUM_WORKERS = 0,     /* > 0: force the number of split workers; 0 = auto         */
  MLA_KNOB_MIN_PAGES = 1,       /* > 0: minimum pages per worker; 0 = auto                  */
  MLA_KNOB_DECODE_KERNEL = 2,   /* 0 = auto (3); 2 = CTA pair split by latent dims, partial
                                   scores exchanged through distributed shared memory;
                                   3 = CTA pair split by heads, pair-wide tcgen05 MMAs       */
  MLA_KNOB_WAIT_LIMIT = 3,      /* > 0: time limit of bounded device waits in ms; 0 = 2000  */
  MLA_KNOB_WITHHOLD_ARRIVE = 4, /* 1: the decode kernel's producer skips one load, so the
                                   consumer's bounded wait must run out (timeout test)      */
  MLA_KNOB_SPLIT_POLICY = 5,    /* 0 = auto: one whole sequence per worker when batch <= the
                                   worker count and the longest sequence is at most 16 pages
                                   above the split quota, else split; 1 = always split;
                                   2 = whole sequences whenever batch <= the worker count.
                                   A forced MLA_KNOB_NUM_WORKERS always splits.             */
  MLA_KNOB_PIECE_COST = 6       /* pages a split charges each sequence for its fixed cost
                                   (q' staging, pipeline fill, epilogue) when it lays the
                                   sequences end to end and cuts equal shares: 0 = auto (8,
                                   a multiple of the 4-page step, so pieces of step-aligned
                                   sequences stay aligned); k > 0: min(k - 1, 256) pages 
                                   (1 = split by pages alone)                               */
} mla_knob_t;
mla_status_t mla_set_knob(mla_knob_t knob, int value);
int mla_get_knob(mla_knob_t knob);
/* Which decode kernel mla_decode runs for `heads` under the current knobs:
   2 or 3 (MLA_KNOB_DECODE_KERNEL's numbering), -1 = none handles it. */
int mla_selected_decode_kernel(int heads);

/*
 * Per-launch device timing.  While enabled, every mla_decode records CUDA events
 * around each of its launches on its stream.  mla_timing_read synchronises on the
 * last event and writes the summed milliseconds since enabling into ms[0..2] --
 * ms[0] the split schedule (no launch of its own: every decode CTA derives its page
 * range from the lengths, so this is the empty interval between two events), ms[1]
 * the decode, ms[2] the combine -- and the number of recorded calls into *calls; it
 * then clears the record.
 */
mla_status_t mla_timing_enable(int enable);
mla_status_t mla_timing_read(float ms[3], int* calls);

#ifdef __cplusplus
}
#endif
#endif /* MLA_H_ */
