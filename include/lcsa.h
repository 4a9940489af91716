/*
 * lcsa.h - C ABI of liblcsa.so, a B200 (sm_100a) implementation of the
 * locality-constrained sparse attention (LCSA) call of FlashVSR's streaming
 * video DiT.
 *
 * What one call computes (sources are page title + section):
 *   For every batch b, head h and query block qb of a T x H' x W' latent token
 *   grid (12 heads, head_dim 128, QK-norm with a norm that spans the heads of a
 *   token, factored 3D RoPE: "Add FlashVSR contrib model ... on Neuron", Model
 *   Information and Additional Information):
 *     1. q^, k^ = RoPE3D(RMSNorm(x) * gamma)               (prologue)
 *     2. pooled block means of q^ and k^                     (prologue)
 *     3. score = pooled_q . pooled_k, restricted to the KV blocks inside the
 *        local window, keep the best k blocks, ties to the lower block index,
 *        emitted as a CSR list ("FlashVSR: From 17.2 FPS to 57.3 FPS at
 *        768x1408", What Was Actually Slow and Rebuild sparse attention for
 *        Hopper: pooling, mask selection, fused CSR construction)
 *     4. out = softmax(q^ k^T * scale) v over the tokens of the kept blocks
 *        (block-sparse flash attention, same section).
 *   Parameters follow the "FlashVSR Inference" skill, Non-Negotiable Streaming
 *   Contract: local_range 11 or 9, KV window = kv_ratio (3.0) x query frames,
 *   topk_ratio = sparse_ratio * 768 * 1280 / (H * W), sizes divisible by 128,
 *   bf16 tensors; and "FlashVSR - Real-Time Diffusion-Based Video
 *   Super-Resolution", How it works: attention limited to local patches.
 *
 * Readings where the pages are silent: the RMSNorm spans heads*head_dim
 * (LCSA_NORM_TOKEN; LCSA_NORM_HEAD is offered), eps 1e-6; RoPE rotates pairs
 * (2i, 2i+1), first d-4*(d/6) dims by frame, next 2*(d/6) by token row, last
 * 2*(d/6) by token column (44/42/42 for d = 128, 24/20/20 for d = 64), pair
 * j of an n-dim axis turning by
 * pos * 10000^(-2j/n); the block score is the raw dot product of block means;
 * local_range is an odd window diameter in blocks applied as a Chebyshev
 * distance over (block row, block column), clipped at the frame edge and the
 * same in every frame of the KV window; the budget in blocks is
 * k = floor(topk_ratio * blocks per latent frame) with H = 16 H', W = 16 W';
 * query frames are the last q_frames of the KV window.
 *
 * Layouts (all row-major, no padding):
 *   q    bf16 [batch][q_frames*grid_h*grid_w][heads*head_dim]   (device)
 *   k, v bf16 [batch][kv_frames*grid_h*grid_w][heads*head_dim]  (device)
 *   out  bf16 [batch][q_frames*grid_h*grid_w][heads*head_dim]   (device)
 *   gamma_q, gamma_k fp32 [heads*head_dim]                      (device)
 *   Token index inside a frame group is raster: (t*grid_h + y)*grid_w + x.
 *   Blocks are numbered (frame group, block row, block column); tokens in a
 *   block (frame, row, column). CSR rows are numbered (b, h, qb), qb fastest.
 *
 * Ownership: the caller owns q, k, v, gains and out. The plan owns every
 * intermediate (normalised q^/k^, pooled values, CSR, RoPE table, error word,
 * optional host-IO staging), all allocated in lcsa_plan_create and freed in
 * lcsa_plan_destroy. lcsa_forward allocates nothing, is asynchronous on the
 * given stream and must not run concurrently with another call on the same
 * plan (the intermediates are shared).
 *
 * Errors: every entry point returns a status; none aborts, throws or falls
 * back to another implementation. lcsa_last_error_message() gives a one-line
 * detail for the calling thread. Failures inside a kernel set the plan's
 * device error word, read by lcsa_check_device_error.
 */
#ifndef LCSA_H
#define LCSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LCSA_ABI_VERSION 2  /* 2: lcsa_config_t.heads_total, head-sharded entry points */

#if defined(__GNUC__)
#define LCSA_API __attribute__((visibility("default")))
#else
#define LCSA_API
#endif

typedef enum {
  LCSA_OK = 0,
  LCSA_ERR_INVALID_ARG = 1,     /* null pointer, negative size, even local_range ... */
  LCSA_ERR_SHAPE = 2,           /* grid not divisible by the block, kv_frames < q_frames ... */
  LCSA_ERR_ALIGNMENT = 3,       /* a tensor pointer is not 16-byte aligned */
  LCSA_ERR_UNSUPPORTED = 4,     /* valid but outside what the kernels implement */
  LCSA_ERR_OOM = 5,             /* device allocation failed in lcsa_plan_create */
  LCSA_ERR_CUDA = 6,            /* a CUDA runtime call failed (no device, launch error) */
  LCSA_ERR_DEVICE_TIMEOUT = 7,  /* a kernel gave up a bounded wait */
  LCSA_ERR_DEVICE_BOUNDS = 8    /* a kernel found an index outside its buffers */
} lcsa_status_t;

#define LCSA_UNBOUNDED 0        /* local_range value that disables the window */
#define LCSA_NORM_TOKEN 0       /* RMSNorm over heads*head_dim of a token */
#define LCSA_NORM_HEAD 1        /* RMSNorm over head_dim of each head */

typedef struct lcsa_config {
  int batch;            /* >= 1 */
  int heads;            /* 1 .. 16 */
  int head_dim;         /* 128 (the pages' size) or 64 */
  int q_frames;         /* >= 1; the last q_frames of the KV window */
  int kv_frames;        /* >= q_frames (equal: self-attention over the chunk) */
  int grid_h, grid_w;   /* latent token grid per frame (H' = H/16, W' = W/16) */
  int block_t, block_h, block_w;  /* block shape; tokens per block must be 64 or 128,
                                     block_t*block_h <= 8 */
  int local_range;      /* odd window diameter in blocks, or LCSA_UNBOUNDED */
  int topk;             /* > 0: budget in blocks; 0: derive from sparse_ratio */
  float sparse_ratio;   /* used when topk == 0 (1.5 or 2.0 on the pages): finite, > 0;
                           a budget beyond 2^30 blocks keeps every admissible block */
  int kv_frame_offset;  /* absolute latent frame index of KV frame 0 (RoPE) */
  int norm_scope;       /* LCSA_NORM_TOKEN or LCSA_NORM_HEAD */
  float rms_eps;        /* finite, > 0 */
  float softmax_scale;  /* 0: 1/sqrt(head_dim) */
  int host_io;          /* 1: also allocate device staging for lcsa_forward_host */
  int heads_total;      /* 0, or the heads of the whole layer when this plan holds
                           `heads` of them (head-sharded; see lcsa_forward_sharded) */
} lcsa_config_t;

/* Sizes derived from a configuration (host-side, no device needed). */
typedef struct lcsa_geometry {
  int64_t q_tokens, kv_tokens;       /* per batch element */
  int64_t channels;                  /* heads*head_dim */
  int64_t block_tokens;              /* n_b */
  int64_t blocks_per_frame;          /* per frame group */
  int64_t q_blocks, kv_blocks;       /* per batch and head */
  int64_t rows;                      /* batch*heads*q_blocks */
  int64_t nnz;                       /* total kept blocks over all rows */
  int topk;                          /* resolved budget in blocks */
  int window_radius;                 /* r = (local_range-1)/2, -1 when unbounded */
  int min_window, max_window;        /* smallest / largest admissible-set size */
  double selected_flops;             /* sum over rows of kept * 4 * n_b^2 * head_dim */
  double prologue_bytes;             /* bytes the prologue must move (q,k in; q^,k^ out) */
  double attention_min_bytes;        /* q^ + out + each touched k^/v block once */
  size_t workspace_bytes;            /* device bytes the plan allocates (at most) */
} lcsa_geometry_t;

typedef struct lcsa_plan* lcsa_plan_t;

/* Fill *cfg with the stream-chunk defaults (12 heads, d 128, 2 of 6 frames,
   48x80 grid, 1x8x16 blocks, local_range 11, sparse_ratio 2.0, eps 1e-6). */
LCSA_API void lcsa_config_default(lcsa_config_t* cfg);

/* Validate *cfg and derive its sizes. Host only: touches no device.
   Returns LCSA_ERR_INVALID_ARG (a size < 1, an even or negative local_range,
   topk < 0, a non-finite or non-positive sparse_ratio (when used) or rms_eps,
   a negative or non-finite softmax_scale, kv_frame_offset < 0, a budget of 0
   blocks, heads_total < heads), LCSA_ERR_SHAPE (kv_frames < q_frames, or a
   token grid the block does not divide) or LCSA_ERR_UNSUPPORTED (head_dim
   other than 64 or 128, more heads than the kernels take, blocks of other than 64
   or 128 tokens or more than 8 token rows, a tensor of more than 2^40
   elements, a window larger than the selection's candidate limit). Sizes are
   bounded before any product of them is formed. */
LCSA_API lcsa_status_t lcsa_config_resolve(const lcsa_config_t* cfg, lcsa_geometry_t* out);

/* Validate, then allocate every intermediate on `cuda_device` and build the
   constant tables. *out is set only on LCSA_OK. */
LCSA_API lcsa_status_t lcsa_plan_create(const lcsa_config_t* cfg, int cuda_device, lcsa_plan_t* out);

/* Free everything the plan owns (synchronises the device). Null is a no-op. */
LCSA_API void lcsa_plan_destroy(lcsa_plan_t plan);

/* One LCSA call: prologue, block selection and block-sparse attention,
   launched on `stream` (a cudaStream_t; null = legacy default stream).
   q, k, v, out: device bf16 as laid out above, 16-byte aligned. gamma_q,
   gamma_k: device fp32 [heads*head_dim], 16-byte aligned. Asynchronous.
   Deterministic: the same inputs give the same output bits on every call,
   however the attention's work is spread over the SMs (with 64-token blocks
   and at least as many query-block pairs as SMs, the last pairs are cut into
   parts run by different CTAs and merged in a fixed part order). */
LCSA_API lcsa_status_t lcsa_forward(lcsa_plan_t plan, const void* q, const void* k, const void* v,
                           const float* gamma_q, const float* gamma_k, void* out, void* stream);

/* Same call from HOST buffers: copies q, k, v and the gains into plan-owned
   device staging, runs the call and copies out back. Needs a plan created
   with host_io = 1 (which also creates a plan-owned copy stream and five
   events). The gains, q and k go up on `stream`, v on the copy stream once
   they are in, so the prologue and the selection run while v uploads; with
   batch 1 and at least two heads the attention runs as two launches over
   the first and the second half of the heads, v goes up in those two halves
   of its channels (each launch waits only for its own), and the first
   half's output channels come back on the copy stream while the second half
   computes.
   The result equals lcsa_forward's bit for bit. Host buffers should be pinned
   for asynchronous copies; the call returns once `out` holds the result,
   after reading the plan's device error word as lcsa_check_device_error does
   (LCSA_ERR_DEVICE_TIMEOUT / LCSA_ERR_DEVICE_BOUNDS: `out` is not valid). */
LCSA_API lcsa_status_t lcsa_forward_host(lcsa_plan_t plan, const void* q, const void* k, const void* v,
                                const float* gamma_q, const float* gamma_k, void* out, void* stream);

/* Streaming, the pages' steady state ("FlashVSR: From 17.2 FPS to 57.3 FPS at
   768x1408", Rebuild sparse attention for Hopper: incremental pooled-K
   caching; "FlashVSR Inference", Non-Negotiable Streaming Contract: the KV
   window is kv_ratio x the query frames). A stream plan keeps the last
   kv_frames frames of k^, pooled k and raw v in a ring, so each call
   normalises, rotates and pools only the new frames.
   lcsa_plan_create_stream: as lcsa_plan_create (host_io must be 0), plus a
     plan-owned v ring of batch * kv_frames frames. Absolute frame positions
     (RoPE) start at cfg->kv_frame_offset for the first frame pushed.
   lcsa_stream_push: appends `frames` frames of k and v ([batch][frames][H'][W']
     [heads*d] bf16, device) to the window without attention (to fill it before
     the first chunk); frames is a multiple of block_t, at most kv_frames.
   lcsa_forward_stream: appends the chunk's q_frames new frames of k and v, and
     computes attention for its q ([batch][q_frames][H'][W'][heads*d]) over the
     window of the last kv_frames frames (the new ones last). The window must be
     full (LCSA_ERR_INVALID_ARG otherwise). The result equals lcsa_forward on
     that window with kv_frame_offset = the absolute index of its first frame.
   A stream plan rejects lcsa_forward; calls on one plan must not overlap. */
LCSA_API lcsa_status_t lcsa_plan_create_stream(const lcsa_config_t* cfg, int cuda_device, lcsa_plan_t* out);
LCSA_API lcsa_status_t lcsa_stream_push(lcsa_plan_t plan, const void* k, const void* v, const float* gamma_k,
                                        int frames, void* stream);
LCSA_API lcsa_status_t lcsa_forward_stream(lcsa_plan_t plan, const void* q, const void* k, const void* v,
                                           const float* gamma_q, const float* gamma_k, void* out, void* stream);

/* Head-sharded layers: the tensor-parallel form of the pages ("Add FlashVSR
   contrib model with video super-resolution on Neuron", Model Information
   and Additional Information: the QK RMSNorm all-reduces across the ranks
   that hold a layer's heads, so it spans all heads of a token). A plan with
   heads_total > heads holds `heads` consecutive heads of a layer of
   heads_total heads: q, k, v, out and the gains are the plan's slice
   ([batch][tokens][heads*d], gains [heads*d]). With token-scope norm the
   RMS mean runs over heads_total*head_dim channels, so each rank:
     1. lcsa_sumsq writes ssq (device fp32, 16-byte aligned,
        batch*(q_tokens + kv_tokens) entries): per token the sum of squares of
        its own q channels (batch-major, first batch*q_tokens entries), then of
        its own k channels;
     2. sums ssq over the ranks (an all-reduce, by the caller: NCCL);
     3. lcsa_forward_sharded runs lcsa_forward with the norm taken from the
        reduced ssq (it must hold the sums over all heads_total heads).
   lcsa_forward rejects such a plan (LCSA_ERR_INVALID_ARG). With head-scope
   norm no exchange is needed and lcsa_forward serves sharded plans directly
   (lcsa_forward_sharded then returns LCSA_ERR_INVALID_ARG). Stream plans and
   lcsa_forward_noalloc are not head-sharded (LCSA_ERR_UNSUPPORTED). */
LCSA_API lcsa_status_t lcsa_sumsq(lcsa_plan_t plan, const void* q, const void* k, float* ssq, void* stream);
LCSA_API lcsa_status_t lcsa_forward_sharded(lcsa_plan_t plan, const void* q, const void* k, const void* v,
                                            const float* gamma_q, const float* gamma_k, const float* ssq, void* out,
                                            void* stream);

/* Threshold reuse: the mask-generation threshold of the previous steady
   chunk reused per DiT block ("FlashVSR: From 17.2 FPS to 57.3 FPS at
   768x1408", Remove the remaining control-plane tax and Measured Results; a
   plan is one DiT block's attention). Every call that selects records, per
   query block, the score of its k-th best block. With reuse on, later calls
   (lcsa_forward, lcsa_forward_stream, lcsa_forward_sharded) skip the top-k
   selection and keep every admissible block whose score is at least the
   recorded one (ascending order; a query block where none reaches it keeps
   its best block), so a query block may keep more or fewer than k blocks: an
   approximation the caller gates on quality. A call with reuse on and no
   recorded thresholds selects (and records). on: 1 reuse, 0 select every call.
   lcsa_selection_nnz: total kept blocks of the last call (synchronises). */
LCSA_API lcsa_status_t lcsa_plan_set_threshold_reuse(lcsa_plan_t plan, int on);
LCSA_API lcsa_status_t lcsa_selection_nnz(lcsa_plan_t plan, int64_t* nnz);

/* Size of the static device workspace used by lcsa_forward_noalloc (64 MiB).
   A GPU holds this array from the first lcsa_forward_noalloc call made on it
   (when the CUDA module that holds it is loaded) until the process exits. */
#define LCSA_NOALLOC_WORKSPACE_BYTES (64u << 20)

/* The LCSA call without a plan and without any allocation, for callers that
   may not allocate device memory once running (for instance a real-time
   video pipeline or a plugin whose device memory is fully reserved at start-up,
   where cudaMalloc/cudaFree would synchronise the device and stall the other
   streams, or could fail). This entry point has no counterpart in the paper.
   Arguments are those of lcsa_forward, with the configuration passed directly
   (host_io must be 0; the checks are lcsa_config_resolve's, shared code).
   All intermediates live in one file-scope static device array of
   LCSA_NOALLOC_WORKSPACE_BYTES.
   Set-up: the first call in a CUDA context looks up that array's address in
   that context and clears its error word. Under CUDA's default lazy module
   loading this first call also loads the module that holds the array, which
   reserves its device memory: make it at start-up, before any stream capture
   (or set CUDA_MODULE_LOADING=EAGER so every module loads with the context).
   Later calls allocate nothing. Addresses are kept per context (by its
   unique ID), so a new context on the same device (after cudaDeviceReset,
   say) repeats the set-up.
   All calls share the array and it keeps the last call's contents: calls that
   overlap on the GPU race and must be serialised by the caller. Returns
   LCSA_ERR_UNSUPPORTED when the problem's intermediates do not fit in the
   array (create a plan instead), and the codes of lcsa_config_resolve for a
   bad configuration; no detail message is set. No device or host memory is
   allocated and no allocating library routine is called. Asynchronous on
   `stream`. A kernel's bounded-wait timeout or index-check failure is kept in
   the array's error word (calls do not clear it) until
   lcsa_noalloc_check_device_error reads it. */
LCSA_API lcsa_status_t lcsa_forward_noalloc(const lcsa_config_t* cfg, const void* q, const void* k, const void* v,
                                            const float* gamma_q, const float* gamma_k, void* out, void* stream);

/* Device-error status of the lcsa_forward_noalloc calls made in the current
   context since the last check: synchronises `stream`, reads the static
   array's error word into host stack memory and clears it. Returns LCSA_OK,
   LCSA_ERR_DEVICE_TIMEOUT (a kernel gave up a bounded wait; that call's output
   is incomplete), LCSA_ERR_DEVICE_BOUNDS, or LCSA_ERR_CUDA (the stream or the
   copy failed). LCSA_OK too when no call has run in this context. Allocates
   nothing. No counterpart in the paper, like lcsa_forward_noalloc. */
LCSA_API lcsa_status_t lcsa_noalloc_check_device_error(void* stream);

/* Resolved geometry of a plan. */
LCSA_API lcsa_status_t lcsa_plan_geometry(lcsa_plan_t plan, lcsa_geometry_t* out);

/* Resolved budget k in blocks. */
LCSA_API lcsa_status_t lcsa_plan_topk(lcsa_plan_t plan, int* k_out);

/* Copy the last call's CSR to host: row_ptr [rows+1], col_idx [nnz] (nnz:
   the geometry's, or lcsa_selection_nnz after a threshold-reuse call). The
   capacities are element counts; too small -> LCSA_ERR_INVALID_ARG.
   Synchronises the device. */
LCSA_API lcsa_status_t lcsa_get_selection(lcsa_plan_t plan, int32_t* row_ptr, size_t row_ptr_cap,
                                 int32_t* col_idx, size_t col_idx_cap);

/* Copy the last call's prologue outputs to host (any pointer may be null):
   qhat bf16 [batch][heads][q_blocks][n_b][head_dim], khat likewise with
   kv_blocks, pooled_q fp32 [batch][heads][q_blocks][head_dim], pooled_k
   likewise. Synchronises the device. */
LCSA_API lcsa_status_t lcsa_get_intermediates(lcsa_plan_t plan, void* qhat, void* khat, float* pooled_q,
                                     float* pooled_k);

/* Synchronise `stream`, then read and clear the plan's device error word:
   LCSA_OK, LCSA_ERR_DEVICE_TIMEOUT or LCSA_ERR_DEVICE_BOUNDS (or
   LCSA_ERR_CUDA if the stream itself failed). */
LCSA_API lcsa_status_t lcsa_check_device_error(lcsa_plan_t plan, void* stream);

/* Kernel timing. capacity > 0: create `capacity` sets of CUDA events and,
   from now on, record one set around the three kernels of every lcsa_forward
   (the ring wraps after `capacity` calls); capacity = 0: stop recording and
   free the events. Any call resets what was recorded so far. */
LCSA_API lcsa_status_t lcsa_plan_set_timing(lcsa_plan_t plan, int capacity);

/* Mean device milliseconds of the three kernels (ms[0] prologue, ms[1]
   select, ms[2] attention) over the forwards recorded since the last
   lcsa_plan_set_timing (at most `capacity` most recent); *count receives how
   many were averaged. Synchronises on the newest recorded event. */
LCSA_API lcsa_status_t lcsa_get_kernel_times(lcsa_plan_t plan, float ms[3], int* count);

/* Self-test of the attention kernel's FMA-pipe exponential: y[i] = 2^x[i]
   computed exactly as the softmax does for one exponential in four
   (Cody-Waite reduction and a degree-3 minimax polynomial; relative error
   below 7.5e-5 for -125 <= x <= 8). x, y: device fp32 [n]. Asynchronous.
   The pages' FFMA-form softmax math ("FlashVSR: From 17.2 FPS to 57.3 FPS at
   768x1408", Rebuild sparse attention for Hopper) is the source of the idea. */
LCSA_API lcsa_status_t lcsa_selftest_exp2(const float* x, float* y, int n, void* stream);

/* Static text of a status code. */
LCSA_API const char* lcsa_status_string(lcsa_status_t status);

/* Detail of the last failure on the calling thread ("" if none). */
LCSA_API const char* lcsa_last_error_message(void);

/* LCSA_ABI_VERSION of the loaded library. */
LCSA_API int lcsa_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LCSA_H */
