/*
 * hga.h -- C ABI of libhga.so, the B200 (sm_100a) kernels of the HGA
 * per-segment attention step.
 *
 * Source of the method: "Low-VRAM Long-Context Fine-Tuning: Hierarchical
 * Global Attention and Segmented Backpropagation in Practice" (sns.style; the
 * ja/de/ko editions share one text, the fr edition is a rewrite):
 *   Background (背景と概要 / Hintergrund / 배경): a long sequence is cut into
 *     segments; only the active segment is differentiable and kept on the GPU;
 *     the history KV is offloaded to system RAM (or NVMe); each query block
 *     attends to a bounded, exact set of history tokens rather than the dense
 *     history, so per-token cost stays roughly constant.
 *   Deep analysis (深掘り分析 / Tiefenanalyse / 심층 분석): per-block summaries
 *     stay resident in VRAM and grow slowly with the context.
 *   fr edition, Contexte: history tokens are loaded dynamically and precisely
 *     per query block; Analyse approfondie: the KV of finished segments is
 *     offloaded right away and decoupled from the active graph.
 * The article leaves the summary, the score, K and the block size open.  This
 * library fixes them as follows (the plainest reading the text supports):
 *   summary[b,h,n]  = mean over the block's tokens of K_hist[b,t,h,:] (fp32)
 *   score[b,h,i,n]  = max over the query heads hq of KV head h of
 *                     mean_{t in query block i}(Q[b,t,hq,:]) . summary / sqrt(d)
 *   selection       = the min(K, n_hist_blocks) highest scores, equal scores
 *                     resolved to the lower block index, listed in ascending
 *                     block order, unused slots = -1
 *   attention       = softmax over [tokens of the selected history blocks] U
 *                     [segment tokens at positions <= the query's], scale
 *                     1/sqrt(d), fp32 statistics
 *   backward        = dQ, dK_seg, dV_seg of <O, dO>; the history, the summaries
 *                     and the selection get no gradient.
 *
 * Notation: B batch, Hq query heads, Hkv KV heads (Hq % Hkv == 0, query head hq
 * uses KV head hq / (Hq/Hkv)), d head dim, `block` tokens per history block,
 * q_block rows per query block (dims.q_block, 0 = block), S segment tokens
 * (S % block == 0 and S % q_block == 0), Nqb = S / q_block.
 *
 * Layouts (row-major, token-major as QKV projections produce them):
 *   q, o, d_o           [B, S, Hq, d]          dtype
 *   k_seg, v_seg        [B, S, Hkv, d]         dtype
 *   k_hist, v_hist      [B, n_kv_blocks*block, Hkv, d] dtype; block n = tokens
 *                       [n*block, (n+1)*block)
 *   summ                [B, n_hist_blocks, Hkv, d] fp32 (block-major, so a growing
 *                       history appends: the first n blocks of a larger array
 *                       are a valid summary array of n blocks when B == 1)
 *   idx                 [B, Hkv, Nqb, topk]    int32
 *   lse                 [B, Hq, S]             fp32 (natural log)
 *   dq                  [B, S, Hq, d]          fp32
 *   dk_seg, dv_seg      [B, S, Hkv, d]         fp32
 *
 * Conventions:
 *   - Ownership: the caller owns every buffer (device memory unless stated).
 *     The library allocates no device or pinned memory; scratch space is
 *     passed in by the caller (hga_attn_bwd_workspace_size).  It creates one
 *     side stream and two events per device, once, for the two-stream
 *     backward (hga_attn_bwd).
 *   - Asynchrony: every call enqueues work on `stream` and returns; errors in
 *     arguments are reported before anything is enqueued.  The fetch calls are
 *     the exception: they wait (bounded by timeout_ms) for a small index copy.
 *   - Device-side faults that a kernel can detect (an out-of-range idx entry,
 *     an expired pipeline wait) set a per-device flag instead of trapping;
 *     hga_device_status() synchronizes the stream and reports and clears it.
 *   - Paths: bf16 with d == 128 and block == 128 and an even group size runs
 *     on the tcgen05 tensor-core kernels; every other supported shape (fp32,
 *     d in {64,128}, block in {16,32,64,128}) runs on CUDA-core kernels.  Both
 *     are GPU code; there is no CPU path.
 *   - Thread safety: calls are independent; hga_last_error() is thread-local.
 */
#ifndef HGA_H
#define HGA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define HGA_API __attribute__((visibility("default")))
#else
#define HGA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HGA_OK = 0,
  HGA_ERR_INVALID_ARG = 1, /* null pointer, bad enum, bad size */
  HGA_ERR_SHAPE = 2,       /* dimensions outside the supported set */
  HGA_ERR_UNSUPPORTED = 3, /* valid request that the library does not implement */
  HGA_ERR_INDEX = 4,       /* a kernel met an out-of-range block index */
  HGA_ERR_TIMEOUT = 5,     /* a bounded wait expired (host or device) */
  HGA_ERR_CUDA = 6         /* a CUDA runtime call failed; see hga_last_error */
} hga_status;

typedef enum { HGA_F32 = 0, HGA_BF16 = 1 } hga_dtype;

/* Shape of one attention step.  n_hist_blocks: history blocks that exist
 * (what selection ranks); topk: K. */
typedef struct {
  int B, Hq, Hkv, d, block, S, n_hist_blocks, topk;
  hga_dtype dtype;
  /* Query-block size: the segment rows that share one selection.  0 = block
   * (one size for history blocks and query blocks).  Otherwise in
   * {16, 32, 64, 128}, S % q_block == 0; a query block's mean is over its
   * q_block rows, and each of its rows attends to the `block` tokens of every
   * block selected for it.  idx and qblock_mask have S / q_block query
   * blocks; a finished segment still becomes S / block history blocks. */
  int q_block;
} hga_dims;

/* A CUDA stream (cudaStream_t); NULL = legacy default stream. */
typedef struct CUstream_st* hga_stream_t;
/* A CUDA event (cudaEvent_t). */
typedef struct CUevent_st* hga_event_t;

/* Human-readable name of a status code (static string). */
HGA_API const char* hga_status_string(hga_status s);
/* Details of the last failure in this thread (static per-thread buffer). */
HGA_API const char* hga_last_error(void);

/* Synchronizes `stream`, then reports (and clears) the device-side error flag
 * of the current device: HGA_ERR_INDEX if a kernel saw an idx entry outside
 * [-1, n_kv_blocks), HGA_ERR_TIMEOUT if a pipeline wait expired, else HGA_OK. */
HGA_API hga_status hga_device_status(hga_stream_t stream);

/*
 * Block summaries (article, Deep analysis: resident per-block summaries).
 *   summ[b,n,h,:] = (1/block) * sum_{t<block} k_hist[b, n*block+t, h, :]
 * for blocks n in [blk_begin, blk_end) of a history of dims->n_hist_blocks
 * blocks; other entries of summ are left untouched, so summaries can be added
 * as blocks enter the history.  k_hist: dtype; summ: fp32 device buffer
 * [B, n_hist_blocks, Hkv, d].  Accumulation in fp32.
 * Errors: HGA_ERR_INVALID_ARG (null pointers, bad range), HGA_ERR_SHAPE.
 */
HGA_API hga_status hga_block_summaries(const hga_dims* dims, const void* k_hist, int blk_begin, int blk_end, float* summ,
                               hga_stream_t stream);

/*
 * Summaries of a finished segment's blocks, as they enter the history
 * (article, Deep analysis: summaries stay resident and grow with the context;
 * fr Analyse approfondie: the segment's KV leaves the active window).
 *   summ[b, at_block + t, h, :] = (1/block) * sum_{u<block} k_seg[b, t*block+u, h, :]
 * for the S/block blocks t of the segment.  Here dims->n_hist_blocks is the
 * capacity (in blocks) of the summ array [B, n_hist_blocks, Hkv, d];
 * at_block + S/block must not exceed it.  Other entries are untouched.
 * Errors: HGA_ERR_INVALID_ARG (null pointers, range), HGA_ERR_SHAPE.
 */
HGA_API hga_status hga_segment_summaries(const hga_dims* dims, const void* k_seg, int at_block, float* summ,
                                         hga_stream_t stream);

/*
 * Per-query-block history selection (article, Background: bounded exact
 * history set per query block; fr Contexte: precise historical tokens per
 * query block).  For every (b, KV head h, query block i):
 *   qm[g]     = mean over the block's `block` rows of q[b, row, h*G+g, :] (fp32)
 *   score[n]  = max_g (qm[g] . summ[b,n,h,:]) / sqrt(d)                   (fp32)
 *   idx[b,h,i,:] = the K_eff = min(topk, n_hist_blocks) best n (ties to the
 *                  lower n), ascending, then -1 up to topk.
 * scores_or_null (optional, fp32 [B,Hkv,Nqb,topk]) receives the selected
 * blocks' scores in the same order (-inf for padding).
 * Limits: n_hist_blocks <= 4096.
 * Errors: HGA_ERR_INVALID_ARG, HGA_ERR_SHAPE.
 */
HGA_API hga_status hga_select_topk(const hga_dims* dims, const void* q_seg, const float* summ, int32_t* idx,
                           float* scores_or_null, hga_stream_t stream);

/*
 * Attention forward over [selected history blocks] U [causal segment]
 * (article, Background: exact attention over a bounded history set; only
 * the active segment is computed on).  For query row p of head hq (KV head h,
 * query block i = p / block), keys J = tokens of blocks idx[b,h,i,:] (entries
 * >= 0) of k_hist/v_hist, plus segment tokens 0..p:
 *   s_j = q.k_j / sqrt(d);  O = sum_j softmax(s)_j v_j;  lse = log sum_j exp(s_j)
 * k_hist/v_hist hold n_kv_blocks blocks: the history itself (n_kv_blocks =
 * n_hist_blocks) or a staging pool filled by hga_fetch_blocks (idx then holds
 * pool slots).  o has the input dtype; lse fp32.  q, k_seg, v_seg, k_hist,
 * v_hist and o must start on a 16-byte boundary.
 * Errors: HGA_ERR_INVALID_ARG (null or misaligned pointers), HGA_ERR_SHAPE
 * (host checks); an idx entry outside [-1, n_kv_blocks) is skipped and flags
 * HGA_ERR_INDEX on the device.
 */
HGA_API hga_status hga_attn_fwd(const hga_dims* dims, const void* q, const void* k_seg, const void* v_seg,
                        const void* k_hist, const void* v_hist, int n_kv_blocks, const int32_t* idx, void* o,
                        float* lse, hga_stream_t stream);

/* 1 when hga_attn_fwd / hga_attn_bwd run these dims on the tcgen05
 * tensor-core kernels (bf16, d in {64, 128}, q_block 128, block 128, 64, 32
 * or 16 -- 128/block selected history blocks per 128-key tile -- an even
 * group size, K <= 64, at most 128 query blocks; with block 64 also
 * n_kv_blocks < 32767, as a tile entry holds two 15-bit block indices), 0 when
 * they run on the CUDA-core kernels, -1 for dims the library rejects.
 * Host-only; no device work. */
HGA_API int hga_attn_uses_tensor_cores(const hga_dims* dims, int n_kv_blocks);

/* Query heads per CTA of the tensor-core forward, for later calls from the
 * calling thread (a per-thread setting, like hga_last_error): 2 (a CTA serves
 * a pair of query heads of one KV head, sharing each K/V tile), 1 (one head
 * per CTA, its tiles split over the CTA's two softmax warpgroups: twice the
 * CTAs), or 0 (the default: a pair, unless B * Hkv * (G/2) * Nqb is below the
 * device's SM count, then one).  The results are the same either way; this is
 * a throughput knob.  Host-only, no device work; HGA_ERR_INVALID_ARG for other
 * values. */
HGA_API hga_status hga_set_forward_heads_per_cta(int heads);

/* Bytes of device scratch hga_attn_bwd needs for these dims (256-byte
 * aligned start required). */
HGA_API size_t hga_attn_bwd_workspace_size(const hga_dims* dims);

/*
 * Attention backward for the active segment only (article, Background and
 * fr Analyse approfondie: only the active segment is differentiable; history
 * KV is detached).  With P the forward softmax (recomputed from lse),
 * dP_j = dO.v_j, Dr = dO.O:
 *   dS_j  = P_j (dP_j - Dr)
 *   dq    = sum_{j in J} dS_j k_j / sqrt(d)                 (history + segment)
 *   dk_seg[j] = sum over rows and the G heads of dS_j q / sqrt(d)  (segment j)
 *   dv_seg[j] = sum over rows and the G heads of P_j dO            (segment j)
 * No gradient is produced for k_hist, v_hist, summaries or idx.
 * o and lse are the forward outputs; d_o has the input dtype; dq, dk_seg and
 * dv_seg are fp32 and fully overwritten.  ws: device scratch of at least
 * hga_attn_bwd_workspace_size(dims) bytes, owned by the caller; its contents
 * need no initialisation and are undefined afterwards.
 * On the tensor-core path the dQ kernel runs on `stream` and the dK/dV kernel
 * on a side stream the library creates once per device, forked from `stream`
 * after the preprocess and joined back into it with events: work queued on
 * `stream` after the call sees all three outputs, and the call records into
 * a CUDA graph under stream capture (as two branches).  The same holds for
 * hga_attn_bwd_sparse and hga_attn_bwd_noalloc.
 * Errors: as hga_attn_fwd, plus HGA_ERR_INVALID_ARG for a short workspace.
 */
HGA_API hga_status hga_attn_bwd(const hga_dims* dims, const void* q, const void* k_seg, const void* v_seg,
                        const void* k_hist, const void* v_hist, int n_kv_blocks, const int32_t* idx, const void* o,
                        const float* lse, const void* d_o, float* dq, float* dk_seg, float* dv_seg, void* ws,
                        size_t ws_bytes, hga_stream_t stream);

/*
 * hga_attn_bwd for callers that cannot allocate device memory.  The article
 * has no counterpart to this call; it exists for integration.
 *
 * Some callers cannot call cudaMalloc at the point where they run the
 * backward: code that runs under a framework-owned memory pool (an allocator
 * that owns every device byte and forbids outside allocations), host code
 * driving a pre-planned memory budget, or a plugin that only receives the
 * tensors it reads and writes.  Such a caller has no workspace to pass.  This
 * variant takes the same inputs and outputs as hga_attn_bwd, minus ws and
 * ws_bytes, and keeps its scratch (Dr = rowsum(dO * O), B*Hq*S floats) in a
 * fixed array inside the library instead.
 *
 * Limit: B*Hq*S <= 1,048,576 (a 4 MiB array, held on every GPU that loads
 * the library until the process exits).  Larger problems return
 * HGA_ERR_SHAPE; use hga_attn_bwd with a caller-owned workspace for them.
 * The call allocates nothing (no cudaMalloc or allocating library routine).
 * Set-up: the first call on each device looks up the array's device address
 * with the device current; make that first call before any stream capture.
 * All calls share the one array and it keeps the last call's contents (the
 * stage that reads it first overwrites every element it reads, so nothing
 * needs clearing); two calls that overlap on the GPU (different streams, no
 * ordering between them) race on it.
 * Results, errors and asynchrony otherwise as hga_attn_bwd.
 */
HGA_API hga_status hga_attn_bwd_noalloc(const hga_dims* dims, const void* q, const void* k_seg, const void* v_seg,
                                        const void* k_hist, const void* v_hist, int n_kv_blocks,
                                        const int32_t* idx, const void* o, const float* lse, const void* d_o,
                                        float* dq, float* dk_seg, float* dv_seg, hga_stream_t stream);

/*
 * Sparse segment backward in the manner of SpaCO ("Training Long-Context LLMs
 * Efficiently via Chunk-wise Optimization", proposed method: only a fixed
 * number of chunks is backpropagated per step, each scaled by a correction
 * factor that keeps the gradient estimate unbiased, with a cap for
 * stability).  With the HGA history detached, a gradient path never leaves
 * the active segment, so the estimator is the backward of
 *   L = scale * sum over the rows of the chosen query blocks of <O, dO>:
 * the hga_attn_bwd result with d_o replaced by scale * d_o on rows of query
 * blocks i with qblock_mask[b*Nqb + i] != 0 and by 0 elsewhere.  dq rows of
 * unchosen blocks are exactly 0.  qblock_mask: device uint8 [B, Nqb]; scale:
 * finite (for k of t blocks sampled uniformly, t/k makes the estimate
 * unbiased; the caller applies any cap).  Work for unchosen blocks is skipped
 * (dQ CTAs of unchosen blocks only write zeros; dK/dV walk chosen blocks only).
 * Other arguments, results and errors as hga_attn_bwd.
 */
HGA_API hga_status hga_attn_bwd_sparse(const hga_dims* dims, const void* q, const void* k_seg, const void* v_seg,
                                       const void* k_hist, const void* v_hist, int n_kv_blocks, const int32_t* idx,
                                       const void* o, const float* lse, const void* d_o, const uint8_t* qblock_mask,
                                       float scale, float* dq, float* dk_seg, float* dv_seg, void* ws,
                                       size_t ws_bytes, hga_stream_t stream);

/*
 * The three stages of hga_attn_bwd as separate calls (same arguments, same
 * results), for callers that schedule or time them individually.  ws is the
 * same caller-owned scratch; its first B*Hq*S floats hold Dr = rowsum(dO * O)
 * [B, Hq, S] between the stages.
 *   hga_attn_bwd_preprocess: Dr from o and d_o.
 *   hga_attn_bwd_dkdv:       dk_seg, dv_seg (fully overwritten), needs Dr.
 *   hga_attn_bwd_dq:         dq (fully overwritten), needs Dr.
 * dkdv and dq read only inputs and Dr, so they may run concurrently on two
 * streams once the preprocess has completed.
 */
HGA_API hga_status hga_attn_bwd_preprocess(const hga_dims* dims, const void* o, const void* d_o, void* ws,
                                           size_t ws_bytes, hga_stream_t stream);
HGA_API hga_status hga_attn_bwd_dkdv(const hga_dims* dims, const void* q, const void* k_seg, const void* v_seg,
                                     const float* lse, const void* d_o, const void* ws, size_t ws_bytes,
                                     float* dk_seg, float* dv_seg, hga_stream_t stream);
HGA_API hga_status hga_attn_bwd_dq(const hga_dims* dims, const void* q, const void* k_seg, const void* v_seg,
                                   const void* k_hist, const void* v_hist, int n_kv_blocks, const int32_t* idx,
                                   const float* lse, const void* d_o, const void* ws, size_t ws_bytes, float* dq,
                                   hga_stream_t stream);

/*
 * Decode step (article, Industry impact; fr edition, Impact: HGA also serves
 * generation and retrieval).  One step processes n_q new query tokens
 * (1 <= n_q <= q_block) at active-segment positions t0 .. t0+n_q-1; they form
 * one partial query block.  Here dims->S is the CAPACITY of the active
 * segment's KV buffer (k_seg/v_seg [B, S, Hkv, d], positions 0 .. t0+n_q-1
 * already written by the caller, the new tokens' K/V included), and
 * dims->n_hist_blocks the history that selection ranks.
 *
 * hga_decode_select: for every (b, KV head h)
 *   qm[g]     = mean over the n_q new rows of q_new[b, u, h*G+g, :]   (fp32)
 *   score[n]  = max_g (qm[g] . summ[b,n,h,:]) / sqrt(d)
 *   idx[b,h,:] = the K_eff = min(topk, n_hist_blocks) best n (ties to the
 *                lower n), ascending, then -1 up to topk.
 * q_new [B, n_q, Hq, d] dtype; summ as for hga_select_topk; idx [B, Hkv, topk]
 * int32; scores_or_null fp32 [B, Hkv, topk] (the selected blocks' scores,
 * -inf for padding).  With n_q = q_block and t0 a multiple of q_block this is
 * exactly hga_select_topk's result for that query block (up to fp32 rounding
 * of the mean near ties).  The blocks are scored in parallel into ws, then
 * selected per (b, KV head); ws as for hga_decode_attn (the same buffer may
 * serve both calls when they run in order on one stream).
 *
 * hga_decode_attn: new query u (position p = t0 + u) of head hq attends to the
 * tokens of blocks idx[b, hq/G, :] (entries >= 0) of k_hist/v_hist (the
 * history or a pool of n_kv_blocks blocks, as for hga_attn_fwd) and to
 * segment positions 0 .. p; scale 1/sqrt(d), fp32 statistics.
 *   o [B, n_q, Hq, d] dtype;  lse [B, Hq, n_q] fp32 (natural log)
 * ws: device scratch of at least hga_decode_workspace_size(dims, n_q) bytes
 * (16-byte aligned; contents need no initialisation), owned by the caller.
 * With n_q = q_block and t0 a multiple of q_block the result equals hga_attn_fwd's
 * rows of that query block.
 * A finished segment joins the history as in the prefill: hga_segment_summaries
 * appends its blocks' summaries, hga_offload_segment moves its K/V to the tier.
 * Errors: HGA_ERR_SHAPE (n_q outside [1, q_block], new tokens outside the
 * buffer, n_hist_blocks > 4096 for the selection, topk + S/block > 512 for the
 * attention), HGA_ERR_INVALID_ARG (null
 * or misaligned pointers, short workspace); an idx entry outside
 * [-1, n_kv_blocks) is skipped and flags HGA_ERR_INDEX on the device.
 */
HGA_API hga_status hga_decode_select(const hga_dims* dims, int n_q, const void* q_new, const float* summ,
                                     int32_t* idx, float* scores_or_null, void* ws, size_t ws_bytes,
                                     hga_stream_t stream);
/* Bytes of device scratch hga_decode_select and hga_decode_attn need for these
 * dims and n_q (0 if they are invalid). */
HGA_API size_t hga_decode_workspace_size(const hga_dims* dims, int n_q);
HGA_API hga_status hga_decode_attn(const hga_dims* dims, int n_q, int t0, const void* q_new, const void* k_seg,
                                   const void* v_seg, const void* k_hist, const void* v_hist, int n_kv_blocks,
                                   const int32_t* idx, void* o, float* lse, void* ws, size_t ws_bytes,
                                   hga_stream_t stream);

/*
 * Targeted loading of the selected history (fr edition, Contexte: dynamic
 * loading of precise historical tokens per query block; Background: history
 * KV lives in system RAM).  host_k/host_v: pinned host memory (cudaHostAlloc)
 * of one layer's history tier [B, host_capacity_blocks*block, Hkv, d] in
 * dtype, of which the first n_hist_blocks blocks are valid.  idx_dev:
 * device idx from hga_select_topk.  The call
 *   1. copies idx to the host on compute_stream (after the work already
 *      queued there) and waits for it, at most timeout_ms.  Pinned scratch
 *      mapped into the device (any cudaHostAlloc / cudaHostRegister memory
 *      with unified addressing) is written by a small kernel through that
 *      mapping, so the copy does not wait behind large device-to-host copies
 *      queued on other streams; other host memory takes cudaMemcpyAsync;
 *   2. forms the sorted set of distinct selected blocks (at most pool_slots);
 *   3. on copy_stream, ordered after that idx copy (so after every kernel
 *      queued on compute_stream before the call), copies each of those
 *      blocks' K and V (all B and Hkv) from host to the device pool (pool_k/
 *      pool_v [B, pool_slots*block, Hkv, d]), and writes idx_pool_dev = idx
 *      with each block number replaced by its pool slot (-1 kept);
 *   4. records `done` on copy_stream; compute work that reads the pool must
 *      wait on it (cudaStreamWaitEvent).
 * host_idx_scratch: pinned host buffer of B*Hkv*Nqb*topk int32 owned by the
 * caller; it must stay untouched until `done` (the pool idx is uploaded from
 * it).  *n_unique_out receives the number of distinct blocks fetched.
 * Errors: HGA_ERR_TIMEOUT (idx copy did not finish in time), HGA_ERR_INDEX
 * (an idx entry out of range), HGA_ERR_INVALID_ARG (more distinct blocks than
 * pool_slots, null pointers), HGA_ERR_CUDA.
 * After HGA_ERR_TIMEOUT no pool copy has been queued, but the idx copy into
 * host_idx_scratch is still pending on compute_stream: the caller must not
 * reuse or free that buffer until compute_stream has drained
 * (cudaStreamSynchronize).
 */
HGA_API hga_status hga_fetch_blocks(const hga_dims* dims, const void* host_k, const void* host_v, int host_capacity_blocks,
                            const int32_t* idx_dev,
                            int32_t* host_idx_scratch, void* pool_k, void* pool_v, int pool_slots,
                            int32_t* idx_pool_dev, int* n_unique_out, hga_stream_t compute_stream,
                            hga_stream_t copy_stream, hga_event_t done, int timeout_ms);

/*
 * hga_fetch_blocks without the host: the distinct selected blocks are read by
 * the GPU itself from the pinned host tier, mapped into the device's address
 * space (zero copy), and the whole call is ordered on `stream` with no host
 * wait (so it can be captured in a CUDA graph and queued ahead).  Same
 * result as hga_fetch_blocks: pool slot k holds the k-th smallest selected
 * block (K and V, all B and Hkv), idx_pool_dev = idx with block numbers
 * replaced by slots (-1 kept).  host_k/host_v: pinned host memory
 * (cudaHostAlloc, or registered as mapped) [B, host_capacity_blocks*block,
 * Hkv, d], checked to be mapped over its whole extent; pool_k/pool_v device
 * [B, pool_slots*block, Hkv, d].  A selected block ranked at or beyond
 * pool_slots gets no slot: its idx_pool entries are -1 and the device error
 * flag reports HGA_ERR_INDEX.  n_hist_blocks <= 32768.  The copies are made
 * by the SMs over the host link (PCIe / C2C), not by the copy engines.
 * Errors: HGA_ERR_INVALID_ARG (NULL or misaligned pointers, a tier that is not
 * mapped pinned memory, tier smaller than the history), HGA_ERR_SHAPE.
 */
HGA_API hga_status hga_gather_blocks_mapped(const hga_dims* dims, const void* host_k, const void* host_v,
                                            int host_capacity_blocks, const int32_t* idx_dev, void* pool_k,
                                            void* pool_v, int pool_slots, int32_t* idx_pool_dev,
                                            hga_stream_t stream);

/*
 * Device block cache: history blocks stay in a layer's device pool across
 * calls, so a block selected again (by the next segment, or by the backward
 * of the same segment) is not copied over the host link again (article,
 * Outlook; fr Perspectives: faster VRAM <-> RAM <-> NVMe transfer is the
 * open problem).  The history tier's blocks never change once offloaded, so
 * a resident copy stays valid.
 *
 * hga_block_cache is host memory owned by the caller and kept across calls:
 *   slot_of_block  [host_capacity_blocks] int32: pool slot holding block n, or -1
 *   block_of_slot  [pool_slots] int32: block held by slot, or -1
 *   last_use       [pool_slots] int64: tick of the last call that needed the slot
 *   tick           calls planned so far
 * hga_block_cache_reset empties it (needed when the tier or pool is reused for
 * another sequence).  Both functions are host-only (no GPU work).
 *
 * hga_block_cache_plan: need[0..n_need) are distinct block numbers in
 * [0, host_capacity_blocks), ascending.  Each gets a slot: a resident block
 * keeps its own (a hit); a missing block takes an empty slot, else the least
 * recently used slot whose block this call does not need (ties: the lowest
 * slot).  slot_out[k] is need[k]'s slot; miss_out[0..*n_miss) lists the
 * missing blocks (ascending), the ones to copy.  The cache records the
 * assignment and advances its tick.  Errors: HGA_ERR_INVALID_ARG (NULL
 * pointers, out-of-range or unsorted need, more distinct blocks than slots;
 * the cache is then unchanged).
 */
typedef struct {
  int32_t* slot_of_block;
  int32_t* block_of_slot;
  int64_t* last_use;
  int host_capacity_blocks;
  int pool_slots;
  int64_t tick;
} hga_block_cache;

HGA_API hga_status hga_block_cache_reset(hga_block_cache* cache);
HGA_API hga_status hga_block_cache_plan(hga_block_cache* cache, const int32_t* need, int n_need, int32_t* slot_out,
                                        int32_t* miss_out, int* n_miss);

/*
 * hga_fetch_blocks through a device block cache: as hga_fetch_blocks, except
 * that the pool (pool_k/pool_v [B, cache->pool_slots*block, Hkv, d]) keeps its
 * contents between calls and only the selected blocks that are not resident
 * are copied (hga_block_cache_plan decides).  idx_pool_dev receives idx with
 * block numbers replaced by their slots.  *n_unique_out: distinct selected
 * blocks; *n_fetched_out: blocks copied by this call.  The copies run on
 * copy_stream after the work already queued on compute_stream, so a slot is
 * never overwritten while earlier kernels may still read it.  host tier
 * capacity: cache->host_capacity_blocks.  Errors as hga_fetch_blocks.
 * The cache is updated only once every copy of the call has been queued: on
 * any error it is left exactly as it was, so no block is recorded as
 * resident whose bytes were never sent.  After HGA_ERR_TIMEOUT the idx copy
 * into host_idx_scratch is still pending on compute_stream, as for
 * hga_fetch_blocks.
 */
HGA_API hga_status hga_fetch_blocks_cached(const hga_dims* dims, const void* host_k, const void* host_v,
                                           const int32_t* idx_dev, int32_t* host_idx_scratch, void* pool_k,
                                           void* pool_v, hga_block_cache* cache, int32_t* idx_pool_dev,
                                           int* n_unique_out, int* n_fetched_out, hga_stream_t compute_stream,
                                           hga_stream_t copy_stream, hga_event_t done, int timeout_ms);

/*
 * Keep a finished segment's blocks resident in a layer's device block cache
 * as they enter the history: plans slots for history blocks [at_block,
 * at_block + S/block) by the hga_block_cache_plan rules (they become the most
 * recently used) and copies the segment's K/V (device, [B, S, Hkv, d]) into
 * those slots of pool_k/pool_v (device-to-device, on `stream`; queue it after
 * every kernel that may still read the pool).  With hga_offload_segment the
 * blocks then exist in both tiers, and a later selection of them copies
 * nothing over the host link.  Errors: HGA_ERR_INVALID_ARG (NULL pointers,
 * blocks outside the cache's host capacity, a pool smaller than a segment),
 * HGA_ERR_CUDA; on any error the cache is unchanged.
 */
HGA_API hga_status hga_cache_segment(const hga_dims* dims, const void* k_seg, const void* v_seg, void* pool_k,
                                     void* pool_v, hga_block_cache* cache, int at_block, hga_stream_t stream);

/*
 * A finished segment enters the history in ONE pass over its K and V
 * (article, Deep analysis: the summaries stay resident and grow with the
 * context; fr edition, Analyse approfondie: a finished segment's KV is
 * offloaded right away).  For the S/block blocks t of the segment
 * (k_seg/v_seg [B, S, Hkv, d], device):
 *   summ[b, at_block+t, h, :] = mean of the block's keys (fp32; as
 *       hga_segment_summaries; dims->n_hist_blocks = the capacity of summ);
 *   with a device block cache (cache != NULL): blocks at_block .. get slots
 *       by the hga_block_cache_plan rules (as hga_cache_segment) and their K
 *       and V are written into pool_k/pool_v [B, cache->pool_slots*block,
 *       Hkv, d] by the same kernel that forms the summaries;
 *   with a host tier (host_k/host_v != NULL, pinned, [B,
 *       tier_capacity_blocks*block, Hkv, d]): the segment's K/V are copied
 *       to the tier at block at_block on copy_stream (ordered after the work
 *       already queued on `stream`; NULL copy_stream = `stream`), running
 *       alongside the kernel; k_seg/v_seg must stay valid until copy_stream
 *       has passed the copies.
 * The kernel runs on `stream`; queue it after every kernel that may still read
 * the pool slots it overwrites.  Replaces hga_segment_summaries +
 * hga_cache_segment + hga_offload_segment (three passes over K) with one.
 * S/block <= 128.  Errors: HGA_ERR_INVALID_ARG (NULL or misaligned pointers,
 * blocks outside summ, the cache or the tier), HGA_ERR_SHAPE, HGA_ERR_CUDA; on
 * any error the cache is unchanged.
 */
HGA_API hga_status hga_append_segment(const hga_dims* dims, const void* k_seg, const void* v_seg, int at_block,
                                      float* summ, void* pool_k, void* pool_v, hga_block_cache* cache, void* host_k,
                                      void* host_v, int tier_capacity_blocks, hga_stream_t stream,
                                      hga_stream_t copy_stream);

/*
 * idx -> pool slots on the device, for a cache that holds every selectable
 * block (then no host round trip is needed):
 *   idx_pool[k] = slot_of_block_dev[idx[k]]   (-1 kept)
 * slot_of_block_dev: device int32 [n_hist_blocks], a copy of the cache's
 * slot_of_block.  An idx entry outside [-1, n_hist_blocks) or a block that is
 * not resident (slot -1) sets the device error flag (HGA_ERR_INDEX at the next
 * hga_device_status) and gives -1, so the attention kernels skip it.
 * Errors: HGA_ERR_INVALID_ARG (NULL pointers), HGA_ERR_SHAPE.
 */
HGA_API hga_status hga_remap_idx(const hga_dims* dims, const int32_t* idx_dev, const int32_t* slot_of_block_dev,
                                 int32_t* idx_pool_dev, hga_stream_t stream);

/*
 * Segment-end offload (fr edition, Analyse approfondie: the KV of a finished
 * segment is offloaded right away).  Copies the segment's K and V (device,
 * [B, S, Hkv, d]) into the pinned host tier at history block `at_block`
 * (host_k/host_v [B, capacity_blocks*block, Hkv, d]) on `stream`, one copy per
 * (batch, tensor).  The summaries of the new blocks are computed on the device
 * with hga_segment_summaries.  Errors: HGA_ERR_INVALID_ARG, HGA_ERR_SHAPE.
 */
HGA_API hga_status hga_offload_segment(const hga_dims* dims, const void* k_seg, const void* v_seg, void* host_k,
                               void* host_v, int capacity_blocks, int at_block, hga_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* HGA_H */
