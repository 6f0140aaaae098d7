/*
 * lf.h — C ABI of liblf, a B200 (sm_100a) implementation of Light Forcing's hierarchical
 * sparse attention (HSA) for chunk-wise autoregressive video diffusion.
 *
 * The method (sources named by page title and section):
 *   [LF-gist] "Light Forcing: Accelerating Autoregressive Video Diffusion via Sparse
 *             Attention" (gist.science explainer), section 2.2 Hierarchical Sparse
 *             Attention — token compression by mean pooling per block and per frame,
 *             two-stage mask selection (frames, then blocks inside chosen frames),
 *             attention only on the chosen frame-block pairs.
 *   [LF-yly]  "南洋理工大学AI新突破 视频生成引擎模仿人脑高效学习" (m.youleyou.com),
 *             section 三 — the same three stages; frames retrieved by inner products;
 *             section 四 — the one-dimensional block-sparse attention it is compared with.
 *   [LF-gist 2.1] the same explainer, section 2.1 — sparsity grown chunk by chunk.
 *   [SF]      Self Forcing article, rolling KV cache paragraph — cache of the last L
 *             frames, oldest evicted first.
 *   [RF]      "南洋理工大学突破：AI实现实时流式视频生成" (163.com, Rolling Forcing),
 *             section 三 — first frames kept as permanent anchors (sink frames).
 *
 * One call of the attention layer = (a) lf_compress, (b) lf_select_frames,
 * (c) lf_select_blocks, (d) lf_block_sparse_attn; lf_forward_chunk chains all four.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  Tensors.  bf16 tensors are token-major [tokens, H, d], contiguous:
 *      q, k_cur, v_cur   : [n_cur_frames*T, H, d]  (the current chunk, raster order)
 *      k_cache, v_cache  : [n_slots, T, H, d]      (one latent frame per slot)
 *      out               : [n_cur_frames*T, H, d]
 *    Pooled and score tensors are fp32, index tensors int32, all contiguous:
 *      q_blk  [H, n_qb, d]           k_blk [H, n_hist, n_bpf, d]    k_frm [H, n_hist, d]
 *      frame_idx [H, n_qb, kf]       block_idx [H, n_qb, kf*kb]      lse [H, n_cur_frames*T]
 *      cur_idx [H, n_qb, kc]
 *    with T = tokens_per_frame, B = block, n_bpf = ceil(T/B), n_qb = n_cur_frames*n_bpf,
 *    kf = min(k_f, n_hist), kb = min(k_b, n_bpf), kc = min(k_c, n_qb).
 *  Blocks.  Block b of a frame covers tokens [b*B, min((b+1)*B, T)); the last block of a
 *    frame is shorter when B does not divide T.  Query block qb = frame*n_bpf + b.
 *    A global history block id is g = f*n_bpf + b, f being the history position.
 *  Frame lists.  hist_slots[n_hist] and sink_slots[n_sink] are HOST int32 arrays giving
 *    the cache slot of each history / sink frame, oldest first; they are read during
 *    the call only.  Rolling the cache means rewriting slot ids; nothing is copied.
 *  Memory.  Every other pointer is caller-owned DEVICE memory on the current device.
 *    The library never allocates or frees.  bf16 tensors and fp32 tensors must be
 *    16-byte aligned; int32 tensors 4-byte aligned.
 *  Streams.  Work is enqueued on `stream` and is asynchronous; a return of LF_OK means
 *    the arguments were valid and the launches were accepted.  Device-detected errors
 *    (an index out of range in a caller-supplied list, a device wait that ran out of
 *    time) are recorded in a per-device status word read by lf_device_status().
 *  Validation.  Every argument check happens before the first launch; on error nothing
 *    is enqueued.
 *  Determinism.  Identical inputs give bit-identical outputs (no float atomics).
 */
#ifndef LF_H_
#define LF_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LF_ABI_VERSION 2

/* status codes */
#define LF_OK               0
#define LF_ERR_INVALID_ARG  1   /* null/misaligned pointer, inconsistent sizes          */
#define LF_ERR_UNSUPPORTED  2   /* d or block outside {64,128}, or a size limit exceeded */
#define LF_ERR_CUDA         3   /* a CUDA runtime or launch error                        */
#define LF_ERR_TIMEOUT      4   /* a bounded device wait expired (from lf_device_status) */
#define LF_ERR_WORKSPACE    5   /* workspace pointer null or smaller than required       */
#define LF_ERR_BAD_INDEX    6   /* device found an index out of range (lf_device_status) */

/* size limits checked by every entry point */
#define LF_MAX_FRAMES       256     /* n_sink + n_hist                                  */
#define LF_MAX_T            16384   /* tokens per frame                                 */
#define LF_MAX_SELECTED     1024    /* kf * kb per query block                          */
#define LF_MAX_PLAN         2048    /* key blocks per 128-row query tile:
                                       n_sink * n_bpf + (block == 64 ? 2 : 1) * (kc + kf*kb) */
#define LF_MAX_CUR_BLOCKS   256     /* n_qb when the current chunk is sparse (k_c > 0)    */

typedef struct lf_shape {
    int32_t H;                /* heads, >= 1                                              */
    int32_t d;                /* head dimension: 64 or 128                                */
    int32_t tokens_per_frame; /* T, 1..LF_MAX_T                                           */
    int32_t block;            /* B, block size in tokens: 64 or 128                       */
    int32_t n_cur_frames;     /* F_c, frames in the current chunk, >= 1                   */
    int32_t n_hist;           /* F, selectable history frames, >= 0                       */
    int32_t n_sink;           /* S_k, always-dense sink frames, >= 0                      */
    int32_t n_slots;          /* frames the cache tensors hold; slot ids are < n_slots    */
    int32_t k_f;              /* frames kept per query block (>= 1 when n_hist > 0)       */
    int32_t k_b;              /* blocks kept per chosen frame (>= 1 when n_hist > 0)      */
    float   scale;            /* softmax scale applied to q.k, normally 1/sqrt(d)         */
    int32_t k_c;              /* current-chunk blocks kept per query block; 0 = the whole
                                 current chunk (dense); kc = min(k_c, n_qb) otherwise      */
} lf_shape;

/* (a) Token compression [LF-gist 2.2 "token compression"; LF-yly 三, first stage].
 * q_blk[h, qb]   = mean of the query tokens of block qb of the current chunk;
 * k_blk[h, f, b] = mean of the keys of block b of history frame f;
 * k_frm[h, f]    = mean of all T keys of history frame f.
 * Accumulation is fp32 in a fixed order.  With n_hist == 0 only q_blk is written and
 * k_cache / k_blk / k_frm may be NULL. */
int lf_compress(const lf_shape* shape, const void* q, const void* k_cache,
                const int32_t* hist_slots, float* q_blk, float* k_blk, float* k_frm,
                cudaStream_t stream);

/* (b) Frame-level selection [LF-gist 2.2, mask selection step 1; LF-yly 三].
 * score[h, qb, f] = q_blk[h, qb] . k_frm[h, f]; frame_idx[h, qb] = the kf frames with the
 * largest scores, ties to the lower index, written in ascending order.
 * frame_score (nullable) receives all scores [H, n_qb, n_hist].  Requires n_hist >= 1. */
int lf_select_frames(const lf_shape* shape, const float* q_blk, const float* k_frm,
                     int32_t* frame_idx, float* frame_score, cudaStream_t stream);

/* (c) Block-level selection inside the chosen frames [LF-gist 2.2, mask selection step 2].
 * For each chosen frame f of (h, qb): score[b] = q_blk[h, qb] . k_blk[h, f, b]; keep the
 * kb largest (ties to the lower index).  block_idx[h, qb] lists the kf*kb global block
 * ids g = f*n_bpf + b in ascending order.  block_score (nullable) receives the scores of
 * the chosen frames [H, n_qb, kf, n_bpf].  frame_idx entries must be ascending and
 * < n_hist (violations are recorded as LF_ERR_BAD_INDEX and the entry is skipped). */
int lf_select_blocks(const lf_shape* shape, const float* q_blk, const float* k_blk,
                     const int32_t* frame_idx, int32_t* block_idx, float* block_score,
                     cudaStream_t stream);

/* (a)+(b)+(c) in one call [LF-gist 2.2; LF-yly 三]: pooling, frame top-k and block top-k.
 * block_idx (device, [H, n_qb, kf*kb]) receives the selected global block ids, ascending
 * per (h, qb), exactly as lf_compress + lf_select_frames + lf_select_blocks define them
 * (frame scores use the identity q_blk . k_frm = sum_b len_b (q_blk . k_blk[b]) / T).
 * workspace: at least lf_select_workspace_size(shape) bytes, 256-byte aligned.
 * Requires n_hist >= 1. */
size_t lf_select_workspace_size(const lf_shape* shape);
int lf_select_chunk(const lf_shape* shape, const void* q, const void* k_cache,
                    const int32_t* hist_slots, int32_t* block_idx, void* workspace,
                    size_t workspace_bytes, cudaStream_t stream);

/* One-dimensional block selection, the ablation the pages compare the hierarchical
 * selection with [LF-yly 四]: (a) pooling as in lf_select_chunk, then no frame stage:
 * block_idx[h, qb] (device, [H, n_qb, kf*kb] with the effective kf = min(k_f, n_hist),
 * kb = min(k_b, n_bpf)) receives the kf*kb history blocks with the largest scores
 * q_blk . k_blk over ALL n_hist * n_bpf blocks, equal scores to the lower global id
 * f*n_bpf + b, in ascending order -- the same layout lf_block_sparse_attn consumes.
 * Same workspace as lf_select_chunk.  LF_ERR_UNSUPPORTED when n_hist * n_bpf > 2048.
 * Requires n_hist >= 1. */
int lf_select_chunk_1d(const lf_shape* shape, const void* q, const void* k_cache,
                       const int32_t* hist_slots, int32_t* block_idx, void* workspace,
                       size_t workspace_bytes, cudaStream_t stream);

/* Pooled-key cache (incremental compression).  A frame's keys do not change once it is
 * in the KV cache [SF, rolling KV cache paragraph], so its block means [LF-gist 2.2,
 * token compression] can be computed once, when the frame enters, instead of on every
 * call.  The pages describe no such cache; it changes no result: the cached path
 * selects bit-identically to lf_select_chunk.
 *
 * k_pool (device, caller-owned, fp32 [n_slots, H, n_bpf, d], lf_pooled_cache_bytes):
 * row (slot, h, b) holds the mean of block b of the keys in cache slot `slot`, computed
 * exactly as lf_compress computes k_blk.
 *
 * lf_pool_frames: pools the keys of the n cache slots slots[0..n) (HOST array, each in
 * [0, n_slots)) of k_cache [n_slots, T, H, d] bf16 into their rows of k_pool; other rows
 * are untouched.  0 <= n <= LF_MAX_FRAMES; n == 0 does nothing.
 *
 * lf_select_chunk_cached: lf_select_chunk with the history block means read from k_pool
 * through hist_slots (their rows must have been written by lf_pool_frames since the
 * slots' keys last changed); only the current chunk's queries are pooled.  Same
 * workspace as lf_select_chunk.  Returns LF_ERR_UNSUPPORTED for shapes beyond the fused
 * selection's limits (n_hist * n_bpf > 2048 or k_f * k_b > 256).  Requires n_hist >= 1. */
size_t lf_pooled_cache_bytes(const lf_shape* shape);
int lf_pool_frames(const lf_shape* shape, const void* k_cache, const int32_t* slots,
                   int32_t n, float* k_pool, cudaStream_t stream);
int lf_select_chunk_cached(const lf_shape* shape, const void* q, const float* k_pool,
                           const int32_t* hist_slots, int32_t* block_idx, void* workspace,
                           size_t workspace_bytes, cudaStream_t stream);

/* Sparse current chunk [LF-yly 一: the first chunk, which has no history, tested at 80%
 * sparsity, so the sparsity reaches the current chunk's own keys; LF-gist 2.2 token
 * compression and inner-product block selection].  Requires shape->k_c >= 1 and
 * n_qb <= LF_MAX_CUR_BLOCKS.  The current chunk's keys are mean-pooled per block exactly
 * as the queries are (fp32, fixed order); query block qb keeps its own block qb and the
 * kc - 1 other current blocks with the largest q_blk[h, qb] . kc_blk[h, c] (ties to the
 * lower index).  cur_idx (device, [H, n_qb, kc]) receives the block ids c = frame*n_bpf
 * + b, ascending.  workspace: at least lf_forward_workspace_size(shape) bytes, 256-byte
 * aligned. */
int lf_select_current(const lf_shape* shape, const void* q, const void* k_cur,
                      int32_t* cur_idx, void* workspace, size_t workspace_bytes,
                      cudaStream_t stream);

/* Workspace bytes lf_block_sparse_attn needs for this shape (its per-tile key plans). */
size_t lf_attn_workspace_size(const lf_shape* shape);

/* (d) Block-sparse attention [LF-gist 2.2 "execution"; LF-yly 三, last stage].
 * For every query token of query block qb and head h, one joint softmax over
 *   - the keys of the current chunk (k_cur): all of them (dense, no causal mask) when
 *     shape->k_c == 0, else those of the current blocks listed in cur_idx[h, qb],
 *   - every key of every sink frame (k_cache at sink_slots) [RF],
 *   - the keys of the history blocks listed in block_idx[h, qb] (k_cache at hist_slots)
 * of scale * q.k, applied to the matching values.  out receives bf16; lse (nullable)
 * receives the natural-log normaliser log(sum exp(scale*q.k)) in fp32.
 * block_idx: [H, n_qb, kf*kb] ascending global ids (ignored, may be NULL, when
 * n_hist == 0).  cur_idx: [H, n_qb, kc] ascending current block ids (ignored, may be
 * NULL, when k_c == 0).  Ids out of range or not ascending are recorded as
 * LF_ERR_BAD_INDEX and that list is dropped.  Compute: tcgen05 bf16 MMAs with fp32
 * accumulation in tensor memory, fp32 online softmax. */
int lf_block_sparse_attn(const lf_shape* shape, const void* q, const void* k_cur,
                         const void* v_cur, const void* k_cache, const void* v_cache,
                         const int32_t* hist_slots, const int32_t* sink_slots,
                         const int32_t* block_idx, const int32_t* cur_idx, void* out,
                         float* lse, void* workspace, size_t workspace_bytes,
                         cudaStream_t stream);

/* FP8 (e4m3) variant of (d) [LF-yly 五 deploys the video model with FP8, activations
 * quantised per token; using e4m3 for the attention's QK^T operands is this library's
 * extension].  The same attention as lf_block_sparse_attn (d = 128 only) on dequantised
 * queries and keys: q8 [n_cur_frames*T, H, d] and k_cur8 / k_cache8 (k_cur / k_cache
 * layouts) are e4m3 codes as written by lf_quantize_e4m3; q_scale [n_cur_frames*T, H]
 * holds one power-of-two scale per (token, head), k_scale [H] one per head for every key
 * the call can attend to; v_cur and v_cache stay bf16.  S = Q K^T runs on tcgen05.mma
 * kind::f8f6f4 (exact products, fp32 accumulation); the scales enter the softmax's
 * per-row factor, so the result is that of the dequantised operands within the bf16
 * path's rounding.  Workspace: lf_attn_workspace_size.  LF_ERR_UNSUPPORTED for d != 128. */
int lf_block_sparse_attn_e4m3(const lf_shape* shape, const void* q8, const float* q_scale,
                              const void* k_cur8, const void* v_cur, const void* k_cache8,
                              const void* v_cache, const float* k_scale,
                              const int32_t* hist_slots, const int32_t* sink_slots,
                              const int32_t* block_idx, const int32_t* cur_idx, void* out,
                              float* lse, void* workspace, size_t workspace_bytes,
                              cudaStream_t stream);

/* e4m3 quantisation of a bf16 tensor x [rows, H, d] (d in {64, 128}) into x8 (same layout,
 * one byte per element): each value is divided by its group's scale (a power of two, so
 * exactly) and rounded to the nearest e4m3 value, ties to the even code.  head_scale
 * non-null: the groups are the heads, with the given scales [H] (powers of two large
 * enough that |x| / scale <= 448; larger values saturate to 448); else the groups are the
 * (row, head) pairs and their scales -- the smallest 2^e with max|x| <= 448 * 2^e, 1 for an
 * all-zero row -- are written to row_scale [rows, H]. */
int lf_quantize_e4m3(const void* x, int64_t rows, int32_t H, int32_t d, const float* head_scale,
                     uint8_t* x8, float* row_scale, cudaStream_t stream);

/* Per-head power-of-two scales over n (1..16) bf16 tensors xs[i] [rows[i], H, d] (HOST
 * arrays of device pointers and row counts): head_scale[h] (device, [H]) = the smallest
 * 2^e with max |x[., h, .]| <= 448 * 2^e over all of them (1 when all are zero). */
int lf_e4m3_head_scales(const void* const* xs, const int64_t* rows, int32_t n, int32_t H,
                        int32_t d, float* head_scale, cudaStream_t stream);

/* lf_block_sparse_attn for callers that cannot allocate device memory.
 *
 * No counterpart in the paper: this is a packaging variant of (d).  Some callers cannot
 * provide the workspace lf_block_sparse_attn asks for: code embedded in a host runtime
 * that exposes no allocator or scratch hook to it, or a latency-critical loop that allows
 * no device allocation after start-up (cudaMalloc may synchronise the device).  This
 * entry point takes the same arguments minus the workspace and uses instead a fixed
 * scratch array in device global memory that lives in the library: at most
 * lf_noalloc_scratch_bytes() bytes (16 MiB), reserved on a device once the library's
 * module is loaded there (with lazy module loading, at its first use on that device) and
 * held until the process exits.  It allocates nothing and calls no allocating routine.
 *
 *  - The first call on a device looks up the array's device address (cudaGetSymbolAddress,
 *    with that device current) and caches it with the current context; a call in a new
 *    context (after cudaDeviceReset) looks it up again.  Make the first call on a device
 *    before any stream capture on it.
 *  - All calls on a device share the one array, which keeps the last call's contents
 *    (nothing in it needs to start at zero).  Calls whose work may overlap on the GPU —
 *    on different streams, or from different host threads — race on it; serialise them.
 *  - A shape whose workspace (lf_attn_workspace_size) exceeds the array returns
 *    LF_ERR_WORKSPACE without launching anything.
 *  - It takes no current-chunk list: a shape with k_c > 0 returns LF_ERR_INVALID_ARG.
 * Results are those of lf_block_sparse_attn. */
size_t lf_noalloc_scratch_bytes(void);
int lf_block_sparse_attn_noalloc(const lf_shape* shape, const void* q, const void* k_cur,
                                 const void* v_cur, const void* k_cache, const void* v_cache,
                                 const int32_t* hist_slots, const int32_t* sink_slots,
                                 const int32_t* block_idx, void* out, float* lse,
                                 cudaStream_t stream);

/* Workspace bytes lf_forward_chunk needs: pooled tensors, index lists and key plans. */
size_t lf_forward_workspace_size(const lf_shape* shape);

/* (a)->(b)->(c)->(d) in one call (and, with k_c > 0, the current-chunk choice of
 * lf_select_current).  block_idx_out (nullable) receives the selected block ids
 * [H, n_qb, kf*kb], cur_idx_out (nullable) the kept current blocks [H, n_qb, kc]; lse is
 * nullable.  With n_hist == 0 no history selection runs and the attention covers the
 * current chunk and the sink frames. */
int lf_forward_chunk(const lf_shape* shape, const void* q, const void* k_cur,
                     const void* v_cur, const void* k_cache, const void* v_cache,
                     const int32_t* hist_slots, const int32_t* sink_slots,
                     void* workspace, size_t workspace_bytes, void* out, float* lse,
                     int32_t* block_idx_out, int32_t* cur_idx_out, cudaStream_t stream);

/* Test hook, not part of the attention path (process-wide, not thread-safe; call it only
 * while no library work is queued).  Sets, for the attention launches that follow:
 *   wait_limit_ns  the limit of every bounded device wait (0 = the default, 2 s; at most
 *                  20 s);
 *   stall          nonzero: the first CTA of each attention launch never arms its query
 *                  barrier, so its waits run out after wait_limit_ns; the launch then
 *                  drains, frees its tensor memory, returns, and lf_device_status()
 *                  reports LF_ERR_TIMEOUT (that launch's output is undefined);
 *   tail_split     zero: every query tile is computed whole (no split of the last partial
 *                  wave into key ranges), so each tile's rounding is independent of how
 *                  many tiles a launch has.
 * lf_debug_configure(0, 0, 1) restores the defaults.  LF_ERR_INVALID_ARG for a limit
 * above 20 s. */
int lf_debug_configure(uint64_t wait_limit_ns, int stall, int tail_split);

/* Chunk-aware growth of the sparsity [LF-gist 2.1, consistency-aware growth]: the sparsity
 * of chunk i rises as the noise level alpha_i falls, s_i = s_base - alpha_i * beta, here
 * with alpha_i = 1/sqrt(i).  Chunks first..n_chunks are sparse; beta and s_base are
 * solved so that the mean of s_i over them is mean_sparsity and s_{n_chunks} is
 * final_sparsity (first == n_chunks needs mean == final).  Host only, no device work.
 * Outputs per chunk i = 1..n_chunks (HOST arrays of n_chunks entries):
 *   keep[i-1] = 1 - s_i, clamped to [0, 1] (1 for chunks before `first`);
 *   if n_hist, k_f and k_b are given, the top-k budget of a chunk with F = n_hist[i-1]
 *   history frames of n_bpf blocks: (0, 0) when F = 0; (F, n_bpf) (dense) before
 *   `first`; else k_f = min(kf_max, F), k_b = floor(keep * F * n_bpf / k_f + 1/2)
 *   (halves round up) clamped to [1, n_bpf], so that k_f * k_b / (F * n_bpf) ~ keep.
 * LF_ERR_INVALID_ARG for n_chunks outside [1, 4096], first outside [1, n_chunks],
 * sparsities outside [0, 1), n_bpf or kf_max < 1, or missing outputs. */
int lf_cag_schedule(int32_t n_chunks, int32_t first, float mean_sparsity, float final_sparsity,
                    const int32_t* n_hist, int32_t n_bpf, int32_t kf_max, float* keep,
                    int32_t* k_f, int32_t* k_b);

/* Reads (synchronising the current device) and optionally clears the device status word
 * of the current device: LF_OK, LF_ERR_BAD_INDEX or LF_ERR_TIMEOUT.  Returns LF_ERR_CUDA
 * if the read itself fails. */
int lf_device_status(int reset);

/* Static text for a status code. */
const char* lf_status_string(int status);

/* LF_ABI_VERSION of the loaded library. */
int lf_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* LF_H_ */
