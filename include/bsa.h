/*
 * bsa.h -- C ABI of the block-sparse global attention layer for multi-view geometry
 * transformers, built for NVIDIA B200 (sm_100a).
 *
 * The layer and its five steps are those of "Block-Sparse Global Attention for
 * Efficient Multi-View Geometry Transformers" (CVPR 2026 paper notes):
 *   - 方法详解 / 整体框架 (flowchart): split the special tokens X_s from the patch
 *     tokens X_p; predict a block mask on X_p; block-sparse attention on the selected
 *     Q-K blocks; dense attention for X_s; merge the outputs;
 *   - 关键设计 1: average pooling P_b(Q), P_b(K) by block size b, softmax of
 *     P_b(Q) P_b(K)^T; Eq. (1) dense attention; Eq. (2) masked attention;
 *   - 关键设计 2: Top-K + CDF dual threshold with k = floor(B (1 - rho));
 *   - 关键设计 3: the 1 camera + 4 register tokens of each frame stay dense.
 * Per-head budgets follow "HeSS: Head Sensitivity Score for Sparsity Redistribution
 * in VGGT", 提案手法 (iterative capped redistribution of the layer budget).
 *
 * Conventions for every call:
 *   - Token layout: Q, K, V and out are row-major [N, H, d] with N = F * T tokens
 *     (frame-major), row stride H * d elements. The first S tokens of each frame are
 *     the special tokens; the remaining P = T - S are patch tokens. The patch tokens
 *     of all frames, concatenated in frame order, form X_p with Np = F * P rows; patch
 *     token p (0 <= p < Np) is row (p / P) * T + S + (p % P).
 *   - Blocks: block j covers patch tokens [j b, min((j+1) b, Np)); B = ceil(Np / b).
 *     Blocks may straddle frames; the last block may be short (ragged).
 *   - Pointers named *_dev or documented as device memory are CUDA device pointers;
 *     host arrays are documented as such. The caller owns and allocates every buffer;
 *     the library never allocates, frees or synchronises (except bsa_check_status).
 *     Device pointers must be 16-byte aligned.
 *   - Every device call is asynchronous and ordered on `stream` (NULL = legacy stream).
 *   - status_dev: optional device int32 (NULL allowed). Kernels write the first device-
 *     side error (BSA_ERR_TIMEOUT, BSA_ERR_DEVICE_BOUNDS, BSA_ERR_RANGE) there and skip
 *     the faulty access instead of faulting; read it with bsa_check_status. Zero it
 *     before use.
 *   - Host-side validation happens before any launch; on error nothing is launched.
 *     A failed launch returns BSA_ERR_CUDA.
 */
#ifndef BSA_H
#define BSA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BSA_API __attribute__((visibility("default")))
#else
#define BSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* bsa_stream_t; /* same type as cudaStream_t */

typedef enum {
    BSA_OK = 0,
    BSA_ERR_INVALID_ARG = 1,   /* null pointer, bad shape or value, misaligned pointer */
    BSA_ERR_UNSUPPORTED = 2,   /* valid arguments outside what the kernels implement */
    BSA_ERR_CUDA = 3,          /* a CUDA runtime or driver call failed */
    BSA_ERR_TIMEOUT = 4,       /* device: a bounded wait ran out */
    BSA_ERR_DEVICE_BOUNDS = 5, /* device: an out-of-range index was rejected */
    BSA_ERR_RANGE = 6          /* device: an input value outside the range the kernels take
                                  (a bf16 V element of magnitude >= 65536, inf or NaN: the
                                  fp16 operand of the P.V product cannot hold it) */
} bsa_status;

typedef enum { BSA_F32 = 0, BSA_BF16 = 1 } bsa_dtype;

typedef struct {
    int32_t frames;            /* F >= 1 */
    int32_t tokens_per_frame;  /* T = P + S, P >= 1 */
    int32_t special_per_frame; /* S >= 0, prefix of every frame (1 camera + 4 register: 5) */
    int32_t heads;             /* H >= 1 */
    int32_t head_dim;          /* d; only 64 is implemented */
    int32_t block;             /* b >= 1 */
    bsa_dtype dtype;           /* element type of Q, K, V and out */
} bsa_layout;

/* Limits of the implementation (BSA_ERR_UNSUPPORTED beyond them). */
#define BSA_HEAD_DIM 64
#define BSA_MAX_BLOCKS 8192       /* B, bounded by the per-row selection buffer */
#define BSA_MAX_HEADS 128
#define BSA_F32_MAX_TOKENS 65536  /* f32 inputs run on CUDA cores; meant for small layers */

/* ---------------------------------------------------------------------------------
 * Step 1 -- block pooling P_b (关键设计 1).
 * pq[h, j, :] = mean of Q[row(p), h, :] over the patch tokens p of block j (the
 * divisor is the block's real token count); the same for pk from K.
 *   q, k    : device, [N, H, d] of layout->dtype
 *   pq      : device, float32 [H, B, d]
 *   pk      : device, float32 [H, d, B] (dimension-major: the score pass of
 *             bsa_predict_mask reads 32 consecutive blocks of one dimension per load)
 */
BSA_API bsa_status bsa_pool_qk(const bsa_layout* layout, const void* q, const void* k,
                       float* pq, float* pk, int32_t* status_dev, bsa_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Steps 2-3 -- pooled softmax and dual-threshold block selection (关键设计 1, 2).
 * For every head h and query block i: s_ij = <pq[h,i], pk[h,j]> / sqrt(d),
 * p_ij = softmax_j(s_ij); rank the blocks by p (descending, ties to the lower index),
 * C(n) = cumulative mass of the first n; keep n = min(B, max(k_h, n_tau)) blocks where
 * n_tau = min{n >= 1 : C(n) >= tau} (0 if tau <= 0, B if never reached).
 * k_h = floor(B (1 - rho) + 1e-9) for every head when head_density is NULL; otherwise
 * k_h = clamp(floor(B head_density[h] + 1e-9), 1, B) and rho only validates that
 * sum_h head_density[h] = H (1 - rho) within 1e-9 * H.
 *   pq, pk        : device, float32 [H, B, d] and [H, d, B] (from bsa_pool_qk)
 *   rho, tau      : in [0, 1]
 *   head_density  : host, double [H] in [0, 1], or NULL
 *   mask_bits     : device, uint32 [H, B, ceil(B/32)] (bit j%32 of word j/32 = block j
 *                   kept), or NULL
 *   kv_idx        : device, uint16 [H, B, B]; row (h, i) holds the kept blocks in
 *                   ascending order in its first kv_cnt[h, i] entries (rest untouched)
 *   kv_cnt        : device, int32 [H, B]
 */
BSA_API bsa_status bsa_predict_mask(const bsa_layout* layout, const float* pq, const float* pk,
                            double rho, double tau, const double* head_density,
                            uint32_t* mask_bits, uint16_t* kv_idx, int32_t* kv_cnt,
                            int32_t* status_dev, bsa_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Alternative block selectors. Each writes the same outputs as bsa_predict_mask (mask_bits
 * optional, kv_idx ascending in the first kv_cnt entries of each row, kv_cnt), so that the
 * same attention entry points compute the layer under them. k_h is computed as in
 * bsa_predict_mask from rho and the optional host head_density (validated the same way).
 *
 * Random selection -- the "Random" rows of the ablation in "Block-Sparse Global Attention
 * for Efficient Multi-View Geometry Transformers", 消融实验 (图 10): every row (h, i) keeps
 * k_h blocks drawn uniformly without replacement. Block j of row (h, i) gets the 32-bit key
 * word 0 of Philox4x32-10 (Salmon et al., "Parallel Random Numbers: As Easy as 1, 2, 3",
 * SC 2011) at counter (j, i, h, 0) under key (seed mod 2^32, seed >> 32); the row keeps the
 * k_h blocks of smallest (key, j). Deterministic in (layout, k_h, seed).
 */
BSA_API bsa_status bsa_random_mask(const bsa_layout* layout, double rho, const double* head_density,
                                   uint64_t seed, uint32_t* mask_bits, uint16_t* kv_idx, int32_t* kv_cnt,
                                   int32_t* status_dev, bsa_stream_t stream);

/* Fixed-stride uniform sampling -- "SAF3R: Dynamic Sparse Attention for Feed-Forward 3D
 * Reconstruction Transformers", 四、1. 均匀采样核 (scanning heads): every row keeps the patch
 * key blocks j = 0, stride, 2 stride, ... (ceil(B / stride) blocks).
 *   stride : >= 1 */
BSA_API bsa_status bsa_uniform_mask(const bsa_layout* layout, int32_t stride, uint32_t* mask_bits,
                                    uint16_t* kv_idx, int32_t* kv_cnt, int32_t* status_dev,
                                    bsa_stream_t stream);

/* Query-probe Top-K -- the same page, 四、1. Query-Probe Top-K 核 and its acceleration in 四、3.:
 * q_bar_h = the mean of the patch queries of head h (taken from the pooled means weighted by
 * the block sizes, in fp64); block j's probe score is q_bar_h . pk[h, :, j] / sqrt(d) (the
 * column means of Q K^T / sqrt(d) averaged over the block's keys), rounded to fp32; the k_h
 * blocks of highest score (ties to the lower index) are kept by every query block of head h.
 *   pq, pk : device, float32 [H, B, d] and [H, d, B] (from bsa_pool_qk / bsa_pack_pool_qkv) */
BSA_API bsa_status bsa_probe_mask(const bsa_layout* layout, const float* pq, const float* pk, double rho,
                                  const double* head_density, uint32_t* mask_bits, uint16_t* kv_idx,
                                  int32_t* kv_cnt, int32_t* status_dev, bsa_stream_t stream);

/* Drift-score selection -- "ReSS: Residual-Restoring Sparse Attention for 3D Vision
 * Transformers" (摘要, 技术框架, 关键设计: blocks chosen by the drift their removal leaves in the
 * residual stream, refined by iterative residual restoration), read at the pooled resolution of
 * bsa_predict_mask. Per head h and query block i, in fp64 from the fp32 pooled means:
 *   p_j = softmax_j(pq[h,i] . pk[h,:,j] / sqrt(d)), o = sum_j p_j pv[h,:,j],
 *   delta_j = p_j (o - pv[h,:,j]),
 *   drift(D) = |sum_{j in D} delta_j| / (1 - sum_{j in D} p_j) for a dropped set D (the exact
 *   shift of the renormalised pooled output).
 * Keep the k_h blocks of largest |delta_j| (ties to the lower index); then, at most `rounds`
 * times, restore the dropped block with the smallest resulting drift and drop the kept block
 * (other than it) with the smallest resulting drift, keeping the swap only if the drift fell.
 *   pq, pk : device, float32 [H, B, d] and [H, d, B] (bsa_pool_qk)
 *   pv        : device, float32 [H, d, B] (bsa_pool_v)
 *   rounds    : 0 .. BSA_RESS_MAX_ROUNDS
 *   workspace : device, 16-byte aligned, at least bsa_ress_workspace_size() bytes (the fp64
 *               Gram matrix of pv per head, H B B doubles; overwritten)
 * Needs P_b(V) of one head in shared memory: BSA_ERR_UNSUPPORTED above about B = 800 blocks. */
#define BSA_RESS_MAX_ROUNDS 1024
BSA_API bsa_status bsa_ress_mask(const bsa_layout* layout, const float* pq, const float* pk, const float* pv,
                                 double rho, const double* head_density, int32_t rounds, void* workspace,
                                 size_t workspace_bytes, uint32_t* mask_bits, uint16_t* kv_idx, int32_t* kv_cnt,
                                 int32_t* status_dev, bsa_stream_t stream);
/* Bytes of bsa_ress_mask's workspace: H B B 8. */
BSA_API bsa_status bsa_ress_workspace_size(const bsa_layout* layout, size_t* bytes);

/* Block pooling of V for bsa_ress_mask: pv[h, :, j] = the mean of V over the patch tokens of
 * block j, fp32, dimension-major [H, d, B] (as pk).
 *   v  : device, [N, H, d] of layout->dtype;  pv : device, float32 [H, d, B] */
BSA_API bsa_status bsa_pool_v(const bsa_layout* layout, const void* v, float* pv, int32_t* status_dev,
                              bsa_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Packing (prepares steps 4 and 5 for bf16 layers; the token split of 关键设计 3 made
 * physical). Copies the patch tokens and the special tokens of Q, K and V into a
 * head-major workspace: per head, rows of d = 64 elements, patch rows padded to a
 * multiple of 128 and special rows padded likewise, padding zeroed; Q and K stay bf16,
 * V is converted to fp16 (the operand type of the P.V product; exact for |v| in
 * [2^-14, 65504], smaller magnitudes lose precision, larger ones overflow).
 * A V element of magnitude >= 65536 (or inf / NaN), which fp16 cannot hold, is reported
 * as BSA_ERR_RANGE through status_dev (the layer's output is then not valid); magnitudes
 * below 2^-14 become fp16 subnormals, with an absolute error below 2^-25.
 * Must run after Q, K, V hold the layer's values and before bsa_block_sparse_attn /
 * bsa_special_dense on the same stream. Not needed (no-op) for f32 layouts.
 *   q, k, v          : device, [N, H, d] bf16
 *   workspace        : device, at least bsa_workspace_size() bytes, 1024-byte aligned
 */
BSA_API bsa_status bsa_pack_qkv(const bsa_layout* layout, const void* q, const void* k, const void* v,
                        void* workspace, size_t workspace_bytes, int32_t* status_dev,
                        bsa_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Packing and step 1 in one pass: the packed workspace of bsa_pack_qkv and the pooled
 * pq, pk of bsa_pool_qk (same layouts and values up to fp32 summation order), reading
 * Q and K from HBM once for both. For f32 layouts only the pooling runs (workspace
 * ignored, may be NULL). V values outside the fp16 range are reported as in bsa_pack_qkv.
 *   q, k, v          : device, [N, H, d] of layout->dtype
 *   workspace        : bf16: device, at least bsa_workspace_size() bytes, 1024-byte aligned
 *   pq, pk           : device, float32 [H, B, d] and [H, d, B]
 */
BSA_API bsa_status bsa_pack_pool_qkv(const bsa_layout* layout, const void* q, const void* k,
                             const void* v, void* workspace, size_t workspace_bytes,
                             float* pq, float* pk, int32_t* status_dev, bsa_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Step 4 -- block-sparse attention over the selected blocks (关键设计 1, Eq. (2)).
 * For every head h and patch token p of query block i:
 *   o_pp[p, h, :] = softmax over the patch keys of the blocks kv_idx[h, i, :kv_cnt[h,i]]
 *                   of (q . k / sqrt(d)), times V;
 *   lse_pp[h, p]  = ln sum exp(q . k / sqrt(d)) over those keys.
 * Keys of unselected blocks are excluded (not zeroed). A row with no kept block gets
 * o_pp = 0 and lse_pp = -inf. Block indices >= B are skipped and reported as
 * BSA_ERR_DEVICE_BOUNDS through status_dev. Listed indices are expected to be distinct
 * (as bsa_predict_mask writes them).
 *   q, k, v   : device, [N, H, d] of layout->dtype (read directly for f32 layouts)
 *   workspace : bf16 layouts: the packed copy written by bsa_pack_qkv (read only);
 *               f32 layouts: ignored (may be NULL)
 *   kv_idx, kv_cnt : device, as written by bsa_predict_mask
 *   o_pp      : device, float32 [Np, H, d];  lse_pp : device, float32 [H, Np]
 * bf16 runs on the tensor cores (tcgen05 MMA, TMEM accumulators, TMA tile loads, P in
 * fp16) and needs block in {64, 128}; f32 runs on CUDA cores in fp32.
 */
BSA_API bsa_status bsa_block_sparse_attn(const bsa_layout* layout, const void* q, const void* k,
                                 const void* v, const void* workspace, size_t workspace_bytes,
                                 const uint16_t* kv_idx, const int32_t* kv_cnt,
                                 float* o_pp, float* lse_pp, int32_t* status_dev,
                                 bsa_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Step 5 -- dense path of the special tokens (关键设计 3).
 *   (i)  every special token attends over all N tokens: out[special rows] (final);
 *   (ii) every patch token attends over the Ns = F * S special tokens:
 *        o_ps[p, h, :] and lse_ps[h, p] (as for step 4; -inf and 0 when S = 0).
 *   q, k, v   : device, [N, H, d] of layout->dtype (read directly for f32 layouts)
 *   workspace : bf16: the packed copy written by bsa_pack_qkv; f32: ignored (may be NULL)
 *   out       : device, [N, H, d] of layout->dtype; only the special rows are written
 *   o_ps    : device, float32 [Np, H, d], or NULL to skip (ii) (lse_ps then ignored)
 *   lse_ps  : device, float32 [H, Np]
 */
BSA_API bsa_status bsa_special_dense(const bsa_layout* layout, const void* q, const void* k,
                             const void* v, const void* workspace, size_t workspace_bytes,
                             void* out, float* o_ps, float* lse_ps, int32_t* status_dev,
                             bsa_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Step 6 -- merge (flowchart "合并输出"): one softmax over the special keys and the
 * selected patch keys, assembled exactly from the two partial results:
 *   L = ln(exp(lse_pp) + exp(lse_ps));
 *   out[row(p), h, :] = exp(lse_pp - L) o_pp[p, h, :] + exp(lse_ps - L) o_ps[p, h, :].
 * Rows where both lse are -inf get 0.
 *   o_pp, o_ps : device, float32 [Np, H, d];  lse_pp, lse_ps : device, float32 [H, Np]
 *   out        : device, [N, H, d] of layout->dtype; only the patch rows are written
 */
BSA_API bsa_status bsa_merge(const bsa_layout* layout, const float* o_pp, const float* lse_pp,
                     const float* o_ps, const float* lse_ps, void* out,
                     int32_t* status_dev, bsa_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Steps 4, 5(ii) and 6 in one pass (bf16 only): for every patch token p of query block i
 * and head h, out[row(p), h, :] = one softmax over the special keys and the patch keys of
 * the kept blocks kv_idx[h, i, :kv_cnt[h, i]] -- the same result as bsa_block_sparse_attn
 * + bsa_special_dense (ii) + bsa_merge, without the fp32 partials. The special rows of out
 * are not touched (bsa_special_dense with o_ps = NULL writes them).
 *   q, k, v   : unused (the packed copies in workspace are read); may be NULL
 *   workspace : the packed copy written by bsa_pack_qkv
 *   out       : device, [N, H, d] bf16
 */
BSA_API bsa_status bsa_block_sparse_attn_fused(const bsa_layout* layout, const void* q, const void* k,
                                               const void* v, const void* workspace,
                                               size_t workspace_bytes, const uint16_t* kv_idx,
                                               const int32_t* kv_cnt, void* out,
                                               int32_t* status_dev, bsa_stream_t stream);

/* ---------------------------------------------------------------------------------
 * The steps on either side of the layer. The pages put the global attention inside an
 * aggregator that alternates frame-wise and global multi-head attention ("Block-Sparse Global
 * Attention for Efficient Multi-View Geometry Transformers", 研究背景与动机; "SAF3R: Dynamic Sparse
 * Attention for Feed-Forward 3D Reconstruction Transformers", 图2). bf16 layouts only (BSA_ERR_UNSUPPORTED otherwise); fp32 accumulation, bf16 results
 * rounded to nearest even. C = heads * head_dim channels.
 *
 * QKV projection: [q | k | v] = x W_qkv^T + b_qkv, channel c of each third = head c / d,
 * dimension c % d (the usual multi-head split); written as three [N, H, d] tensors.
 *   x      : device, bf16 [N, C] (row stride C)
 *   w_qkv  : device, bf16 [3C, C] (output features x input features, row-major)
 *   b_qkv  : device, float32 [3C], or NULL for no bias
 *   q, k, v: device, bf16 [N, H, d] each
 * tcgen05 MMA on CTA pairs (256 x 256 output tiles, TMEM accumulators, TMA operand tiles). */
BSA_API bsa_status bsa_qkv_project(const bsa_layout* layout, const void* x, const void* w_qkv, const float* b_qkv,
                                   void* q, void* k, void* v, int32_t* status_dev, bsa_stream_t stream);

/* Output projection: y = o W_o^T + b_o with o's heads concatenated ([N, H, d] read as [N, C]).
 *   o   : device, bf16 [N, H, d];  w_o : device, bf16 [C, C];  b_o : device, float32 [C] or NULL
 *   y   : device, bf16 [N, C] (must not overlap o) */
BSA_API bsa_status bsa_out_project(const bsa_layout* layout, const void* o, const void* w_o, const float* b_o,
                                   void* y, int32_t* status_dev, bsa_stream_t stream);

/* Frame-wise attention, two calls. bsa_pack_frames copies Q, K and V per (head, frame) into
 * the workspace: the frame's T tokens, special tokens included, padded with zero rows to a
 * multiple of 128 (V as fp16, range-checked as in bsa_pack_qkv). bsa_frame_attention then
 * lets every token attend densely (Eq. (1)) over the T tokens of its own frame on the tensor
 * cores, reading only the workspace, and writes every row of out.
 *   q, k, v, out : device, bf16 [N, H, d]
 *   workspace    : device, at least bsa_frame_workspace_size() bytes, 1024-byte aligned */
BSA_API bsa_status bsa_pack_frames(const bsa_layout* layout, const void* q, const void* k, const void* v,
                                   void* workspace, size_t workspace_bytes, int32_t* status_dev,
                                   bsa_stream_t stream);
BSA_API bsa_status bsa_frame_attention(const bsa_layout* layout, const void* workspace, size_t workspace_bytes,
                                       void* out, int32_t* status_dev, bsa_stream_t stream);
/* Bytes of the frame-wise attention's workspace: 3 H F ceil(T / 128) 128 rows of 128 bytes
 * (0 for f32 layouts). */
BSA_API bsa_status bsa_frame_workspace_size(const bsa_layout* layout, size_t* bytes);

/* ---------------------------------------------------------------------------------
 * Allocation-free attention (bf16). The pages have no counterpart: this entry point
 * exists for callers that cannot allocate device memory -- code running under a host
 * framework whose memory pool owns every device allocation, or latency-critical loops in
 * which cudaMalloc/cudaFree are not allowed because they may synchronize the device.
 * It does what bsa_pack_qkv + bsa_special_dense (o_ps = NULL) + bsa_block_sparse_attn_fused
 * do (every row of out: the special rows dense, the patch rows over the special keys and
 * the kept blocks), but keeps the packed copy and the partial results in one static
 * device array of BSA_NOALLOC_SCRATCH_BYTES inside the library instead of a workspace.
 * The array exists on every GPU that loads the library until the process exits.
 *   - V values outside the fp16 range are reported through status_dev as in bsa_pack_qkv.
 *   - Layers whose packed data (bsa_workspace_size) exceed BSA_NOALLOC_SCRATCH_BYTES are
 *     rejected with BSA_ERR_UNSUPPORTED before anything is launched.
 *   - No memory is allocated or freed. The first call on a device looks up the device
 *     address of the array (cudaGetSymbolAddress) with that device current; make that
 *     first call before any stream capture.
 *   - All calls share the array and it keeps the last call's contents; every byte a call
 *     reads is written earlier by the same call, so nothing needs clearing. Calls that
 *     overlap on the GPU (other streams, other threads) race on the array: serialize them.
 *   q, k, v : device, [N, H, d] bf16;  kv_idx, kv_cnt : as written by bsa_predict_mask
 *   out     : device, [N, H, d] bf16, every row written
 */
#define BSA_NOALLOC_SCRATCH_BYTES (64u << 20)
BSA_API bsa_status bsa_attention_noalloc(const bsa_layout* layout, const void* q, const void* k,
                                         const void* v, const uint16_t* kv_idx, const int32_t* kv_cnt,
                                         void* out, int32_t* status_dev, bsa_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Self-check of the bounded device waits (no counterpart on the pages). Launches one
 * thread that waits, with the same bounded wait as the attention kernels, on an
 * mbarrier that nothing arrives on. After limit_us microseconds the wait gives up and
 * writes BSA_ERR_TIMEOUT to *status_dev; the kernel then returns normally and the
 * context stays usable. Read the result with bsa_check_status.
 *   status_dev : device int32, required
 *   limit_us   : 1 .. 10,000,000
 */
BSA_API bsa_status bsa_selftest_wait_timeout(int32_t* status_dev, uint32_t limit_us, bsa_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Host helpers (no device work).
 */
/* B = ceil(F P / b). */
BSA_API bsa_status bsa_num_blocks(const bsa_layout* layout, int32_t* num_blocks);
/* Bytes of the packed workspace of bsa_pack_qkv (0 for f32 layouts). */
BSA_API bsa_status bsa_workspace_size(const bsa_layout* layout, size_t* bytes);
/* k = floor(B (1 - rho) + 1e-9), rho in [0, 1]. */
BSA_API bsa_status bsa_k_from_rho(int32_t num_blocks, double rho, int32_t* k);
/* k = clamp(floor(B density + 1e-9), 1, B), density in [0, 1]. */
BSA_API bsa_status bsa_k_from_density(int32_t num_blocks, double density, int32_t* k);
/* Capped redistribution of the layer budget H (1 - rho) across heads in proportion to
 * positive scores (HeSS 提案手法): repeat d_h = (budget - cap #capped) s_h / sum of the
 * uncapped s, capping every head above `cap`, until no new head is capped.
 *   scores : host double [H] > 0;  density : host double [H] (output)
 *   needs H (1 - rho) <= H cap. */
BSA_API bsa_status bsa_head_budgets(const double* scores, int32_t heads, double rho, double cap,
                            double* density);
/* Waits for `stream`, reads *status_dev into the returned code and resets it to 0. */
BSA_API bsa_status bsa_check_status(int32_t* status_dev, bsa_stream_t stream);
BSA_API const char* bsa_status_string(bsa_status status);

#ifdef __cplusplus
}
#endif

#endif /* BSA_H */
