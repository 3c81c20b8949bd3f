/*
 * sparse_attn.h — C ABI of the block-sparse video attention library
 * (libsparse_attn.so, CUDA for sm_100a / B200).
 *
 * The library computes non-causal softmax attention over the 3D
 * (frame x height x width) token grid of a video diffusion transformer, where
 * only selected (q-block, k-block) tiles are executed.  Entry points:
 *   sa_build_mask           mean-pooled block scores -> tau-mass mask (per row
 *                           or per head) or PSA level map
 *   sa_build_mask_noalloc   the same without a caller workspace
 *   sa_radial_mask          static radial mask (window halves as frame
 *                           distance doubles)
 *   sa_pyramid_pool         PSA pyramid: mean-pooled K/V at 2, 4 and 8 tokens
 *   sa_sparse_attn_fwd      FlashAttention-style forward over kept tiles, with
 *                           the LiteAttention skip-mask update fused in
 *   sa_sparse_attn_fwd_host the same with Q/K/V/O in host memory, streamed
 *   sa_pyramid_attn_fwd     PSA multi-level attention over a level map
 *   sa_sparse_attn_bwd      gradients of sa_sparse_attn_fwd for Q, K and V
 *   sa_token_permute        PARO axis orders / VMoBA cell partitions of the grid
 *   sa_get_device_status    read and clear the device error word
 *   sa_self_test_timeout    make one bounded wait run out on purpose
 *
 * Conventions shared by every entry point
 *   - Tensors are caller-owned DEVICE memory.  Q, K, V and O are bf16,
 *     contiguous [B, H, N, d] (d fastest), tokens in raster (t, h, w) order:
 *     n = (t*Hh + h)*Ww + w.  Base pointers must be 16-byte aligned.
 *   - Blocks are runs of `block` consecutive tokens; Nb = ceil(N / block).
 *     The last block may be partial; means, maxima and softmax use its valid
 *     tokens only.
 *   - Block masks are uint8 [B, H, Nb, Nb] (q-block i, k-block j; j fastest).
 *   - Every call is asynchronous on `stream` (a cudaStream_t, NULL = legacy
 *     default stream).  Arguments are validated on the host before any launch;
 *     a rejected call launches nothing and returns SA_ERR_INVALID_ARG or
 *     SA_ERR_UNSUPPORTED.  No call falls back to another implementation.
 *   - Device-side waits are bounded.  A wait that runs out records
 *     SA_ERR_TIMEOUT in a per-device error word that sa_get_device_status
 *     reads; the kernel then returns without hanging the GPU.
 *   - The library allocates no device memory at run time.  Scratch memory
 *     is passed in by the caller (the workspace arguments); the one
 *     exception, sa_build_mask_noalloc, uses a static device array.
 *     sa_sparse_attn_fwd_host creates and destroys its own copy streams and
 *     events inside the call.
 *   - Every device entry point only launches kernels on `stream` (no copy,
 *     allocation or synchronisation), so it can be captured in a CUDA graph
 *     (after one eager call on the device, which sets kernel attributes).
 *     sa_build_mask launches its scores and selection kernels with
 *     programmatic stream serialization: each may start while the kernel
 *     before it finishes, and waits for that kernel's results on the device.
 *
 * Citations name the web page the operation comes from and its section.
 */
#ifndef SPARSE_ATTN_H
#define SPARSE_ATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SA_API __attribute__((visibility("default")))
#else
#define SA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SA_OK = 0,
  SA_ERR_INVALID_ARG = 1,   /* bad pointer, alignment, size or value        */
  SA_ERR_UNSUPPORTED = 2,   /* valid but not built (e.g. d not in {64,128}) */
  SA_ERR_CUDA = 3,          /* a CUDA runtime call failed                   */
  SA_ERR_TIMEOUT = 4        /* a device-side bounded wait ran out           */
} sa_status;

/* Order in which sa_sparse_attn_fwd visits the kept k-blocks of a q-block
 * (it decides only the skip update; the output is the same up to rounding). */
typedef enum {
  SA_ORDER_ASCENDING = 0,   /* ascending j                                   */
  SA_ORDER_RADIAL = 1       /* radial-centric, see sa_sparse_attn_fwd         */
} sa_visit_order;

enum { SA_MASK_TAU = 0, SA_MASK_LEVELS = 1, SA_MASK_GLOBAL = 2 };

/* Human-readable name of a status code (static string, never NULL). */
SA_API const char* sa_status_string(sa_status s);

/* Library version, major*10000 + minor*100 + patch. */
SA_API int sa_version(void);

/*
 * sa_get_device_status — synchronise `stream`, then read and clear the
 * current device's error word.  Returns SA_OK, SA_ERR_TIMEOUT (a kernel's
 * bounded wait ran out; its outputs are undefined) or SA_ERR_CUDA (the
 * synchronisation itself failed).
 */
SA_API sa_status sa_get_device_status(void* stream);

/*
 * sa_self_test_timeout — exercise the failure-detection path on purpose.
 *   No page counterpart: the pages describe no error handling.  This entry
 *   point lets a caller (or a test) check, without faulting or hanging the
 *   GPU, that a device-side wait which runs out is reported.
 *
 * Launches one CTA on `stream` whose single thread waits, through the same
 * bounded mbarrier wait the kernels use, on an mbarrier that nothing arrives
 * on.  The wait gives up after wait_ns nanoseconds of the global timer (plus
 * at most 0.1 ms), records SA_ERR_TIMEOUT in the device error word and the
 * kernel returns; no copy or MMA is left in flight.  The next
 * sa_get_device_status on the device returns SA_ERR_TIMEOUT and clears the
 * word, after which the library works as before.
 *   wait_ns   1 .. 1,000,000,000 (1 s); anything else is SA_ERR_INVALID_ARG.
 * Returns SA_OK once the kernel is queued.
 */
SA_API sa_status sa_self_test_timeout(uint64_t wait_ns, void* stream);

/*
 * sa_build_mask_workspace — bytes of device scratch sa_build_mask needs:
 * the block means of Q and K, each as two fp32 arrays (tf32 high and low
 * parts for the tensor-core scores: 4 * B*H*Nb*d floats), plus the fp32 block
 * scores (B*H*Nb*Nb floats).  The caller allocates it (any 256-byte aligned
 * buffer of at least this size).
 */
SA_API size_t sa_build_mask_workspace(int B, int H, int N, int d, int block);

/*
 * sa_build_mask — dynamic block mask from mean-pooled block scores.
 *   VMoBA write-up (arXiv 2506.23858), "threshold dynamic selection" and
 *   "global block selection" paragraphs: block importance from pooled
 *   query/key blocks scored with one matrix product, blocks kept until the
 *   selected attention mass reaches a threshold; PSA page (arXiv 2512.04025),
 *   multi-level mask generator paragraph, for SA_MASK_LEVELS.
 *
 * Computes q_i = mean of Q rows in block i, k_j likewise (fp32), the score
 * S_ij = q_i . k_j / sqrt(d) (on tensor cores as three tf32 passes of a
 * high / low split of the means: within about 2e-5 of each score's magnitude,
 * close to an fp32 dot product), then per row (b, h, i):
 *   SA_MASK_TAU:    P_i = softmax_j(S_i); visit j by descending S (ties: lower
 *                   j first); mask[j] = 1 iff the mass of the blocks visited
 *                   before j is < tau (the block that crosses tau is kept).
 *   SA_MASK_GLOBAL: P as for SA_MASK_TAU, but the pairs of a head compete
 *                   with each other (VMoBA's global selection; the threshold
 *                   then adapts the count to the head's concentration):
 *                   visit all (i, j) of the head by descending P_ij (ties:
 *                   lower i * Nb + j first); mask[i][j] = 1 iff the mass
 *                   visited before it is < tau * Nb.  A row may keep nothing.
 *   SA_MASK_LEVELS: rank r_j of S_ij in the same order; with quotas
 *                   c_l = ceil(level_frac[l] * Nb) (cumulative fractions,
 *                   non-decreasing; a product within 1e-3 above an integer
 *                   counts as that integer, so that 0.1f * 1000 gives 100
 *                   although 0.1f is slightly above 0.1), code = 1 if
 *                   r < c_0, 2 if r < c_1, 3 if r < c_2, else 4 (code =
 *                   pyramid level + 1).
 * Arguments
 *   q, k        bf16 [B,H,N,d] device, read only.
 *   tau         (0, 1]; used for SA_MASK_TAU and SA_MASK_GLOBAL.
 *   level_frac  HOST pointer to 3 floats in [0,1]; used for SA_MASK_LEVELS.
 *   mask_out    uint8 [B,H,Nb,Nb] device, written in full.
 *   scores_out  optional fp32 [B,H,Nb,Nb] device, 16-byte aligned (NULL:
 *               kept in workspace).
 *   workspace   device scratch of sa_build_mask_workspace() bytes.
 * Limits: d in {64,128}, block in {64,128}, Nb <= 4096.
 */
SA_API sa_status sa_build_mask(const void* q, const void* k, int B, int H, int N, int d, int block,
                        int mode, float tau, const float* level_frac,
                        uint8_t* mask_out, float* scores_out,
                        void* workspace, size_t workspace_bytes, void* stream);

/*
 * sa_build_mask_noalloc — sa_build_mask without a caller-provided workspace.
 *   The pages have no counterpart to this entry point.  It serves callers
 *   that cannot allocate device memory when they need a mask: serving
 *   runtimes that reserve all device memory up front in their own pool and
 *   do not let a library allocate beside it, and latency-critical loops that
 *   cannot afford cudaMalloc / cudaFree (they can synchronise the device).
 *
 * Same arguments, computation and results as sa_build_mask, minus the
 * workspace.  The scratch comes from one static device array of 32 MiB
 * (33,554,432 bytes) that every GPU loading this library holds until the
 * process exits.  Rules:
 *   - Size limit: sizes whose sa_build_mask_workspace(B, H, N, d, block)
 *     exceeds 32 MiB are rejected with SA_ERR_UNSUPPORTED before any launch
 *     (the other arguments are checked first, with sa_build_mask's codes).
 *   - Set-up: the first call on a device, with that device current, looks up
 *     the array's device address (cudaGetSymbolAddress) and keeps it; a
 *     lookup that fails returns SA_ERR_CUDA and is tried again on the next
 *     call.  Make that first call before any stream capture.
 *   - Sharing: all calls on a device share the one array, and it keeps the
 *     previous call's contents.  What has to start at zero (the histograms
 *     and search state of SA_MASK_GLOBAL) is cleared by each call itself;
 *     every other byte it reads was written earlier in the same call.  Calls
 *     whose kernels overlap on the GPU (different streams, no ordering
 *     between them) race on the array and give wrong masks: serialise them.
 *   - No memory is allocated or freed by this call.
 */
SA_API sa_status sa_build_mask_noalloc(const void* q, const void* k, int B, int H, int N, int d, int block,
                                       int mode, float tau, const float* level_frac,
                                       uint8_t* mask_out, float* scores_out, void* stream);

/*
 * sa_radial_mask — static radial mask for a T x Hh x Ww grid.
 *   "MIT实验室推出Radial Attention" (arXiv 2506.19852), spatio-temporal energy
 *   decay and static-mask paragraphs: attention concentrates on nearby frames,
 *   the spatial window shrinks exponentially with temporal distance, and the
 *   mask is precomputed once (O(n log n) kept pairs).
 *
 * Block i's frame f_i and in-frame block position p_i are those of its first
 * token (f = floor(i*block / F), p = floor((i*block mod F) / block),
 * F = Hh*Ww), S = ceil(F / block).  mask[i][j] = 1 iff |f_i - f_j| <= 1 or
 * |p_i - p_j| < S / 2^floor(log2 |f_i - f_j|).
 *   mask_out  uint8 [Nb, Nb] device (broadcast over B and H by passing
 *             batch/head strides of 0 to sa_sparse_attn_fwd).
 */
SA_API sa_status sa_radial_mask(int T, int Hh, int Ww, int block, uint8_t* mask_out, void* stream);

/*
 * sa_pyramid_pool — PSA pyramid KV construction.
 *   PSA page ("浙江大学突破视频AI瓶颈:金字塔方法提升视频AI效率10倍",
 *   arXiv 2512.04025), pyramid KV paragraph: the bottom level keeps the
 *   original keys/values, each level up is an average pooling of the one below.
 *
 * For c in {2, 4, 8} (level 1, 2, 3): pooled[g] = mean of rows c*g ..
 * min(N, c*g+c)-1 (fp32 sum of the bf16 inputs, rounded to bf16).  Groups
 * never cross a block edge because block is a multiple of 8.
 *   k, v            bf16 [B,H,N,d] device, read only.
 *   k_pool, v_pool  HOST arrays of 3 device pointers, each bf16
 *                   [B,H,ceil(N/c),d] for c = 2, 4, 8.
 */
SA_API sa_status sa_pyramid_pool(const void* k, const void* v, int B, int H, int N, int d, int block,
                          void* const* k_pool, void* const* v_pool, void* stream);

/*
 * sa_sparse_attn_fwd — block-sparse attention forward with the LiteAttention
 * skip update.
 *   Block-sparse keep/drop attention: PSA page, block-sparse attention
 *   paragraph.  Skip rule and persistent skip mask: LiteAttention write-up
 *   (arXiv 2511.11062), sections 3 (full-iteration skips), 5 (skip condition)
 *   and 6 (persistent tile-level skip mask; producer loads only non-skipped
 *   tiles; per-warp recording with the cross-warp reduction at kernel end).
 *
 * For each row r of q-block i:  O_r = sum_c softmax(s_rc) v_c over the key
 * columns c of every k-block j with mask[b,h,i,j] != 0 and skip_in[b,h,i,j]
 * == 0, where s_rc = scale * q_r . k_c.  LSE_r = ln sum_c exp(s_rc).  A row
 * with no visited block gets O = 0 and LSE = -inf.
 * Skip update (only when skip_out != NULL): visited k-blocks are taken in
 * the visit order; block j (not the first visited) gets skip_out = 1 iff
 * max_c s_rc over block j < (running max of row r over the blocks visited
 * before j) - eps for every valid row r of the q-block.  Block j still
 * contributes to this call's O.  Every other byte of the row is written as
 * skip_in's byte (0 when skip_in is NULL), so skip_out = skip_in | new bits;
 * skip_out may alias skip_in.
 * Arguments
 *   q, k, v       bf16 [B,H,N,d] device.
 *   mask          uint8 device, element (b,h,i,j) at b*mask_sb + h*mask_sh +
 *                 i*mask_si + j; strides of 0 broadcast (e.g. a radial mask
 *                 [Nb,Nb]: 0, 0, Nb).  NULL keeps every block.  Any nonzero
 *                 byte keeps the block at full resolution.
 *   skip_in       NULL or uint8 [B,H,Nb,Nb] device.
 *   skip_out      NULL or uint8 [B,H,Nb,Nb] device (may equal skip_in).
 *   eps           skip threshold in natural-log logit units (>= 0; +inf
 *                 never skips).
 *   scale         logit scale; 0 selects 1/sqrt(d).
 *   order         SA_ORDER_ASCENDING, or SA_ORDER_RADIAL: the radial-centric
 *                 ordering of the LiteAttention write-up (section 5; section
 *                 10 expects 10-20 % more skips from it), read as follows.
 *                 Keys are cut into tiles of 128, query rows into bands of
 *                 256; the k-blocks of q-block i are visited by ascending
 *                 distance of their tile from the two diagonal tiles of the
 *                 band holding row i*block (distance 0 for both), ties by
 *                 ascending tile, ascending j inside a tile.  Any other
 *                 value is SA_ERR_INVALID_ARG.
 *   causal        0, or 1: key c is visible to row r only if c <= r (token
 *                 index in the sequence as given).  The PSA page notes the
 *                 method serves causal video generation as well as
 *                 bidirectional understanding; read as: the effective mask
 *                 is mask AND (j <= i), and inside the diagonal block the
 *                 key must not come after the row.  Blocks j > i are neither
 *                 visited nor tested; their skip_out bytes copy skip_in.
 *   o             bf16 [B,H,N,d] device, written for every valid row.
 *   lse           NULL or fp32 [B,H,N] device.
 * Limits: d in {64,128}, block in {64,128}, ceil(N/128) <= 4096, B*H <= 65535.
 */
SA_API sa_status sa_sparse_attn_fwd(const void* q, const void* k, const void* v,
                             int B, int H, int N, int d, int block,
                             const uint8_t* mask, int64_t mask_sb, int64_t mask_sh, int64_t mask_si,
                             const uint8_t* skip_in, uint8_t* skip_out, float eps, float scale, int order,
                             int causal, void* o, float* lse, void* stream);

/*
 * sa_pyramid_attn_fwd — PSA multi-level attention forward.
 *   PSA page, adaptive pyramid attention paragraph (pooled keys weighted so
 *   that the probability distribution stays consistent) and decoupled
 *   block-tile kernel paragraph (logical block size independent of the
 *   hardware tile).
 *
 * levels is a uint8 [B,H,Nb,Nb] code map (strides as for `mask`): 0 drops
 * k-block j, 1 attends to its original keys, 2/3/4 attend to its keys pooled
 * by c = 2/4/8 (k_pool/v_pool from sa_pyramid_pool).  A pooled key of a group
 * holding n tokens gets logit scale * q . k_pooled + ln(n).
 *   k_pool, v_pool  HOST arrays of 3 device pointers (c = 2, 4, 8).
 *   causal          0, or 1 (PSA page: the method serves causal generation
 *                   too).  Read as: k-blocks j > i are dropped; block i itself,
 *                   if kept, is attended at level 0 (pooled keys of that block
 *                   would mix in later tokens) with key c visible to row r
 *                   only if c <= r; blocks j < i keep their codes.
 * Limits: as sa_sparse_attn_fwd, block == 64 or 128.
 */
SA_API sa_status sa_pyramid_attn_fwd(const void* q, const void* k, const void* v,
                              int B, int H, int N, int d, int block,
                              const uint8_t* levels, int64_t lv_sb, int64_t lv_sh, int64_t lv_si,
                              const void* const* k_pool, const void* const* v_pool,
                              float scale, int causal, void* o, float* lse, void* stream);

/*
 * sa_sparse_attn_bwd — gradients of sa_sparse_attn_fwd with respect to Q, K, V.
 *   Needed by the LoRA length extension of the Radial Attention write-up
 *   ("MIT实验室推出Radial Attention", arXiv 2506.19852, training-cost
 *   paragraph), which trains through the sparse attention.  The formulas are
 *   the derivative of the forward's definition; no page states them:
 *     P_rc = exp(s_rc - LSE_r) on the kept columns of row r (0 elsewhere),
 *     D_r  = dO_r . O_r,
 *     dV_c = sum_r P_rc dO_r,
 *     dS   = P * (dO V^T - D),
 *     dQ_r = scale sum_c dS_rc k_c,   dK_c = scale sum_r dS_rc q_r.
 * Arguments
 *   q, k, v       bf16 [B,H,N,d] device, the forward's inputs.
 *   o, lse        the forward's outputs for the same q, k, v, mask and scale
 *                 (bf16 [B,H,N,d]; fp32 [B,H,N], natural log).  A row with no
 *                 kept block (LSE = -inf) gets dQ = 0.
 *   dout          bf16 [B,H,N,d] device, the gradient of the loss w.r.t. O.
 *   mask, mask_s* as sa_sparse_attn_fwd (NULL keeps every block; any nonzero
 *                 byte keeps).  Pass the forward's effective mask (mask AND
 *                 NOT skip_in when the forward skipped blocks).
 *   scale         logit scale; 0 selects 1/sqrt(d).
 *   causal        as sa_sparse_attn_fwd (use the forward's value).
 *   dq, dk, dv    bf16 [B,H,N,d] device, written for every valid row (zero
 *                 where the row or key takes part in no kept block).
 *   workspace     device scratch of at least sa_sparse_attn_bwd_workspace()
 *                 bytes (16-byte aligned): holds D_r as fp32 [B,H,N].
 * Deterministic: no atomics; dK/dV and dQ come from separate passes.
 * Limits: as sa_sparse_attn_fwd.
 */
SA_API size_t sa_sparse_attn_bwd_workspace(int B, int H, int N);
SA_API sa_status sa_sparse_attn_bwd(const void* q, const void* k, const void* v, const void* o,
                             const void* dout, const float* lse, int B, int H, int N, int d, int block,
                             const uint8_t* mask, int64_t mask_sb, int64_t mask_sh, int64_t mask_si,
                             float scale, int causal, void* dq, void* dk, void* dv, void* workspace,
                             size_t workspace_bytes, void* stream);

/*
 * sa_sparse_attn_fwd_host — sa_sparse_attn_fwd with Q, K, V and O in HOST memory.
 *   No page counterpart: the pages run attention inside a model on the GPU.
 *   This entry point serves callers whose tensors live in host memory; it
 *   streams the (b, h) rows through the device so the transfers overlap the
 *   attention.
 *
 * q, k, v, o are HOST bf16 [B,H,N,d] (page-locked memory makes the copies
 * asynchronous; pageable memory works but serialises them).  Every other
 * argument is as sa_sparse_attn_fwd (mask, skip_in, skip_out, lse: device).
 * The heads go through the device in chunks of heads_per_chunk heads of one
 * batch entry, two chunk buffers in turn: the copies in of chunk c + 1, the
 * attention of chunk c (on `stream`) and the copy out of chunk c - 1 run
 * concurrently (the copies on two streams this call creates and releases).
 * Work queued on `stream` before the call completes before the first copy;
 * work queued after it starts after the last copy out.  Each chunk gives the
 * same results as one sa_sparse_attn_fwd call over all heads.
 *   workspace     device scratch of sa_sparse_attn_fwd_host_workspace(N, d,
 *                 min(heads_per_chunk, H)) bytes, 16-byte aligned.
 * Returns the first error; a call that fails part way may have written some
 * chunks.
 */
SA_API size_t sa_sparse_attn_fwd_host_workspace(int N, int d, int heads_per_chunk);
SA_API sa_status sa_sparse_attn_fwd_host(const void* q, const void* k, const void* v,
                                  int B, int H, int N, int d, int block,
                                  const uint8_t* mask, int64_t mask_sb, int64_t mask_sh, int64_t mask_si,
                                  const uint8_t* skip_in, uint8_t* skip_out, float eps, float scale,
                                  int order, int causal, void* o, float* lse, void* workspace,
                                  size_t workspace_bytes, int heads_per_chunk, void* stream);

/*
 * sa_token_permute — reorder the tokens of the (t, h, w) grid, per head.
 *   PAROAttention write-up (pattern-aware reordering paragraphs: 6 orders of
 *   the three axes, one chosen per head, so that scattered attention becomes
 *   blocks) and VMoBA write-up (layer-wise recurrent 1D / 2D / 3D block
 *   partition of the video into temporal, spatial and spatio-temporal cells).
 *
 * Tokens are ordered by (cell coordinates, coordinates inside the cell), both
 * tuples in the head's axis order, slowest axis first.  Axis order codes:
 * 0 t,h,w (raster)  1 t,w,h  2 h,t,w  3 h,w,t  4 w,t,h  5 w,h,t.  Cells are
 * ct x ch x cw and must divide the grid; 1 x 1 x 1 cells give the pure axis
 * orders, order 0 with cells (ct, Hh, Ww) / (T, ch, cw) / (ct, ch, cw) the 1D
 * / 2D / 3D partitions.  The blocks of the attention calls are then runs of
 * `block` consecutive tokens of the permuted sequence.
 * Arguments
 *   src, dst      HOST arrays of n_tensors (1..4) device pointers, each bf16
 *                 [B,H,N,d], N = T*Hh*Ww, 16-byte aligned; dst[i] != src[i].
 *   order         axis order code of every head when head_order is NULL.
 *   head_order    NULL, or uint8 [H] device array of per-head codes (0..5).
 *   inverse       0: dst holds the permuted sequence of src (raster order);
 *                 1: src is permuted, dst gets raster order back.
 * Limits: d in {64,128}, N <= 2^30, B*H <= 65535.  Invalid codes in head_order are not
 * checked on the device; they read as code 5.
 */
SA_API sa_status sa_token_permute(const void* const* src, void* const* dst, int n_tensors, int B, int H,
                           int T, int Hh, int Ww, int d, int order, const uint8_t* head_order,
                           int ct, int ch, int cw, int inverse, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SPARSE_ATTN_H */
