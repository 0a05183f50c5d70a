/*
 * rettention.h -- C ABI of the B200 (sm_100a) Re-ttention attention library.
 *
 * Re-ttention ("Re-ttention: Ultra Sparse Visual Generation via Attention
 * Statistical Reshape", project page) keeps only a few percent of the keys in
 * each DiT attention step and corrects the sparse result with statistics
 * cached at an earlier full-attention denoising step: the ratio between the
 * full and the sparse softmax denominators, and the residual contribution of
 * the masked-out tokens (project page, teaser and mechanism highlight).
 *
 * Three calls make up one attention layer's denoising cycle:
 *   rt_build_block_mask     which key blocks each query block keeps;
 *   rt_attn_full_capture    full attention at a capture step, plus the cache;
 *   rt_attn_sparse_reshape  block-sparse attention reshaped with the cache.
 * A fourth, rt_pair_query_blocks, only schedules: it groups query blocks
 * into the sparse kernel's 128-row tiles so that a tile's blocks keep mostly
 * the same key blocks, which makes the sparse step faster without changing
 * its result.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Q, K, V and the attention output are bf16 tensors [B, H, N, D],
 *    contiguous, in device memory.  Only the first d = head_dim columns carry
 *    data; columns d..D-1 (D = head_dim_padded) must be zero on input and are
 *    written as zero on output.  The softmax scale is passed by the caller
 *    (normally 1/sqrt(d)).
 *  - Tokens are grouped into blocks of block_size tokens, for queries and
 *    keys alike; n_blocks = ceil(N / block_size) and the last block may be
 *    short (ragged tail).
 *  - The kept-block list is a CSR over the B*H*n_blocks query blocks
 *    (row index (b*H + h)*n_blocks + query_block): row_ptr int32
 *    [B*H*n_blocks + 1] holds global offsets into col_idx, col_idx int32 holds
 *    head-local key-block indices, each row sorted ascending without
 *    duplicates.
 *  - Statistics are fp32: stat_m, stat_zfull, stat_zkept [B, H, N] and
 *    stat_u [B, H, N, D] (columns d..D-1 zero).
 *  - Every pointer argument except the shape is device memory, 16-byte
 *    aligned, owned by the caller and never freed or retained by the library.
 *    Calls are asynchronous on `stream` (NULL = the legacy default stream);
 *    nothing is synchronised.
 *  - Supported: head_dim_padded in {64, 80, 128}, 1 <= head_dim <= head_dim_padded,
 *    block_size in {64, 128}, n_blocks <= 2048.
 *
 * Errors
 * ------
 * Arguments are validated on the host before any CUDA call: a null pointer,
 * a negative or zero size, a bad keep count or a misaligned pointer gives
 * RT_ERR_INVALID_ARGUMENT, a head dim or block size outside the supported set
 * gives RT_ERR_UNSUPPORTED, and nothing is launched.  A failed launch gives
 * RT_ERR_CUDA.  Kernels never trap: every wait inside a kernel is bounded;
 * when one runs out the kernel records RT_ERR_TIMEOUT in a device status word
 * (read it with rt_take_device_error), leaves its outputs unspecified and
 * returns.  The CSR must be readable where row_ptr points: row_ptr holds
 * B*H*n_blocks + 1 entries and 0 <= row_ptr[r] <= row_ptr[r+1] <= the length
 * of col_idx (the library cannot see that length).  Beyond that, malformed
 * contents (block indices out of range, unsorted or repeated entries, rows
 * longer than n_blocks) never make a kernel read or write out of bounds;
 * their results are unspecified.
 */
#ifndef RETTENTION_H
#define RETTENTION_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define RT_ABI_VERSION 7

typedef enum rt_status {
    RT_OK = 0,
    RT_ERR_INVALID_ARGUMENT = 1,
    RT_ERR_UNSUPPORTED = 2,
    RT_ERR_CUDA = 3,
    RT_ERR_TIMEOUT = 4
} rt_status;

/* Same type as cudaStream_t, spelled without the CUDA headers. */
typedef struct CUstream_st *rt_stream_t;

/* Problem shape, passed by host pointer. */
typedef struct rt_shape {
    int32_t batch;            /* B */
    int32_t heads;            /* H */
    int32_t seq_len;          /* N tokens */
    int32_t head_dim;         /* d: logical head dim */
    int32_t head_dim_padded;  /* D: stored head dim, >= d */
    int32_t block_size;       /* tokens per query block and per key block */
} rt_shape;

/*
 * rt_build_block_mask -- choose the key blocks each query block keeps.
 *
 * The project page's Abstract has the sparse step attend to a small subset of
 * the tokens, down to 3.1% of them; it does not say how the subset is chosen.
 * This call uses block mean pooling and a per-query-block top-k:
 *   pooled_q[b,h,qb] = mean of q over the real tokens of query block qb
 *                      (logical columns only); pooled_k likewise;
 *   score[qb,kb]     = scale * <pooled_q[qb], pooled_k[kb]>;
 *   kept(qb)         = every key block overlapping tokens [0, forced_prefix_tokens)
 *                      plus the keep_blocks - |forced| other blocks with the
 *                      largest score (equal scores: lower block index first),
 *                      written sorted ascending.
 *
 * q, k          bf16 [B,H,N,D] device.
 * scale         softmax scale used for the block scores.
 * keep_blocks   kept key blocks per query block, 1..n_blocks, and at least
 *               the number of forced blocks.
 * forced_prefix_tokens  >= 0; 0 forces nothing.
 * row_ptr       out, int32 [B*H*n_blocks + 1] device; row r starts at r*keep_blocks.
 * col_idx       out, int32 [B*H*n_blocks*keep_blocks] device.
 * block_scores  optional out (may be NULL), fp32 [B,H,n_blocks,n_blocks] device:
 *               the scores the selection used.
 * Takes a transient device workspace of 2*B*H*n_blocks*D*4 bytes (the pooled
 * block means) on `stream` and returns it on the same stream.  Transient
 * workspaces come from a stream-ordered memory pool the library creates once
 * per device; it keeps freed memory cached for later calls.
 */
rt_status rt_build_block_mask(const rt_shape *shape, const void *q, const void *k, float scale,
                              int32_t keep_blocks, int32_t forced_prefix_tokens,
                              int32_t *row_ptr, int32_t *col_idx, float *block_scores,
                              rt_stream_t stream);

/*
 * rt_attn_full_capture -- full attention at a capture step, and the cache.
 *
 * The teaser corrects sparse attention with statistics kept from an earlier
 * denoising step; the mechanism highlight names the cached quantities: the
 * ratio of the two softmax denominators (sparse over full), which stays
 * nearly constant across steps, and what the masked keys add to the output.
 * For every query row i, with s_ij = scale * q_i . k_j over all keys j < N and
 * K(i) the keys of the blocks that i's query block keeps:
 *   m_i      = max_j s_ij                  (the cache's reference, see below)
 *   Z_full_i = sum_j exp(s_ij - m_i)
 *   Z_kept_i = sum_{j in K(i)} exp(s_ij - m_i)
 *   U_i      = sum_{j not in K(i)} exp(s_ij - m_i) * v_j
 *   out_i    = sum_j exp(s_ij - m_i) * v_j / Z_full_i       (full attention, bf16)
 *
 * m_i is the reference the three cached sums share, and the reshape does not
 * depend on it.  It is the row max, except on a row whose kept keys carry less
 * than 2^-64 of the mass at the max (a masked key far above every kept one):
 * there Z_kept_i would leave fp32's range, and m_i is lowered by the integer
 * number of binades that balances the exponents of Z_kept_i and Z_full_i (by
 * at most 100 binades).  A kept part below ~2^-226 of the mass at the max
 * still reads Z_kept_i = 0; the sparse step then takes that row's kept mass as
 * unchanged since the capture (see rt_attn_sparse_reshape).  Ratios such as
 * Z_full/Z_kept, m + log Z_full and U/Z_full are what to compare across
 * implementations.
 *
 * The P V products take the probabilities in f16 with an f16 copy of V, made
 * by the call in a device workspace of B*H*N*D*2 + B*H*4 bytes (see
 * rt_workspace_bytes).  The kept and the masked keys of a row are summed as
 * two separate online softmaxes, each against a reference of its own, and p
 * enters f16 as p * 2^7 with p <= 2^8: every term of U down to 2^-21 of the
 * row's largest masked term keeps 11 mantissa bits (a relative error below
 * 2^-12, plus at most 7.5e-5 for the one exponential in eight computed on the
 * FMA pipe, see rt_selftest_exp2_poly), smaller ones an absolute error below
 * 2^-32 of that term, however far the row's maximum lies above its masked
 * scores.  The copy is scaled per
 * (batch, head) by the power of two that puts max |v| in [2^14, 2^15) and the
 * scale is taken out exactly afterwards, so any finite V keeps 11 mantissa
 * bits down to 2^-30 of its head's largest |v|.
 *
 * q, k, v       bf16 [B,H,N,D] device.
 * row_ptr, col_idx  CSR of kept blocks (for example from rt_build_block_mask).
 * out           out, bf16 [B,H,N,D] device.
 * stat_m, stat_zfull, stat_zkept  out, fp32 [B,H,N] device.
 * stat_u        out, fp32 [B,H,N,D] device.
 * workspace     optional (may be NULL), device, 16-byte aligned, at least the
 *               capture size rt_workspace_bytes gives (workspace_bytes says
 *               how large it is; a smaller one is RT_ERR_INVALID_ARGUMENT).
 *               Used only while the call's work runs on `stream`.  NULL takes
 *               a transient buffer from the library's stream-ordered pool.
 */
rt_status rt_attn_full_capture(const rt_shape *shape, const void *q, const void *k, const void *v,
                               float scale, const int32_t *row_ptr, const int32_t *col_idx,
                               void *out, float *stat_m, float *stat_zfull, float *stat_zkept,
                               float *stat_u, void *workspace, size_t workspace_bytes,
                               rt_stream_t stream);

/*
 * rt_attn_sparse_reshape -- block-sparse attention with the statistical reshape.
 *
 * The Abstract reshapes the sparse attention scores using the softmax
 * statistics of an earlier step, to undo the shift in normalisation that a
 * softmax over part of the keys causes; the mechanism highlight reconstructs the full
 * distribution from the reused denominator ratio and the cached residual.
 * For every query row i, over the kept keys K(i) of the current Q, K, V:
 *   m'_i = max_{j in K(i)} s_ij,  Z'_i = sum_{K(i)} exp(s_ij - m'_i),
 *   N'_i = sum_{K(i)} exp(s_ij - m'_i) * v_j
 *   out_i = (N'_i + exp(m_i - m'_i) * U_i) / (Z'_i * Z_full_i / Z_kept_i)
 * with m, Z_full, Z_kept, U from the latest capture step (same CSR).  If all
 * four statistics pointers are NULL the call computes plain block-sparse
 * attention out_i = N'_i / Z'_i.  A row whose query block keeps no key block
 * gets out_i = 0.  The product is formed so that no intermediate leaves fp32's
 * range when the kept keys lie far below the cached reference (where
 * exp(m_i - m'_i) * U_i and Z_full_i / Z_kept_i can each exceed it); a row that
 * keeps keys but has a cached Z_kept_i of 0 (a kept mass below the capture's
 * range, see rt_attn_full_capture) gets out_i = U_i / Z_full_i, the reshape
 * with its kept mass taken as unchanged, exact when the inputs are.
 *
 * q, k, v       bf16 [B,H,N,D] device (the current step's inputs).
 * row_ptr, col_idx  the CSR used at the capture step.
 * tile_blocks   optional (may be NULL), int32 [B*H][n_tiles][2] device,
 *               n_tiles = ceil(N / 128): which query blocks the kernel computes
 *               together in each 128-row tile, as written by
 *               rt_pair_query_blocks (block size 64: two blocks per tile;
 *               block size 128: one, the second entry unused).  NULL means
 *               the neighbouring blocks (tile t = blocks 2t, 2t+1 at block
 *               size 64).  Every row's result is the same for any table in
 *               which each query block of a head appears exactly once (-1 or
 *               an out-of-range entry is an empty half); a block that appears
 *               in no tile leaves its output rows unwritten, one that appears
 *               twice is computed twice.
 * stat_*        fp32 statistics written by rt_attn_full_capture, or all NULL.
 * out           out, bf16 [B,H,N,D] device.
*/
rt_status rt_attn_sparse_reshape(const rt_shape *shape, const void *q, const void *k,
                                 const void *v, float scale, const int32_t *row_ptr,
                                 const int32_t *col_idx, const int32_t *tile_blocks,
                                 const float *stat_m, const float *stat_zfull,
                                 const float *stat_zkept, const float *stat_u, void *out,
                                 rt_stream_t stream);

/*
 * rt_attn_full_capture_u16, rt_attn_sparse_reshape_u16 -- the same two steps
 * with a compressed residual cache.
 *
 * The mechanism highlight caches the residual contribution of the masked-out
 * tokens; at a few per cent of kept keys that cache (U, D values per row) is
 * the largest stream the sparse step reads.  These variants store U as f16
 * with one power-of-two scale per row instead of fp32, which halves it:
 *   U_i = stat_u16_i * stat_u_scale_i,
 * where stat_u_scale_i = 2^-k is chosen so that the row's largest |U_i[c]|
 * times 2^k lies in [2^14, 2^15) (a row without masked keys gets scale 1 and
 * zeros).  Every element down to 2^-28 of its row's largest keeps 11 mantissa
 * bits (relative error below 2^-12, inside the 1e-3 statistics tolerance).
 * m, Z_full and Z_kept stay fp32.  Everything else -- arguments, layouts,
 * results, errors -- is as for rt_attn_full_capture and rt_attn_sparse_reshape.
 *
 * stat_u16      f16 bits [B,H,N,D] device (16-byte aligned; columns d..D-1 zero):
 *               written by the capture call, read by the sparse call.
 * stat_u_scale  fp32 [B,H,N] device: written / read likewise.
 * The sparse variant requires all five statistics pointers (plain block-sparse
 * attention is rt_attn_sparse_reshape with NULL statistics).
 */
rt_status rt_attn_full_capture_u16(const rt_shape *shape, const void *q, const void *k,
                                   const void *v, float scale, const int32_t *row_ptr,
                                   const int32_t *col_idx, void *out, float *stat_m,
                                   float *stat_zfull, float *stat_zkept, uint16_t *stat_u16,
                                   float *stat_u_scale, void *workspace, size_t workspace_bytes,
                                   rt_stream_t stream);
rt_status rt_attn_sparse_reshape_u16(const rt_shape *shape, const void *q, const void *k,
                                     const void *v, float scale, const int32_t *row_ptr,
                                     const int32_t *col_idx, const int32_t *tile_blocks,
                                     const float *stat_m, const float *stat_zfull,
                                     const float *stat_zkept, const uint16_t *stat_u16,
                                     const float *stat_u_scale, void *out, rt_stream_t stream);

/*
 * rt_build_block_mask_exact -- choose the kept key blocks by their exact
 * attention mass.
 *
 * The Abstract reshapes the sparse scores with the softmax distribution of an
 * earlier step; the capture step computes every score, so the mask can be
 * chosen from that distribution itself instead of from pooled block means.
 * For every query block qb and key block kb of a head:
 *   mass[qb,kb] = sum over the real query rows i of qb and keys j of kb of
 *                 exp(s_ij - m_i) / Z_full_i,   s_ij = scale * q_i . k_j
 * (the softmax probability the block's rows give the key block, over all N
 * keys), and kept(qb) is selected from these masses by the same rule as in
 * rt_build_block_mask: the forced prefix blocks, then the largest masses
 * (equal masses: lower block index first), sorted ascending.
 *
 * The call makes one full-attention pass over Q and K (the capture kernel
 * with no key block kept and no output stored: the cost of about one capture
 * step), which writes each row's per-64-key-tile log-sum-exp, then reduces
 * those to block masses and selects.  Use the CSR with rt_attn_full_capture
 * on the same Q, K, V to get the statistics for it.
 *
 * q, k, v       bf16 [B,H,N,D] device (v feeds the pass but not the masses).
 * keep_blocks, forced_prefix_tokens, row_ptr, col_idx  as for rt_build_block_mask.
 * block_mass    optional out (may be NULL), fp32 [B,H,n_blocks,n_blocks] device.
 * workspace     optional (may be NULL), device, 256-byte aligned, at least
 *               rt_exact_mask_workspace_bytes (about 4*B*H*N*(ceil(N/64) + 3)
 *               + 2*B*H*N*D bytes: 1.07 GB for B*H = 48, N = 17776, D = 64);
 *               NULL takes a transient buffer from the library's pool.
 */
rt_status rt_build_block_mask_exact(const rt_shape *shape, const void *q, const void *k,
                                    const void *v, float scale, int32_t keep_blocks,
                                    int32_t forced_prefix_tokens, int32_t *row_ptr,
                                    int32_t *col_idx, float *block_mass, void *workspace,
                                    size_t workspace_bytes, rt_stream_t stream);

/* Workspace size of rt_build_block_mask_exact for a shape (validates the shape). */
rt_status rt_exact_mask_workspace_bytes(const rt_shape *shape, size_t *bytes);

/*
 * rt_hilbert_order, rt_permute_tokens -- Hilbert-curve token order.
 *
 * HilbertA blog page, "Introducing HilbertA", first component (Reordering):
 * tokens are put in the order of a Hilbert curve over the patch grid, so
 * tokens that are close on the grid stay close in the sequence.  Run the
 * attention path on Q, K, V permuted this way and map the output back with
 * the inverse: a 64-token block of a 64 x 64 image grid is then an 8 x 8 patch
 * square instead of one patch row, so the block mask pools and keeps
 * spatially coherent blocks.  The results of every call are those of the same
 * calls on the permuted tensors (attention commutes with a common permutation
 * of its tokens); the cached statistics stay in the permuted order.
 *
 * rt_hilbert_order (host only, no CUDA call) writes perm[t], int32, for
 * t < prefix_tokens + frames*grid_h*grid_w: position t of the reordered
 * sequence takes token perm[t] of the row-major one, where cell (x, y) of
 * frame f is token prefix_tokens + f*grid_h*grid_w + y*grid_w + x.  The
 * prefix tokens (text) keep their places; each frame's cells follow the
 * Hilbert curve of the smallest power-of-two square holding the grid
 * (starting at (0, 0), ending at (2^k - 1, 0)), the square's cells outside
 * the grid skipped.  grid sides up to 32768.  perm: host memory.
 *
 * rt_permute_tokens copies a bf16 [B,H,N,D] tensor: inverse = 0 gathers
 * dst[b,h,t] = src[b,h,perm[t]], inverse != 0 scatters dst[b,h,perm[t]] =
 * src[b,h,t].  perm: int32 [N] device, a permutation of 0..N-1 (entries
 * outside [0, N) are skipped; a gather writes that row as zeros).  src and
 * dst are distinct, 16-byte aligned device buffers.  HBM-bound: one read and
 * one write of the tensor.
 */
rt_status rt_hilbert_order(int32_t prefix_tokens, int32_t frames, int32_t grid_h, int32_t grid_w,
                           int32_t *perm);
rt_status rt_permute_tokens(const rt_shape *shape, const void *src, const int32_t *perm,
                            int32_t inverse, void *dst, rt_stream_t stream);

/*
 * rt_pair_query_blocks -- group the query blocks of each head into the
 * sparse kernel's 128-row tiles.
 *
 * Not part of the method (the pages describe no kernel): a schedule for
 * rt_attn_sparse_reshape.  A 128-row tile is computed against the union of
 * its query blocks' kept key blocks, so at block size 64 a key block kept by
 * only one of the two costs the other a wasted step.  This call pairs blocks
 * that keep many of the same key blocks, deterministically:
 *   1. for each query block i, its 8 best partners j with |i - j| <= 224 in
 *      the order (overlap desc, |i - j| asc, j asc), where overlap is the
 *      number of key blocks both rows keep (entries outside [0, n_blocks)
 *      ignored, a row cut to its first n_blocks entries);
 *   2. 8 rounds in which every unpaired block picks its first unpaired
 *      candidate and two blocks that pick each other become a pair;
 *   3. tiles: the pairs in order of their lower block, then the unpaired
 *      blocks two by two in ascending order (-1 for an odd last half).
 * At block size 128 a tile is one block: tile t = (t, -1).  Compute it once
 * per mask (at the capture step) and pass it to every sparse step that uses
 * that mask.
 *
 * row_ptr, col_idx  the CSR (as for rt_attn_sparse_reshape).
 * tile_blocks   out, int32 [B*H][ceil(N / 128)][2] device.
 * workspace     optional (may be NULL), device, 16-byte aligned: at block size
 *               64 the candidates of step 1 need B*H*n_blocks*16 bytes (the
 *               pairing size rt_workspace_bytes gives; a smaller workspace is
 *               RT_ERR_INVALID_ARGUMENT).  NULL takes a transient buffer from
 *               the library's stream-ordered pool.
 * Malformed CSR contents give a valid table of unspecified quality.
 */
rt_status rt_pair_query_blocks(const rt_shape *shape, const int32_t *row_ptr,
                               const int32_t *col_idx, int32_t *tile_blocks, void *workspace,
                               size_t workspace_bytes, rt_stream_t stream);

/*
 * rt_workspace_bytes -- device workspace sizes for a shape.
 *
 * *capture_bytes (if not NULL) receives what rt_attn_full_capture needs,
 * *pairing_bytes (if not NULL) what rt_pair_query_blocks needs (0 at block
 * size 128).  With these passed in, rt_build_block_mask_static,
 * rt_pair_query_blocks, rt_attn_full_capture and rt_attn_sparse_reshape run a
 * whole denoising cycle without the library allocating device memory.
 * Validates the shape like the other calls; launches nothing.
 */
rt_status rt_workspace_bytes(const rt_shape *shape, size_t *capture_bytes, size_t *pairing_bytes);

/* Human-readable name of a status code (static string, never NULL). */
const char *rt_status_string(rt_status status);

/* RT_ABI_VERSION of the loaded library. */
int32_t rt_abi_version(void);

/*
 * rt_take_device_error -- read and clear the device status word of the
 * current CUDA device.  Waits for all work on the device to finish first.
 * *code receives RT_OK or the first error a kernel recorded (RT_ERR_TIMEOUT).
 * While the word holds an error, this library's kernels return at once
 * without touching their outputs, so clear it before going on.
 */
rt_status rt_take_device_error(int32_t *code);

/*
 * rt_selftest_wait_timeout -- failure-detection self test.  Launches one
 * block that waits, bounded by timeout_ns nanoseconds, on a barrier that
 * nothing completes; the kernel then records RT_ERR_TIMEOUT in the device
 * status word and returns.  Faults nothing and leaves the context usable.
 */
rt_status rt_selftest_wait_timeout(int64_t timeout_ns, rt_stream_t stream);

/*
 * rt_selftest_exp2_poly -- evaluates, for the tests, the FMA-pipe 2^x that the
 * capture kernel uses for one exponential pair in eight (Cody-Waite range
 * reduction and a degree-3 minimax polynomial on [-1/2, 1/2]; maximum relative
 * error 7.5e-5; inputs below -125, -inf included, give 2^-125).
 *
 * x  in, fp32 [n] device.   y  out, fp32 [n] device (y[i] = 2^x[i]).
 * n = 0 does nothing; a NULL or misaligned pointer is RT_ERR_INVALID_ARGUMENT.
 */
rt_status rt_selftest_exp2_poly(const float *x, float *y, int32_t n, rt_stream_t stream);

/*
 * rt_build_block_mask_static -- rt_build_block_mask for callers that must not
 * allocate device memory.
 *
 * The pages describe no such call; it exists for deployment.  Some callers
 * cannot let a library call cudaMalloc or the stream-ordered allocator: code
 * running under a framework that owns every byte of device memory through its
 * own pool, real-time loops that must never block in an allocator, and
 * processes whose memory budget is fixed up front.  This variant computes
 * exactly what rt_build_block_mask computes (same arguments, same outputs,
 * same kernels), but keeps its pooled-mean workspace in a fixed array that
 * the library places in device memory when it is loaded, instead of taking a
 * transient buffer from the allocator.
 *
 * Limit: the workspace holds 2*B*H*n_blocks*D fp32 values and is 8 MiB, so
 * 2*B*H*n_blocks*D must not exceed 2097152 (the video 5B shape, 48 heads x 278
 * blocks x 64, needs 1708032).  Larger shapes return RT_ERR_UNSUPPORTED and
 * launch nothing.  Every GPU that loads the library holds those 8 MiB until the
 * process exits.
 *
 * The first call on a device looks up the workspace's device address on that
 * device (with the device current); make that first call before capturing
 * the stream into a CUDA graph.  The address is remembered per CUDA context:
 * after cudaDeviceReset (a new primary context, the module loaded again at a
 * new address) the next call looks it up again.  The library's first call of
 * any kind on a device loads its module there (under CUDA's lazy loading),
 * and that load is what places the 8 MiB array and the kernels in device
 * memory; a caller whose memory budget is fixed later, or who must never see
 * a call allocate, should make one call (this one, or rt_workspace_bytes
 * followed by this one) at start-up.  All calls on a device share the one
 * workspace and it keeps the last call's contents; nothing in it needs to
 * start at zero (every call overwrites what it reads).  Calls that overlap on
 * the GPU (different streams, or different host threads, without ordering
 * between them) race on the workspace and give wrong masks: serialise them.
 */
rt_status rt_build_block_mask_static(const rt_shape *shape, const void *q, const void *k, float scale,
                                     int32_t keep_blocks, int32_t forced_prefix_tokens,
                                     int32_t *row_ptr, int32_t *col_idx, float *block_scores,
                                     rt_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* RETTENTION_H */
