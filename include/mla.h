/*
 * mla.h -- C ABI of the B200 (sm_100a) absorbed Multi-head Latent Attention library.
 *
 * The operation is attention over a latent cache in its absorbed form, as derived
 * on the page "Module 05 -- MLA: Compressing Per-Token History" (jared-hpc.com,
 * GLM-5.3-Flash Architecture Mastery, Lecture-05):
 *   section 1  every cached token keeps one shared latent c_j (width R = 512);
 *              per head h the key/value are k = U_h^K c_j and v = U_h^V c_j,
 *              U_h in R^{D x R} with D = 256 and H = 64 heads (NoPE);
 *   section 3  q~_h = (U_h^K)^T q_h  (mla_absorb_q),
 *              score_j = scale * q~_h . c_j, softmax, o_h = sum_j a_j c_j
 *              (mla_attend_*), out_h = U_h^V o_h (mla_up_proj);
 *              the scale is the original q.k temperature (1/sqrt(256) = 1/16);
 *   section 4  causal masking: a query at position t sees positions j <= t.
 * Multi-token-prediction verification (page dimsnsums.com/models/glm-5-3-flash/mtp)
 * scores all q_len = 1 + drafts positions of a proposed run in one pass: with the
 * q_len new latents already appended to a cache of L_b rows, query i sits at
 * position t_i = L_b - q_len + i and sees rows 0..t_i.
 *
 * Conventions for every entry point
 *  - bf16 tensors are passed as uint16_t bit patterns; all tensors are dense,
 *    row-major (last index fastest) and 16-byte aligned.
 *  - Every data pointer is a DEVICE pointer owned by the caller.  The library never
 *    allocates, frees, synchronises or throws; work is enqueued on `stream`
 *    (a cudaStream_t, NULL = legacy default stream) and runs asynchronously.
 *  - Host-detectable errors (null pointers, bad sizes, unsupported H/D/R,
 *    misalignment, workspace too small) return an error code and enqueue nothing.
 *  - Device-detectable errors (page id or index out of range, a bounded wait that
 *    expired) are written to *status (a device int32, may be NULL) only if it is still
 *    MLA_OK, so the first error is kept; the caller zeroes it and reads it after its
 *    own synchronisation.  Outputs are unspecified when *status != MLA_OK.
 *  - Supported sizes in this version: H = 64, D = 256, R = 512.
 *  - Launch chaining: each kernel may start while the previous kernel on the stream is
 *    still running and waits for it (griddepcontrol.wait) before it reads that kernel's
 *    results.  The one exception is the projection weights: mla_absorb_q and mla_up_proj
 *    start streaming w_uk / w_uv before that wait, so the weights must not be written by
 *    the kernel launched immediately before them on the same stream.  Weights written
 *    earlier (or on another stream followed by an event wait, or by a memcpy) are safe.
 */
#ifndef MLA_B200_H
#define MLA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t mla_status;

#define MLA_OK 0
#define MLA_ERR_ARG 1          /* null pointer, non-positive or inconsistent size */
#define MLA_ERR_UNSUPPORTED 2  /* H, D or R other than 64, 256, 512; misaligned pointer */
#define MLA_ERR_CUDA 3         /* a CUDA runtime/driver call failed (launch, tensor map) */
#define MLA_ERR_WORKSPACE 4    /* workspace pointer null or ws_bytes too small */
#define MLA_ERR_INDEX 5        /* device: page id / cache index / length out of range */
#define MLA_ERR_TIMEOUT 6      /* device: a bounded pipeline wait expired */

/* Human-readable name of a status code (static string, never NULL). */
const char *mla_status_string(mla_status s);

/* Message of the last CUDA runtime error seen by an entry point on the calling thread
 * (the reason behind an MLA_ERR_CUDA return), or "no error".  Static string. */
const char *mla_last_error_string(void);

/*
 * Query absorption, Module 05 section 3:  q_tilde[n,h,:] = U_h^K^T q[n,h,:].
 *   q       [n, H, D] bf16     query heads (n = batch * q_len rows)
 *   w_uk    [H, D, R] bf16     U^K per head, k = U_h^K c  (row d, column r)
 *   q_tilde [n, H, R] bf16     output, fp32 accumulation, rounded to nearest even
 * n >= 1.  Errors: MLA_ERR_ARG, MLA_ERR_UNSUPPORTED, MLA_ERR_CUDA.
 */
mla_status mla_absorb_q(const uint16_t *q, const uint16_t *w_uk, uint16_t *q_tilde,
                        int n, int H, int D, int R, void *stream);

/*
 * Latent attention over a contiguous cache, Module 05 sections 3-4 (+ MTP window).
 *   q_tilde  [B, Q, H, R] bf16   absorbed queries (output of mla_absorb_q)
 *   cache    [B, Lmax, R] bf16   latent rows c_j of each sequence
 *   seq_lens [B] int32 or NULL   rows L_b of sequence b, INCLUDING the Q newly appended
 *                                query rows; NULL means every sequence has Lmax rows.
 *                                0 <= L_b <= Lmax (else MLA_ERR_INDEX on *status).
 *   scale                         softmax scale applied to q~.c (1/16 for these heads)
 *   workspace, ws_bytes           caller scratch, >= mla_attend_workspace_bytes(B, Q, H, R)
 *   o_latent [B, Q, H, R] bf16   o = sum_j a_j c_j (normalised), the input of mla_up_proj
 *   lse      [B, Q, H] fp32      natural-log sum-exp of the scaled scores, or NULL
 * Query i of sequence b sees rows 0 .. L_b - Q + i; an empty window gives o = 0 and
 * lse = -inf.  Rows beyond L_b may hold any bits (they are never used).
 */
mla_status mla_attend_dense(const uint16_t *q_tilde, const uint16_t *cache, const int32_t *seq_lens,
                            int B, int Q, int H, int R, int Lmax, float scale,
                            void *workspace, size_t ws_bytes, uint16_t *o_latent, float *lse,
                            int32_t *status, void *stream);

/*
 * Same as mla_attend_dense over a paged cache: logical row j of sequence b is
 *   pool[page_table[b * max_pages + j / page_size]][j % page_size][:].
 *   pool       [num_pages, page_size, R] bf16
 *   page_table [B, max_pages] int32   entries for pages past the end are ignored;
 *                                     max_pages * page_size and num_pages * page_size < 2^31
 *   seq_lens   [B] int32 (required)   0 <= L_b <= max_pages * page_size
 * page_size must be 64.  A used entry outside [0, num_pages) sets MLA_ERR_INDEX.
 * The result is bit-identical to mla_attend_dense on the same logical rows.
 */
mla_status mla_attend_paged(const uint16_t *q_tilde, const uint16_t *pool, const int32_t *page_table,
                            const int32_t *seq_lens, int B, int Q, int H, int R, int page_size,
                            int max_pages, int num_pages, float scale, void *workspace, size_t ws_bytes,
                            uint16_t *o_latent, float *lse, int32_t *status, void *stream);

/*
 * Attention of each query over a given list of cache positions (a sparse selection
 * such as the DSA indexer's): query i of sequence b attends exactly to the rows
 * cache[b, indices[b, i, k]] for k < K.
 *   indices  [B, Q, K] int32   positions, each in [0, L_b - Q + i] (causally visible);
 *                              order does not matter, a repeated entry counts twice;
 *                              an entry of -1 is unused and contributes nothing (lists of a
 *                              fixed width K that hold fewer positions, as the k-pool index
 *                              producer below emits).
 *   seq_lens [B] int32 or NULL  as for mla_attend_dense (used to validate indices)
 * An out-of-range entry sets MLA_ERR_INDEX.  K >= 1.
 * Each list is split over C = min(SMs / (B * Q), ceil(K / 64)) CTAs.  When C <= 8 and a
 * cluster of C CTAs per list fits the device for every list at once (32 lists of 2,048
 * entries on a B200: clusters of 4), the CTAs of a list run as one thread-block cluster
 * and merge their partials inside the attend kernel: one kernel per call.  Otherwise a
 * combine kernel follows, as for mla_attend_dense.  The workspace is used either way, and
 * the results are the same bits.
 */
mla_status mla_attend_indexed(const uint16_t *q_tilde, const uint16_t *cache, const int32_t *indices,
                              const int32_t *seq_lens, int B, int Q, int H, int R, int Lmax, int K,
                              float scale, void *workspace, size_t ws_bytes, uint16_t *o_latent,
                              float *lse, int32_t *status, void *stream);

/*
 * Value up-projection, Module 05 section 3:  out[n,h,:] = U_h^V o_latent[n,h,:].
 *   o_latent [n, H, R] bf16, w_uv [H, D, R] bf16 (v = U_h^V c), out [n, H, D] bf16.
 */
mla_status mla_up_proj(const uint16_t *o_latent, const uint16_t *w_uv, uint16_t *out,
                       int n, int H, int D, int R, void *stream);

/*
 * Attention with the value up-projection fused into its split-L merge, Module 05 section 3:
 * "the latent-space sum is expanded once, at the end" -- out_h = U_h^V o_h with
 * o_h = sum_j a_j c_j, computed without o making a round trip through global memory.
 * Same inputs and semantics as mla_attend_dense / _paged / _indexed, plus
 *   w_uv     [H, D, R] bf16   U^V per head (as for mla_up_proj), D = 256
 *   out      [B, Q, H, D] bf16  the attention output (what mla_up_proj returns)
 *   o_latent [B, Q, H, R] bf16 or NULL: also store the normalised latent output
 *   lse      [B, Q, H] fp32 or NULL
 * The workspace is the same as the unfused call's (mla_attend_workspace_bytes).  The merge
 * and the projection run in one kernel launched after the attend kernel: clusters of four
 * CTAs per head split the latent into chunks of 128, merge their chunk of the partials
 * into the tensor-core operand and sum the four partial products through distributed
 * shared memory.  w_uv is read before that kernel waits for the attend kernel (see the
 * launch-chaining note above).  Results match mla_attend_* followed by mla_up_proj to
 * rounding (here o is rounded to bf16 per 128-wide chunk, exactly as mla_up_proj's input).
 */
mla_status mla_attend_up_dense(const uint16_t *q_tilde, const uint16_t *cache, const int32_t *seq_lens, int B, int Q,
                               int H, int R, int Lmax, float scale, const uint16_t *w_uv, int D, void *workspace,
                               size_t ws_bytes, uint16_t *out, uint16_t *o_latent, float *lse, int32_t *status,
                               void *stream);
mla_status mla_attend_up_paged(const uint16_t *q_tilde, const uint16_t *pool, const int32_t *page_table,
                               const int32_t *seq_lens, int B, int Q, int H, int R, int page_size, int max_pages,
                               int num_pages, float scale, const uint16_t *w_uv, int D, void *workspace,
                               size_t ws_bytes, uint16_t *out, uint16_t *o_latent, float *lse, int32_t *status,
                               void *stream);
mla_status mla_attend_up_indexed(const uint16_t *q_tilde, const uint16_t *cache, const int32_t *indices,
                                 const int32_t *seq_lens, int B, int Q, int H, int R, int Lmax, int K, float scale,
                                 const uint16_t *w_uv, int D, void *workspace, size_t ws_bytes, uint16_t *out,
                                 uint16_t *o_latent, float *lse, int32_t *status, void *stream);

/*
 * Prefill in the expanded form, Module 05 section 5 ("prefill and decode may want different
 * algebra"): when every token of a sequence is a query, the pass is compute-heavy and the
 * naive algebra -- expand keys and values once, then ordinary attention over 256-wide heads
 * -- does half the attention arithmetic of the absorbed form (whose scores and value sums
 * run over the 512-wide latent).  The absorbed form of the same prefill is
 * mla_absorb_q -> mla_attend_dense (q_len = L, cache = the sequence's own latents) ->
 * mla_up_proj; these two calls are the expanded one, for measuring which form wins.
 *
 * mla_expand_kv, Module 05 section 1: k[n, h, :] = U_h^K c[n, :], v[n, h, :] = U_h^V c[n, :].
 *   c [n, R] bf16 latents; w_uk, w_uv [H, D, R] bf16; k, v [n, H, D] bf16 (fp32 accumulation).
 * mla_prefill_expanded: causal attention of B sequences of L tokens over themselves,
 *   out[b, t, h, :] = sum_{j <= t} softmax_j(scale * q[b, t, h] . k[b, j, h]) v[b, j, h]
 *   q, k, v, out [B, L, H, D] bf16 (token-major, as mla_expand_kv writes k and v with
 *   n = B * L); lse [B, L, H] fp32 natural-log sum-exp or NULL.  k and v must be finite
 *   (rows past a sequence's last query are read but weighted zero).  B * L * H < 2^31.
 */
mla_status mla_expand_kv(const uint16_t *c, const uint16_t *w_uk, const uint16_t *w_uv, uint16_t *k, uint16_t *v,
                         int n, int H, int D, int R, void *stream);
mla_status mla_prefill_expanded(const uint16_t *q, const uint16_t *k, const uint16_t *v, int B, int L, int H, int D,
                                float scale, uint16_t *out, float *lse, int32_t *status, void *stream);

/*
 * mla_attend_dense for callers that cannot allocate device memory (for example a plugin
 * inside a host runtime that owns all device memory and passes its plugins no workspace,
 * or a runtime whose memory plan is fixed at start-up).  There is no counterpart on the
 * pages: it is a packaging variant of mla_attend_dense, with the same arguments minus
 * the workspace and the same results.
 *  - Scratch comes from a 32 MiB array inside the library.  Sizes whose
 *    mla_attend_workspace_bytes(B, Q, H, R) exceeds 32 MiB return MLA_ERR_WORKSPACE and
 *    enqueue nothing.
 *  - No call allocates: no cudaMalloc, cudaFree or allocating library call.  The array
 *    itself is device memory that the CUDA runtime reserves when it loads the library's
 *    code module holding it on a device.  With the default lazy module loading that
 *    happens in the first call of this entry point on that device (which looks the array's
 *    address up with cudaGetSymbolAddress, with that device current); it is then held
 *    until the process exits.  A caller with a fixed memory plan makes that first call at
 *    start-up, or sets CUDA_MODULE_LOADING=EAGER so that every device reserves the array
 *    when the context is created.  If the reservation fails, the call returns MLA_ERR_CUDA.
 *    Make the first call before any stream capture.
 *  - All calls share the one array, so calls whose kernels overlap on the GPU (different
 *    streams, or several host threads) race and corrupt each other's results; serialise
 *    them.  No part of the array has to start at zero.
 */
mla_status mla_attend_dense_noalloc(const uint16_t *q_tilde, const uint16_t *cache, const int32_t *seq_lens,
                                    int B, int Q, int H, int R, int Lmax, float scale, uint16_t *o_latent,
                                    float *lse, int32_t *status, void *stream);

/*
 * Latent-cache bookkeeping around a speculative verify step.  Page "Module 08 -- Vision,
 * MTP, and Hybrid Serving State" (jared-hpc.com, GLM-5.3-Flash Architecture Mastery,
 * Lecture-08), section 3: the MLA latent cache is indexed by token position, so it is
 * rolled back by truncating it to the accepted prefix, and the state after rollback must
 * equal the state of a run that never generated the rejected tokens.
 *
 * mla_cache_append_*: write the Q latent rows of a verify window after each sequence's
 * current length and advance the length:
 *   rows     [B, Q, R] bf16     rows[b, i] goes to position seq_lens[b] + i
 *   seq_lens [B] int32, in/out  seq_lens[b] += Q
 *   dense:   cache [B, Lmax, R] bf16, position j of sequence b is cache[b, j]
 *   paged:   pool [num_pages, page_size = 64, R] bf16, page_table [B, max_pages] int32;
 *            position j is pool[page_table[b, j / 64], j % 64].  The caller maps the pages
 *            first: every position written must land on an entry in [0, num_pages).
 * mla_cache_truncate_*: keep the first keep[b] (0..Q) of the last Q rows of sequence b:
 *   seq_lens[b] becomes seq_lens[b] - Q + keep[b] and the discarded rows are set to zero,
 *   so a cache whose unused rows are zero ends identical to one that never held them.
 *   Pages that become empty stay mapped; releasing them is the caller's business.
 * A sequence whose positions would fall outside the cache (or on an unmapped or
 * out-of-range page), or whose keep[b] is outside 0..Q, is left untouched and sets
 * MLA_ERR_INDEX; the other sequences proceed.  Q >= 1, R = 512.
 */
mla_status mla_cache_append_dense(uint16_t *cache, int32_t *seq_lens, const uint16_t *rows, int B, int Q, int R,
                                  int Lmax, int32_t *status, void *stream);
mla_status mla_cache_append_paged(uint16_t *pool, const int32_t *page_table, int32_t *seq_lens, const uint16_t *rows,
                                  int B, int Q, int R, int page_size, int max_pages, int num_pages, int32_t *status,
                                  void *stream);
mla_status mla_cache_truncate_dense(uint16_t *cache, int32_t *seq_lens, const int32_t *keep, int B, int Q, int R,
                                    int Lmax, int32_t *status, void *stream);
mla_status mla_cache_truncate_paged(uint16_t *pool, const int32_t *page_table, int32_t *seq_lens, const int32_t *keep,
                                    int B, int Q, int R, int page_size, int max_pages, int num_pages, int32_t *status,
                                    void *stream);

/*
 * k-pool index producer for mla_attend_indexed.  Page "GLM-5.3-Flash engine (c/glm53.c)"
 * (colibri docs), Architecture notes, DSA with k-pooling: keys are grouped into pools of
 * `pool` consecutive positions, a pool's key is a per-channel softmax mixture of its
 * members, only complete and causally visible pools are selectable, the incomplete tail is
 * appended when asked for, and ties go to the lower index.  The pages give no indexer
 * projections: here the key of a position is its cached latent c_j and the indexer query
 * is a given vector w[b, i] of width R.
 *
 * mla_kpool_keys: pooled[b, p, d] = sum_j softmax_j(c[b, p*pool + j, d]) * c[b, p*pool + j, d]
 *   for every complete pool of sequence b (p < seq_lens[b] / pool); other rows untouched.
 *   cache [B, Lmax, R] bf16, seq_lens [B] int32 or NULL (all Lmax), pooled [B, Lmax / pool, R]
 *   fp32 (caller-owned; may be reused across calls while the cache only grows).
 * mla_kpool_select: for query i of sequence b at position t = seq_lens[b] - Q + i, writes
 *   indices[b, i, 0 .. W) =
 *     the positions of the topk / pool best pools among those ending at or before t
 *     (score = w[b, i] . pooled[b, p] in fp32; ties to the lower pool), in ascending order,
 *     then -1 up to topk; with_tail != 0 appends the positions of the incomplete pool up
 *     to t, then -1 up to W = topk + pool - 1 (W = topk without the tail).
 *   w_query [B, Q, R] bf16.  topk a positive multiple of pool, topk / pool <= 1024,
 *   Lmax / pool <= 51200, B * Q < 2^31 (mla_kpool_keys: B <= 65535).  The list feeds
 *   mla_attend_indexed with K = W (-1 entries unused).
 */
mla_status mla_kpool_keys(const uint16_t *cache, const int32_t *seq_lens, int B, int R, int Lmax, int pool,
                          float *pooled, void *stream);
mla_status mla_kpool_select(const float *pooled, const uint16_t *w_query, const int32_t *seq_lens, int B, int Q, int R,
                            int Lmax, int pool, int topk, int with_tail, int32_t *indices, int W, void *stream);

/*
 * Bytes of workspace the mla_attend_* calls need for B sequences of Q queries on the
 * current device (split-L partial results and their max/sum terms).  0 on bad sizes.
 */
size_t mla_attend_workspace_bytes(int B, int Q, int H, int R);

/*
 * Test aid: copy the latent rows the attend kernels would address, with the same
 * address computation, so that page-table and index handling can be compared bit
 * for bit.  For request r = (req[3r], req[3r+1], req[3r+2]) = (b, i, k):
 *   mode 0 (dense):   out[r] = cache[b, k]
 *   mode 1 (paged):   out[r] = pool[page_table[b, k / 64], k % 64]
 *   mode 2 (indexed): out[r] = cache[b, indices[b, i, k]]
 * `src` is the cache (modes 0, 2) or the pool (mode 1); sizes as in the attend calls
 * (Lmax is unused in mode 1, num_pages unused in modes 0 and 2).  A request whose
 * address is out of range writes a zero row and sets MLA_ERR_INDEX on *status.
 */
mla_status mla_debug_gather(int mode, const uint16_t *src, const int32_t *page_table, const int32_t *indices,
                            int B, int Q, int R, int Lmax, int max_pages, int num_pages, int K,
                            const int32_t *req, int n_req, uint16_t *out, int32_t *status, void *stream);

/*
 * Test aid for failure detection: runs the bounded mbarrier wait that every pipeline role
 * of the attend kernel uses, on a barrier that nothing ever completes, with a limit of
 * `limit_cycles` SM cycles (1 .. 2e9).  The wait gives up, writes MLA_ERR_TIMEOUT to
 * *status (a device int32, required) if it is still MLA_OK, and the kernel returns: the
 * context stays usable.  No counterpart on the pages.
 */
mla_status mla_debug_wait_timeout(long long limit_cycles, int32_t *status, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* MLA_B200_H */
