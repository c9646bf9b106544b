/*
 * calibatt.h -- C ABI of libcalibatt.so: calibrated block-sparse attention on one
 * NVIDIA B200 (sm_100a).
 *
 * The method is the one described in the summaries of "Accelerating Text-to-Video
 * Generation with Calibrated Sparse Attention" (gist.science pages in Chinese, German,
 * Portuguese and French): offline, energy-based block selection aggregated over
 * calibration inputs into a static per-(timestep, layer, head) block mask and skip list;
 * at inference, attention that computes only the kept (query block, key block) tiles,
 * plus a spatial-repetition mode that computes anchor rows and broadcasts their output.
 * Section citations below use the tags [zh] technical summary §2.1/§2.2A/§2.2B,
 * [de] "Technische Zusammenfassung" §2A/§2B, [pt] "Resumo técnico" §2A/§2B,
 * [fr] "Résumé technique" §2.A/§2.B/§2.C, and [AdaSpa] for the page "Training-free and
 * Adaptive Sparse Attention for Efficient Long Video Generation" §2.
 *
 * Conventions shared by every call:
 *  - Every pointer is a DEVICE pointer unless its comment says "host".  The caller
 *    allocates and owns all memory; the library allocates nothing and keeps no state
 *    other than one device-side status word per device (see calib_device_check).
 *  - `stream` is a cudaStream_t passed as void*; NULL means the legacy default stream.
 *    Calls are asynchronous: they validate arguments on the host, enqueue kernels on
 *    `stream` and return.  No call synchronises, except calib_device_check.
 *  - Q, K, V, O are bf16, shape [H, N, D] for batch 1, contiguous with D innermost
 *    (row n of head h starts at element (h*N + n)*D).  Pointers must be 16-byte aligned.
 *  - Blocks: block size B in {64, 128}; block i covers rows [iB, min((i+1)B, len)).
 *    nq = ceil(Nq / B) query blocks, nk = ceil(N / B) key blocks; the last one may be
 *    ragged.
 *  - Masks are uint8 [H, nq, nk] (0 = skip, 1 = keep), row (h, i) at (h*nq + i)*nk.
 *  - Errors: CALIB_ERR_INVALID for a null or misaligned pointer or an out-of-range size,
 *    CALIB_ERR_UNSUPPORTED for a size or device this build does not handle (D not in
 *    {64,128}, nk > 1024 in selection, a device other than sm_100), CALIB_ERR_CUDA for
 *    a failed launch.  On an error nothing is enqueued.  Device-side waits are bounded:
 *    a kernel that gives up records CALIB_ERR_TIMEOUT in the status word and returns.
 */
#ifndef CALIBATT_H
#define CALIBATT_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Flags of the attention calls. */
#define CALIB_ATTN_OUT_F32 1u   /* o is fp32 [H, N, D] instead of bf16 */

typedef enum calib_status {
    CALIB_OK = 0,
    CALIB_ERR_INVALID = 1,
    CALIB_ERR_UNSUPPORTED = 2,
    CALIB_ERR_CUDA = 3,
    CALIB_ERR_TIMEOUT = 4
} calib_status;

/* Skip list of one (timestep, layer) slice: the kept key blocks of every (head, query
 * block) row in CSR form ([zh] §2.2B, [pt] §2A.5, [fr] §2.C: the mask is converted into
 * the list of block intervals to compute, precomputed before inference).
 * Row r = h*nq + i holds col_idx[row_ptr[r] .. row_ptr[r+1]) in ascending order.
 * `work` (optional) is the order in which rows are processed: entries h << 16 | i,
 * longest rows first (calib_build_schedule); NULL processes rows in index order.
 * All arrays are device memory owned by the caller. */
typedef struct calib_block_list {
    int32_t H, nq, nk, block;
    const int32_t* row_ptr;   /* [H*nq + 1], row_ptr[0] = 0, non-decreasing */
    const int16_t* col_idx;   /* [row_ptr[H*nq]], each in [0, nk) */
    const int32_t* work;      /* [n_work] or NULL */
    int32_t n_work;           /* entries in `work` (ignored when work == NULL) */
} calib_block_list;

/* Human-readable name of a status code (static storage). */
const char* calib_status_string(calib_status s);

/* Synchronises `stream`, then reads and clears the status word of the current device.
 * Returns CALIB_ERR_TIMEOUT if any kernel since the last check gave up on a bounded
 * wait; CALIB_ERR_INVALID if a selection kernel met a negative or non-finite energy
 * (treated as 0) or an attention kernel met a work item outside the call (head >= H or
 * query block >= nq) or a skip-list row with a negative start, decreasing pointers or
 * more than nk blocks (that item is skipped, its output rows are not written);
 * CALIB_ERR_CUDA on a CUDA error; else CALIB_OK. */
calib_status calib_device_check(void* stream);

/* Row log-sum-exp and block energies, fused ([zh] §2.2A, [de] §2A.1, [fr] §2.B.1: split
 * the post-softmax attention matrix P into B x B blocks and sum each block):
 *   energy[h, i, j] (+)= sum_{r in I_i, c in J_j} exp(scale * q_r.k_c - LSE_r)
 * where LSE_r = log sum_c exp(scale * q_r.k_c) over all N keys.
 *   q, k     : bf16 [H, N, D].
 *   lse      : NULL, or a cached natural-log LSE fp32 [H, Nq] (e.g. sparse_attn_fwd's
 *              lse_opt of a dense call; [AdaSpa] §2 caches the LSE this way).  NULL makes
 *              the kernel compute it first, in registers, with a second pass over K.
 *   q_rows   : NULL (query rows are the N tokens) or int32 [n_q] token indices in
 *              compacted order -- the anchor rows of a spatial-repetition head
 *              (calib_anchor_rows); then Nq = n_q and blocks are over that sequence.
 *   energy   : fp32 [H, ceil(Nq/B), ceil(N/B)].  accumulate != 0 adds to it (the sum
 *              over calibration inputs, which calib_energy_mean then divides by their
 *              count); 0 overwrites.
 * P is never written to memory.  N <= 131072 (CALIB_ERR_UNSUPPORTED beyond: the per-block
 * partial sums of one query block are kept in shared memory). */
calib_status calib_block_energy(const void* q, const void* k, const float* lse,
                                int H, int N, int D, int block, float scale,
                                const int32_t* q_rows, int n_q,
                                float* energy, int accumulate, void* stream);

/* Minimal tau-energy selection ([fr] §2.B.1: per query block, the fewest key blocks whose
 * cumulative energy reaches the threshold; [zh] §2.2A, [de] §2A.2), one warp per row.
 * Equivalent to calib_select_mask_batched with one batch entry:
 *   energy     : fp32 [H, nq, nk], finite and >= 0.
 *   tau        : in (0, 1]; the per-timestep threshold eps(t).
 *   force_keep : NULL or uint8 [H, nq, nk]; forced blocks are kept first and count
 *                toward the threshold (text rows/columns of joint attention).
 *   mask_out   : uint8 [H, nq, nk].
 *   count_accum: NULL or int32 [H, nq, nk]; when given, mask_out is also added to it
 *                (the per-input masks of the cross-prompt vote).
 * Arithmetic is exact integer: each row is scaled by a power of two into integers
 * q_j < 2^53 (rounded half-even), T = max(1, ceil(tau * sum q)) with one IEEE double
 * multiply, and the kept set is forced blocks plus the largest q_j (lower key index
 * first on ties) until the sum reaches T.  A row whose energies are all 0 keeps block
 * i (block 0 if i >= nk) and its forced blocks.  nk <= 1024. */
calib_status calib_select_mask(const float* energy, int H, int nq, int nk, double tau,
                               const uint8_t* force_keep, uint8_t* mask_out,
                               int32_t* count_accum, void* stream);

/* Minimal tau-energy selection over a batch of energy matrices in one launch: the rows of
 * every (calibration input, timestep) pair of a calibration slice or sweep ([fr] §2.B.1:
 * one selection per query block at the timestep's threshold eps(t)).
 *   energy      : fp32 [nb, H, nq, nk], finite and >= 0; entry b is selected at tau[b].
 *   nb          : 1 .. 256 entries.
 *   tau         : HOST double [nb], each in (0, 1].
 *   force_keep  : NULL or uint8 [H, nq, nk], shared by every entry.
 *   mask_out    : NULL or uint8 [nb, H, nq, nk], the mask of every entry.
 *   count_accum : NULL or int32 [H, nq, nk]; each (h, i, j) is incremented by the number of
 *                 entries that keep it (the vote counts of calib_aggregate_masks when the
 *                 entries are one slice's calibration inputs).  Increments are atomic, so
 *                 the result does not depend on the order in which entries are processed.
 * At least one of mask_out and count_accum must be given.  The rule and its integer
 * arithmetic are those of calib_select_mask, row by row and entry by entry.  Energy and
 * count_accum pointers must be 4-byte aligned.  nk <= 1024. */
calib_status calib_select_mask_batched(const float* energy, int nb, int H, int nq, int nk,
                                       const double* tau, const uint8_t* force_keep,
                                       uint8_t* mask_out, int32_t* count_accum, void* stream);

/* Energy-mean aggregation over calibration inputs: the block energies averaged over the
 * inputs, then selected once (the alternative to the pages' vote over per-input masks,
 * calib_aggregate_masks; with one input both give that input's mask):
 *   mean_out[x] = energy_sum[x] / n_inputs,  x < count,
 * in fp32 with a correctly rounded division.  energy_sum is the fp32 sum of the inputs'
 * energies, as calib_block_energy(accumulate = 1) leaves it; mean_out may be energy_sum
 * (in place).  Pointers 4-byte aligned; 1 <= n_inputs <= 2^24. */
calib_status calib_energy_mean(const float* energy_sum, int64_t count, int n_inputs,
                               float* mean_out, void* stream);

/* Cross-input vote ([zh] §2.2A, [de] §2A.3, [fr] §2.B.2): keep (h, i, j) iff
 * counts[h,i,j] * rho_den > rho_num * n_inputs (frequency strictly above rho =
 * rho_num/rho_den).  A row left empty keeps its most frequent block (lowest index on
 * ties).  counts: int32 [H, nq, nk] in [0, n_inputs]; mask_out: uint8 [H, nq, nk]. */
calib_status calib_aggregate_masks(const int32_t* counts, int H, int nq, int nk,
                                   int n_inputs, int rho_num, int rho_den,
                                   uint8_t* mask_out, void* stream);

/* Skip list from a mask: row_ptr_out int32 [H*nq + 1], col_idx_out int16 with capacity
 * for every kept block (H*nq*nk always suffices).  nk <= 32767. */
calib_status calib_mask_to_csr(const uint8_t* mask, int H, int nq, int nk,
                               int32_t* row_ptr_out, int16_t* col_idx_out, void* stream);

/* Interval form of a skip list ([zh] §2.2B and [fr] §2.C describe the per-query-block
 * list as the block intervals to compute): every row's ascending kept key blocks grouped
 * into maximal runs of consecutive indices.
 *   row_ptr, col_idx : a CSR skip list (calib_mask_to_csr), col_idx ascending per row.
 *   iv_ptr_out       : int32 [H*nq + 1], runs of row r at [iv_ptr[r], iv_ptr[r+1]).
 *   iv_start_out     : int16, first key block of each run; iv_len_out: int16, its length.
 *                      Capacity: the number of kept blocks (row_ptr[H*nq]) always suffices.
 * Exact integer work; rows in order, runs in ascending order within a row. */
calib_status calib_csr_to_intervals(const int32_t* row_ptr, const int16_t* col_idx, int H, int nq,
                                    int32_t* iv_ptr_out, int16_t* iv_start_out,
                                    int16_t* iv_len_out, void* stream);

/* Inverse of calib_csr_to_intervals: expands runs back into the CSR skip list the
 * attention kernel walks.  row_ptr_out int32 [H*nq + 1]; col_idx_out int16 with capacity
 * for every kept block (the sum of all run lengths), or NULL: then only row_ptr_out is
 * written, and its last entry sizes the list for a second call. */
calib_status calib_intervals_to_csr(const int32_t* iv_ptr, const int16_t* iv_start,
                                    const int16_t* iv_len, int H, int nq,
                                    int32_t* row_ptr_out, int16_t* col_idx_out, void* stream);

/* Spatial-repetition detection, similarity step ([zh] §2.2A, [de] §2A.4, [fr] §2.B.3: the
 * cosine similarity of attention vectors of different spatial rows of one frame):
 *   cos_out[h, i] = cos(P_h[a(b_i)], P_h[b_i]) for every sampled token b_i, where P_h is
 *   the post-softmax attention of head h over all N keys and a(b) = (f, floor(y/s)*s, x) is
 *   the anchor of b = (f, y, x) at stride s (text tokens are their own anchor).
 *   q, k     : bf16 [H, N, D], device, 16-byte aligned; token n = (f*Hl + y)*Wl + x for
 *              the F*Hl*Wl video tokens, text tokens after them.
 *   lse      : NULL (the row LSEs are computed: two passes over K) or fp32 [H, N].
 *   members  : int32 [n] sampled token indices, shared by all heads (the caller draws them).
 *   cos_out  : fp32 [H, n].
 * P is never written to memory.  D in {64, 128}, block in {64, 128}. */
calib_status calib_repeat_similarity(const void* q, const void* k, const float* lse,
                                     int H, int N, int D, int block, float scale,
                                     int F, int Hl, int Wl, int stride,
                                     const int32_t* members, int n, float* cos_out, void* stream);

/* Spatial-repetition detection, decision step: per head the mean of cos[h, i] over the
 * samples that are not their own anchor, and flag = mean > gamma ("exceeds", [zh] §2.2A),
 * taken in fp32.  A head with no such sample gets mean 0.  mean_out fp32 [H], flag_out
 * uint8 [H]. */
calib_status calib_repeat_flags(const float* cos, const int32_t* members, int H, int n,
                                int F, int Hl, int Wl, int stride, float gamma,
                                float* mean_out, uint8_t* flag_out, void* stream);

/* Processing order ([AdaSpa] §2 balances kernel load across heads of different
 * sparsity): work_out int32 [H*nq] = every row h << 16 | i, heads ascending and, within
 * a head, kept count descending (longest first), ties by i ascending.  Head-major order
 * keeps the K/V blocks read by concurrently running tiles within one or two heads, so
 * they stay in L2.  H < 32768, nq < 65536. */
calib_status calib_build_schedule(const int32_t* row_ptr, int H, int nq,
                                  int32_t* work_out, void* stream);

/* Number of anchor tokens of a spatial-repetition head: F * ceil(Hl/stride) * Wl +
 * n_text (host computation, no device work).  Returns -1 for invalid sizes. */
int64_t calib_anchor_count(int F, int Hl, int Wl, int n_text, int stride);

/* Anchor token indices in compacted order ([zh] §2.1, [fr] §2.A.4, §2.C: only anchor rows
 * of a frame are computed and broadcast to the other rows of the frame): latent rows
 * y = 0, s, 2s, ... of each frame, all columns, then the text tokens.
 * rows_out: int32 [calib_anchor_count(...)]. */
calib_status calib_anchor_rows(int F, int Hl, int Wl, int n_text, int stride,
                               int32_t* rows_out, void* stream);

/* Block-sparse attention forward ([zh] §2.2B, [de] §2B, [pt] §2B, [fr] §2.C: compute the
 * kept blocks densely, skip the rest):
 *   O_r = sum_{c in K(i)} softmax_{c in K(i)}(scale * q_r.k_c) v_c
 * with K(i) the union of the key blocks kept for r's query block i (list row h*nq+i).
 *   q, k, v, o : bf16 [H, N, D]; D in {64, 128}; list->block in {64, 128};
 *                list->nq == list->nk == ceil(N/B).
 *   lse_opt    : NULL or fp32 [H, N], natural-log LSE over the kept keys.
 *   scale      : > 0 (typically 1/sqrt(D)).
 *   flags      : 0, or CALIB_ATTN_OUT_F32 to write o as fp32 (no output rounding).
 * Arithmetic: S = QK^T and O += PV on the tensor cores with fp32 accumulation; P is
 * rounded to bf16 for the PV product and O is divided by the sum of those rounded
 * weights.
 * A row with no kept block writes O = 0 and LSE = -inf.  With an all-kept list this is
 * dense attention.  The list is trusted: calib_validate_block_list_host checks one that
 * comes from outside the library's own builders. */
calib_status sparse_attn_fwd(const void* q, const void* k, const void* v, void* o,
                             float* lse_opt, int H, int N, int D, float scale,
                             const calib_block_list* list, uint32_t flags, void* stream);

/* sparse_attn_fwd on HOST tensors, with the transfers overlapped with the attention: the
 * heads are processed in chunks of heads_per_chunk; chunk c's Q/K/V go host -> device on
 * h2d_stream while the kernel of chunk c-1 runs on `stream`, and each chunk's O goes
 * device -> host on d2h_stream once its kernel is done.
 *   q_host, k_host, v_host : bf16 [H, N, D] in host memory (page-locked for the copies to
 *                overlap; pageable memory gives the same result without overlap).
 *   o_host     : host [H, N, D], bf16 (fp32 with CALIB_ATTN_OUT_F32).
 *   q_dev, k_dev, v_dev, o_dev : caller-owned device buffers of the same shapes, used as
 *                staging; their previous contents are overwritten.
 *   lse_opt    : NULL or a DEVICE fp32 [H, N] buffer (it stays on the device).
 *   heads_per_chunk >= 1.  Chunks follow the work list, which must then hold each head's nq
 *                items contiguously in head order (as calib_build_schedule writes it);
 *                with list->work == NULL or n_work != H*nq the call runs as one chunk.
 *                When there are several chunks, the heads of the last one go one head per
 *                chunk: the kernel and copy-back after the last host-to-device copy are
 *                then one head's.
 *   h2d_stream, d2h_stream : copy streams (NULL: `stream`, no overlap).
 * Ordering: the copies start after the work already queued on `stream`, and `stream` is
 * ordered after the last copy of O, so synchronising `stream` makes o_host complete.
 * Other arguments, results and errors as sparse_attn_fwd; host pointers must be non-NULL.
 * Argument errors are reported before anything is enqueued; a CUDA error met while
 * enqueueing (CALIB_ERR_CUDA) can leave the earlier chunks' copies and kernels queued.
 * The copies are one cudaMemcpyAsync per tensor and chunk. */
calib_status sparse_attn_fwd_host(const void* q_host, const void* k_host, const void* v_host, void* o_host,
                                  void* q_dev, void* k_dev, void* v_dev, void* o_dev, float* lse_opt,
                                  int H, int N, int D, float scale, const calib_block_list* list,
                                  uint32_t flags, int heads_per_chunk, void* stream, void* h2d_stream,
                                  void* d2h_stream);

/* sparse_attn_fwd_repeat on HOST tensors, transfers overlapped per head chunk as in
 * sparse_attn_fwd_host (a repeat head's broadcast stays inside its own head, so chunks of
 * heads are independent).  Repeat arguments as sparse_attn_fwd_repeat; host, staging,
 * chunk and stream arguments as sparse_attn_fwd_host. */
calib_status sparse_attn_fwd_repeat_host(const void* q_host, const void* k_host, const void* v_host,
                                         void* o_host, void* q_dev, void* k_dev, void* v_dev, void* o_dev,
                                         float* lse_opt, int H, int D, int F, int Hl, int Wl, int n_text,
                                         int stride, const uint8_t* head_repeat, float scale,
                                         const calib_block_list* list, uint32_t flags, int heads_per_chunk,
                                         void* stream, void* h2d_stream, void* d2h_stream);

/* Block-sparse attention with spatial repetition ([zh] §2.2B, [fr] §2.C): heads flagged
 * in head_repeat (HOST uint8 [H]) compute only their anchor tokens (calib_anchor_rows
 * order) and write each anchor's output (and LSE) to every token it stands for -- token
 * (f, y, x) takes anchor (f, floor(y/stride)*stride, x); text tokens are their own
 * anchors.  For a flagged head, list rows i < ceil(N_a/B) are in anchor block space and
 * rows beyond are ignored; unflagged heads behave as in sparse_attn_fwd.
 * N = F*Hl*Wl + n_text; q, k, v, o, lse_opt, D, scale and flags as in sparse_attn_fwd.
 * H <= 1024, stride >= 1 (stride 1 makes every token its own anchor). */
calib_status sparse_attn_fwd_repeat(const void* q, const void* k, const void* v, void* o,
                                    float* lse_opt, int H, int D, int F, int Hl, int Wl,
                                    int n_text, int stride, const uint8_t* head_repeat,
                                    float scale, const calib_block_list* list,
                                    uint32_t flags, void* stream);

/* Checks a skip list held in HOST memory (copied back from the device by the caller) before
 * it is given to the attention calls, which trust the list's structure: row_ptr[0] == 0;
 * for every row r < H*nq, row_ptr[r] <= row_ptr[r+1] <= col_capacity and the row keeps at
 * most nk blocks; each row's col_idx strictly ascending in [0, nk); and, when `work` is
 * given, every entry h << 16 | i with 0 <= h < H and 0 <= i < nq.  ([fr] §2.C: the lists
 * are precomputed and held in memory before inference; a list that comes from elsewhere is
 * checked here.)
 *   row_ptr     : HOST int32 [H*nq + 1].
 *   col_idx     : HOST int16, col_capacity entries (may be NULL when the list is empty).
 *   work        : HOST int32 [n_work] or NULL.
 * Pure host code, no device work: returns CALIB_OK or CALIB_ERR_INVALID.  The attention
 * kernels themselves skip (and report through calib_device_check) items whose head, query
 * block or row pointers are out of range, but they cannot see col_idx's capacity. */
calib_status calib_validate_block_list_host(int H, int nq, int nk, const int32_t* row_ptr,
                                            const int16_t* col_idx, int64_t col_capacity,
                                            const int32_t* work, int n_work);

/* Failure-detection self-test: launches one kernel that waits, with the library's bounded
 * wait, on an mbarrier that nothing ever completes, giving up after timeout_us
 * microseconds.  Returns what calib_device_check then reports: CALIB_ERR_TIMEOUT when
 * the bound works (the GPU context stays usable).  Synchronises `stream`. */
calib_status calib_selftest_wait_timeout(uint32_t timeout_us, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* CALIBATT_H */
