/*
 * nsa_sel.h -- C ABI of the B200 (sm_100a) selected-block attention library
 * (Native Sparse Attention, selection branch: each query attends only to the
 * KV blocks chosen for its sequence and KV head).
 *
 * Sources for the operation:
 *  - "Relaxed-System-Lab/Flash-Sparse-Attention" project page, Quick-start section:
 *    block_size (64), topk (16), init_blocks (1), local_blocks (2), GQA head counts,
 *    head_dim 128, and varlen packing through cu_seqlens (int32 cumulative lengths
 *    with a leading 0).  Same page, Limitations section: Q, K and V share one head
 *    dimension.  Same page, key-features table: a main query-to-KV kernel plus
 *    reduction and online-softmax kernels with no atomics; forward-only prefill and
 *    full backward.
 *  - "FSA: Efficient Implementation of Native Sparse Attention" blog page, second
 *    paragraph: the kernel swaps the loop order so that small GQA groups still fill
 *    the hardware tiles.
 *
 * Definition computed (token t of sequence s, local position i, query block
 * qb = i / block_size, query head h, KV head g = h / (hq / hkv)):
 *     Sel  = { block_idx[t, g, j] : 0 <= value <= qb }        (-1 pads)
 *     J    = { keys j of the blocks in Sel : j <= i }        (causal)
 *     O[t, h]   = softmax_j(scale * q[t,h] . k[j,g]) . v[j,g]
 *     LSE[h, t] = natural log of sum_j exp(scale * q[t,h] . k[j,g])
 * An empty J gives O = 0 and LSE = -inf.  Block numbers are local to each sequence.
 * Indices in one (t, g) row must be distinct (nsa_sel_validate_indices checks).
 *
 * Conventions for every call:
 *  - All tensor pointers are DEVICE pointers, contiguous, in the layouts stated.
 *    16-bit tensors and the workspace must be 16-byte aligned, int32/fp32 ones
 *    4-byte aligned.
 *  - The caller owns every buffer, including the workspace; the library allocates
 *    nothing and keeps no state between calls.
 *  - Work is enqueued on `stream` (a cudaStream_t); no call synchronises except
 *    nsa_sel_validate_indices and nsa_sel_check_status.
 *  - Argument errors are detected on the host before any launch and leave the
 *    outputs untouched.  Launch failures return NSA_ERR_CUDA.  Device-side
 *    problems (a bounded wait that expired, malformed cu_seqlens) are recorded
 *    in the status block at the start of the workspace and read with
 *    nsa_sel_check_status.  No C++ exception crosses this interface.
 *  - Supported domain: bf16 (fp16 through the _ex calls' NSA_F16); head_dim 64, 128
 *    or 256 in the forward (256 with block_size 64 only: its Q stages fill the shared
 *    memory), 64 or 128 in the backward (64 runs the 128-column backward with columns
 *    64..127 read as zeros); block_size in {64, 128},
 *    1 <= topk <= 64, hq % hkv == 0 with hq / hkv a divisor of 128 (a 128-row tile
 *    holds whole query-head groups), total_tokens < 2^25, and (for 32-bit row
 *    coordinates) total_tokens * hkv * topk < 2^31, total_tokens * hq < 2^31 and
 *    fewer than 2^31 forward partial rows (about total_tokens * hq * topk; far
 *    beyond any device memory).  Anything else returns NSA_ERR_UNSUPPORTED.
 */
#ifndef NSA_SEL_H
#define NSA_SEL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define NSA_API __attribute__((visibility("default")))
#else
#define NSA_API
#endif

typedef struct CUstream_st *nsa_stream_t; /* the same type as cudaStream_t */

typedef enum {
    NSA_OK = 0,
    NSA_ERR_INVALID_ARG = 1,  /* null / misaligned pointer, negative size, bad shape */
    NSA_ERR_UNSUPPORTED = 2,  /* outside the supported domain above */
    NSA_ERR_WORKSPACE = 3,    /* workspace smaller than nsa_sel_attn_workspace_size() */
    NSA_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
    NSA_ERR_TIMEOUT = 5,      /* a bounded device-side wait expired (kernel returned) */
    NSA_ERR_BAD_INDEX = 6,    /* block_idx or cu_seqlens content is invalid */
    NSA_ERR_NO_DEVICE = 7     /* no sm_100 device is current */
} nsa_status_t;

/* Bytes of workspace that nsa_sel_attn_fwd (for_bwd = 0) or nsa_sel_attn_bwd
 * (for_bwd = 1) needs for these sizes; 0 when the sizes are unsupported.  The first
 * 256 bytes are the device status block. */
NSA_API size_t nsa_sel_attn_workspace_size(int total_tokens, int num_seqs, int hq, int hkv,
                                   int head_dim, int topk, int block_size, int for_bwd);

/* Forward selected-block attention (definition in the file header).
 *   q   bf16 [total_tokens, hq, head_dim]        k, v bf16 [total_tokens, hkv, head_dim]
 *   cu_seqlens int32 [num_seqs + 1], cu_seqlens[0] = 0, non-decreasing,
 *              cu_seqlens[num_seqs] = total_tokens
 *   block_idx  int32 [total_tokens, hkv, topk], block numbers local to the sequence
 *   out  bf16 [total_tokens, hq, head_dim] (written)
 *   lse  fp32 [hq, total_tokens] (written; natural log), or null for a forward
 *        that will have no backward (nothing is stored then)
 * Steps on `stream`: block-index inversion, the tensor-core tile kernel over
 * (KV block, gathered query rows), and the log-sum-exp merge of the per-block
 * partial results. */
NSA_API nsa_status_t nsa_sel_attn_fwd(const void *q, const void *k, const void *v,
                              const int32_t *cu_seqlens, int num_seqs, int total_tokens,
                              int hq, int hkv, int head_dim, const int32_t *block_idx,
                              int topk, int block_size, float scale, void *out, float *lse,
                              void *workspace, size_t workspace_bytes, nsa_stream_t stream);

/* Backward of the forward above for the loss gradient dout = dL/dO.
 *   out, lse   the forward's outputs (same layouts)
 *   dout       bf16 [total_tokens, hq, head_dim]
 *   dq         bf16 [total_tokens, hq, head_dim] (written)
 *   dk, dv     bf16 [total_tokens, hkv, head_dim] (written; keys that no query
 *              attends get 0)
 * Uses D = rowsum(dout * out) from the bf16 `out`.  Deterministic: the sums over
 * query rows run in a fixed order. */
NSA_API nsa_status_t nsa_sel_attn_bwd(const void *q, const void *k, const void *v, const void *out,
                              const float *lse, const void *dout, const int32_t *cu_seqlens,
                              int num_seqs, int total_tokens, int hq, int hkv, int head_dim,
                              const int32_t *block_idx, int topk, int block_size, float scale,
                              void *dq, void *dk, void *dv, void *workspace,
                              size_t workspace_bytes, nsa_stream_t stream);

/* Instrumented forms of the two calls above, used for measurement.  Identical work;
 * in addition, when events is non-null, events[i] (cudaEvent_t, created by the caller)
 * is recorded on `stream` at phase boundary i, for i < num_events:
 *   forward:  0 start, 1 inversion done, 2 tile kernel done, 3 merge done
 *   backward: 0 start, 1 inversion done, 2 D = rowsum(dO * O) done, 3 tile kernel
 *             done, 4 dQ merge done, 5 dK / dV reduction done
 * and *num_launches (when non-null) receives the number of kernels launched. */
NSA_API nsa_status_t nsa_sel_attn_fwd_profiled(
    const void *q, const void *k, const void *v, const int32_t *cu_seqlens, int num_seqs,
    int total_tokens, int hq, int hkv, int head_dim, const int32_t *block_idx, int topk,
    int block_size, float scale, void *out, float *lse, void *workspace, size_t workspace_bytes,
    nsa_stream_t stream, void *const *events, int num_events, int *num_launches);
NSA_API nsa_status_t nsa_sel_attn_bwd_profiled(
    const void *q, const void *k, const void *v, const void *out, const float *lse,
    const void *dout, const int32_t *cu_seqlens, int num_seqs, int total_tokens, int hq, int hkv,
    int head_dim, const int32_t *block_idx, int topk, int block_size, float scale, void *dq,
    void *dk, void *dv, void *workspace, size_t workspace_bytes, nsa_stream_t stream,
    void *const *events, int num_events, int *num_launches);

/* Option flags of the _ex calls below (OR-ed). */
#define NSA_BWD_REUSE_INDEX 1u
#define NSA_F16 2u
/* Test-only options of nsa_sel_attn_fwd_ex, for the failure-detection tests (no
 * counterpart in the pages).  NSA_TEST_SHORT_WAITS limits every bounded wait of the
 * call's kernels to 0x01010101 SM cycles (about 8.6 ms at 1.965 GHz) instead of about
 * one second.  NSA_TEST_SKIP_ARRIVE makes one Q loader warp of the first CTA of the
 * tile kernel withhold its arrival on the first tile's Q barrier (its copies still
 * complete and nothing reads the stage), so that the MMA issuer's wait expires: the
 * call then records NSA_ERR_TIMEOUT in the status block, every CTA drains its own
 * copies and tensor-core work and frees its tensor memory, the later kernels of the
 * call leave out and lse untouched, and the device stays usable. */
#define NSA_TEST_SHORT_WAITS 0x100u
#define NSA_TEST_SKIP_ARRIVE 0x200u
/* The forward with options: flags = NSA_F16 makes q, k, v and out fp16 instead of bf16
 * (same layouts; the partials stay fp16 and all arithmetic fp32, as for bf16);
 * NSA_TEST_SHORT_WAITS and NSA_TEST_SKIP_ARRIVE as above.  Other flag bits return
 * NSA_ERR_INVALID_ARG.
 *   window_size  0: no window.  W > 0: a sliding window of W keys as well: the token at
 *       local position i attends key j only if j lies in a selected block, j <= i and
 *       j > i - W (the window_size of the sliding branch in the quick start of the
 *       "Relaxed-System-Lab/Flash-Sparse-Attention" project page; with block_idx
 *       selecting the blocks qb - ceil(W / block_size) .. qb this is that branch).
 *       Blocks wholly before the window contribute nothing; a row left with no key
 *       gets out = 0, lse = -inf.  Negative values return NSA_ERR_INVALID_ARG.
 * events / num_events / num_launches as in nsa_sel_attn_fwd_profiled (null / 0 for
 * none). */
NSA_API nsa_status_t nsa_sel_attn_fwd_ex(
    const void *q, const void *k, const void *v, const int32_t *cu_seqlens, int num_seqs,
    int total_tokens, int hq, int hkv, int head_dim, const int32_t *block_idx, int topk,
    int block_size, float scale, void *out, float *lse, void *workspace, size_t workspace_bytes,
    nsa_stream_t stream, unsigned flags, int window_size, void *const *events, int num_events,
    int *num_launches);

/* The backward with options (flags, OR-ed):
 *   NSA_BWD_REUSE_INDEX  the workspace holds the block-index inversion that
 *       nsa_sel_attn_fwd (or _profiled) computed in it for the same cu_seqlens and
 *       block_idx pointers and sizes, with workspace_bytes at least the backward size,
 *       and no other call used the workspace since; the backward then skips the
 *       inversion (a training step uses one index for both passes).  The status block
 *       is kept as the forward left it.  If the workspace was last inverted for other
 *       inputs (pointers or sizes), the call records NSA_ERR_INVALID_ARG in the device
 *       status (nsa_sel_check_status) and the outputs are undefined; the index contents
 *       themselves are not compared.
 *   NSA_F16  q, k, v, out, dout, dq, dk, dv are fp16 instead of bf16 (the forward was
 *       called with NSA_F16 too).
 * Other flag bits return NSA_ERR_INVALID_ARG.  window_size as in nsa_sel_attn_fwd_ex
 * (the forward's value; a reused inversion made with another window_size is reported
 * like other inputs).  events / num_events / num_launches as in
 * nsa_sel_attn_bwd_profiled (null / 0 for none).  Otherwise identical to
 * nsa_sel_attn_bwd. */
NSA_API nsa_status_t nsa_sel_attn_bwd_ex(
    const void *q, const void *k, const void *v, const void *out, const float *lse,
    const void *dout, const int32_t *cu_seqlens, int num_seqs, int total_tokens, int hq, int hkv,
    int head_dim, const int32_t *block_idx, int topk, int block_size, float scale, void *dq,
    void *dk, void *dv, void *workspace, size_t workspace_bytes, nsa_stream_t stream,
    unsigned flags, int window_size, void *const *events, int num_events, int *num_launches);

/* The block-index inversion on its own (the loop swap named in the file header):
 * for KV head g and global block B (blocks of earlier sequences first), the list of
 * entries token * 64 + slot with block_idx[token, g, slot] = local block of B and
 * 0 <= value <= qb(token), ascending.
 *   offsets  int32 [hkv * NB + 1], NB = sum_s ceil(L_s / block_size); exclusive
 *            prefix sums over (g major, B minor).  Room for
 *            hkv * (total_tokens / block_size + num_seqs) + 1 values is required.
 *   entries  int32 [total_tokens * hkv * topk] room; the first offsets[hkv*NB] are set.
 *   counts   int32 [2] (written): NB and the number of entries.
 * Uses the forward workspace size. */
NSA_API nsa_status_t nsa_sel_invert_index(const int32_t *cu_seqlens, int num_seqs, int total_tokens,
                                  int hkv, const int32_t *block_idx, int topk, int block_size,
                                  int32_t *offsets, int32_t *entries, int32_t *counts,
                                  void *workspace, size_t workspace_bytes, nsa_stream_t stream);

/* Bytes of scratch the block-index inversion needs for these sizes (0 when they are
 * outside the supported domain): 256-byte-aligned regions of about 16.25 bytes per
 * (token, KV head, slot) entry (two key and two value buffers of the radix sort and
 * its digit histograms) plus 12 bytes per (KV head, block) and 4 per sequence.
 * nsa_sel_invert_index_noalloc accepts exactly the sizes for which this is at most
 * nsa_sel_invert_index_noalloc_max_bytes().  Host only; no device work. */
NSA_API size_t nsa_sel_invert_index_scratch_bytes(int total_tokens, int num_seqs, int hkv,
                                                  int topk, int block_size);

/* The block-index inversion above, for callers that cannot allocate device memory
 * (for example a plug-in whose host framework owns all device memory and offers no
 * allocation hook, or a loop where cudaMalloc's possible device synchronisation is
 * not allowed).  The pages have no counterpart for this entry point.
 *   Arguments and outputs are those of nsa_sel_invert_index, without the workspace:
 *   the scratch is a fixed array in the library's device data, of
 *   nsa_sel_invert_index_noalloc_max_bytes() bytes (64 MiB) per device, held until
 *   the process exits.  Problems whose inversion scratch
 *   (nsa_sel_invert_index_scratch_bytes; at topk 16 and block 64 roughly
 *   T * hkv <= 250,000) would not fit return NSA_ERR_WORKSPACE before any device work.
 *   The first call on a device (and the first after the device's context was
 *   replaced) looks up the array's device address with that device current; make
 *   that first call before any stream capture.
 *   All calls share the array and it keeps the last call's contents; everything a
 *   call reads from it is first written by the same call, but calls whose work
 *   overlaps on the GPU (other streams, other host threads) race: serialise them. */
NSA_API nsa_status_t nsa_sel_invert_index_noalloc(const int32_t *cu_seqlens, int num_seqs,
                                                  int total_tokens, int hkv,
                                                  const int32_t *block_idx, int topk,
                                                  int block_size, int32_t *offsets,
                                                  int32_t *entries, int32_t *counts,
                                                  nsa_stream_t stream);
/* Size in bytes of the scratch array used by nsa_sel_invert_index_noalloc. */
NSA_API size_t nsa_sel_invert_index_noalloc_max_bytes(void);

/* Host-synchronous check of block_idx: counts values outside {-1} U [0, NB_s) and
 * repeated non-negative values within one (token, KV head) row.  Returns
 * NSA_ERR_BAD_INDEX when either count is non-zero, NSA_OK otherwise.  Future blocks
 * (qb < value < NB_s) are allowed and contribute nothing. */
NSA_API nsa_status_t nsa_sel_validate_indices(const int32_t *cu_seqlens, int num_seqs,
                                      int total_tokens, int hkv, const int32_t *block_idx,
                                      int topk, int block_size, long long *n_out_of_range,
                                      long long *n_duplicates, void *workspace,
                                      size_t workspace_bytes, nsa_stream_t stream);

/* Block-selection step, the stage that produces block_idx: compression, block scores
 * from attention over the compressed keys, top-k.
 * The quick start of the "Relaxed-System-Lab/Flash-Sparse-Attention" project page
 * sets kernel_size 32, kernel_stride 16, init_blocks 1, local_blocks 2; the pages
 * print no formula, so compressed keys / values are the means of the covered rows
 * and the top-k breaks score ties toward the lower block.
 *
 * nsa_sel_compress_kv: for each sequence s (length L_s), compressed block c covers
 * its tokens [c * kernel_stride, c * kernel_stride + kernel_size); there are
 * floor((L_s - kernel_size) / kernel_stride) + 1 of them (0 if L_s < kernel_size).
 *   k, v      bf16 (fp16 with flags = NSA_F16) [total_tokens, hkv, head_dim]
 *   k_cmp, v_cmp  same type, [floor(total_tokens / kernel_stride), hkv, head_dim] room;
 *             block c of sequence s at row cu_cmp[s] + c (written): the mean of the
 *             covered rows, accumulated in fp32
 *   cu_cmp    int32 [num_seqs + 1] (written on the device): exclusive prefix sums of
 *             the per-sequence block counts
 * Requires kernel_stride <= kernel_size <= 4096 and head_dim 128; other flag bits
 * return NSA_ERR_INVALID_ARG. */
NSA_API nsa_status_t nsa_sel_compress_kv(const void *k, const void *v, const int32_t *cu_seqlens,
                                         int num_seqs, int total_tokens, int hkv, int head_dim,
                                         int kernel_size, int kernel_stride, unsigned flags,
                                         void *k_cmp, void *v_cmp, int32_t *cu_cmp,
                                         nsa_stream_t stream);

/* nsa_sel_block_scores: the scores of the selection blocks from attention over the
 * compressed keys (kernel_size 32, kernel_stride 16 only).  The token at local
 * position i sees compressed block c when c * 16 + 31 <= i; its probabilities are the
 * softmax of scale * q . k_cmp[c] over those blocks (none seen: all 0).  The score of
 * selection block b for (token, KV head g) is the sum, over the G = hq / hkv query
 * heads of g and over the compressed blocks whose span meets block b, of those
 * probabilities.
 *   q          bf16 [total_tokens, hq, head_dim], head_dim 128, G dividing 32
 *   k_cmp      bf16 [k_cmp_rows, hkv, head_dim] and cu_cmp int32 [num_seqs + 1], as
 *              nsa_sel_compress_kv wrote them (k_cmp_rows = its room)
 *   scores     fp32 [total_tokens, hkv, nb_stride] (written for blocks
 *              b < nb_stride up to the block of the row's own token; later entries of
 *              a row are left as they were)
 *   block_size 64 or 128; workspace of nsa_sel_block_scores_workspace_size(num_seqs)
 *   bytes, 256-byte aligned (its status block is read by nsa_sel_check_status). */
NSA_API size_t nsa_sel_block_scores_workspace_size(int num_seqs);
NSA_API nsa_status_t nsa_sel_block_scores(const void *q, const void *k_cmp, int k_cmp_rows,
                                          const int32_t *cu_seqlens, const int32_t *cu_cmp,
                                          int num_seqs, int total_tokens, int hq, int hkv,
                                          int head_dim, int block_size, int kernel_size,
                                          int kernel_stride, float scale, int nb_stride,
                                          float *scores, void *workspace, size_t workspace_bytes,
                                          nsa_stream_t stream);

/* nsa_sel_select_topk: block_idx row of (token at local position i, KV head g), with
 * qb = i / block_size: blocks 0 .. init_blocks - 1, then qb, qb - 1, .. (local_blocks
 * of them), each within [0, qb] and listed once, then the other blocks b <= qb in
 * descending scores[t, g, b] (ties: the lower block first), at most topk in all, the
 * rest -1.
 *   scores     fp32 [total_tokens, hkv, nb_stride], finite; nb_stride >= the largest
 *              qb + 1 (a row whose qb does not fit records NSA_ERR_INVALID_ARG in the
 *              status block and is written as -1), nb_stride <= 1024
 *   block_idx  int32 [total_tokens, hkv, topk] (written), 1 <= topk <= 64
 *   workspace  at least 256 bytes, 256-byte aligned: its status block is cleared and
 *              then read by nsa_sel_check_status. */
NSA_API nsa_status_t nsa_sel_select_topk(const float *scores, const int32_t *cu_seqlens,
                                         int num_seqs, int total_tokens, int hkv, int nb_stride,
                                         int block_size, int topk, int init_blocks,
                                         int local_blocks, int32_t *block_idx, void *workspace,
                                         size_t workspace_bytes, nsa_stream_t stream);

/* Threshold-pruned block attention (BSFA; the "Block Sparse Flash Attention" news
 * pages): every score is exact; key block b (64 keys of the token's sequence) is kept
 * for row (token at local position i, query head h) iff
 * max_{j in b, j <= i} scale * q . k_j >= tau[h]; the output is softmax attention
 * over the keys of the kept blocks only (no kept block: out = 0, lse = -inf).
 *   q bf16 [total_tokens, hq, 128]; k, v bf16 [total_tokens, hkv, 128]
 *   tau   fp32 [hq] device array of thresholds (natural units of scale * q . k)
 *   out   bf16 [total_tokens, hq, 128] (written); lse fp32 [hq, total_tokens] or null
 *   block_size 64; hq / hkv must divide 128; workspace of
 *   nsa_sel_bsfa_workspace_size(num_seqs) bytes, 256-byte aligned. */
NSA_API size_t nsa_sel_bsfa_workspace_size(int num_seqs);
NSA_API nsa_status_t nsa_sel_bsfa_fwd(const void *q, const void *k, const void *v,
                                  const int32_t *cu_seqlens, int num_seqs, int total_tokens,
                                  int hq, int hkv, int head_dim, int block_size, float scale,
                                  const float *tau, void *out, float *lse, void *workspace,
                                  size_t workspace_bytes, nsa_stream_t stream);

/* Synchronises `stream` and returns the device-side status of the last call that
 * used this workspace (NSA_OK, NSA_ERR_TIMEOUT or NSA_ERR_BAD_INDEX). */
NSA_API nsa_status_t nsa_sel_check_status(const void *workspace, nsa_stream_t stream);

/* Static string for a status code. */
NSA_API const char *nsa_sel_status_string(nsa_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* NSA_SEL_H */
