// nsa_kernels.h -- internal launch interface between the C ABI (api.cu) and the
// kernels.  Not installed; the public interface is include/nsa_sel.h.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace nsa {

struct DevStatus;

// Everything the index inversion reads and writes.
struct InvertPlan {
    const int32_t* cu;       // [nseq + 1]
    int nseq;
    int T;
    int hkv;
    const int32_t* bidx;     // [T, hkv, topk]
    int topk;
    int bs;
    int swin;                // sliding window in keys (0: none); drops blocks before it
    int tokens_per_tile;     // 128 / G (query heads per KV head)
    int chunk_tiles;         // tiles per backward work unit
    long long nent;          // T * hkv * topk
    int nbk_cap;             // hkv * (T / bs + nseq): bound on buckets
    int key_bits;            // bits of the bucket key
    int sort_tiles;          // ceil(nent / kSortTile)
    // workspace views
    int32_t* blkoff;         // [nseq + 1]
    uint32_t* keys[2];       // [nent] ping-pong
    uint32_t* vals[2];       // [nent] ping-pong
    uint32_t* hist;          // [256 * sort_tiles]
    uint32_t* digit_tot;     // [256]
    int32_t* offsets;        // [nbk_cap + 1]
    int32_t* tile_off;       // [nbk_cap + 1]
    int32_t* chunk_off;      // [nbk_cap + 1]
    // forward only (null otherwise): the start of every (bucket, token window) run,
    // [hkv * NB * nwin + 1], windows of wtok tokens
    int32_t* wstart;
    int nwin, wtok;
    DevStatus* st;
    unsigned long long tag;  // written to st->index_tag by the inversion
    // result: the sorted values live in vals[final_buf]
    int final_buf;
};

// vals buffer that holds the sorted entries after launch_invert
int invert_final_buf(const InvertPlan& p);

constexpr int kSortTile = 4096;  // entries per sort tile (256 threads x 16)

// Window split of the (g, B) lists for the forward's tile order (g, window, B).
struct WindowPlan {
    int nwin;                // number of token windows
    int wtok;                // tokens per window
    int nb_stride;           // row stride of the tables: T / bs + nseq >= NB
    int32_t* tile_off;       // [hkv * nwin * (nb_stride + 1)]: tile offsets within a row
    int32_t* row_tiles;      // [hkv * nwin]
    int32_t* row_off;        // [hkv * nwin + 1]
    int4* tile_desc;         // [tiles_cap]: (key0, e0, nrows | g << 8, g * NB + B)
    long long tiles_cap;     // bound on the number of forward tiles
};

// Runs the inversion on `stream`; returns the first launch error.
cudaError_t launch_invert(InvertPlan& p, cudaStream_t stream);
cudaError_t launch_window_split(const InvertPlan& p, const WindowPlan& w, cudaStream_t stream);
// posmap[(t * hkv + g) * topk + j] = tile * (128 / G) + (position of the entry's token
// in its forward tile) for every valid entry; the partial rows are posmap * G + head.
cudaError_t launch_posmap(const InvertPlan& p, const WindowPlan& w, int32_t* posmap,
                          cudaStream_t stream);
// check_tag: the inversion is reused from an earlier call; a workspace whose
// st->index_tag differs from p.tag records NSA_ERR_INVALID_ARG (where 80).
cudaError_t launch_unit_desc(const InvertPlan& p, long long units_cap, int4* udesc, int* ubucket,
                             bool check_tag, cudaStream_t stream);
// Units ordered by tile count, largest first, for the snake deal of the backward kernel.
cudaError_t launch_unit_order(const DevStatus* st, const int4* udesc, int* uorder,
                              cudaStream_t stream);

struct FwdPlan {
    const void* q;
    const int32_t* cu;
    int nseq, T, hq, hkv, topk, bs, G;
    int d;                   // head dimension: 64, 128 or 256 (256 with block 64 only)
    int f16;                 // 1: q, k, v, out (dout, dq, dk, dv) are fp16; 0: bf16
    int swin;                // sliding window in keys (0: none)
    float scale_log2;        // scale * log2(e)
    const int32_t* blkoff;
    const int32_t* offsets;  // bucket offsets into entries
    const int32_t* tile_off; // bucket tile offsets
    const uint32_t* entries; // token * 64 + slot
    int nbk_cap;
    // window order of the tiles (see WindowPlan)
    int nwin, nb_stride;
    const int32_t* wtile_off;
    const int32_t* row_off;
    const int4* tile_desc;
    void* part_o;            // fp16 [tiles * 128, d]: the block's O over f, row tile * 128 + r
    float2* part_meta;       // [tiles * 128]: (lse_B, f)
    const int32_t* vexp;     // [hkv * NB]: exponent e of each (g, B) block's V
    DevStatus* st;
    int num_sms;
    int test_skip_arrive;    // test-only fault injection (NSA_TEST_SKIP_ARRIVE), 0 normally
};

// vexp[g * NB + B] = 0, or the exponent that brings max |V_B| under 2^15
cudaError_t launch_vblock_exp(const FwdPlan& p, const void* v, int nb_stride, int32_t* vexp,
                              cudaStream_t stream);
// omap[0], omap[1]: tensor maps over part_o (fp16 [tiles_cap * 128, d], 128B swizzle)
// with boxes of 64 columns x 8 rows and 64 columns x 32 rows
cudaError_t launch_fwd_tiles(const FwdPlan& p, const CUtensorMap* kmap, const CUtensorMap* vmap,
                             const CUtensorMap* omap, cudaStream_t stream);

struct MergePlan {
    const int32_t* cu;
    int nseq, T, hq, hkv, topk, bs, G;
    int d;                   // head dimension: 64, 128 or 256
    int f16;                 // 1: out is fp16; 0: bf16
    int swin;                // sliding window in keys (0: none)
    const int32_t* bidx;
    const int32_t* posmap;   // tile position of each KV-major (t, g, j) entry
    const void* part_o;      // KV-major partials
    const float2* part_meta;
    void* out;
    float* lse;              // may be null
    const DevStatus* st;
};

// O and LSE of every row from its KV-major partials
cudaError_t launch_merge(const MergePlan& p, cudaStream_t stream);

struct BwdPlan {
    const void* q;
    const void* dout;
    int f16;                 // 1: the attention tensors are fp16; 0: bf16
    const float* lse;        // [hq, T]
    float* delta;            // [hq, T]  rowsum(dout * out)
    const int32_t* cu;
    int nseq, T, hq, hkv, topk, bs, G;
    int d;                   // head dimension of q, k, v, dout, dq, dk, dv (64 or 128); the
                             // tile kernel and its partials work at 128 columns
    int swin;                // sliding window in keys (0: none)
    float scale, scale_log2;
    const int32_t* blkoff;
    const int32_t* offsets;
    const int32_t* tile_off;
    const int32_t* chunk_off;
    const uint32_t* entries;
    int nbk_cap;
    int chunk_tiles;
    const int4* udesc;       // per unit: (key0, first entry, list end, ntiles | g << 8)
    const int* ubucket;      // per unit: g * NB + B
    const int* uorder;       // units by tile count, largest first (k_unit_order)
    void* part_dq;           // bf16 [T * hq * topk, 128]
    float* part_dkdv;        // fp32 [chunks, 2, bs, 128]
    DevStatus* st;
    int num_sms;
};

cudaError_t launch_bwd_preprocess(const void* out, const void* dout, float* delta, int T, int hq,
                                  int d, int f16, cudaStream_t stream);
// qmap / domap: 2D maps over Q and dO viewed as [T * hq, 128], box 64 columns x 1 row,
// 128-byte swizzle (the tile kernel's gather4 loads)
cudaError_t launch_bwd_tiles(const BwdPlan& p, const CUtensorMap* kmap, const CUtensorMap* vmap,
                             const CUtensorMap* qmap, const CUtensorMap* domap,
                             cudaStream_t stream);
cudaError_t launch_bwd_dq_merge(const BwdPlan& p, const int32_t* bidx, void* dq,
                                cudaStream_t stream);
cudaError_t launch_bwd_dkdv_reduce(const BwdPlan& p, void* dk, void* dv, cudaStream_t stream);

// Block-selection step (select.cu): cu_cmp[nseq + 1] and the mean-pooled compressed
// K and V ([floor(T / stride) rows room, hkv, 128]); the top-k of the block scores
// ([T, hkv, nb_stride] fp32) into block_idx [T, hkv, topk].
cudaError_t launch_compress_kv(const void* k, const void* v, const int32_t* cu, int nseq, int T,
                               int hkv, int ksize, int stride, int f16, int32_t* cu_cmp, void* kc,
                               void* vc, cudaStream_t stream);
// Block scores from attention over the compressed keys (kernel 32, stride 16):
// scores [T, hkv, nb_stride] fp32; tile_off [nseq + 1] scratch; qmap over Q [T, hq, 128]
// with box (64 columns, G heads, 128 / G tokens), kcmap over k_cmp [kc_rows, hkv, 128]
// with box (64 columns, 1 head, 64 rows), both 128-byte swizzled.
cudaError_t launch_cmp_scores(const void* q, const void* kc, long long kc_rows, const int32_t* cu,
                              const int32_t* cu_cmp, int nseq, int T, int hq, int hkv,
                              int nb_stride, int bs, float scale, float* scores,
                              int32_t* tile_off, DevStatus* st, int num_sms,
                              const CUtensorMap* qmap, const CUtensorMap* kcmap,
                              cudaStream_t stream);
// Threshold-pruned block attention (bsfa.cu): out bf16 [T, hq, 128], lse [hq, T] (or
// null); tau fp32 [hq]; qmap as for the block scores, kmap / vmap as for the forward.
cudaError_t launch_bsfa_fwd(const int32_t* cu, int nseq, int T, int hq, int hkv, float scale,
                            const float* tau, void* out, float* lse, int32_t* tile_off,
                            DevStatus* st, int num_sms, const CUtensorMap* qmap,
                            const CUtensorMap* kmap, const CUtensorMap* vmap,
                            cudaStream_t stream);
cudaError_t launch_select_topk(const float* scores, const int32_t* cu, int nseq, int T, int hkv,
                               int nb_stride, int bs, int topk, int init_blocks, int local_blocks,
                               int32_t* bidx, DevStatus* st, cudaStream_t stream);

cudaError_t launch_validate(const int32_t* cu, int nseq, int T, int hkv, const int32_t* bidx,
                            int topk, int bs, DevStatus* st, cudaStream_t stream);

}  // namespace nsa
