// api.cu -- the C ABI declared in include/nsa_sel.h.
//
// Host side only: argument checks (before any launch), the workspace layout, the
// TMA tensor maps for K and V, and the launch sequences of the forward and backward
// passes.  All work is enqueued on the caller's stream; nothing is allocated.
#include <cudaTypedefs.h>
#include <string.h>

#include <algorithm>
#include <mutex>

#include "nsa_common.cuh"
#include "nsa_kernels.h"

using namespace nsa;

namespace {

constexpr int kChunkTiles = 32;   // tiles per backward work unit
constexpr int kWindowRows = 131072; // query rows per forward token window (tokens x group)

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct Dims {
    int T, nseq, hq, hkv, d, topk, bs, G;
    long long nent;
    int nbk_cap;
    int key_bits;
    int sort_tiles;
    long long tiles_cap, units_cap;
    int wtok, nwin, nb_stride;   // forward token windows
    long long fwd_tiles_cap;     // bound on the number of forward tiles
};

struct Layout {
    size_t status, blkoff, keys0, keys1, vals0, vals1, hist, digit_tot, offsets, tile_off, chunk_off;
    size_t inv_end;   // end of the regions the index inversion (InvertPlan) uses
    size_t wstart, wtile_off, row_tiles, row_off, tile_desc, posmap, vexp;
    size_t part_o, part_lse, delta, part_dkdv, udesc, ubucket, uorder;
    size_t total;
};

// Head dimensions: 64, 128 and 256 in the forward (256 with block 64: its Q and K / V
// tiles fill the shared memory); 128 in the backward (bwd = true).
nsa_status_t check_dims(int T, int nseq, int hq, int hkv, int d, int topk, int bs, Dims* D,
                        bool bwd = false) {
    if (T < 0 || nseq < 1 || hq < 1 || hkv < 1 || d < 1 || topk < 1 || bs < 1)
        return NSA_ERR_INVALID_ARG;
    if (hq % hkv != 0) return NSA_ERR_INVALID_ARG;
    if ((bs != 64 && bs != 128) || topk > kMaxTopk) return NSA_ERR_UNSUPPORTED;
    if (d != 64 && d != kHeadDim && d != 256) return NSA_ERR_UNSUPPORTED;
    // the backward runs d = 64 as d = 128 with the upper half read as zeros; d = 256 has no
    // shared memory for its Q / dO stages
    if ((d == 256 && bs != 64) || (bwd && d == 256)) return NSA_ERR_UNSUPPORTED;
    const int G = hq / hkv;
    if (G > kMaxGroup || kTileRows % G != 0) return NSA_ERR_UNSUPPORTED;
    if (T >= (1 << 25)) return NSA_ERR_UNSUPPORTED;
    const long long nent = (long long)T * hkv * topk;
    if (nent >= (1ll << 31)) return NSA_ERR_UNSUPPORTED;
    const long long nbk_cap = (long long)hkv * ((long long)T / bs + nseq);
    if (nbk_cap >= (1ll << 30)) return NSA_ERR_UNSUPPORTED;
    if ((long long)T * hq >= (1ll << 31)) return NSA_ERR_UNSUPPORTED;   // TMA row coordinate
    D->T = T; D->nseq = nseq; D->hq = hq; D->hkv = hkv; D->d = d; D->topk = topk; D->bs = bs;
    D->G = G;
    D->nent = nent;
    D->nbk_cap = (int)nbk_cap;
    int bits = 1;
    while ((1ll << bits) <= nbk_cap) ++bits;   // 2^bits > nbk_cap
    D->key_bits = bits;
    D->sort_tiles = (int)((nent + kSortTile - 1) / kSortTile);
    const int tpt = kTileRows / G;
    D->tiles_cap = (nent + tpt - 1) / tpt + nbk_cap;
    D->units_cap = (D->tiles_cap + kChunkTiles - 1) / kChunkTiles + nbk_cap;
    D->wtok = kWindowRows / G;
    D->nwin = std::max(1, (T + D->wtok - 1) / D->wtok);
    D->nb_stride = (int)((long long)T / bs + nseq);
    if ((long long)hkv * D->nwin * (D->nb_stride + 1) >= (1ll << 31)) return NSA_ERR_UNSUPPORTED;
    D->fwd_tiles_cap = (nent + tpt - 1) / tpt +
                       std::min<long long>(nent, (long long)hkv * D->nwin * D->nb_stride);
    // forward partial rows are addressed by 32-bit TMA row coordinates and row indices
    if (D->fwd_tiles_cap * kTileRows >= (1ll << 31)) return NSA_ERR_UNSUPPORTED;
    return NSA_OK;
}

Layout make_layout(const Dims& D, bool bwd) {
    Layout L{};
    size_t o = 0;
    auto take = [&](size_t bytes) { size_t at = o; o = align256(o + bytes); return at; };
    L.status = take(sizeof(DevStatus));
    L.blkoff = take(sizeof(int32_t) * (D.nseq + 1));
    L.keys0 = take(sizeof(uint32_t) * (size_t)std::max<long long>(D.nent, 1));
    L.keys1 = take(sizeof(uint32_t) * (size_t)std::max<long long>(D.nent, 1));
    L.vals0 = take(sizeof(uint32_t) * (size_t)std::max<long long>(D.nent, 1));
    L.vals1 = take(sizeof(uint32_t) * (size_t)std::max<long long>(D.nent, 1));
    L.hist = take(sizeof(uint32_t) * 256 * (size_t)std::max(D.sort_tiles, 1));
    L.digit_tot = take(sizeof(uint32_t) * 256);
    L.offsets = take(sizeof(int32_t) * ((size_t)D.nbk_cap + 1));
    L.tile_off = take(sizeof(int32_t) * ((size_t)D.nbk_cap + 1));
    L.chunk_off = take(sizeof(int32_t) * ((size_t)D.nbk_cap + 1));
    L.inv_end = o;   // everything the inversion alone touches lies below this offset
    const size_t wrows = (size_t)D.hkv * D.nwin;
    L.wstart = take(sizeof(int32_t) * (wrows * (size_t)D.nb_stride + 1));
    L.wtile_off = take(sizeof(int32_t) * wrows * ((size_t)D.nb_stride + 1));
    L.row_tiles = take(sizeof(int32_t) * wrows);
    L.row_off = take(sizeof(int32_t) * (wrows + 1));
    L.tile_desc = take(sizeof(int4) * (size_t)std::max<long long>(D.fwd_tiles_cap, 1));
    L.posmap = take(sizeof(int32_t) * (size_t)std::max<long long>(D.nent, 1));
    L.vexp = take(sizeof(int32_t) * ((size_t)D.nbk_cap + 1));
    // forward: one 128-row slot per tile; backward: one row per (token, head, slot)
    const size_t rows = std::max((size_t)D.T * D.hq * D.topk,
                                 (size_t)std::max<long long>(D.fwd_tiles_cap, 1) * kTileRows);
    // fp16 partial O (forward, d columns) / bf16 dQ (backward, 128 columns)
    L.part_o = take(rows * (size_t)(bwd ? std::max(D.d, kHeadDim) : D.d) * 2);
    L.part_lse = take(rows * sizeof(float2));  // (lse, exponent) per partial
    if (bwd) {
        L.delta = take(sizeof(float) * (size_t)D.hq * D.T);
        L.part_dkdv = take(sizeof(float) * 2 * (size_t)D.bs * kHeadDim * (size_t)D.units_cap);
        L.udesc = take(sizeof(int4) * (size_t)D.units_cap);
        L.ubucket = take(sizeof(int) * (size_t)D.units_cap);
        L.uorder = take(sizeof(int) * (size_t)D.units_cap);
    }
    L.total = o;
    return L;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// The current device must be an sm_100 part, and `stream` (when it is not one of the
// default-stream handles) must belong to it: the launches, the scratch of the
// no-allocation entry point and the SM count are all taken from the current device.
nsa_status_t check_device(int* num_sms, nsa_stream_t stream_) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NSA_ERR_NO_DEVICE;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (stream != nullptr && stream != cudaStreamLegacy && stream != cudaStreamPerThread) {
        int sdev = -1;
        if (cudaStreamGetDevice(stream, &sdev) != cudaSuccess) return NSA_ERR_INVALID_ARG;
        if (sdev != dev) return NSA_ERR_INVALID_ARG;
    }
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
        return NSA_ERR_NO_DEVICE;
    if (major != 10 || minor != 0) return NSA_ERR_NO_DEVICE;
    if (cudaDeviceGetAttribute(num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return NSA_ERR_NO_DEVICE;
    return NSA_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// Tensor map over a bf16 [T, hkv, 128] tensor; box = (64 columns, 1 head, bs keys),
// 128-byte swizzle (the layout the tensor-core descriptors expect).
bool make_kv_map(CUtensorMap* map, const void* base, int T, int hkv, int bs, bool f16,
                 int d = kHeadDim) {
    auto enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)hkv, (cuuint64_t)(T > 0 ? T : 1)};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)hkv * d * 2};
    cuuint32_t box[3] = {64, 1, (cuuint32_t)bs};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                     3, const_cast<void*>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Tensor map over a bf16 Q [T, hq, 128]; box = (64 columns, G heads, 128 / G tokens):
// one 128-row tile of G heads of consecutive tokens, rows token-major, 128-byte swizzle.
bool make_q_group_map(CUtensorMap* map, const void* base, int T, int hq, int G, bool f16 = false) {
    auto enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)kHeadDim, (cuuint64_t)hq, (cuuint64_t)(T > 0 ? T : 1)};
    cuuint64_t strides[2] = {(cuuint64_t)kHeadDim * 2, (cuuint64_t)hq * kHeadDim * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)G, (cuuint32_t)(kTileRows / G)};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                     3, const_cast<void*>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Tensor map over a bf16 / fp16 [rows, d] tensor (Q or dO viewed as [T * hq, d]); box =
// (64 columns, 1 row), 128-byte swizzle: the gather4 loads of the tile kernels.
bool make_row_map(CUtensorMap* map, const void* base, long long rows, bool f16, int d = kHeadDim) {
    auto enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)(rows > 0 ? rows : 1)};
    cuuint64_t strides[1] = {(cuuint64_t)d * 2};
    cuuint32_t box[2] = {64, 1};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                     2, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Tensor map over a bf16 / fp16 [T, hq, d] tensor as (d columns, hq heads, T tokens);
// box = (64 columns, G heads, 1 token), 128-byte swizzle: one token's G rows of a KV
// group (G >= 8: whole 1 KB swizzle atoms).
bool make_token_map(CUtensorMap* map, const void* base, int T, int hq, int G, bool f16,
                    int d = kHeadDim) {
    auto enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)hq, (cuuint64_t)(T > 0 ? T : 1)};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)hq * d * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)G, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                     3, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Tensor map over the forward partials, fp16 [rows, 128]; box = (64 columns, box_rows),
// 128-byte swizzle: the epilogue's TMA stores of 8-row groups and of whole warps.
bool make_part_map(CUtensorMap* map, void* base, long long rows, int box_rows, int d = kHeadDim) {
    auto enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)d * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, base, dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

struct Carved {
    DevStatus* st;
    InvertPlan inv;
    uint8_t* base;
    Layout L;
};

Carved carve(const Dims& D, const Layout& L, void* ws, const int32_t* cu, const int32_t* bidx,
             int swin = 0) {
    Carved c{};
    uint8_t* b = static_cast<uint8_t*>(ws);
    c.base = b;
    c.L = L;
    c.st = reinterpret_cast<DevStatus*>(b + L.status);
    InvertPlan& p = c.inv;
    p.cu = cu;
    p.nseq = D.nseq;
    p.T = D.T;
    p.hkv = D.hkv;
    p.bidx = bidx;
    p.topk = D.topk;
    p.bs = D.bs;
    p.swin = swin;
    p.tokens_per_tile = kTileRows / D.G;
    p.chunk_tiles = kChunkTiles;
    p.nent = D.nent;
    p.nbk_cap = D.nbk_cap;
    p.key_bits = D.key_bits;
    p.sort_tiles = D.sort_tiles;
    p.blkoff = reinterpret_cast<int32_t*>(b + L.blkoff);
    p.keys[0] = reinterpret_cast<uint32_t*>(b + L.keys0);
    p.keys[1] = reinterpret_cast<uint32_t*>(b + L.keys1);
    p.vals[0] = reinterpret_cast<uint32_t*>(b + L.vals0);
    p.vals[1] = reinterpret_cast<uint32_t*>(b + L.vals1);
    p.hist = reinterpret_cast<uint32_t*>(b + L.hist);
    p.digit_tot = reinterpret_cast<uint32_t*>(b + L.digit_tot);
    p.offsets = reinterpret_cast<int32_t*>(b + L.offsets);
    p.tile_off = reinterpret_cast<int32_t*>(b + L.tile_off);
    p.chunk_off = reinterpret_cast<int32_t*>(b + L.chunk_off);
    p.wstart = nullptr;   // set by the forward, which needs the window runs
    p.nwin = 1;
    p.wtok = 1;
    p.st = c.st;
    // identity of the inversion's inputs: the index arrays and every size it depends on
    unsigned long long h = 1469598103934665603ull;
    for (unsigned long long x : {(unsigned long long)(uintptr_t)cu, (unsigned long long)(uintptr_t)bidx,
                                 (unsigned long long)D.T, (unsigned long long)D.nseq,
                                 (unsigned long long)D.hkv, (unsigned long long)D.topk,
                                 (unsigned long long)D.bs, (unsigned long long)D.G,
                                 (unsigned long long)kChunkTiles, (unsigned long long)swin}) {
        h ^= x;
        h *= 1099511628211ull;
    }
    p.tag = h;
    p.final_buf = 0;
    return c;
}

nsa_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? NSA_OK : NSA_ERR_CUDA; }

// Common checks of the index inputs and the workspace; returns NSA_OK and fills D.
nsa_status_t check_common(const int32_t* cu, int nseq, int T, int hq, int hkv, int d,
                          const int32_t* bidx, int topk, int bs, void* ws, size_t ws_bytes,
                          bool bwd, Dims* D) {
    nsa_status_t s = check_dims(T, nseq, hq, hkv, d, topk, bs, D, bwd);
    if (s != NSA_OK) return s;
    if (!cu || !ws || (T > 0 && !bidx)) return NSA_ERR_INVALID_ARG;
    if (!aligned(cu, 4) || !aligned(bidx, 4) || !aligned(ws, 256)) return NSA_ERR_INVALID_ARG;
    if (ws_bytes < make_layout(*D, bwd).total) return NSA_ERR_WORKSPACE;
    return NSA_OK;
}

}  // namespace

extern "C" {

size_t nsa_sel_attn_workspace_size(int total_tokens, int num_seqs, int hq, int hkv, int head_dim,
                                   int topk, int block_size, int for_bwd) {
    Dims D;
    if (check_dims(total_tokens, num_seqs, hq, hkv, head_dim, topk, block_size, &D, for_bwd != 0) !=
        NSA_OK)
        return 0;
    return make_layout(D, for_bwd != 0).total;
}

const char* nsa_sel_status_string(nsa_status_t s) {
    switch (s) {
        case NSA_OK: return "ok";
        case NSA_ERR_INVALID_ARG: return "invalid argument";
        case NSA_ERR_UNSUPPORTED: return "unsupported shape or parameter";
        case NSA_ERR_WORKSPACE: return "workspace too small";
        case NSA_ERR_CUDA: return "CUDA error";
        case NSA_ERR_TIMEOUT: return "device-side wait timed out";
        case NSA_ERR_BAD_INDEX: return "invalid block_idx or cu_seqlens";
        case NSA_ERR_NO_DEVICE: return "no sm_100 device is current";
    }
    return "unknown status";
}

}  // extern "C"

namespace {

// Records ev[i] (when given) on the stream at phase boundary i.
struct PhaseMarks {
    void* const* ev;
    int n;
    cudaStream_t stream;
    int* launches;
    void mark(int i) const {
        if (ev && i < n && ev[i]) cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), stream);
    }
    void add(int k) const {
        if (launches) *launches += k;
    }
};

int invert_launches(const Dims& D) {
    const int passes = D.key_bits <= 8 ? 1 : (D.key_bits + 7) / 8;
    return 1 + 3 * passes + 2;
}

nsa_status_t fwd_impl(const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                      int num_seqs, int total_tokens, int hq, int hkv, int head_dim,
                      const int32_t* block_idx, int topk, int block_size, float scale, void* out,
                      float* lse, void* workspace, size_t workspace_bytes, nsa_stream_t stream_,
                      void* const* events, int num_events, int* launches, bool f16, int swin,
                      bool test_short_waits = false, bool test_skip_arrive = false) {
    Dims D;
    nsa_status_t s = check_common(cu_seqlens, num_seqs, total_tokens, hq, hkv, head_dim,
                                  block_idx, topk, block_size, workspace, workspace_bytes, false, &D);
    if (s != NSA_OK) return s;
    if (total_tokens > 0 && (!q || !k || !v || !out)) return NSA_ERR_INVALID_ARG;   // lse may be null
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
        !aligned(lse, 4))
        return NSA_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !(scale < 1e30f) || swin < 0) return NSA_ERR_INVALID_ARG;
    int num_sms = 0;
    if ((s = check_device(&num_sms, stream_)) != NSA_OK) return s;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    const Layout L = make_layout(D, false);
    Carved c = carve(D, L, workspace, cu_seqlens, block_idx, swin);
    const PhaseMarks pm{events, num_events, stream, launches};
    if (launches) *launches = 0;
    pm.mark(0);
    if (cudaMemsetAsync(c.st, 0, sizeof(DevStatus), stream) != cudaSuccess) return NSA_ERR_CUDA;
    if (test_short_waits &&   // low four bytes 0x01 each: a budget of 0x01010101 cycles
        cudaMemsetAsync(&c.st->wait_budget, 0x01, 4, stream) != cudaSuccess)
        return NSA_ERR_CUDA;
    if (total_tokens == 0) {
        for (int i = 1; i < 4; ++i) pm.mark(i);
        return NSA_OK;
    }

    CUtensorMap kmap, vmap;
    if (!make_kv_map(&kmap, k, D.T, D.hkv, D.bs, f16, D.d) ||
        !make_kv_map(&vmap, v, D.T, D.hkv, D.bs, f16, D.d))
        return NSA_ERR_CUDA;
    c.inv.wstart = reinterpret_cast<int32_t*>(c.base + L.wstart);
    c.inv.nwin = D.nwin;
    c.inv.wtok = D.wtok;
    if ((s = cuda_status(launch_invert(c.inv, stream))) != NSA_OK) return s;
    WindowPlan wp{};
    wp.nwin = D.nwin;
    wp.wtok = D.wtok;
    wp.nb_stride = D.nb_stride;
    wp.tile_off = reinterpret_cast<int32_t*>(c.base + L.wtile_off);
    wp.row_tiles = reinterpret_cast<int32_t*>(c.base + L.row_tiles);
    wp.row_off = reinterpret_cast<int32_t*>(c.base + L.row_off);
    wp.tile_desc = reinterpret_cast<int4*>(c.base + L.tile_desc);
    wp.tiles_cap = D.fwd_tiles_cap;
    if ((s = cuda_status(launch_window_split(c.inv, wp, stream))) != NSA_OK) return s;
    int32_t* posmap = reinterpret_cast<int32_t*>(c.base + L.posmap);
    if ((s = cuda_status(launch_posmap(c.inv, wp, posmap, stream))) != NSA_OK) return s;
    pm.add(invert_launches(D) + 4);
    pm.mark(1);

    FwdPlan fp{};
    fp.q = q;
    fp.cu = cu_seqlens;
    fp.nseq = D.nseq; fp.T = D.T; fp.hq = D.hq; fp.hkv = D.hkv; fp.topk = D.topk; fp.bs = D.bs;
    fp.G = D.G;
    fp.d = D.d;
    fp.f16 = f16 ? 1 : 0;
    fp.swin = swin;
    fp.scale_log2 = scale * 1.4426950408889634f;
    fp.blkoff = c.inv.blkoff;
    fp.offsets = c.inv.offsets;
    fp.tile_off = c.inv.tile_off;
    fp.entries = c.inv.vals[c.inv.final_buf];
    fp.nbk_cap = D.nbk_cap;
    fp.nwin = wp.nwin;
    fp.nb_stride = wp.nb_stride;
    fp.wtile_off = wp.tile_off;
    fp.row_off = wp.row_off;
    fp.tile_desc = wp.tile_desc;
    fp.part_o = c.base + L.part_o;
    fp.part_meta = reinterpret_cast<float2*>(c.base + L.part_lse);
    fp.st = c.st;
    fp.num_sms = num_sms;
    fp.test_skip_arrive = test_skip_arrive ? 1 : 0;
    int32_t* vexp = reinterpret_cast<int32_t*>(c.base + L.vexp);
    fp.vexp = vexp;
    if ((s = cuda_status(launch_vblock_exp(fp, v, D.nb_stride, vexp, stream))) != NSA_OK) return s;
    CUtensorMap omap[2];
    const long long prow = std::max<long long>(D.fwd_tiles_cap, 1) * kTileRows;
    if (!make_part_map(&omap[0], fp.part_o, prow, 8, D.d) ||
        !make_part_map(&omap[1], fp.part_o, prow, 32, D.d))
        return NSA_ERR_CUDA;
    if ((s = cuda_status(launch_fwd_tiles(fp, &kmap, &vmap, omap, stream))) != NSA_OK) return s;
    pm.add(2);
    pm.mark(2);

    MergePlan mp{};
    mp.cu = cu_seqlens;
    mp.nseq = D.nseq; mp.T = D.T; mp.hq = D.hq; mp.hkv = D.hkv; mp.topk = D.topk; mp.bs = D.bs;
    mp.G = D.G;
    mp.d = D.d;
    mp.f16 = f16 ? 1 : 0;
    mp.swin = swin;
    mp.bidx = block_idx;
    mp.posmap = posmap;
    mp.part_o = fp.part_o;
    mp.part_meta = fp.part_meta;
    mp.out = out;
    mp.lse = lse;
    mp.st = c.st;
    if ((s = cuda_status(launch_merge(mp, stream))) != NSA_OK) return s;
    pm.add(1);
    pm.mark(3);
    return NSA_OK;
}

nsa_status_t bwd_impl(const void* q, const void* k, const void* v, const void* out,
                      const float* lse, const void* dout, const int32_t* cu_seqlens, int num_seqs,
                      int total_tokens, int hq, int hkv, int head_dim, const int32_t* block_idx,
                      int topk, int block_size, float scale, void* dq, void* dk, void* dv,
                      void* workspace, size_t workspace_bytes, nsa_stream_t stream_,
                      void* const* events, int num_events, int* launches, bool reuse_index,
                      bool f16, int swin) {
    Dims D;
    nsa_status_t s = check_common(cu_seqlens, num_seqs, total_tokens, hq, hkv, head_dim,
                                  block_idx, topk, block_size, workspace, workspace_bytes, true, &D);
    if (s != NSA_OK) return s;
    if (total_tokens > 0 && (!q || !k || !v || !out || !lse || !dout || !dq || !dk || !dv))
        return NSA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
        !aligned(dout, 16) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) ||
        !aligned(lse, 4))
        return NSA_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !(scale < 1e30f) || swin < 0) return NSA_ERR_INVALID_ARG;
    int num_sms = 0;
    if ((s = check_device(&num_sms, stream_)) != NSA_OK) return s;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    const Layout L = make_layout(D, true);
    Carved c = carve(D, L, workspace, cu_seqlens, block_idx, swin);
    const PhaseMarks pm{events, num_events, stream, launches};
    if (launches) *launches = 0;
    pm.mark(0);
    // a reused inversion keeps the status block the forward left (its counts, any error)
    if (!reuse_index && cudaMemsetAsync(c.st, 0, sizeof(DevStatus), stream) != cudaSuccess)
        return NSA_ERR_CUDA;
    if (total_tokens == 0) {
        for (int i = 1; i < 6; ++i) pm.mark(i);
        return NSA_OK;
    }

    CUtensorMap kmap, vmap;
    // d = 64: the maps cover the d columns, and the kernel's loads of columns 64..127 lie
    // outside them and read as zeros
    if (!make_kv_map(&kmap, k, D.T, D.hkv, D.bs, f16, D.d) ||
        !make_kv_map(&vmap, v, D.T, D.hkv, D.bs, f16, D.d))
        return NSA_ERR_CUDA;
    if (reuse_index) {
        c.inv.final_buf = invert_final_buf(c.inv);
    } else {
        if ((s = cuda_status(launch_invert(c.inv, stream))) != NSA_OK) return s;
        pm.add(invert_launches(D));
    }
    int4* udesc = reinterpret_cast<int4*>(c.base + L.udesc);
    int* ubucket = reinterpret_cast<int*>(c.base + L.ubucket);
    if ((s = cuda_status(launch_unit_desc(c.inv, D.units_cap, udesc, ubucket, reuse_index,
                                          stream))) != NSA_OK)
        return s;
    int* uorder = reinterpret_cast<int*>(c.base + L.uorder);
    if ((s = cuda_status(launch_unit_order(c.st, udesc, uorder, stream))) != NSA_OK) return s;
    pm.add(2);
    pm.mark(1);

    BwdPlan bp{};
    bp.q = q;
    bp.dout = dout;
    bp.lse = lse;
    bp.delta = reinterpret_cast<float*>(c.base + L.delta);
    bp.cu = cu_seqlens;
    bp.nseq = D.nseq; bp.T = D.T; bp.hq = D.hq; bp.hkv = D.hkv; bp.topk = D.topk; bp.bs = D.bs;
    bp.G = D.G;
    bp.d = D.d;
    bp.f16 = f16 ? 1 : 0;
    bp.swin = swin;
    bp.scale = scale;
    bp.scale_log2 = scale * 1.4426950408889634f;
    bp.blkoff = c.inv.blkoff;
    bp.offsets = c.inv.offsets;
    bp.tile_off = c.inv.tile_off;
    bp.chunk_off = c.inv.chunk_off;
    bp.entries = c.inv.vals[c.inv.final_buf];
    bp.nbk_cap = D.nbk_cap;
    bp.chunk_tiles = kChunkTiles;
    bp.udesc = udesc;
    bp.ubucket = ubucket;
    bp.uorder = uorder;
    bp.part_dq = c.base + L.part_o;
    bp.part_dkdv = reinterpret_cast<float*>(c.base + L.part_dkdv);
    bp.st = c.st;
    bp.num_sms = num_sms;
    if ((s = cuda_status(launch_bwd_preprocess(out, dout, bp.delta, D.T, D.hq, D.d, bp.f16, stream))) != NSA_OK)
        return s;
    pm.add(1);
    pm.mark(2);
    // G >= 8: 3D maps (columns, heads, tokens) with a box of one token's G heads, whole
    // swizzle atoms; otherwise 2D row maps for the four-row gathers
    CUtensorMap qmap, domap;
    if (D.G >= 8) {
        if (!make_token_map(&qmap, q, D.T, D.hq, D.G, f16, D.d) ||
            !make_token_map(&domap, dout, D.T, D.hq, D.G, f16, D.d))
            return NSA_ERR_CUDA;
    } else if (!make_row_map(&qmap, q, (long long)D.T * D.hq, f16, D.d) ||
               !make_row_map(&domap, dout, (long long)D.T * D.hq, f16, D.d)) {
        return NSA_ERR_CUDA;
    }
    if ((s = cuda_status(launch_bwd_tiles(bp, &kmap, &vmap, &qmap, &domap, stream))) != NSA_OK) return s;
    pm.add(1);
    pm.mark(3);
    if ((s = cuda_status(launch_bwd_dq_merge(bp, block_idx, dq, stream))) != NSA_OK) return s;
    pm.add(1);
    pm.mark(4);
    if ((s = cuda_status(launch_bwd_dkdv_reduce(bp, dk, dv, stream))) != NSA_OK) return s;
    pm.add(1);
    pm.mark(5);
    return NSA_OK;
}

}  // namespace

extern "C" {

nsa_status_t nsa_sel_attn_fwd(const void* q, const void* k, const void* v,
                              const int32_t* cu_seqlens, int num_seqs, int total_tokens, int hq,
                              int hkv, int head_dim, const int32_t* block_idx, int topk,
                              int block_size, float scale, void* out, float* lse, void* workspace,
                              size_t workspace_bytes, nsa_stream_t stream) {
    return fwd_impl(q, k, v, cu_seqlens, num_seqs, total_tokens, hq, hkv, head_dim, block_idx,
                    topk, block_size, scale, out, lse, workspace, workspace_bytes, stream, nullptr,
                    0, nullptr, false, 0);
}

nsa_status_t nsa_sel_attn_fwd_profiled(const void* q, const void* k, const void* v,
                                       const int32_t* cu_seqlens, int num_seqs, int total_tokens,
                                       int hq, int hkv, int head_dim, const int32_t* block_idx,
                                       int topk, int block_size, float scale, void* out,
                                       float* lse, void* workspace, size_t workspace_bytes,
                                       nsa_stream_t stream, void* const* events, int num_events,
                                       int* num_launches) {
    return fwd_impl(q, k, v, cu_seqlens, num_seqs, total_tokens, hq, hkv, head_dim, block_idx,
                    topk, block_size, scale, out, lse, workspace, workspace_bytes, stream, events,
                    num_events, num_launches, false, 0);
}

nsa_status_t nsa_sel_attn_fwd_ex(const void* q, const void* k, const void* v,
                                 const int32_t* cu_seqlens, int num_seqs, int total_tokens, int hq,
                                 int hkv, int head_dim, const int32_t* block_idx, int topk,
                                 int block_size, float scale, void* out, float* lse,
                                 void* workspace, size_t workspace_bytes, nsa_stream_t stream,
                                 unsigned flags, int window_size, void* const* events,
                                 int num_events, int* num_launches) {
    if (flags & ~(unsigned)(NSA_F16 | NSA_TEST_SHORT_WAITS | NSA_TEST_SKIP_ARRIVE))
        return NSA_ERR_INVALID_ARG;
    return fwd_impl(q, k, v, cu_seqlens, num_seqs, total_tokens, hq, hkv, head_dim, block_idx,
                    topk, block_size, scale, out, lse, workspace, workspace_bytes, stream, events,
                    num_events, num_launches, (flags & NSA_F16) != 0, window_size,
                    (flags & NSA_TEST_SHORT_WAITS) != 0, (flags & NSA_TEST_SKIP_ARRIVE) != 0);
}

nsa_status_t nsa_sel_attn_bwd(const void* q, const void* k, const void* v, const void* out,
                              const float* lse, const void* dout, const int32_t* cu_seqlens,
                              int num_seqs, int total_tokens, int hq, int hkv, int head_dim,
                              const int32_t* block_idx, int topk, int block_size, float scale,
                              void* dq, void* dk, void* dv, void* workspace,
                              size_t workspace_bytes, nsa_stream_t stream) {
    return bwd_impl(q, k, v, out, lse, dout, cu_seqlens, num_seqs, total_tokens, hq, hkv,
                    head_dim, block_idx, topk, block_size, scale, dq, dk, dv, workspace,
                    workspace_bytes, stream, nullptr, 0, nullptr, false, false, 0);
}

nsa_status_t nsa_sel_attn_bwd_profiled(const void* q, const void* k, const void* v,
                                       const void* out, const float* lse, const void* dout,
                                       const int32_t* cu_seqlens, int num_seqs, int total_tokens,
                                       int hq, int hkv, int head_dim, const int32_t* block_idx,
                                       int topk, int block_size, float scale, void* dq, void* dk,
                                       void* dv, void* workspace, size_t workspace_bytes,
                                       nsa_stream_t stream, void* const* events, int num_events,
                                       int* num_launches) {
    return bwd_impl(q, k, v, out, lse, dout, cu_seqlens, num_seqs, total_tokens, hq, hkv,
                    head_dim, block_idx, topk, block_size, scale, dq, dk, dv, workspace,
                    workspace_bytes, stream, events, num_events, num_launches, false, false, 0);
}

nsa_status_t nsa_sel_attn_bwd_ex(const void* q, const void* k, const void* v, const void* out,
                                 const float* lse, const void* dout, const int32_t* cu_seqlens,
                                 int num_seqs, int total_tokens, int hq, int hkv, int head_dim,
                                 const int32_t* block_idx, int topk, int block_size, float scale,
                                 void* dq, void* dk, void* dv, void* workspace,
                                 size_t workspace_bytes, nsa_stream_t stream, unsigned flags,
                                 int window_size, void* const* events, int num_events,
                                 int* num_launches) {
    if (flags & ~(unsigned)(NSA_BWD_REUSE_INDEX | NSA_F16)) return NSA_ERR_INVALID_ARG;
    return bwd_impl(q, k, v, out, lse, dout, cu_seqlens, num_seqs, total_tokens, hq, hkv,
                    head_dim, block_idx, topk, block_size, scale, dq, dk, dv, workspace,
                    workspace_bytes, stream, events, num_events, num_launches,
                    (flags & NSA_BWD_REUSE_INDEX) != 0, (flags & NSA_F16) != 0, window_size);
}

nsa_status_t nsa_sel_invert_index(const int32_t* cu_seqlens, int num_seqs, int total_tokens,
                                  int hkv, const int32_t* block_idx, int topk, int block_size,
                                  int32_t* offsets, int32_t* entries, int32_t* counts,
                                  void* workspace, size_t workspace_bytes, nsa_stream_t stream_) {
    Dims D;
    // hq = hkv (group 1) fixes the tile geometry; it does not change the inversion.
    nsa_status_t s = check_common(cu_seqlens, num_seqs, total_tokens, hkv, hkv, kHeadDim,
                                  block_idx, topk, block_size, workspace, workspace_bytes, false, &D);
    if (s != NSA_OK) return s;
    if (!offsets || !entries || !counts || !aligned(offsets, 4) || !aligned(entries, 4) ||
        !aligned(counts, 4))
        return NSA_ERR_INVALID_ARG;
    int num_sms = 0;
    if ((s = check_device(&num_sms, stream_)) != NSA_OK) return s;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    const Layout L = make_layout(D, false);
    Carved c = carve(D, L, workspace, cu_seqlens, block_idx);
    if (cudaMemsetAsync(c.st, 0, sizeof(DevStatus), stream) != cudaSuccess) return NSA_ERR_CUDA;
    if (total_tokens == 0) {
        if (cudaMemsetAsync(counts, 0, 2 * sizeof(int32_t), stream) != cudaSuccess ||
            cudaMemsetAsync(offsets, 0, sizeof(int32_t) * ((size_t)D.nbk_cap + 1), stream) !=
                cudaSuccess)
            return NSA_ERR_CUDA;
        return NSA_OK;
    }
    if ((s = cuda_status(launch_invert(c.inv, stream))) != NSA_OK) return s;
    cudaError_t e = cudaMemcpyAsync(offsets, c.inv.offsets, sizeof(int32_t) * ((size_t)D.nbk_cap + 1),
                                    cudaMemcpyDeviceToDevice, stream);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(entries, c.inv.vals[c.inv.final_buf], sizeof(int32_t) * (size_t)D.nent,
                            cudaMemcpyDeviceToDevice, stream);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(counts, &c.st->nblocks_total, sizeof(int32_t), cudaMemcpyDeviceToDevice,
                            stream);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(counts + 1, &c.st->nentries, sizeof(int32_t), cudaMemcpyDeviceToDevice,
                            stream);
    return cuda_status(e);
}

nsa_status_t nsa_sel_validate_indices(const int32_t* cu_seqlens, int num_seqs, int total_tokens,
                                      int hkv, const int32_t* block_idx, int topk, int block_size,
                                      long long* n_out_of_range, long long* n_duplicates,
                                      void* workspace, size_t workspace_bytes,
                                      nsa_stream_t stream_) {
    if (!workspace || workspace_bytes < sizeof(DevStatus) || !aligned(workspace, 256))
        return NSA_ERR_WORKSPACE;
    if (!cu_seqlens || num_seqs < 1 || total_tokens < 0 || hkv < 1 || topk < 1 ||
        block_size < 1 || (total_tokens > 0 && !block_idx))
        return NSA_ERR_INVALID_ARG;
    int num_sms = 0;
    nsa_status_t s;
    if ((s = check_device(&num_sms, stream_)) != NSA_OK) return s;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    DevStatus* st = static_cast<DevStatus*>(workspace);
    if (cudaMemsetAsync(st, 0, sizeof(DevStatus), stream) != cudaSuccess) return NSA_ERR_CUDA;
    if ((s = cuda_status(launch_validate(cu_seqlens, num_seqs, total_tokens, hkv, block_idx, topk,
                                         block_size, st, stream))) != NSA_OK)
        return s;
    DevStatus h;
    if (cudaMemcpyAsync(&h, st, sizeof(DevStatus), cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
        return NSA_ERR_CUDA;
    if (n_out_of_range) *n_out_of_range = h.bad_range;
    if (n_duplicates) *n_duplicates = h.bad_dup;
    return (h.bad_range || h.bad_dup) ? NSA_ERR_BAD_INDEX : NSA_OK;
}

nsa_status_t nsa_sel_compress_kv(const void* k, const void* v, const int32_t* cu_seqlens,
                                 int num_seqs, int total_tokens, int hkv, int head_dim,
                                 int kernel_size, int kernel_stride, unsigned flags, void* k_cmp,
                                 void* v_cmp, int32_t* cu_cmp, nsa_stream_t stream_) {
    if (flags & ~(unsigned)NSA_F16) return NSA_ERR_INVALID_ARG;
    if (total_tokens < 0 || num_seqs < 1 || hkv < 1 || kernel_stride < 1 ||
        kernel_size < kernel_stride)
        return NSA_ERR_INVALID_ARG;
    if (head_dim != kHeadDim || kernel_size > 4096 || total_tokens >= (1 << 25))
        return NSA_ERR_UNSUPPORTED;
    if (!cu_seqlens || !cu_cmp || (total_tokens >= kernel_stride && (!k || !v || !k_cmp || !v_cmp)))
        return NSA_ERR_INVALID_ARG;
    if (!aligned(cu_seqlens, 4) || !aligned(cu_cmp, 4) || !aligned(k, 16) || !aligned(v, 16) ||
        !aligned(k_cmp, 16) || !aligned(v_cmp, 16))
        return NSA_ERR_INVALID_ARG;
    int num_sms = 0;
    nsa_status_t s = check_device(&num_sms, stream_);
    if (s != NSA_OK) return s;
    return cuda_status(launch_compress_kv(k, v, cu_seqlens, num_seqs, total_tokens, hkv, kernel_size,
                                          kernel_stride, (flags & NSA_F16) ? 1 : 0, cu_cmp, k_cmp,
                                          v_cmp, reinterpret_cast<cudaStream_t>(stream_)));
}

size_t nsa_sel_block_scores_workspace_size(int num_seqs) {
    return num_seqs < 1 ? 0 : align256(sizeof(DevStatus)) + align256(sizeof(int32_t) * ((size_t)num_seqs + 1));
}

nsa_status_t nsa_sel_block_scores(const void* q, const void* k_cmp, int k_cmp_rows,
                                  const int32_t* cu_seqlens, const int32_t* cu_cmp, int num_seqs,
                                  int total_tokens, int hq, int hkv, int head_dim, int block_size,
                                  int kernel_size, int kernel_stride, float scale, int nb_stride,
                                  float* scores, void* workspace, size_t workspace_bytes,
                                  nsa_stream_t stream_) {
    if (total_tokens < 0 || num_seqs < 1 || hq < 1 || hkv < 1 || hq % hkv != 0 ||
        nb_stride < 1 || k_cmp_rows < 1)
        return NSA_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !(scale < 1e30f)) return NSA_ERR_INVALID_ARG;
    const int G = hq / hkv;
    if (head_dim != kHeadDim || kernel_size != 32 || kernel_stride != 16 ||
        (block_size != 64 && block_size != 128) || G > 32 || 32 % G != 0 ||
        total_tokens >= (1 << 25) || (long long)total_tokens * hkv * nb_stride >= (1ll << 40))
        return NSA_ERR_UNSUPPORTED;
    if (!cu_seqlens || !cu_cmp || !workspace || !k_cmp || (total_tokens > 0 && (!q || !scores)))
        return NSA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k_cmp, 16) || !aligned(cu_seqlens, 4) || !aligned(cu_cmp, 4) ||
        !aligned(scores, 4) || !aligned(workspace, 256))
        return NSA_ERR_INVALID_ARG;
    if (workspace_bytes < nsa_sel_block_scores_workspace_size(num_seqs)) return NSA_ERR_WORKSPACE;
    int num_sms = 0;
    nsa_status_t s = check_device(&num_sms, stream_);
    if (s != NSA_OK) return s;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    DevStatus* st = static_cast<DevStatus*>(workspace);
    int32_t* tile_off = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(workspace) +
                                                   align256(sizeof(DevStatus)));
    if (cudaMemsetAsync(st, 0, sizeof(DevStatus), stream) != cudaSuccess) return NSA_ERR_CUDA;
    if (total_tokens == 0) return NSA_OK;
    CUtensorMap qmap, kcmap;
    if (!make_q_group_map(&qmap, q, total_tokens, hq, G) ||
        !make_kv_map(&kcmap, k_cmp, k_cmp_rows, hkv, 64, false))
        return NSA_ERR_CUDA;
    return cuda_status(launch_cmp_scores(q, k_cmp, k_cmp_rows, cu_seqlens, cu_cmp, num_seqs,
                                         total_tokens, hq, hkv, nb_stride, block_size, scale,
                                         scores, tile_off, st, num_sms, &qmap, &kcmap, stream));
}

size_t nsa_sel_bsfa_workspace_size(int num_seqs) { return nsa_sel_block_scores_workspace_size(num_seqs); }

nsa_status_t nsa_sel_bsfa_fwd(const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                          int num_seqs, int total_tokens, int hq, int hkv, int head_dim,
                          int block_size, float scale, const float* tau, void* out, float* lse,
                          void* workspace, size_t workspace_bytes, nsa_stream_t stream_) {
    if (total_tokens < 0 || num_seqs < 1 || hq < 1 || hkv < 1 || hq % hkv != 0)
        return NSA_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !(scale < 1e30f)) return NSA_ERR_INVALID_ARG;
    const int G = hq / hkv;
    if (head_dim != kHeadDim || block_size != 64 || kTileRows % G != 0 ||
        total_tokens >= (1 << 25) || (long long)total_tokens * hq >= (1ll << 31))
        return NSA_ERR_UNSUPPORTED;
    if (!cu_seqlens || !workspace || (total_tokens > 0 && (!q || !k || !v || !tau || !out)))
        return NSA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
        !aligned(cu_seqlens, 4) || !aligned(tau, 4) || !aligned(lse, 4) || !aligned(workspace, 256))
        return NSA_ERR_INVALID_ARG;
    if (workspace_bytes < nsa_sel_bsfa_workspace_size(num_seqs)) return NSA_ERR_WORKSPACE;
    int num_sms = 0;
    nsa_status_t s = check_device(&num_sms, stream_);
    if (s != NSA_OK) return s;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    DevStatus* st = static_cast<DevStatus*>(workspace);
    int32_t* tile_off = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(workspace) +
                                                   align256(sizeof(DevStatus)));
    if (cudaMemsetAsync(st, 0, sizeof(DevStatus), stream) != cudaSuccess) return NSA_ERR_CUDA;
    if (total_tokens == 0) return NSA_OK;
    CUtensorMap qmap, kmap, vmap;
    if (!make_q_group_map(&qmap, q, total_tokens, hq, G) ||
        !make_kv_map(&kmap, k, total_tokens, hkv, 64, false) ||
        !make_kv_map(&vmap, v, total_tokens, hkv, 64, false))
        return NSA_ERR_CUDA;
    return cuda_status(launch_bsfa_fwd(cu_seqlens, num_seqs, total_tokens, hq, hkv, scale, tau, out,
                                       lse, tile_off, st, num_sms, &qmap, &kmap, &vmap, stream));
}

nsa_status_t nsa_sel_select_topk(const float* scores, const int32_t* cu_seqlens, int num_seqs,
                                 int total_tokens, int hkv, int nb_stride, int block_size,
                                 int topk, int init_blocks, int local_blocks, int32_t* block_idx,
                                 void* workspace, size_t workspace_bytes, nsa_stream_t stream_) {
    if (total_tokens < 0 || num_seqs < 1 || hkv < 1 || nb_stride < 1 || block_size < 1 ||
        topk < 1 || init_blocks < 0 || local_blocks < 0)
        return NSA_ERR_INVALID_ARG;
    if (topk > kMaxTopk || nb_stride > 1024 || total_tokens >= (1 << 25) ||
        (long long)total_tokens * hkv * nb_stride >= (1ll << 40))
        return NSA_ERR_UNSUPPORTED;
    if (!cu_seqlens || !workspace || (total_tokens > 0 && (!scores || !block_idx)))
        return NSA_ERR_INVALID_ARG;
    if (!aligned(cu_seqlens, 4) || !aligned(scores, 4) || !aligned(block_idx, 4) ||
        !aligned(workspace, 256))
        return NSA_ERR_INVALID_ARG;
    if (workspace_bytes < sizeof(DevStatus)) return NSA_ERR_WORKSPACE;
    int num_sms = 0;
    nsa_status_t s = check_device(&num_sms, stream_);
    if (s != NSA_OK) return s;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    DevStatus* st = static_cast<DevStatus*>(workspace);
    if (cudaMemsetAsync(st, 0, sizeof(DevStatus), stream) != cudaSuccess) return NSA_ERR_CUDA;
    return cuda_status(launch_select_topk(scores, cu_seqlens, num_seqs, total_tokens, hkv, nb_stride,
                                          block_size, topk, init_blocks, local_blocks, block_idx,
                                          st, stream));
}

nsa_status_t nsa_sel_check_status(const void* workspace, nsa_stream_t stream_) {
    if (!workspace || !aligned(workspace, 256)) return NSA_ERR_INVALID_ARG;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    int code = 0;
    if (cudaMemcpyAsync(&code, workspace, sizeof(int), cudaMemcpyDeviceToHost, stream) !=
            cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
        return NSA_ERR_CUDA;
    return static_cast<nsa_status_t>(code);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Index inversion with library-owned scratch.
//
// For callers that cannot allocate device memory themselves -- a plug-in running
// inside a framework that owns every byte of device memory and gives plug-ins no
// allocation hook, or a latency-critical loop where cudaMalloc (which may
// synchronise the device) is not allowed -- this entry point takes its scratch from
// a fixed array in the library's own device data instead of a caller workspace.
//
// The array (kInvertScratchBytes, 64 MiB) exists once per device that loads the
// library and stays allocated until the process exits.  Its device address is looked
// up with cudaGetSymbolAddress the first time the entry point runs on a device (with
// that device current); make that first call before any stream capture.  All calls
// share the array and it keeps the last call's contents (everything a call reads is
// first written by the same call, and its status block is cleared on entry), so
// calls whose work overlaps on the GPU -- on different streams, or from different
// host threads -- race with one another: serialise them.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kInvertScratchBytes = size_t(64) << 20;
__device__ __align__(256) unsigned char g_invert_scratch[kInvertScratchBytes];

constexpr int kMaxScratchDevices = 64;
std::mutex g_scratch_mutex;
struct ScratchSlot {
    unsigned long long ctx_id;   // the context the address was resolved in (0: none yet)
    void* ptr;
};
ScratchSlot g_scratch[kMaxScratchDevices] = {};

// Driver-API context identity (through the runtime's entry-point query, so that the
// library links no driver library): a device's primary context that was torn down and
// created again gets a new id, and the module (with its array) is loaded anew.
using PfnCtxGetCurrent = CUresult (*)(CUcontext*);
using PfnCtxGetId = CUresult (*)(CUcontext, unsigned long long*);
bool current_context_id(unsigned long long* id) {
    static std::once_flag once;
    static PfnCtxGetCurrent get_current = nullptr;
    static PfnCtxGetId get_id = nullptr;
    std::call_once(once, [] {
        void* a = nullptr;
        void* b = nullptr;
        cudaDriverEntryPointQueryResult qa, qb;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) == cudaSuccess &&
            qa == cudaDriverEntryPointSuccess &&
            cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) == cudaSuccess &&
            qb == cudaDriverEntryPointSuccess) {
            get_current = reinterpret_cast<PfnCtxGetCurrent>(a);
            get_id = reinterpret_cast<PfnCtxGetId>(b);
        }
    });
    CUcontext ctx = nullptr;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of the current device's scratch array.  It is resolved with
// cudaGetSymbolAddress once per device and context, and looked up again only if that
// context was replaced (or its identity cannot be read).
nsa_status_t scratch_for_current_device(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return NSA_ERR_NO_DEVICE;
    if (dev < 0 || dev >= kMaxScratchDevices) return NSA_ERR_UNSUPPORTED;
    unsigned long long id = 0;
    const bool have_id = current_context_id(&id) && id != 0;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    ScratchSlot& slot = g_scratch[dev];
    if (!have_id || slot.ctx_id != id || !slot.ptr) {
        // first use on this device (or in a new context): the lookup also makes the
        // device's primary context current if nothing did before
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_invert_scratch) != cudaSuccess || !ptr) return NSA_ERR_CUDA;
        unsigned long long id2 = 0;
        slot.ptr = ptr;
        slot.ctx_id = (current_context_id(&id2) && id2 != 0) ? id2 : 0;
    }
    *out = slot.ptr;
    return NSA_OK;
}

}  // namespace

extern "C" {

size_t nsa_sel_invert_index_noalloc_max_bytes(void) { return kInvertScratchBytes; }

size_t nsa_sel_invert_index_scratch_bytes(int total_tokens, int num_seqs, int hkv, int topk,
                                          int block_size) {
    Dims D;
    // hq = hkv (group 1) fixes the tile geometry; it does not change the inversion.
    if (check_dims(total_tokens, num_seqs, hkv, hkv, kHeadDim, topk, block_size, &D) != NSA_OK)
        return 0;
    return make_layout(D, false).inv_end;
}

nsa_status_t nsa_sel_invert_index_noalloc(const int32_t* cu_seqlens, int num_seqs,
                                          int total_tokens, int hkv, const int32_t* block_idx,
                                          int topk, int block_size, int32_t* offsets,
                                          int32_t* entries, int32_t* counts,
                                          nsa_stream_t stream_) {
    Dims D;
    // hq = hkv (group 1) fixes the tile geometry; it does not change the inversion.
    nsa_status_t s = check_dims(total_tokens, num_seqs, hkv, hkv, kHeadDim, topk, block_size, &D);
    if (s != NSA_OK) return s;
    if (!cu_seqlens || (total_tokens > 0 && !block_idx) || !offsets || !entries || !counts)
        return NSA_ERR_INVALID_ARG;
    if (!aligned(cu_seqlens, 4) || !aligned(block_idx, 4) || !aligned(offsets, 4) ||
        !aligned(entries, 4) || !aligned(counts, 4))
        return NSA_ERR_INVALID_ARG;
    const Layout L = make_layout(D, false);
    if (L.inv_end > kInvertScratchBytes) return NSA_ERR_WORKSPACE;   // too large for the array
    int num_sms = 0;
    if ((s = check_device(&num_sms, stream_)) != NSA_OK) return s;
    void* scratch = nullptr;
    if ((s = scratch_for_current_device(&scratch)) != NSA_OK) return s;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    Carved c = carve(D, L, scratch, cu_seqlens, block_idx);
    if (cudaMemsetAsync(c.st, 0, sizeof(DevStatus), stream) != cudaSuccess) return NSA_ERR_CUDA;
    if (total_tokens == 0) {
        if (cudaMemsetAsync(counts, 0, 2 * sizeof(int32_t), stream) != cudaSuccess ||
            cudaMemsetAsync(offsets, 0, sizeof(int32_t) * ((size_t)D.nbk_cap + 1), stream) !=
                cudaSuccess)
            return NSA_ERR_CUDA;
        return NSA_OK;
    }
    if ((s = cuda_status(launch_invert(c.inv, stream))) != NSA_OK) return s;
    cudaError_t e = cudaMemcpyAsync(offsets, c.inv.offsets, sizeof(int32_t) * ((size_t)D.nbk_cap + 1),
                                    cudaMemcpyDeviceToDevice, stream);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(entries, c.inv.vals[c.inv.final_buf], sizeof(int32_t) * (size_t)D.nent,
                            cudaMemcpyDeviceToDevice, stream);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(counts, &c.st->nblocks_total, sizeof(int32_t), cudaMemcpyDeviceToDevice,
                            stream);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(counts + 1, &c.st->nentries, sizeof(int32_t), cudaMemcpyDeviceToDevice,
                            stream);
    return cuda_status(e);
}

}  // extern "C"
