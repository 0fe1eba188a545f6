// invert.cu -- block-index inversion for selected-block attention.
//
// The FSA pages describe swapping the outer and inner loops of the NSA selection
// kernel so that small GQA groups still fill the hardware tiles ("FSA: Efficient
// Implementation of Native Sparse Attention" blog, second paragraph; the
// "Relaxed-System-Lab/Flash-Sparse-Attention" project page, key-features table: a
// main batched query-to-KV kernel).  Swapping the loops needs, for every
// (KV head g, KV block B), the list of query rows that selected B.  This file builds
// it as a stable counting sort of the (token, KV head, slot) entries by the bucket
// key g * NB + B, so every list comes out in ascending token order and the result is
// deterministic (bit-exact, independent of scheduling).
//
// Steps (all on the caller's stream, no host synchronisation):
//   1. k_seq_blocks      global block offset of every sequence, cu_seqlens check
//   2. per digit (at most 8 bits, the key's bits split evenly over the passes):
//                        k_sort_hist -> k_scan_digits -> k_sort_scatter (LSD radix,
//                        stable: warp-ordered ranks from per-bit ballots)
//   3. k_run_offsets     CSR offsets from the sorted keys (and, for the forward, the
//                        start of every (bucket, token window) run)
//   4. k_tile_offsets    per-bucket 128-row tile and backward-chunk prefix sums
#include "nsa_common.cuh"
#include "nsa_kernels.h"

namespace nsa {
namespace {

constexpr int kSortThreads = 256;
constexpr int kSortWarps = kSortThreads / 32;
constexpr int kItems = kSortTile / kSortThreads;   // 16 entries per thread
constexpr uint32_t kInvalidKey = 0xFFFFFFFFu;

struct SortArgs {
    const int32_t* cu;
    int nseq, T, hkv, topk, bs;
    int bs_log2;             // block sizes are powers of two
    int swin;                // sliding window in keys, 0: none
    const int32_t* bidx;
    long long nent;
    int nbk_cap;
    const int32_t* blkoff;
    const DevStatus* st;
};

// Block-wide inclusive scan of one int64 per thread (blockDim.x <= 1024).
__device__ __forceinline__ unsigned long long block_incl_scan_u64(unsigned long long x,
                                                                  unsigned long long* warp_tot) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
    for (int o = 1; o < 32; o <<= 1) {
        unsigned long long y = __shfl_up_sync(0xFFFFFFFFu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[w] = x;
    __syncthreads();
    if (w == 0) {
        unsigned long long t = lane < nw ? warp_tot[lane] : 0ull;
        for (int o = 1; o < 32; o <<= 1) {
            unsigned long long y = __shfl_up_sync(0xFFFFFFFFu, t, o);
            if (lane >= o) t += y;
        }
        warp_tot[lane] = t;
    }
    __syncthreads();
    unsigned long long r = x + (w > 0 ? warp_tot[w - 1] : 0ull);
    __syncthreads();
    return r;
}

// 1. blkoff[s] = sum_{s' < s} ceil(L_s' / bs); checks cu_seqlens.
__global__ void __launch_bounds__(1024) k_seq_blocks(const int32_t* cu, int nseq, int T, int bs,
                                                     int32_t* blkoff, DevStatus* st,
                                                     unsigned long long tag) {
    __shared__ unsigned long long warp_tot[32];
    __shared__ unsigned long long round_total;
    __shared__ int bad;
    if (threadIdx.x == 0) bad = (cu[0] != 0 || cu[nseq] != T) ? 1 : 0;
    __syncthreads();
    unsigned long long carry = 0;
    for (int base = 0; base < nseq; base += blockDim.x) {
        int s = base + threadIdx.x;
        unsigned long long nb = 0;
        if (s < nseq) {
            int L = cu[s + 1] - cu[s];
            if (L < 0) bad = 1;
            nb = L > 0 ? (unsigned long long)((L + bs - 1) / bs) : 0ull;
        }
        unsigned long long incl = block_incl_scan_u64(nb, warp_tot);
        if (s < nseq) blkoff[s] = (int32_t)(carry + incl - nb);
        // total of this pass of the loop = inclusive value of the last thread
        if (threadIdx.x == blockDim.x - 1) round_total = incl;
        __syncthreads();
        carry += round_total;
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        blkoff[nseq] = (int32_t)carry;
        // invalid cu_seqlens: no blocks, so no later table outgrows its T / bs + nseq rows
        st->nblocks_total = bad ? 0 : (int)carry;
        st->index_tag = tag;
        if (bad) record_error(st, NSA_ERR_BAD_INDEX, 1);
    }
}

// Position of entry e = (t * hkv + g) * topk + j (token-major, then KV head, then
// slot) in its row, and the sequence that holds its token.  A thread walks its entries
// with a fixed stride, so the position advances by a precomputed (dt, dg, dj) with one
// carry per level and the sequence by a forward scan of cu_seqlens: no division and
// no search per entry.
struct EntryCursor {
    int t, g, j;             // token, KV head, slot
    int s, seq0, seq1, blk;  // sequence of t, its token range [seq0, seq1), global block offset
    int dt, dg, dj;          // the stride, decomposed like an entry index

    __device__ __forceinline__ void init(const SortArgs& a, long long e, int stride) {
        const long long rowk = (long long)a.hkv * a.topk;
        t = (int)(e / rowk);
        const int r = (int)(e - (long long)t * rowk);
        g = r / a.topk;
        j = r - g * a.topk;
        dt = stride / (int)rowk;
        const int rs = stride - dt * (int)rowk;
        dg = rs / a.topk;
        dj = rs - dg * a.topk;
        s = t < a.T ? seq_of_token(a.cu, a.nseq, t) : a.nseq - 1;
        seq0 = __ldg(a.cu + s);
        seq1 = __ldg(a.cu + s + 1);
        blk = __ldg(a.blkoff + s);
    }
    __device__ __forceinline__ void advance(const SortArgs& a) {
        j += dj;
        int c = j >= a.topk;
        j -= c ? a.topk : 0;
        g += dg + c;
        c = g >= a.hkv;
        g -= c ? a.hkv : 0;
        t += dt + c;
    }
    // the bucket key g * NB + global block of block b (kInvalidKey if it selects
    // nothing: padding, a future or out-of-range block, or a block wholly before the
    // sliding window); t must be < T
    __device__ __forceinline__ uint32_t key(const SortArgs& a, int b, uint32_t nbtot) {
        while (t >= seq1 && s + 1 < a.nseq) {
            ++s;
            seq0 = seq1;
            seq1 = __ldg(a.cu + s + 1);
            blk = __ldg(a.blkoff + s);
        }
        const int i = t - seq0;
        const int qb = i >> a.bs_log2;
        if (!block_valid(b, qb, i, a.bs, a.swin)) return kInvalidKey;
        const uint32_t k = (uint32_t)g * nbtot + (uint32_t)blk + (uint32_t)b;
        return k < (uint32_t)a.nbk_cap ? k : kInvalidKey;
    }
    __device__ __forceinline__ uint32_t val() const { return (uint32_t)t * 64u + (uint32_t)j; }
};

// 2a. per-tile digit histogram, stored digit-major: hist[d * ntiles + tile].
template <bool kFirst>
__global__ void __launch_bounds__(kSortThreads) k_sort_hist(SortArgs a, const uint32_t* keys_in,
                                                           int shift, uint32_t mask, uint32_t* hist) {
    __shared__ uint32_t h[256];
    h[threadIdx.x] = 0;
    const long long base = (long long)blockIdx.x * kSortTile + threadIdx.x;
    const int nitems = a.nent > base ? (int)min((long long)kItems, (a.nent - base + kSortThreads - 1) / kSortThreads) : 0;
    const uint32_t* src = (kFirst ? reinterpret_cast<const uint32_t*>(a.bidx) : keys_in) + base;
    // every load of the thread first (independent loads in flight together)
    uint32_t x[kItems];
#pragma unroll
    for (int it = 0; it < kItems; ++it) x[it] = it < nitems ? __ldg(src + it * kSortThreads) : 0u;
    __syncthreads();
    if (kFirst) {
        const uint32_t nbtot = (uint32_t)a.st->nblocks_total;
        EntryCursor c;
        c.init(a, base, kSortThreads);
#pragma unroll
        for (int it = 0; it < kItems; ++it) {
            if (it < nitems) atomicAdd(&h[(c.key(a, (int)x[it], nbtot) >> shift) & mask], 1u);
            c.advance(a);
        }
    } else {
#pragma unroll
        for (int it = 0; it < kItems; ++it)
            if (it < nitems) atomicAdd(&h[(x[it] >> shift) & mask], 1u);
    }
    __syncthreads();
    hist[(size_t)threadIdx.x * gridDim.x + blockIdx.x] = h[threadIdx.x];
}

// 2b. per digit (one block each): exclusive scan of hist[d * ntiles + tile] over the
//     tiles, in place, and the digit's total into digit_tot[d].
__global__ void __launch_bounds__(1024) k_scan_digits(uint32_t* hist, int ntiles,
                                                      uint32_t* digit_tot) {
    __shared__ unsigned long long warp_tot[32];
    uint32_t* a = hist + (size_t)blockIdx.x * ntiles;
    const int per = (ntiles + blockDim.x - 1) / blockDim.x;
    const int lo = per * threadIdx.x;
    const int hi = min(lo + per, ntiles);
    unsigned long long sum = 0;
    for (int i = lo; i < hi; ++i) sum += a[i];
    const unsigned long long incl = block_incl_scan_u64(sum, warp_tot);
    unsigned long long run = incl - sum;
    for (int i = lo; i < hi; ++i) {
        const uint32_t x = a[i];
        a[i] = (uint32_t)run;
        run += x;
    }
    if (threadIdx.x == blockDim.x - 1) digit_tot[blockIdx.x] = (uint32_t)incl;
}

// 2c. stable scatter of one tile by the digit (key >> shift) & mask.  Entries are ranked within
//     the tile (warp-ordered ranks from one ballot per digit bit, then the warps in order), put
//     into shared memory in the tile's digit order, and written out from there: thread
//     k stores the tile's k-th entry of that order, so each digit's run of the tile
//     goes to consecutive global addresses (coalesced) instead of one scattered word
//     per entry.
template <bool kFirst>
__global__ void __launch_bounds__(kSortThreads, 3) k_sort_scatter(SortArgs a, const uint32_t* keys_in,
                                                              const uint32_t* vals_in, int shift,
                                                              uint32_t mask,
                                                              const uint32_t* hist_scan,
                                                              const uint32_t* digit_tot,
                                                              uint32_t* keys_out,
                                                              uint32_t* vals_out) {
    __shared__ uint32_t whist[kSortWarps][256];
    __shared__ uint32_t tile_base[256];      // global start of each digit's run of this tile
    __shared__ uint32_t local_start[256];    // start of each digit's run within the tile
    __shared__ unsigned long long warp_tot[32];
    __shared__ uint32_t stage_k[kSortTile];  // keys in the tile's digit order
    __shared__ uint32_t stage_v[kSortTile];  // their values
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const long long tile0 = (long long)blockIdx.x * kSortTile;
    const long long base = tile0 + (long long)w * (kItems * 32) + lane;
    const int nvalid = (int)min((long long)kSortTile, a.nent - tile0);
    const int nitems = a.nent > base ? (int)min((long long)kItems, (a.nent - base + 31) / 32) : 0;
    const uint32_t lt_mask = (1u << lane) - 1u;
    const uint32_t* src = (kFirst ? reinterpret_cast<const uint32_t*>(a.bidx) : keys_in) + base;
    // every key of the lane first (independent loads in flight together, and in flight
    // during the prologue), then the warp-ordered ranks
    uint32_t key[kItems], pos[kItems];
#pragma unroll
    for (int it = 0; it < kItems; ++it) key[it] = it < nitems ? __ldg(src + it * 32) : 0u;
    for (int i = tid; i < kSortWarps * 256; i += kSortThreads) (&whist[0][0])[i] = 0;
    {   // start of digit tid in the output = totals of smaller digits + earlier tiles
        const uint32_t tot = digit_tot[tid];
        const unsigned long long incl = block_incl_scan_u64(tot, warp_tot);
        tile_base[tid] = (uint32_t)(incl - tot) + hist_scan[(size_t)tid * gridDim.x + blockIdx.x];
    }
    __syncthreads();
    if (kFirst) {
        const uint32_t nbtot = (uint32_t)a.st->nblocks_total;
        EntryCursor c;
        c.init(a, base, 32);
#pragma unroll
        for (int it = 0; it < kItems; ++it) {
            if (it < nitems) key[it] = c.key(a, (int)key[it], nbtot);
            c.advance(a);
        }
    }
#pragma unroll
    for (int it = 0; it < kItems; ++it) {
        const uint32_t d = it < nitems ? (key[it] >> shift) & mask : 256u;   // 256: past the end
        // lanes with the same digit: a ballot per digit bit (cheaper than match.any)
        uint32_t peers = __ballot_sync(0xFFFFFFFFu, d < 256u);
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            if ((mask >> b) == 0u) break;
            const uint32_t bit = (d >> b) & 1u;
            const uint32_t ones = __ballot_sync(0xFFFFFFFFu, bit);
            peers &= bit ? ones : ~ones;
        }
        const uint32_t before = __popc(peers & lt_mask);
        if (d < 256u) pos[it] = whist[w][d] + before;
        __syncwarp();
        if (d < 256u && before == 0) whist[w][d] += __popc(peers);
        __syncwarp();
    }
    __syncthreads();
    {   // exclusive prefix of each digit over the warps of the tile, and the digit's
        // start within the tile (a scan over the digits)
        uint32_t run = 0;
        for (int ww = 0; ww < kSortWarps; ++ww) {
            uint32_t cnt = whist[ww][tid];
            whist[ww][tid] = run;
            run += cnt;
        }
        const unsigned long long incl = block_incl_scan_u64(run, warp_tot);
        local_start[tid] = (uint32_t)(incl - run);
    }
    __syncthreads();
    // the keys into their staging slots, then the values (loaded together)
#pragma unroll
    for (int it = 0; it < kItems; ++it) {
        if (it < nitems) {
            const uint32_t d = (key[it] >> shift) & mask;
            pos[it] += local_start[d] + whist[w][d];
            stage_k[pos[it]] = key[it];
        }
    }
    if (kFirst) {
        EntryCursor c;
        c.init(a, base, 32);
#pragma unroll
        for (int it = 0; it < kItems; ++it) {
            if (it < nitems) stage_v[pos[it]] = c.val();
            c.advance(a);
        }
    } else {
        const uint32_t* vsrc = vals_in + base;
#pragma unroll
        for (int it = 0; it < kItems; ++it) key[it] = it < nitems ? __ldg(vsrc + it * 32) : 0u;
#pragma unroll
        for (int it = 0; it < kItems; ++it)
            if (it < nitems) stage_v[pos[it]] = key[it];
    }
    __syncthreads();
    for (int k = tid; k < nvalid; k += kSortThreads) {
        const uint32_t kk = stage_k[k];
        const uint32_t d = (kk >> shift) & mask;
        const uint32_t at = tile_base[d] + (uint32_t)k - local_start[d];
        keys_out[at] = kk;
        vals_out[at] = stage_v[k];
    }
}

// 3. Run offsets of the sorted list.  offsets[B] = number of sorted keys below B, for
//    B in [0, hkv * NB].  With a window table (the forward), also the start of every
//    (bucket, token window) run: entries are sorted by bucket and, within a bucket, by
//    token, so the composite c = bucket * nwin + window of the token is ascending too,
//    and wstart[c] = number of entries whose composite is below c, for c in
//    [0, hkv * NB * nwin].  Entries of invalid key sort last and count as c = the end.
__device__ __forceinline__ int run_code(uint32_t key, uint32_t val, int nbk, int nwin, uint32_t wtok) {
    const int k = (int)min(key, (uint32_t)nbk);
    if (k == nbk || nwin == 1) return k * nwin;
    return k * nwin + min((int)((val >> 6) / wtok), nwin - 1);
}

// Four consecutive entries per thread (one 16-byte load of keys and of values).
__global__ void k_run_offsets(const uint32_t* keys, const uint32_t* vals, long long nent,
                              const DevStatus* st, int hkv, int nwin, int wtok, int32_t* offsets,
                              int32_t* wstart) {
    const long long i0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) * 4;
    if (i0 > nent) return;
    const int nbk = hkv * st->nblocks_total;
    const int cend = nbk * nwin;   // code of the end (and of invalid keys)
    const bool wins = nwin > 1;
    uint32_t k[5], v[5];           // entries i0 - 1 .. i0 + 3
    if (i0 + 4 <= nent) {
        const uint4 kk = __ldg(reinterpret_cast<const uint4*>(keys + i0));
        k[1] = kk.x; k[2] = kk.y; k[3] = kk.z; k[4] = kk.w;
        if (wins) {
            const uint4 vv = __ldg(reinterpret_cast<const uint4*>(vals + i0));
            v[1] = vv.x; v[2] = vv.y; v[3] = vv.z; v[4] = vv.w;
        }
    } else {
#pragma unroll
        for (int q = 1; q < 5; ++q) {
            k[q] = i0 + q - 1 < nent ? __ldg(keys + i0 + q - 1) : 0u;
            v[q] = wins && i0 + q - 1 < nent ? __ldg(vals + i0 + q - 1) : 0u;
        }
    }
    k[0] = i0 > 0 ? __ldg(keys + i0 - 1) : 0u;
    v[0] = wins && i0 > 0 ? __ldg(vals + i0 - 1) : 0u;
    int prev = i0 > 0 ? run_code(k[0], v[0], nbk, nwin, (uint32_t)wtok) : -1;
#pragma unroll
    for (int q = 1; q < 5; ++q) {
        const long long i = i0 + q - 1;
        if (i > nent) break;
        const int cur = i < nent ? run_code(k[q], v[q], nbk, nwin, (uint32_t)wtok) : cend;
        for (int c = prev + 1; c <= cur; ++c) {
            if (wstart) wstart[c] = (int32_t)i;
            if (!wins) offsets[c] = (int32_t)i;
            else if (c % nwin == 0) offsets[c / nwin] = (int32_t)i;
        }
        prev = cur;
    }
}

// 4. tile and chunk prefix sums per bucket; totals into the status block.
__global__ void __launch_bounds__(1024) k_tile_offsets(const int32_t* offsets, DevStatus* st,
                                                       int hkv, int tpt, int chunk_tiles,
                                                       int32_t* tile_off, int32_t* chunk_off) {
    __shared__ unsigned long long warp_tot[32];
    __shared__ unsigned long long round_total;
    const long long nbk = (long long)hkv * st->nblocks_total;
    unsigned long long carry = 0;   // (chunks << 32) | tiles
    for (long long base = 0; base < nbk; base += blockDim.x) {
        long long B = base + threadIdx.x;
        unsigned long long x = 0;
        if (B < nbk) {
            const uint32_t cnt = (uint32_t)(offsets[B + 1] - offsets[B]);
            const uint32_t nt = (cnt + (uint32_t)tpt - 1u) / (uint32_t)tpt;
            const uint32_t nc = (nt + (uint32_t)chunk_tiles - 1u) / (uint32_t)chunk_tiles;
            x = ((unsigned long long)nc << 32) | nt;
        }
        unsigned long long incl = block_incl_scan_u64(x, warp_tot);
        unsigned long long ex = carry + incl - x;
        if (B < nbk) {
            tile_off[B] = (int32_t)(ex & 0xFFFFFFFFull);
            chunk_off[B] = (int32_t)(ex >> 32);
        }
        if (threadIdx.x == blockDim.x - 1) round_total = incl;
        __syncthreads();
        carry += round_total;
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        tile_off[nbk] = (int32_t)(carry & 0xFFFFFFFFull);
        chunk_off[nbk] = (int32_t)(carry >> 32);
        st->ntiles = (int)(carry & 0xFFFFFFFFull);
        st->nchunks = (int)(carry >> 32);
        st->nentries = offsets[nbk];
    }
}

// 5. Window runs for the forward's tile order.  Tokens are cut into windows of `wtok`
//    (packed) tokens; the run of the (g, B) list whose tokens lie in window w is
//    [wstart[c], wstart[c + 1]) with c = (g * NB + B) * nwin + w (k_run_offsets).
__device__ __forceinline__ int2 window_run(const int32_t* wstart, int nbtot, int nwin, int g,
                                           int w, int B) {
    const size_t c = ((size_t)g * nbtot + B) * nwin + w;
    const int a = __ldg(wstart + c);
    return make_int2(a, __ldg(wstart + c + 1) - a);
}

// 6. Per (g, w) row: exclusive scan over B of ceil(count / tpt) tiles, and the row's
//    total.  One block per row.
__global__ void __launch_bounds__(1024) k_window_tiles(const int32_t* wstart, const DevStatus* st,
                                                       int nwin, int nb_stride, int tpt,
                                                       int32_t* tile_off, int32_t* row_tiles) {
    __shared__ unsigned long long warp_tot[32];
    __shared__ unsigned long long round_total;
    const int nbtot = st->nblocks_total;
    const int g = blockIdx.x / nwin, w = blockIdx.x - g * nwin;
    int32_t* out = tile_off + (size_t)blockIdx.x * (nb_stride + 1);
    unsigned long long carry = 0;
    for (int base = 0; base < nbtot; base += blockDim.x) {
        const int B = base + threadIdx.x;
        unsigned long long x = 0;
        if (B < nbtot)
            x = (unsigned long long)((window_run(wstart, nbtot, nwin, g, w, B).y + tpt - 1) / tpt);
        const unsigned long long incl = block_incl_scan_u64(x, warp_tot);
        if (B < nbtot) out[B] = (int32_t)(carry + incl - x);
        if (threadIdx.x == blockDim.x - 1) round_total = incl;
        __syncthreads();
        carry += round_total;
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        out[nbtot] = (int32_t)carry;
        row_tiles[blockIdx.x] = (int32_t)carry;
    }
}

// 7. Exclusive scan of the rows' tile counts; total into the status block.
__global__ void __launch_bounds__(1024) k_row_offsets(const int32_t* row_tiles, int nrows,
                                                      int32_t* row_off, DevStatus* st) {
    __shared__ unsigned long long warp_tot[32];
    __shared__ unsigned long long round_total;
    unsigned long long carry = 0;
    for (int base = 0; base < nrows; base += blockDim.x) {
        const int r = base + threadIdx.x;
        const unsigned long long x = r < nrows ? (unsigned long long)row_tiles[r] : 0ull;
        const unsigned long long incl = block_incl_scan_u64(x, warp_tot);
        if (r < nrows) row_off[r] = (int32_t)(carry + incl - x);
        if (threadIdx.x == blockDim.x - 1) round_total = incl;
        __syncthreads();
        carry += round_total;
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        row_off[nrows] = (int32_t)carry;
        st->ntiles_fwd = (int)carry;
    }
}

// 8. One descriptor per forward tile, so that the tile kernel's roles read a tile's
//    geometry with one load instead of three dependent binary searches:
//    (first key of the block, first entry, nrows | g << 8, g * NB + B).
__global__ void k_tile_desc(const DevStatus* st, const int32_t* row_off, const int32_t* tile_off,
                            const int32_t* wstart, const int32_t* blkoff, const int32_t* cu,
                            int nseq, int hkv, int nwin, int nb_stride, int G, int bs,
                            int4* desc) {
    const int tile = blockIdx.x * blockDim.x + threadIdx.x;
    if (tile >= st->ntiles_fwd) return;
    const int nbtot = st->nblocks_total;
    const int row = upper_index(row_off, hkv * nwin, tile);
    const int tr = tile - row_off[row];
    const int32_t* toff = tile_off + (size_t)row * (nb_stride + 1);
    const int B = upper_index(toff, nbtot, tr);
    const int tpt = kTileRows / G;
    const int g = row / nwin;
    const int2 rng = window_run(wstart, nbtot, nwin, g, row - g * nwin, B);
    const int s = upper_index(blkoff, nseq, B);
    const int key0 = cu[s] + (B - blkoff[s]) * bs;
    const int e0 = rng.x + (tr - toff[B]) * tpt;
    const int nrows = (min(e0 + tpt, rng.x + rng.y) - e0) * G;
    desc[tile] = make_int4(key0, e0, nrows | (g << 8), g * nbtot + B);
}

// 9. One descriptor per backward work unit (up to chunk_tiles consecutive tiles of one
//    (g, B) list): (first key of the block, first entry, end of the list's entries,
//    ntiles | g << 8) and the bucket id g * NB + B.
__global__ void k_unit_desc(DevStatus* st, const int32_t* chunk_off, const int32_t* tile_off,
                            const int32_t* offsets, const int32_t* blkoff, const int32_t* cu,
                            int nseq, int hkv, int tpt, int chunk_tiles, int bs, int4* udesc,
                            int* ubucket, int check_tag, unsigned long long tag) {
    const int u = blockIdx.x * blockDim.x + threadIdx.x;
    if (check_tag && st->index_tag != tag) {   // the workspace holds another inversion
        if (u == 0) record_error(st, NSA_ERR_INVALID_ARG, 80);
        return;
    }
    if (u >= st->nchunks) return;
    const int nbtot = st->nblocks_total;
    const int bucket = upper_index(chunk_off, hkv * nbtot, u);
    const int t0 = tile_off[bucket];
    const int tlo = t0 + (u - chunk_off[bucket]) * chunk_tiles;
    const int thi = min(tlo + chunk_tiles, tile_off[bucket + 1]);
    const int g = bucket / nbtot;
    const int B = bucket - g * nbtot;
    const int s = upper_index(blkoff, nseq, B);
    const int key0 = cu[s] + (B - blkoff[s]) * bs;
    udesc[u] = make_int4(key0, offsets[bucket] + (tlo - t0) * tpt, offsets[bucket + 1],
                         (thi - tlo) | (g << 8));
    ubucket[u] = bucket;
}

// Units sorted by tile count, largest first (a counting sort in one block; units of
// equal count in any order).  The backward tile kernel deals them out in snake order
// (round k: CTA c takes rank k P + c for even k and k P + P - 1 - c for odd k), which
// evens out the tiles per CTA; which CTA runs a unit does not change its arithmetic.
__global__ void __launch_bounds__(1024) k_unit_order(const DevStatus* st, const int4* udesc,
                                                     int* uorder) {
    __shared__ int hist[256];
    if (st->code != 0) return;
    const int n = st->nchunks;
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int u = threadIdx.x; u < n; u += blockDim.x) atomicAdd(&hist[udesc[u].w & 255], 1);
    __syncthreads();
    if (threadIdx.x == 0) {   // exclusive prefix from the largest count down
        int acc = 0;
        for (int c = 255; c >= 0; --c) {
            const int h = hist[c];
            hist[c] = acc;
            acc += h;
        }
    }
    __syncthreads();
    for (int u = threadIdx.x; u < n; u += blockDim.x) uorder[atomicAdd(&hist[udesc[u].w & 255], 1)] = u;
}

// 10. Position map from the forward tiles: the k-th token of tile tau, entry
//     (t, g, j), gets posmap[(t * hkv + g) * topk + j] = tau * tpt + k; its partial
//     rows are posmap * G + head offset, inside the tile's own 128-row slot.
__global__ void k_posmap_tiles(const int4* desc, const uint32_t* entries, const DevStatus* st,
                               int hkv, int topk, int tpt, int32_t* posmap) {
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    int tile, k;
    if (idx <= 0x7FFFFFFFll) {   // 32-bit division where the index allows it
        const uint32_t i32 = (uint32_t)idx;
        tile = (int)(i32 / (uint32_t)tpt);
        k = (int)(i32 - (uint32_t)tile * (uint32_t)tpt);
    } else {
        tile = (int)(idx / tpt);
        k = (int)(idx % tpt);
    }
    if (st->code != 0 || tile >= st->ntiles_fwd) return;
    const int4 d = desc[tile];
    const int G = kTileRows / tpt;
    if (k >= (d.z & 255) / G) return;
    const uint32_t v = entries[d.y + k];
    posmap[((size_t)(v >> 6) * hkv + (d.z >> 8)) * topk + (v & 63u)] = tile * tpt + k;
}

// Range / duplicate check of block_idx (one thread per (token, KV head) row).
__global__ void k_validate(const int32_t* cu, int nseq, int T, int hkv, const int32_t* bidx,
                           int topk, int bs, DevStatus* st) {
    long long r = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= (long long)T * hkv) return;
    int t = (int)(r / hkv);
    int s = seq_of_token(cu, nseq, t);
    int L = cu[s + 1] - cu[s];
    int nb = L > 0 ? (L + bs - 1) / bs : 0;
    const int32_t* row = bidx + r * topk;
    long long bad = 0, dup = 0;
    for (int j = 0; j < topk; ++j) {
        int b = row[j];
        if (b == -1) continue;
        if (b < -1 || b >= nb) ++bad;
        if (b >= 0)
            for (int j2 = 0; j2 < j; ++j2)
                if (row[j2] == b) { ++dup; break; }
    }
    if (bad) atomicAdd(reinterpret_cast<unsigned long long*>(&st->bad_range),
                       (unsigned long long)bad);
    if (dup) atomicAdd(reinterpret_cast<unsigned long long*>(&st->bad_dup),
                       (unsigned long long)dup);
}

}  // namespace

int invert_final_buf(const InvertPlan& p) {
    const int passes = p.key_bits <= 8 ? 1 : (p.key_bits + 7) / 8;
    return (passes - 1) & 1;
}

cudaError_t launch_invert(InvertPlan& p, cudaStream_t stream) {
    k_seq_blocks<<<1, 1024, 0, stream>>>(p.cu, p.nseq, p.T, p.bs, p.blkoff, p.st, p.tag);
    int bs_log2 = 0;
    while ((2 << bs_log2) <= p.bs) ++bs_log2;   // p.bs is a power of two (64 or 128)
    SortArgs a{p.cu, p.nseq, p.T, p.hkv, p.topk, p.bs, bs_log2, p.swin, p.bidx, p.nent,
               p.nbk_cap, p.blkoff, p.st};
    // digits of at most 8 bits, split evenly over the passes (13 bits: 7 + 6), so that
    // every pass scatters runs of similar length
    const int passes = p.key_bits <= 8 ? 1 : (p.key_bits + 7) / 8;
    const uint32_t* kin = nullptr;
    const uint32_t* vin = nullptr;
    int shift = 0;
    // the scatter's 42 KB of static shared memory: ask for the largest carveout so that
    // three CTAs fit on an SM
    cudaFuncSetAttribute(k_sort_scatter<true>, cudaFuncAttributePreferredSharedMemoryCarveout,
                         cudaSharedmemCarveoutMaxShared);
    cudaFuncSetAttribute(k_sort_scatter<false>, cudaFuncAttributePreferredSharedMemoryCarveout,
                         cudaSharedmemCarveoutMaxShared);
    for (int pass = 0; pass < passes; ++pass) {
        const int bits = p.key_bits / passes + (pass < p.key_bits % passes ? 1 : 0);
        const uint32_t mask = (1u << bits) - 1u;
        uint32_t* kout = p.keys[pass & 1];
        uint32_t* vout = p.vals[pass & 1];
        if (pass == 0)
            k_sort_hist<true><<<p.sort_tiles, kSortThreads, 0, stream>>>(a, nullptr, shift, mask, p.hist);
        else
            k_sort_hist<false><<<p.sort_tiles, kSortThreads, 0, stream>>>(a, kin, shift, mask, p.hist);
        k_scan_digits<<<256, 1024, 0, stream>>>(p.hist, p.sort_tiles, p.digit_tot);
        if (pass == 0)
            k_sort_scatter<true><<<p.sort_tiles, kSortThreads, 0, stream>>>(
                a, nullptr, nullptr, shift, mask, p.hist, p.digit_tot, kout, vout);
        else
            k_sort_scatter<false><<<p.sort_tiles, kSortThreads, 0, stream>>>(
                a, kin, vin, shift, mask, p.hist, p.digit_tot, kout, vout);
        kin = kout;
        vin = vout;
        shift += bits;
    }
    p.final_buf = invert_final_buf(p);
    const long long n1 = p.nent + 1;
    const long long nthr = (n1 + 3) / 4;
    k_run_offsets<<<(unsigned)((nthr + 255) / 256), 256, 0, stream>>>(
        p.keys[p.final_buf], p.vals[p.final_buf], p.nent, p.st, p.hkv, p.wstart ? p.nwin : 1,
        p.wtok, p.offsets, p.wstart);
    k_tile_offsets<<<1, 1024, 0, stream>>>(p.offsets, p.st, p.hkv, p.tokens_per_tile,
                                           p.chunk_tiles, p.tile_off, p.chunk_off);
    return cudaGetLastError();
}

cudaError_t launch_window_split(const InvertPlan& p, const WindowPlan& w, cudaStream_t stream) {
    const int nrows = p.hkv * w.nwin;
    if (!p.wstart || p.nwin != w.nwin || p.wtok != w.wtok) return cudaErrorInvalidValue;
    k_window_tiles<<<nrows, 1024, 0, stream>>>(p.wstart, p.st, w.nwin, w.nb_stride,
                                               p.tokens_per_tile, w.tile_off, w.row_tiles);
    k_row_offsets<<<1, 1024, 0, stream>>>(w.row_tiles, nrows, w.row_off, p.st);
    k_tile_desc<<<(unsigned)((w.tiles_cap + 255) / 256), 256, 0, stream>>>(
        p.st, w.row_off, w.tile_off, p.wstart, p.blkoff, p.cu, p.nseq, p.hkv, w.nwin, w.nb_stride,
        kTileRows / p.tokens_per_tile, p.bs, w.tile_desc);
    return cudaGetLastError();
}

cudaError_t launch_posmap(const InvertPlan& p, const WindowPlan& w, int32_t* posmap,
                          cudaStream_t stream) {
    const long long n = w.tiles_cap * p.tokens_per_tile;
    if (n > 0)
        k_posmap_tiles<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(
            w.tile_desc, p.vals[p.final_buf], p.st, p.hkv, p.topk, p.tokens_per_tile, posmap);
    return cudaGetLastError();
}

cudaError_t launch_unit_desc(const InvertPlan& p, long long units_cap, int4* udesc, int* ubucket,
                             bool check_tag, cudaStream_t stream) {
    k_unit_desc<<<(unsigned)((units_cap + 255) / 256), 256, 0, stream>>>(
        p.st, p.chunk_off, p.tile_off, p.offsets, p.blkoff, p.cu, p.nseq, p.hkv,
        p.tokens_per_tile, p.chunk_tiles, p.bs, udesc, ubucket, check_tag ? 1 : 0, p.tag);
    return cudaGetLastError();
}

cudaError_t launch_unit_order(const DevStatus* st, const int4* udesc, int* uorder,
                              cudaStream_t stream) {
    k_unit_order<<<1, 1024, 0, stream>>>(st, udesc, uorder);
    return cudaGetLastError();
}

cudaError_t launch_validate(const int32_t* cu, int nseq, int T, int hkv, const int32_t* bidx,
                            int topk, int bs, DevStatus* st, cudaStream_t stream) {
    long long rows = (long long)T * hkv;
    if (rows > 0)
        k_validate<<<(unsigned)((rows + 255) / 256), 256, 0, stream>>>(cu, nseq, T, hkv, bidx,
                                                                        topk, bs, st);
    return cudaGetLastError();
}

}  // namespace nsa
