// select.cu -- kernels of the block-selection step that produces block_idx.
//
// The step ahead of the selected attention in NSA: keys and values are compressed
// per sequence (block c covers tokens [c * stride, c * stride + kernel_size); the
// quick start of the "Relaxed-System-Lab/Flash-Sparse-Attention" project page sets
// kernel_size 32, kernel_stride 16), the compressed attention scores every selection
// block, and each (token, KV head) row keeps its initial and local blocks plus the
// best scored others (init_blocks 1, local_blocks 2, topk 16 there).  The pages print
// no formula; the compressed key and value are the means of the covered rows, and the
// top-k orders by score with ties to the lower block.
//
//   k_cmp_offsets   cu_cmp[s] = compressed blocks of the sequences before s
//   k_compress_kv   one warp per (compressed block, KV head): mean of kernel_size rows
//                   of K and of V (lane = four columns, 256-byte coalesced rows)
//   k_select_topk   one warp per (token, KV head): forced blocks, then repeated warp
//                   arg-max (two redux operations) over the remaining causal blocks'
//                   scores held in registers
#include <math_constants.h>

#include "nsa_common.cuh"
#include "nsa_kernels.h"

namespace nsa {
namespace {

constexpr int kSelWarps = 8;   // warps per block of the per-row kernels
constexpr int kWgThreadsSel = 128;

// Single block: exclusive prefix sum of the per-sequence compressed block counts.
__global__ void __launch_bounds__(1024) k_cmp_offsets(const int32_t* cu, int nseq, int ksize,
                                                      int stride, int32_t* cu_cmp) {
    __shared__ int warp_tot[32];
    __shared__ int carry_s;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    if (threadIdx.x == 0) carry_s = 0;
    __syncthreads();
    for (int base = 0; base < nseq; base += blockDim.x) {
        const int s = base + threadIdx.x;
        int n = 0;
        if (s < nseq) {
            const int L = __ldg(cu + s + 1) - __ldg(cu + s);
            n = L < ksize ? 0 : (L - ksize) / stride + 1;
        }
        int x = n;                                   // inclusive scan within the warp
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) warp_tot[w] = x;
        __syncthreads();
        if (w == 0) {
            int t = lane < (int)(blockDim.x >> 5) ? warp_tot[lane] : 0;
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, t, o);
                if (lane >= o) t += y;
            }
            warp_tot[lane] = t;                      // inclusive over warps
        }
        __syncthreads();
        const int carry = carry_s;
        const int before = carry + (w > 0 ? warp_tot[w - 1] : 0) + x - n;
        if (s < nseq) cu_cmp[s] = before;
        __syncthreads();
        if (threadIdx.x == blockDim.x - 1) carry_s = carry + warp_tot[(blockDim.x >> 5) - 1];
        __syncthreads();
    }
    if (threadIdx.x == 0) cu_cmp[nseq] = carry_s;
}

template <int F16>
__global__ void __launch_bounds__(kSelWarps * 32) k_compress_kv(const void* k, const void* v,
                                                               const int32_t* cu, int nseq,
                                                               int hkv, int ksize, int stride,
                                                               long long npairs,
                                                               const int32_t* cu_cmp, void* kc,
                                                               void* vc) {
    const int lane = threadIdx.x & 31;
    const long long w = (long long)blockIdx.x * kSelWarps + (threadIdx.x >> 5);
    if (w >= npairs) return;
    const int c = (int)(w / hkv), g = (int)(w - (long long)c * hkv);
    if (c >= __ldg(cu_cmp + nseq)) return;          // past the last compressed block
    const int s = upper_index(cu_cmp, nseq, c);
    const int t0 = __ldg(cu + s) + (c - __ldg(cu_cmp + s)) * stride;
    const uint2* kp = reinterpret_cast<const uint2*>(k) + ((size_t)t0 * hkv + g) * (kHeadDim / 4) + lane;
    const uint2* vp = reinterpret_cast<const uint2*>(v) + ((size_t)t0 * hkv + g) * (kHeadDim / 4) + lane;
    const size_t row = (size_t)hkv * (kHeadDim / 4);
    float ak[4] = {0.f, 0.f, 0.f, 0.f}, av[4] = {0.f, 0.f, 0.f, 0.f};
    for (int r = 0; r < ksize; ++r) {
        const uint2 a = __ldg(kp + r * row), b = __ldg(vp + r * row);
        const float2 a0 = unpack2<F16>(a.x), a1 = unpack2<F16>(a.y);
        const float2 b0 = unpack2<F16>(b.x), b1 = unpack2<F16>(b.y);
        ak[0] += a0.x; ak[1] += a0.y; ak[2] += a1.x; ak[3] += a1.y;
        av[0] += b0.x; av[1] += b0.y; av[2] += b1.x; av[3] += b1.y;
    }
    const float inv = 1.f / (float)ksize;
    uint2* ko = reinterpret_cast<uint2*>(kc) + ((size_t)c * hkv + g) * (kHeadDim / 4) + lane;
    uint2* vo = reinterpret_cast<uint2*>(vc) + ((size_t)c * hkv + g) * (kHeadDim / 4) + lane;
    *ko = make_uint2(pack2<F16>(ak[0] * inv, ak[1] * inv), pack2<F16>(ak[2] * inv, ak[3] * inv));
    *vo = make_uint2(pack2<F16>(av[0] * inv, av[1] * inv), pack2<F16>(av[2] * inv, av[3] * inv));
}

// (score, block) order of the top-k: higher score first, the lower block on ties
__device__ __forceinline__ bool better(float a, int ia, float b, int ib) {
    return a > b || (a == b && ia < ib);
}

// Unsigned key with the order of the float (a -0 counts as +0, as the float compare
// does); finite scores and +-inf map above 0.
__device__ __forceinline__ uint32_t order_key(float x) {
    const uint32_t u = __float_as_uint(x + 0.0f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// J = candidate blocks per lane (nb_stride <= 32 J)
template <int J>
__global__ void __launch_bounds__(kSelWarps * 32) k_select_topk(const float* scores,
                                                               const int32_t* cu, int nseq, int T,
                                                               int hkv, int nb_stride, int bs,
                                                               int topk, int init_blocks,
                                                               int local_blocks, int32_t* bidx,
                                                               DevStatus* st) {
    const int lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * kSelWarps + (threadIdx.x >> 5);
    if (row >= (long long)T * hkv) return;
    const int t = (int)(row / hkv);
    const int s = seq_of_token(cu, nseq, t);
    const int i = t - __ldg(cu + s);
    const int qb = i / bs;
    int32_t* out = bidx + (size_t)row * topk;
    if (qb >= nb_stride) {                          // the score rows are too short
        for (int j = lane; j < topk; j += 32) out[j] = -1;
        if (lane == 0) record_error(st, NSA_ERR_INVALID_ARG, 90, t);
        return;
    }
    // forced blocks: 0 .. init_blocks - 1, then qb, qb - 1, .. (local_blocks of them),
    // within [0, qb], each once, at most topk
    auto forced_at = [&](int n) -> int {           // n-th forced block, or -1
        int m = 0;
        for (int b = 0; b < init_blocks && b <= qb; ++b)
            if (m++ == n) return b;
        for (int b = qb; b > qb - local_blocks && b >= 0; --b) {
            if (b < init_blocks) continue;          // already among the initial blocks
            if (m++ == n) return b;
        }
        return -1;
    };
    int nforced = 0;
    while (nforced < topk && forced_at(nforced) >= 0) ++nforced;
    auto is_forced = [&](int b) {
        return b < init_blocks || (b > qb - local_blocks && b <= qb);
    };
    // lane l holds blocks l, l + 32, ...; excluded ones (forced, future) are -inf
    const float* sr = scores + (size_t)row * nb_stride;
    float v[J];
#pragma unroll
    for (int j = 0; j < J; ++j) {
        const int b = lane + 32 * j;
        v[j] = (b <= qb && !is_forced(b)) ? __ldg(sr + b) : -CUDART_INF_F;
    }
    // this lane's best remaining candidate
    auto local_best = [&](float& bv, int& bb) {
        bv = -CUDART_INF_F;
        bb = 0x7fffffff;
#pragma unroll
        for (int j = 0; j < J; ++j) {
            const int b = lane + 32 * j;
            if (v[j] != -CUDART_INF_F && better(v[j], b, bv, bb)) { bv = v[j]; bb = b; }
        }
    };
    float bv;
    int bb;
    local_best(bv, bb);
    const int nrest = min(topk - nforced, (qb + 1) - nforced);
    // forced slots and padding here; the chosen slots only by lane 0 below (no slot is
    // stored by two lanes)
    for (int j = lane; j < topk; j += 32) {
        if (j < nforced) out[j] = forced_at(j);
        else if (j >= nforced + nrest) out[j] = -1;
    }
    for (int n = 0; n < nrest; ++n) {
        // the warp's best: the highest score (one redux over the order keys), then the
        // lowest block among the lanes holding it (a second redux)
        const uint32_t key = bv == -CUDART_INF_F ? 0u : order_key(bv);
        const uint32_t kmax = __reduce_max_sync(0xffffffffu, key);
        const int wb = __reduce_min_sync(0xffffffffu, key == kmax ? bb : 0x7fffffff);
        if (lane == 0) out[nforced + n] = wb;
        if ((wb & 31) == lane) {                    // the winner drops it and rescans
#pragma unroll
            for (int j = 0; j < J; ++j)
                if (lane + 32 * j == wb) v[j] = -CUDART_INF_F;
            local_best(bv, bb);
        }
    }
}

// ---------------------------------------------------------------- block scores
// Scores of the selection blocks from attention over the compressed keys, for the
// geometry of the quick start: compressed blocks of 32 keys at stride 16, selection
// blocks of BS (64 or 128).  A tile is 128 / G consecutive tokens of one sequence x
// the G query heads of KV head g (rows token-major, one 3D TMA box: no gather); a
// chunk is 64 consecutive compressed keys.  Two passes over the chunks the tile
// needs: pass 1 keeps each row's running max and sum of 2^(c s) (the LSE), pass 2
// turns the scores into probabilities p = 2^(c s - lse) and sums them per selection
// block (compressed key k of a chunk meets the chunk's relative blocks
// 16 k / BS .. (16 k + 31) / BS; the last one may be the next chunk's first block,
// carried over), then over the G heads of each token (lane shuffles), and writes the
// token's block scores.  No O is formed, so no accumulator is ever rescaled.
//
//   warp 0       TMA producer: the Q tile, then the compressed-key chunks (3 stages)
//   warp 1       MMA issuer: S = Q Kc^T (8 x M128 N64 K16) into one of two TMEM slots
//   warps 4-7    one thread per row: pass 1 statistics, pass 2 block sums and stores
constexpr int kScThreads = 256;
constexpr int kScStages = 3;
constexpr int kCmpKs = 32, kCmpStride = 16;    // the only compression geometry supported

struct alignas(1024) ScoreSmem {
    uint8_t q[2][kTileRows * 128];            // Q tile: [64-column half][row]
    uint8_t kc[kScStages][2][64 * 128];       // compressed keys: [stage][half][key]
    uint64_t q_full, q_empty;
    uint64_t kc_full[kScStages], kc_empty[kScStages];
    uint64_t s_full[2], s_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};

struct ScorePlan {
    const int32_t* cu;
    const int32_t* cu_cmp;
    const int32_t* tile_off;   // [nseq + 1]: tiles (of 128 / G tokens) before sequence s
    int nseq, hkv, G, tpt, nb_stride;
    float scale_log2;
    float* scores;             // [T, hkv, nb_stride]
    DevStatus* st;
};

// tile_off[s] = sum over earlier sequences of ceil(L / tpt)
__global__ void __launch_bounds__(1024) k_score_tiles(const int32_t* cu, int nseq, int tpt,
                                                      int32_t* tile_off) {
    if (threadIdx.x != 0) return;
    int acc = 0;
    for (int s = 0; s < nseq; ++s) {           // sequences are few: one thread suffices
        tile_off[s] = acc;
        acc += (__ldg(cu + s + 1) - __ldg(cu + s) + tpt - 1) / tpt;
    }
    tile_off[nseq] = acc;
}

template <int BS>
__global__ void __launch_bounds__(kScThreads, 1)
    k_cmp_scores(const ScorePlan p, const __grid_constant__ CUtensorMap qmap,
                 const __grid_constant__ CUtensorMap kcmap) {
    constexpr int NBC = 64 * kCmpStride / BS;       // selection blocks per chunk (16 or 8)
    extern __shared__ uint8_t smem_raw[];
    ScoreSmem& S = *reinterpret_cast<ScoreSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                 ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    DevStatus* st = p.st;
    if (tid == 0) {
        S.abort_flag = (*reinterpret_cast<volatile int*>(&st->code) != 0);
        mbar_init(&S.q_full, 1);
        mbar_init(&S.q_empty, 1);
        for (int i = 0; i < kScStages; ++i) {
            mbar_init(&S.kc_full[i], 1);
            mbar_init(&S.kc_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.s_full[i], 1);
            mbar_init(&S.s_empty[i], kWgThreadsSel);
        }
        mbar_init(&S.drain, 1);
        fence_barrier_init();
    }
    if (warp == 0) {
        __syncwarp();
        tmem_alloc(&S.tmem_base, 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;
    const int ntiles = S.abort_flag ? 0 : __ldg(p.tile_off + p.nseq) * p.hkv;
    volatile int* abort_flag = &S.abort_flag;
    auto wait = [&](uint64_t* bar, uint32_t parity, int where) -> bool {
        if (*abort_flag) return false;
        if (!mbar_wait(bar, parity, st, where)) {
            *abort_flag = 1;
            return false;
        }
        return true;
    };
    // tile -> (sequence, KV head, first local token, sequence length, chunks per pass)
    struct Tile { int s, g, i0, L, nkb; };
    auto tile_at = [&](int ti) {
        Tile t;
        t.g = ti % p.hkv;
        const int u = ti / p.hkv;
        t.s = upper_index(p.tile_off, p.nseq, u);
        t.i0 = (u - __ldg(p.tile_off + t.s)) * p.tpt;
        t.L = __ldg(p.cu + t.s + 1) - __ldg(p.cu + t.s);
        const int imax = min(t.i0 + p.tpt, t.L) - 1;
        t.nkb = (imax / BS) / NBC + 1;              // chunks up to the block of the last row
        return t;
    };
    const int bid = (int)blockIdx.x, grid = (int)gridDim.x;

    if (warp == 0) {
        // ------------------------------------------------------------- TMA producer
        if (lane == 0) {
            prefetch_tmap(&qmap);
            prefetch_tmap(&kcmap);
            int n = 0, u = 0;
            int qpar = -1, kcpar[kScStages];
            for (int i = 0; i < kScStages; ++i) kcpar[i] = -1;
            for (int ti = bid; ti < ntiles; ti += grid, ++n) {
                const Tile t = tile_at(ti);
                if (!wait(&S.q_empty, (n & 1) ^ 1, 100)) break;
                mbar_arrive_expect_tx(&S.q_full, 2u * kTileRows * 128u);
                const int tok0 = __ldg(p.cu + t.s) + t.i0;
                tma_load_3d(S.q[0], &qmap, &S.q_full, 0, t.g * p.G, tok0);
                tma_load_3d(S.q[1], &qmap, &S.q_full, 64, t.g * p.G, tok0);
                qpar = n & 1;
                const int crow0 = __ldg(p.cu_cmp + t.s);
                bool ok = true;
                for (int pass = 0; pass < 2 && ok; ++pass)
                    for (int kb = 0; kb < t.nkb; ++kb, ++u) {
                        const int stg = u % kScStages;
                        if (!(ok = wait(&S.kc_empty[stg], ((u / kScStages) & 1) ^ 1, 101))) break;
                        mbar_arrive_expect_tx(&S.kc_full[stg], 2u * 64u * 128u);
                        tma_load_3d(S.kc[stg][0], &kcmap, &S.kc_full[stg], 0, t.g, crow0 + 64 * kb);
                        tma_load_3d(S.kc[stg][1], &kcmap, &S.kc_full[stg], 64, t.g, crow0 + 64 * kb);
                        kcpar[stg] = (u / kScStages) & 1;
                    }
                if (!ok) break;
            }
            if (*abort_flag) {   // let copies still in flight land before the CTA exits
                if (qpar >= 0) mbar_wait(&S.q_full, qpar, st, 102);
                for (int i = 0; i < kScStages; ++i)
                    if (kcpar[i] >= 0) mbar_wait(&S.kc_full[i], kcpar[i], st, 103);
            }
        }
    } else if (warp == 1) {
        // -------------------------------------------------------------- MMA issuer
        const uint32_t elected = elect_one();
        constexpr uint32_t kIdescS = idesc_f16kind_f32(false, 128, 64, false, false);
        constexpr uint32_t kQHalf = sizeof(S.q[0]) >> 4;
        constexpr uint32_t kKcStage = sizeof(S.kc[0]) >> 4, kKcHalf = sizeof(S.kc[0][0]) >> 4;
        const uint32_t q_desc0 = (uint32_t)smem_desc_sw128(smem_u32(S.q[0]), 16, 1024);
        const uint32_t k_desc0 = (uint32_t)smem_desc_sw128(smem_u32(S.kc[0][0]), 16, 1024);
        int n = 0, u = 0, j = 0;
        bool ok = true;
        for (int ti = bid; ti < ntiles && ok; ti += grid, ++n) {
            const Tile t = tile_at(ti);
            if (!(ok = wait(&S.q_full, n & 1, 104))) break;
            for (int pass = 0; pass < 2 && ok; ++pass)
                for (int kb = 0; kb < t.nkb; ++kb, ++u, ++j) {
                    const int stg = u % kScStages, slot = j & 1;
                    if (!(ok = wait(&S.kc_full[stg], (u / kScStages) & 1, 105))) break;
                    if (!(ok = wait(&S.s_empty[slot], ((j >> 1) & 1) ^ 1, 106))) break;
                    tc_fence_after();
                    const uint32_t tS = tmem + (uint32_t)slot * 64u;
                    const uint32_t b0 = k_desc0 + (uint32_t)stg * kKcStage;
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        const uint32_t off = (uint32_t)((ks >> 2) * kQHalf + (ks & 3) * 2);
                        const uint32_t offk = (uint32_t)((ks >> 2) * kKcHalf + (ks & 3) * 2);
                        mma_ss_e(tS, q_desc0 + off, b0 + offk, kIdescS, ks > 0 ? 1u : 0u, elected);
                    }
                    mma_commit_e(&S.s_full[slot], elected);
                    mma_commit_e(&S.kc_empty[stg], elected);
                }
            if (ok) mma_commit_e(&S.q_empty, elected);   // the tile's last S has read Q
        }
        // every tcgen05 operation issued above has finished once this commit arrives
        mma_commit_e(&S.drain, elected);
        mbar_wait(&S.drain, 0, st, 107);
    } else if (warp >= 4) {
        // ------------------------------------------------------------------ rows
        const int quad = warp & 3, r = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const int tok = r / p.G, h = r - tok * p.G;
        const float c = p.scale_log2;
        int j = 0;
        bool ok = true;
        for (int ti = bid; ti < ntiles && ok; ti += grid) {
            const Tile t = tile_at(ti);
            const int i = t.i0 + tok;                     // local position of this row
            const bool valid = i < t.L;
            // compressed keys 0 .. clim are visible (their span ends at or before i)
            const int clim = (valid && i >= kCmpKs - 1) ? (i - kCmpKs + 1) / kCmpStride : -1;
            float m = -CUDART_INF_F, l = 0.f, lse2 = -CUDART_INF_F;
            float carry = 0.f;
            float* srow = p.scores + ((size_t)(__ldg(p.cu + t.s) + (valid ? i : 0)) * p.hkv + t.g) * p.nb_stride;
            for (int pass = 0; pass < 2 && ok; ++pass) {
                for (int kb = 0; kb < t.nkb; ++kb, ++j) {
                    const int slot = j & 1;
                    if (!(ok = __all_sync(0xffffffffu, wait(&S.s_full[slot], (j >> 1) & 1, 108)))) break;
                    tc_fence_after();
                    float sv[64];
                    tmem_ld64_sync(tmem + (uint32_t)slot * 64u + lane_off, sv);
                    tc_fence_before();
                    mbar_arrive(&S.s_empty[slot]);
                    const int kvis = clim - 64 * kb;          // keys 0 .. kvis of the chunk
                    if (pass == 0) {
                        float mx = m;
#pragma unroll
                        for (int k = 0; k < 64; ++k) {
                            sv[k] = k <= kvis ? sv[k] * c : -CUDART_INF_F;
                            mx = fmaxf(mx, sv[k]);
                        }
                        if (mx != -CUDART_INF_F) {
                            float acc = 0.f;
#pragma unroll
                            for (int k = 0; k < 64; ++k) acc += ex2_approx(sv[k] - mx);
                            l = l * ex2_approx(m - mx) + acc;
                            m = mx;
                        }
                    } else {
                        float bsum[NBC + 1];
#pragma unroll
                        for (int b = 0; b <= NBC; ++b) bsum[b] = 0.f;
                        bsum[0] = carry;
#pragma unroll
                        for (int k = 0; k < 64; ++k) {
                            const float pk = (k <= kvis && lse2 != -CUDART_INF_F)
                                                 ? ex2_approx(sv[k] * c - lse2) : 0.f;
                            const int b_first = (kCmpStride * k) / BS;
                            const int b_last = (kCmpStride * k + kCmpKs - 1) / BS;
                            bsum[b_first] += pk;
                            if (b_last != b_first) bsum[b_last] += pk;
                        }
                        carry = bsum[NBC];
                        // sum over the G heads of the token (G consecutive lanes)
                        for (int o = 1; o < p.G; o <<= 1)
#pragma unroll
                            for (int b = 0; b < NBC; ++b)
                                bsum[b] += __shfl_xor_sync(0xffffffffu, bsum[b], o);
                        if (valid && h == 0) {
#pragma unroll
                            for (int b = 0; b < NBC; ++b) {
                                const int blk = kb * NBC + b;
                                if (blk < p.nb_stride) srow[blk] = bsum[b];
                            }
                        }
                    }
                }
                if (pass == 0) lse2 = l > 0.f ? m + __log2f(l) : -CUDART_INF_F;
            }
        }
    }

    // ---- teardown: every role has left its loop (all waits are bounded) and the MMA
    //      issuer has drained its tensor-core work
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 128);
}

}  // namespace

cudaError_t launch_cmp_scores(const void* q, const void* kc, long long kc_rows, const int32_t* cu,
                              const int32_t* cu_cmp, int nseq, int T, int hq, int hkv,
                              int nb_stride, int bs, float scale, float* scores,
                              int32_t* tile_off, DevStatus* st, int num_sms,
                              const CUtensorMap* qmap, const CUtensorMap* kcmap,
                              cudaStream_t stream) {
    ScorePlan p{};
    p.cu = cu;
    p.cu_cmp = cu_cmp;
    p.tile_off = tile_off;
    p.nseq = nseq;
    p.hkv = hkv;
    p.G = hq / hkv;
    p.tpt = kTileRows / p.G;
    p.nb_stride = nb_stride;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.scores = scores;
    p.st = st;
    (void)q; (void)kc; (void)kc_rows; (void)T;
    k_score_tiles<<<1, 32, 0, stream>>>(cu, nseq, p.tpt, tile_off);
    const size_t smem = sizeof(ScoreSmem) + 1024;
    if (bs == 64) {
        cudaFuncSetAttribute(k_cmp_scores<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k_cmp_scores<64><<<num_sms, kScThreads, smem, stream>>>(p, *qmap, *kcmap);
    } else {
        cudaFuncSetAttribute(k_cmp_scores<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k_cmp_scores<128><<<num_sms, kScThreads, smem, stream>>>(p, *qmap, *kcmap);
    }
    return cudaGetLastError();
}

cudaError_t launch_compress_kv(const void* k, const void* v, const int32_t* cu, int nseq, int T,
                               int hkv, int ksize, int stride, int f16, int32_t* cu_cmp, void* kc,
                               void* vc, cudaStream_t stream) {
    k_cmp_offsets<<<1, 1024, 0, stream>>>(cu, nseq, ksize, stride, cu_cmp);
    const long long npairs = (long long)(T / stride) * hkv;   // bound on (block, head) pairs
    if (npairs > 0) {
        const unsigned grid = (unsigned)((npairs + kSelWarps - 1) / kSelWarps);
        if (f16)
            k_compress_kv<1><<<grid, kSelWarps * 32, 0, stream>>>(k, v, cu, nseq, hkv, ksize, stride,
                                                                  npairs, cu_cmp, kc, vc);
        else
            k_compress_kv<0><<<grid, kSelWarps * 32, 0, stream>>>(k, v, cu, nseq, hkv, ksize, stride,
                                                                  npairs, cu_cmp, kc, vc);
    }
    return cudaGetLastError();
}

cudaError_t launch_select_topk(const float* scores, const int32_t* cu, int nseq, int T, int hkv,
                               int nb_stride, int bs, int topk, int init_blocks, int local_blocks,
                               int32_t* bidx, DevStatus* st, cudaStream_t stream) {
    const long long rows = (long long)T * hkv;
    if (rows == 0) return cudaGetLastError();
    const unsigned grid = (unsigned)((rows + kSelWarps - 1) / kSelWarps);
#define NSA_TOPK_LAUNCH(J)                                                                     \
    k_select_topk<J><<<grid, kSelWarps * 32, 0, stream>>>(scores, cu, nseq, T, hkv, nb_stride, \
                                                          bs, topk, init_blocks, local_blocks,  \
                                                          bidx, st)
    if (nb_stride <= 32) NSA_TOPK_LAUNCH(1);
    else if (nb_stride <= 128) NSA_TOPK_LAUNCH(4);
    else if (nb_stride <= 512) NSA_TOPK_LAUNCH(16);
    else NSA_TOPK_LAUNCH(32);
#undef NSA_TOPK_LAUNCH
    return cudaGetLastError();
}

}  // namespace nsa
