// bsfa.cu -- threshold-pruned block attention (Block Sparse Flash Attention).
//
// The "Block Sparse Flash Attention" news pages (the aiqbench analysis and the
// marsel.app article, "How it works"): every query-key score is computed exactly;
// for each query and key block the block's largest score is compared with a
// calibrated threshold and blocks below it are skipped.  Reading taken here: blocks
// are the 64-key blocks of each sequence (causal, key j <= query i); block b is kept
// for row (i, h) iff max_{j in b, j <= i} scale q_i . k_j >= tau[h]; the output is
// softmax attention over the keys of the kept blocks only; no kept block gives O = 0,
// LSE = -inf.
//
// A tile is 128 / G consecutive tokens of one sequence x the G query heads of KV head
// g (one 3D TMA box, rows token-major).  Two passes over the tile's key blocks:
//   pass 1  S = Q K^T; each row's block maximum decides the block, and the kept
//           blocks' keys update the row's running max and sum (its LSE);
//   pass 2  S again; P = 2^(c S - lse) on the kept blocks (0 elsewhere), written as
//           bf16 into the S columns of TMEM; O += P V (P read from TMEM).
// Because pass 2 knows the final LSE, O is never rescaled.  Pass 1 also marks, per
// tile, the blocks that at least one row keeps (a bit mask in shared memory, one per
// tile parity); pass 2 loads, multiplies and accumulates only those blocks (rows that
// pruned a block of the mask get P = 0 there).  Tiles with more than kMaskBits blocks
// (sequences beyond 131072 tokens) visit every block in pass 2.
//
//   warp 0       TMA producer: Q tile; K blocks (pass 1), K and V blocks (pass 2)
//   warp 1       MMA issuer: S (8 x M128 N64 K16) into two TMEM slots, PV (4 x M128
//                N128 K16) into the O columns; S(j) waits for PV(j - 2), which reads
//                P(j - 2) from the same slot
//   warps 4-7    one thread per row: block decisions, statistics, P, the O epilogue
#include <math_constants.h>

#include "nsa_common.cuh"
#include "nsa_kernels.h"

namespace nsa {
namespace {

constexpr int kBfThreads = 256;
constexpr int kBfStages = 3;
constexpr int kBfRows = 128;       // threads of the row warpgroup
constexpr int kBfBS = 64;          // keys per block
constexpr int kMaskBits = 2048;    // blocks a tile's keep mask covers

struct alignas(1024) BsfaSmem {
    uint8_t q[2][kTileRows * 128];            // Q tile: [64-column half][row]
    uint8_t kv[kBfStages][2][2][kBfBS * 128]; // [stage][K, V][64-column half][key]
    uint64_t q_full, q_empty;
    uint64_t kv_full[kBfStages], kv_empty[kBfStages];
    uint64_t s_full[2], s_read[2], p_full[2], pv_done[2];
    uint64_t o_full, o_empty, drain;
    uint64_t mask_ready;                      // the rows finished pass 1 of the tile
    uint32_t keep[2][kMaskBits / 32];         // blocks kept by some row, per tile parity
    uint32_t tmem_base;
    int abort_flag;
};

struct BsfaPlan {
    const int32_t* cu;
    const int32_t* tile_off;   // [nseq + 1]: tiles of 128 / G tokens before sequence s
    const float* tau;          // [hq] thresholds
    int nseq, T, hq, hkv, G, tpt;
    float scale_log2;
    __nv_bfloat16* out;        // [T, hq, 128]
    float* lse;                // [hq, T]
    DevStatus* st;
};

__global__ void __launch_bounds__(32) k_bsfa_tiles(const int32_t* cu, int nseq, int tpt,
                                                   int32_t* tile_off) {
    if (threadIdx.x != 0) return;
    int acc = 0;
    for (int s = 0; s < nseq; ++s) {
        tile_off[s] = acc;
        acc += (__ldg(cu + s + 1) - __ldg(cu + s) + tpt - 1) / tpt;
    }
    tile_off[nseq] = acc;
}

__global__ void __launch_bounds__(kBfThreads, 1)
    k_bsfa_fwd(const BsfaPlan p, const __grid_constant__ CUtensorMap qmap,
               const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap) {
    extern __shared__ uint8_t smem_raw[];
    BsfaSmem& S = *reinterpret_cast<BsfaSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    DevStatus* st = p.st;
    constexpr uint32_t kColO = 2 * kBfBS;   // TMEM: S slots at 0, 64; O at 128 .. 255
    if (tid == 0) {
        S.abort_flag = (*reinterpret_cast<volatile int*>(&st->code) != 0);
        mbar_init(&S.q_full, 1);
        mbar_init(&S.q_empty, 1);
        for (int i = 0; i < kBfStages; ++i) {
            mbar_init(&S.kv_full[i], 1);
            mbar_init(&S.kv_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.s_full[i], 1);
            mbar_init(&S.s_read[i], kBfRows);
            mbar_init(&S.p_full[i], kBfRows);
            mbar_init(&S.pv_done[i], 1);
        }
        mbar_init(&S.o_full, 1);
        mbar_init(&S.o_empty, kBfRows);
        mbar_init(&S.mask_ready, kBfRows);
        mbar_init(&S.drain, 1);
        fence_barrier_init();
    }
    if (warp == 0) {
        __syncwarp();
        tmem_alloc(&S.tmem_base, 256);
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
    struct Tile { int s, g, i0, L, nkb; };
    auto tile_at = [&](int ti) {
        Tile t;
        t.g = ti % p.hkv;
        const int u = ti / p.hkv;
        t.s = upper_index(p.tile_off, p.nseq, u);
        t.i0 = (u - __ldg(p.tile_off + t.s)) * p.tpt;
        t.L = __ldg(p.cu + t.s + 1) - __ldg(p.cu + t.s);
        t.nkb = (min(t.i0 + p.tpt, t.L) - 1) / kBfBS + 1;   // key blocks up to the last row's
        return t;
    };
    const int bid = (int)blockIdx.x, grid = (int)gridDim.x;
    // pass 2 visits the blocks kb >= from whose bit is set in the tile's mask (every
    // block when the tile has more blocks than the mask covers); nkb when none is left
    auto next_kept = [&](const Tile& t, int n, int from) -> int {
        if (t.nkb > kMaskBits) return from;
        const volatile uint32_t* km = S.keep[n & 1];
        for (int w = from >> 5; w < (t.nkb + 31) >> 5; ++w) {
            uint32_t bits = km[w];
            if (w == (from >> 5)) bits &= ~0u << (from & 31);
            if (bits) {
                const int kb = w * 32 + __ffs(bits) - 1;
                return kb < t.nkb ? kb : t.nkb;
            }
        }
        return t.nkb;
    };

    if (warp == 0) {
        // ------------------------------------------------------------- TMA producer
        if (lane == 0) {
            prefetch_tmap(&qmap);
            prefetch_tmap(&kmap);
            prefetch_tmap(&vmap);
            int n = 0, u = 0, qpar = -1, kvpar[kBfStages];
            for (int i = 0; i < kBfStages; ++i) kvpar[i] = -1;
            bool ok = true;
            for (int ti = bid; ti < ntiles && ok; ti += grid, ++n) {
                const Tile t = tile_at(ti);
                if (!(ok = wait(&S.q_empty, (n & 1) ^ 1, 120))) break;
                const int tok0 = __ldg(p.cu + t.s) + t.i0;
                mbar_arrive_expect_tx(&S.q_full, 2u * kTileRows * 128u);
                tma_load_3d(S.q[0], &qmap, &S.q_full, 0, t.g * p.G, tok0);
                tma_load_3d(S.q[1], &qmap, &S.q_full, 64, t.g * p.G, tok0);
                qpar = n & 1;
                const int key0 = __ldg(p.cu + t.s);
                for (int pass = 0; pass < 2 && ok; ++pass) {
                    if (pass == 1 && !(ok = wait(&S.mask_ready, n & 1, 136))) break;
                    for (int kb = pass == 0 ? 0 : next_kept(t, n, 0); kb < t.nkb;
                         kb = pass == 0 ? kb + 1 : next_kept(t, n, kb + 1), ++u) {
                        const int stg = u % kBfStages;
                        if (!(ok = wait(&S.kv_empty[stg], ((u / kBfStages) & 1) ^ 1, 121))) break;
                        const int row = key0 + kb * kBfBS;
                        mbar_arrive_expect_tx(&S.kv_full[stg], (pass == 0 ? 2u : 4u) * kBfBS * 128u);
                        tma_load_3d(S.kv[stg][0][0], &kmap, &S.kv_full[stg], 0, t.g, row);
                        tma_load_3d(S.kv[stg][0][1], &kmap, &S.kv_full[stg], 64, t.g, row);
                        if (pass == 1) {
                            tma_load_3d(S.kv[stg][1][0], &vmap, &S.kv_full[stg], 0, t.g, row);
                            tma_load_3d(S.kv[stg][1][1], &vmap, &S.kv_full[stg], 64, t.g, row);
                        }
                        kvpar[stg] = (u / kBfStages) & 1;
                    }
                }
            }
            if (*abort_flag) {   // let copies still in flight land before the CTA exits
                if (qpar >= 0) mbar_wait(&S.q_full, qpar, st, 122);
                for (int i = 0; i < kBfStages; ++i)
                    if (kvpar[i] >= 0) mbar_wait(&S.kv_full[i], kvpar[i], st, 123);
            }
        }
    } else if (warp == 1) {
        // -------------------------------------------------------------- MMA issuer
        const uint32_t elected = elect_one();
        constexpr uint32_t kIdescS = idesc_f16kind_f32(false, 128, kBfBS, false, false);
        constexpr uint32_t kIdescO = idesc_f16kind_f32(false, 128, 128, false, true);
        constexpr uint32_t kQHalf = sizeof(S.q[0]) >> 4;
        constexpr uint32_t kKvStage = sizeof(S.kv[0]) >> 4, kKvHalf = sizeof(S.kv[0][0][0]) >> 4;
        const uint32_t q_desc0 = (uint32_t)smem_desc_sw128(smem_u32(S.q[0]), 16, 1024);
        const uint32_t k_desc0 = (uint32_t)smem_desc_sw128(smem_u32(S.kv[0][0][0]), 16, 1024);
        const uint32_t v_desc0 = (uint32_t)smem_desc_sw128(smem_u32(S.kv[0][1][0]), kBfBS * 128, 1024);
        // per TMEM slot: how its last S was released (0 none, 1 rows read it in pass 1,
        // 2 PV read P in pass 2) and how many releases of each kind it has had
        int last_kind[2] = {0, 0}, nread[2] = {0, 0}, npv[2] = {0, 0};
        int n = 0, u = 0, j = 0;
        bool ok = true;
        auto issue_s = [&](int jj, int stg) -> bool {
            const int slot = jj & 1;
            if (last_kind[slot] == 1 && !wait(&S.s_read[slot], (nread[slot] - 1) & 1, 124)) return false;
            if (last_kind[slot] == 2 && !wait(&S.pv_done[slot], (npv[slot] - 1) & 1, 125)) return false;
            tc_fence_after();
            const uint32_t tS = tmem + (uint32_t)slot * kBfBS;
            const uint32_t b0 = k_desc0 + (uint32_t)stg * kKvStage;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t off = (uint32_t)((ks >> 2) * kQHalf + (ks & 3) * 2);
                const uint32_t offk = (uint32_t)((ks >> 2) * kKvHalf + (ks & 3) * 2);
                mma_ss_e(tS, q_desc0 + off, b0 + offk, kIdescS, ks > 0 ? 1u : 0u, elected);
            }
            mma_commit_e(&S.s_full[slot], elected);
            return true;
        };
        for (int ti = bid; ti < ntiles && ok; ti += grid, ++n) {
            const Tile t = tile_at(ti);
            if (!(ok = wait(&S.q_full, n & 1, 126))) break;
            // pass 1: S of every block; the rows release each slot after reading it
            for (int kb = 0; kb < t.nkb && ok; ++kb, ++u, ++j) {
                const int stg = u % kBfStages;
                if (!(ok = wait(&S.kv_full[stg], (u / kBfStages) & 1, 127))) break;
                if (!(ok = issue_s(j, stg))) break;
                mma_commit_e(&S.kv_empty[stg], elected);
                last_kind[j & 1] = 1;
                ++nread[j & 1];
            }
            if (!ok) break;
            // the previous tile's O has been read out before this tile's first PV
            if (!(ok = wait(&S.o_empty, (n & 1) ^ 1, 128))) break;
            // pass 2 over the kept blocks: S(kb), then once the rows wrote P(kb), O += P(kb) V(kb)
            if (!(ok = wait(&S.mask_ready, n & 1, 134))) break;
            bool first = true;
            for (int kb = next_kept(t, n, 0); kb < t.nkb && ok; kb = next_kept(t, n, kb + 1), ++u, ++j) {
                const int stg = u % kBfStages, slot = j & 1;
                if (!(ok = wait(&S.kv_full[stg], (u / kBfStages) & 1, 129))) break;
                if (!(ok = issue_s(j, stg))) break;
                // P(j) is the rows' k-th write into this slot's p_full barrier
                if (!(ok = wait(&S.p_full[slot], npv[slot] & 1, 130))) break;
                tc_fence_after();
                const uint32_t tS = tmem + (uint32_t)slot * kBfBS, tO = tmem + kColO;
                const uint32_t b0 = v_desc0 + (uint32_t)stg * kKvStage;
#pragma unroll
                for (int ks = 0; ks < kBfBS / 16; ++ks)
                    mma_ts_e(tO, tS + (uint32_t)ks * 8u, b0 + (uint32_t)ks * 128u, kIdescO,
                             (!first || ks > 0) ? 1u : 0u, elected);
                first = false;
                mma_commit_e(&S.pv_done[slot], elected);
                mma_commit_e(&S.kv_empty[stg], elected);
                last_kind[slot] = 2;
                ++npv[slot];
            }
            if (!ok) break;
            mma_commit_e(&S.o_full, elected);
            mma_commit_e(&S.q_empty, elected);
        }
        mma_commit_e(&S.drain, elected);
        mbar_wait(&S.drain, 0, st, 131);
    } else if (warp >= 4) {
        // ------------------------------------------------------------------ rows
        const int quad = warp & 3, r = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const int tok = r / p.G, h = r - tok * p.G;
        const float c = p.scale_log2;
        int j = 0, n = 0, npv_row[2] = {0, 0};
        bool ok = true;
        for (int ti = bid; ti < ntiles && ok; ti += grid, ++n) {
            const Tile t = tile_at(ti);
            const int i = t.i0 + tok;
            const bool valid = i < t.L;
            const int head = t.g * p.G + h;
            const float tau2 = __ldg(p.tau + head) * 1.4426950408889634f;   // log2 units
            float m = -CUDART_INF_F, l = 0.f, lse2 = -CUDART_INF_F;
            // this tile's keep mask starts empty (the producer and the issuer finished
            // with the mask of tile n - 2 before this tile's first S could arrive)
            if (r < kMaskBits / 32) S.keep[n & 1][r] = 0u;
            if (kMaskBits / 32 > kBfRows)
                for (int w = r + kBfRows; w < kMaskBits / 32; w += kBfRows) S.keep[n & 1][w] = 0u;
            asm volatile("bar.sync 1, %0;" ::"n"(kBfRows) : "memory");
            for (int pass = 0; pass < 2 && ok; ++pass) {
                if (pass == 1) {
                    // every row's bits are in the mask once all rows have arrived
                    __threadfence_block();
                    mbar_arrive(&S.mask_ready);
                    if (!(ok = __all_sync(0xffffffffu, wait(&S.mask_ready, n & 1, 135)))) break;
                }
                for (int kb = pass == 0 ? 0 : next_kept(t, n, 0); kb < t.nkb;
                     kb = pass == 0 ? kb + 1 : next_kept(t, n, kb + 1), ++j) {
                    const int slot = j & 1;
                    if (!(ok = __all_sync(0xffffffffu, wait(&S.s_full[slot], (j >> 1) & 1, 132)))) break;
                    tc_fence_after();
                    float sv[64];
                    const uint32_t tS = tmem + (uint32_t)slot * kBfBS + lane_off;
                    tmem_ld64_sync(tS, sv);
                    const int lim = valid ? i - kb * kBfBS : -1;   // keys 0 .. lim are causal
                    float bm = -CUDART_INF_F;
#pragma unroll
                    for (int k = 0; k < 64; ++k) {
                        sv[k] = k <= lim ? sv[k] * c : -CUDART_INF_F;
                        bm = fmaxf(bm, sv[k]);
                    }
                    const bool kept = bm != -CUDART_INF_F && bm >= tau2;
                    if (pass == 0 && t.nkb <= kMaskBits && __any_sync(0xffffffffu, kept) && lane == 0)
                        atomicOr(&S.keep[n & 1][kb >> 5], 1u << (kb & 31));
                    if (pass == 0) {
                        tc_fence_before();
                        mbar_arrive(&S.s_read[slot]);
                        if (kept) {
                            const float mx = fmaxf(m, bm);
                            float acc = 0.f;
#pragma unroll
                            for (int k = 0; k < 64; ++k) acc += ex2_approx(sv[k] - mx);
                            l = l * ex2_approx(m - mx) + acc;
                            m = mx;
                        }
                    } else {
                        uint32_t pk[32];
#pragma unroll
                        for (int k2 = 0; k2 < 32; ++k2) {
                            const float a = kept ? ex2_approx(sv[2 * k2] - lse2) : 0.f;
                            const float b = kept ? ex2_approx(sv[2 * k2 + 1] - lse2) : 0.f;
                            pk[k2] = pack_bf16x2(a, b);
                        }
                        tmem_st32_sync(tS, pk);
                        tc_fence_before();
                        mbar_arrive(&S.p_full[slot]);
                        ++npv_row[slot];
                    }
                }
                if (pass == 0) lse2 = l > 0.f ? m + __log2f(l) : -CUDART_INF_F;
            }
            if (!ok) break;
            // O of this tile: all of its PV products have completed
            if (!(ok = __all_sync(0xffffffffu, wait(&S.o_full, n & 1, 133)))) break;
            tc_fence_after();
            float o[64];
            const uint32_t tO = tmem + kColO + lane_off;
            const int t_glob = __ldg(p.cu + t.s) + (valid ? i : 0);
            uint4* dst = reinterpret_cast<uint4*>(p.out + ((size_t)t_glob * p.hq + head) * kHeadDim);
            // a tile whose mask is empty issued no PV: its O columns are stale, O is 0
            const bool any_pv = next_kept(t, n, 0) < t.nkb;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                tmem_ld64_sync(tO + (uint32_t)half * 64u, o);
                if (!any_pv) {
#pragma unroll
                    for (int x = 0; x < 64; ++x) o[x] = 0.f;
                }
                if (valid) {
#pragma unroll
                    for (int q8 = 0; q8 < 8; ++q8)
                        dst[half * 8 + q8] = make_uint4(pack_bf16x2(o[8 * q8], o[8 * q8 + 1]),
                                                        pack_bf16x2(o[8 * q8 + 2], o[8 * q8 + 3]),
                                                        pack_bf16x2(o[8 * q8 + 4], o[8 * q8 + 5]),
                                                        pack_bf16x2(o[8 * q8 + 6], o[8 * q8 + 7]));
                }
            }
            if (valid && p.lse) p.lse[(size_t)head * p.T + t_glob] = lse2 * 0.69314718055994531f;
            tc_fence_before();
            mbar_arrive(&S.o_empty);
        }
        (void)npv_row;
    }

    // ---- teardown: every role has left its loop (all waits are bounded) and the MMA
    //      issuer has drained its tensor-core work
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

}  // namespace

cudaError_t launch_bsfa_fwd(const int32_t* cu, int nseq, int T, int hq, int hkv, float scale,
                            const float* tau, void* out, float* lse, int32_t* tile_off,
                            DevStatus* st, int num_sms, const CUtensorMap* qmap,
                            const CUtensorMap* kmap, const CUtensorMap* vmap,
                            cudaStream_t stream) {
    BsfaPlan p{};
    p.cu = cu;
    p.tile_off = tile_off;
    p.tau = tau;
    p.nseq = nseq;
    p.T = T;
    p.hq = hq;
    p.hkv = hkv;
    p.G = hq / hkv;
    p.tpt = kTileRows / p.G;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.out = static_cast<__nv_bfloat16*>(out);
    p.lse = lse;
    p.st = st;
    k_bsfa_tiles<<<1, 32, 0, stream>>>(cu, nseq, p.tpt, tile_off);
    const size_t smem = sizeof(BsfaSmem) + 1024;
    cudaFuncSetAttribute(k_bsfa_fwd, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k_bsfa_fwd<<<num_sms, kBfThreads, smem, stream>>>(p, *qmap, *kmap, *vmap);
    return cudaGetLastError();
}

}  // namespace nsa
