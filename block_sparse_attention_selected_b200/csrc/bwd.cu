// bwd.cu -- backward tile kernel of selected-block attention (KV-block major).
//
// The full loss-backward named in the key-features table of the
// "Relaxed-System-Lab/Flash-Sparse-Attention" project page, organised like the
// forward: a work unit is up to `chunk_tiles` consecutive 128-row tiles of one
// (KV head, KV block) list.  Per tile (rows = gathered (token, head) pairs):
//
//   S  = Q K^T,  dP = dO V^T                    tcgen05.mma -> TMEM
//   P  = exp(scale S - LSE) (causal on the diagonal block, and on the block where a
//        sliding window starts),  dS = P (dP - D)
//   dV^T += dO^T P,  dK^T += Q^T dS              accumulate in TMEM over the unit
//   dQ_part = scale * dS K                       per (row, slot), bf16
//
// At the end of a unit dV and scale*dK of its block are written as fp32 partials;
// k_dkdv_reduce sums the units of each block in order and k_dq_merge sums the dQ
// partials of each row over its slots.  No atomics: the result is deterministic.
//
// One persistent CTA per SM takes units (largest first, dealt in snake order); it is
// warp-specialised:
//
//   warps 0-3          loaders: row metadata, TMA gather4 of the Q and dO rows (NQ
//                      stages; rows past the list read as zero, so they add nothing to dV / dK)
//   warp 12            TMA producer: K_B and V_B of each unit
//   warp 13            MMA issuer (one thread): S/dP may run one tile ahead of the
//                      dV/dK/dQ products; it issues whichever of the two is ready first
//   warps 4-11         P / dS, dQ epilogue and unit epilogue of every tile, the two
//                      warpgroups on one half of the columns each
//
// Work descriptors come from k_unit_desc; every wait is bounded (nsa_common.cuh).
#include <math_constants.h>

#include "nsa_common.cuh"
#include "nsa_kernels.h"

namespace nsa {
namespace {

// Warp roles (four warpgroups; warp % 4 = TMEM lane quadrant):
//   warpgroup 0 (warps 0-3)      Q / dO loaders, one tile row per lane
//   warpgroups 1, 2 (4-11)       P / dS and the epilogues, half of the columns each
//   warpgroup 3 (12-15)          TMA producer (12), MMA issuer (13); 14, 15 idle
// The 64 KB of Q and dO rows a tile needs arrive by TMA gather4 (four arbitrary rows of
// one 64-column half per instruction), issued by every fourth loader lane.  setmaxnreg
// rebalances the launch's 128 registers per thread: warpgroups 0 and 3 take 64, the
// P / dS warpgroups 192 (2 x 128 x 64 + 2 x 128 x 192 = 512 x 128).
constexpr int kThreads = 512;
constexpr int kLoaderWarps = 4;
constexpr int kLoaderThreads = kLoaderWarps * 32;
static_assert(kLoaderThreads == kTileRows, "one row per loader lane");
constexpr int kGatherLanes = kTileRows / 4;   // lanes that issue a tile's gathers
constexpr int kTmaWarp = 12, kMmaWarp = 13;
constexpr int kRegsLow = 64, kRegsWg = 192;
constexpr int kWgThreads = 128;

template <int N>
__device__ __forceinline__ void reg_dealloc() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void reg_alloc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

// TMEM slots of [S | dP] (dQ aliases a slot's first 128 columns): a third slot when
// it fits next to the dV^T / dK^T accumulators, so that S / dP of tile i + 1 need not
// wait for the dQ epilogue of tile i - 1, which runs after P / dS of tile i.
template <int BS, int NSLOT>
constexpr int bwd_tmem_slots() {
    return (NSLOT == 2 && 3 * 2 * BS + 2 * BS <= 512) ? 3 : NSLOT;
}

template <int BS, int NQ, int NSLOT>
struct alignas(1024) BwdSmem {
    static constexpr int NTS = bwd_tmem_slots<BS, NSLOT>();
    uint8_t q[NQ][2][kTileRows * 128];        // [stage][64-column half]
    uint8_t dout[NQ][2][kTileRows * 128];
    uint8_t k[2][BS * 128];                   // [half]
    uint8_t v[2][BS * 128];
    uint8_t p[BS / 64][kTileRows * 128];      // P bf16 [row][key], 64-key chunks
    uint8_t ds[BS / 64][kTileRows * 128];     // dS bf16 [row][key]
    int4 meta[NQ][kTileRows];                 // (token or -1, head, slot, causal limit)
    float rlse[NQ][kTileRows];                // row LSE * log2(e)
    float rdelta[NQ][kTileRows];              // row D = rowsum(dO * O)
    uint8_t dqs[8][32 * 64];                  // dQ staging: 32 rows x 32 columns per warp
    uint64_t q_full[NQ], q_empty[NQ], meta_full[NQ], meta_empty[NQ];
    uint64_t kv_full, kv_empty;
    uint64_t sdp_full[NTS], dq_full[NTS], tmem_empty[NTS];
    uint64_t pds_full, pds_empty, acc_full, acc_empty, drain;
    uint32_t tmem_base;
    int abort_flag;
    int nunits;
};

template <int BS, int NQ, int NSLOT>
constexpr size_t bwd_smem_bytes() {
    return sizeof(BwdSmem<BS, NQ, NSLOT>) + 1024;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

template <int BS, int NQ, int NSLOT, int F16>
__global__ void __launch_bounds__(kThreads, 1)
    k_bwd_tiles(const BwdPlan p, const __grid_constant__ CUtensorMap kmap,
                const __grid_constant__ CUtensorMap vmap, const __grid_constant__ CUtensorMap qmap,
                const __grid_constant__ CUtensorMap domap) {
    extern __shared__ uint8_t smem_raw[];
    BwdSmem<BS, NQ, NSLOT>& S = *reinterpret_cast<BwdSmem<BS, NQ, NSLOT>*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    DevStatus* st = p.st;
    constexpr int NTS = BwdSmem<BS, NQ, NSLOT>::NTS;

    if (tid == 0) {
        S.abort_flag = (*reinterpret_cast<volatile int*>(&st->code) != 0);
        S.nunits = *reinterpret_cast<volatile int*>(&st->nchunks);
        for (int i = 0; i < NQ; ++i) {
            // gathering lanes: every fourth (gather4), or one per token for G >= 8
            mbar_init(&S.q_full[i], p.G >= 8 ? kTileRows / p.G : kGatherLanes);
            mbar_init(&S.q_empty[i], 1);
            mbar_init(&S.meta_full[i], kLoaderThreads);
            mbar_init(&S.meta_empty[i], 2 * kWgThreads);
        }
        for (int i = 0; i < NTS; ++i) {
            mbar_init(&S.sdp_full[i], 1);
            mbar_init(&S.dq_full[i], 1);
            mbar_init(&S.tmem_empty[i], 2 * kWgThreads);
        }
        mbar_init(&S.kv_full, 1);
        mbar_init(&S.kv_empty, 1);
        mbar_init(&S.pds_full, 2 * kWgThreads);
        mbar_init(&S.pds_empty, 1);
        mbar_init(&S.acc_full, 1);
        mbar_init(&S.acc_empty, 2 * kWgThreads);
        mbar_init(&S.drain, 1);
        fence_barrier_init();
    }
    if (warp == 0) {
        __syncwarp();
        tmem_alloc(&S.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tmem = S.tmem_base;
    const int nunits = S.nunits;
    // units dealt in snake order over the list sorted by tile count (k_unit_order)
    const int ncta = (int)gridDim.x, cta = (int)blockIdx.x;
    auto rank_of = [&](int k) { return k * ncta + ((k & 1) ? ncta - 1 - cta : cta); };
    const int nfull = nunits / ncta;
    const int nk = S.abort_flag ? 0 : nfull + (rank_of(nfull) < nunits ? 1 : 0);
    auto unit_of = [&](int k) { return __ldg(p.uorder + rank_of(k)); };
    auto ld_unit = [&](int k) {
        return k < nk ? __ldg(p.udesc + unit_of(k)) : make_int4(0, 0, 0, 0);
    };
    auto ld_bucket = [&](int k) { return k < nk ? __ldg(p.ubucket + unit_of(k)) : -1; };
    const int tpt = kTileRows / p.G;
    volatile int* abort_flag = &S.abort_flag;
    auto wait = [&](uint64_t* bar, uint32_t parity, int where) -> bool {
        if (*abort_flag) return false;
        if (!mbar_wait(bar, parity, st, where)) {
            *abort_flag = 1;
            return false;
        }
        return true;
    };
    // TMEM columns: per slot [S | dP] (2*BS, dQ aliases its first 128), then dV^T, dK^T
    constexpr int kSlotCols = 2 * BS;
    constexpr int kColDV = NTS * kSlotCols;
    constexpr int kColDK = kColDV + BS;
    static_assert(kColDK + BS <= 512, "TMEM budget");

    const int wgrp = warp >> 2;
    const int li = wgrp == 0 ? warp : -1;

    if (wgrp == 0 || wgrp == 3) {
        reg_dealloc<kRegsLow>();
        if (li >= 0) {
            // ------------------------------------------------------------------ loaders
            // Loader w fills tile rows [32 w, 32 w + 32); lane l owns row 32 w + l: it
            // writes the row's metadata, LSE (times log2 e) and D into shared memory for the
            // P / dS warps and contributes the row's coordinate in the [T hq, 128] view of
            // Q and dO.  Lanes 4j then gather rows 32 w + 4j .. 32 w + 4j + 3: one gather4
            // per 64-column half and tensor, 2 KB per lane, armed on q_full with their byte
            // count.  A row past the list takes the out-of-range coordinate T hq and reads
            // as zero, so it adds nothing to dV and dK.
            const int w = li;
            const float kLog2e = 1.4426950408889634f;
            int4 u0 = ld_unit(0), u1 = ld_unit(1), u2 = ld_unit(2);
            const int rA = 32 * w + lane;
            auto ld_ent = [&](int e0, int ehi) -> uint32_t {
                return e0 + rA / p.G < ehi ? __ldg(p.entries + e0 + rA / p.G) : 0xFFFFFFFFu;
            };
            uint32_t entA = 0xFFFFFFFFu;
            if (nk > 0) entA = ld_ent(u0.y, u0.z);
            if (lane == 0) {
                prefetch_tmap(&qmap);
                prefetch_tmap(&domap);
            }
            const int oob_row = p.T * p.hq;
            int i = 0, issued = 0;
            bool stopped = false;
            for (int k = 0; k < nk && !stopped; ++k) {
                const int4 d = u0;
                u0 = u1; u1 = u2; u2 = ld_unit(k + 3);
                const int ntl = d.w & 255, g = d.w >> 8;
                for (int tt = 0; tt < ntl; ++tt, ++i) {
                    const int e0 = d.y + tt * tpt;
                    const int stg = i % NQ;
                    const uint32_t ph_empty = ((i / NQ) & 1) ^ 1;
                    const uint32_t ea = entA;
                    // index entries of the next tile (this unit's or the next unit's first)
                    if (tt + 1 < ntl) entA = ld_ent(e0 + tpt, d.z);
                    else if (k + 1 < nk) entA = ld_ent(u0.y, u0.z);
                    // this lane's row: metadata, LSE, D, row coordinate
                    int rowc = oob_row;
                    float lA = 0.f, dA = 0.f;
                    int4 mA = make_int4(-1, 0, 0, -1);
                    if (kChecks) {   // the gathered row must lie inside q and dout
                        const bool row_in = ea == 0xFFFFFFFFu ||
                                            ((int)(ea >> 6) < p.T && (int)(ea & 63u) < p.topk && g < p.hkv);
                        if (!__all_sync(0xffffffffu, check_ok(row_in, st, 142, i))) {
                            *abort_flag = 1;
                            stopped = true;
                            break;
                        }
                    }
                    if (ea != 0xFFFFFFFFu) {
                        mA = make_int4((int)(ea >> 6), g * p.G + rA % p.G, (int)(ea & 63u), (int)(ea >> 6) - d.x);
                        rowc = mA.x * p.hq + mA.y;
                        lA = __ldg(p.lse + (size_t)mA.y * p.T + mA.x) * kLog2e;
                        dA = __ldg(p.delta + (size_t)mA.y * p.T + mA.x);
                    }
                    if (!__all_sync(0xffffffffu, wait(&S.meta_empty[stg], ph_empty, 50))) {
                        stopped = true;
                        break;
                    }
                    S.meta[stg][rA] = mA;
                    S.rlse[stg][rA] = lA;
                    S.rdelta[stg][rA] = dA;
                    mbar_arrive(&S.meta_full[stg]);
                    if (!__all_sync(0xffffffffu, wait(&S.q_empty[stg], ph_empty, 51))) {
                        stopped = true;
                        break;
                    }
                    // gather Q and dO (the stage's previous readers, the products of tile
                    // i - NQ, completed before q_empty)
                    const int r1 = __shfl_down_sync(0xffffffffu, rowc, 1);
                    const int r2 = __shfl_down_sync(0xffffffffu, rowc, 2);
                    const int r3 = __shfl_down_sync(0xffffffffu, rowc, 3);
                    if (p.G >= 8) {
                        // the G rows of a token are adjacent in Q and dO and fill whole
                        // 1 KB swizzle atoms of the tile: one tiled box per token, half and
                        // tensor (the maps are 3D here: columns, heads, tokens), issued by
                        // the token's first lane; a token past the list reads as zero
                        if (rA % p.G == 0) {
                            const uint32_t ro = (uint32_t)rA * 128u;
                            const int tok = ea != 0xFFFFFFFFu ? mA.x : p.T;
                            mbar_arrive_expect_tx(&S.q_full[stg], 4u * (uint32_t)p.G * 128u);
                            tma_load_3d(S.q[stg][0] + ro, &qmap, &S.q_full[stg], 0, g * p.G, tok);
                            tma_load_3d(S.q[stg][1] + ro, &qmap, &S.q_full[stg], 64, g * p.G, tok);
                            tma_load_3d(S.dout[stg][0] + ro, &domap, &S.q_full[stg], 0, g * p.G, tok);
                            tma_load_3d(S.dout[stg][1] + ro, &domap, &S.q_full[stg], 64, g * p.G, tok);
                        }
                    } else if ((lane & 3) == 0) {
                        const uint32_t ro = (uint32_t)rA * 128u;
                        mbar_arrive_expect_tx(&S.q_full[stg], 4u * 4u * 128u);
                        tma_gather4(S.q[stg][0] + ro, &qmap, &S.q_full[stg], 0, rowc, r1, r2, r3);
                        tma_gather4(S.q[stg][1] + ro, &qmap, &S.q_full[stg], 64, rowc, r1, r2, r3);
                        tma_gather4(S.dout[stg][0] + ro, &domap, &S.q_full[stg], 0, rowc, r1, r2, r3);
                        tma_gather4(S.dout[stg][1] + ro, &domap, &S.q_full[stg], 64, rowc, r1, r2, r3);
                    }
                    issued = i + 1;
                }
            }
            // nothing may still be in flight when the CTA exits: after an abort, wait
            // (bounded) for the last gathers into every stage
            if (*abort_flag)
                for (int j = issued - 1; j >= 0 && j >= issued - NQ; --j)
                    mbar_wait(&S.q_full[j % NQ], (j / NQ) & 1, st, 53);
        } else if (warp == kTmaWarp) {
            // ------------------------------------------------------------- K/V producer
            if (lane == 0) {
                prefetch_tmap(&kmap);
                prefetch_tmap(&vmap);
                int prev = -1, loads = 0, last_parity = 0;
                bool loaded = false;
                int4 u0 = ld_unit(0), u1 = ld_unit(1);
                int b0 = ld_bucket(0), b1 = ld_bucket(1);
                for (int k = 0; k < nk; ++k) {
                    const int4 d = u0;
                    const int b = b0;
                    u0 = u1; b0 = b1; u1 = ld_unit(k + 2); b1 = ld_bucket(k + 2);
                    if (b == prev) continue;
                    prev = b;
                    if (!check_ok(d.x >= 0 && d.x < p.T && (d.w >> 8) < p.hkv, st, 143, k)) {
                        *abort_flag = 1;
                        break;
                    }
                    if (!wait(&S.kv_empty, (loads & 1) ^ 1, 52)) break;
                    const int g = d.w >> 8;
                    mbar_arrive_expect_tx(&S.kv_full, 4u * BS * 128u);
                    tma_load_3d(S.k[0], &kmap, &S.kv_full, 0, g, d.x);
                    tma_load_3d(S.k[1], &kmap, &S.kv_full, 64, g, d.x);
                    tma_load_3d(S.v[0], &vmap, &S.kv_full, 0, g, d.x);
                    tma_load_3d(S.v[1], &vmap, &S.kv_full, 64, g, d.x);
                    last_parity = loads & 1;
                    loaded = true;
                    ++loads;
                }
                if (*abort_flag && loaded) mbar_wait(&S.kv_full, last_parity, st, 53);
            }
        } else if (warp == kMmaWarp) {
            // -------------------------------------------------------------- MMA issuer
            // The whole warp runs the issue loop (warp-uniform state and decisions); one
            // elected lane executes the tcgen05 instructions.
            {
                const uint32_t elected = elect_one();
                constexpr uint32_t kIdescS = idesc_f16kind_f32(F16, 128, BS, false, false);  // S, dP
                constexpr uint32_t kIdescT = idesc_f16kind_f32(F16, 128, BS, true, true);    // dV^T, dK^T
                constexpr uint32_t kIdescQ = idesc_f16kind_f32(F16, 128, 128, false, true);  // dQ
                int kv_loads = 0, prev_bucket = -1;
                bool ok = true;
                // Shared-memory descriptors are computed once; an MMA step adds its byte
                // offset / 16 to the start-address field (addresses < 2^18 bytes: no carry
                // out of the 14-bit field).  K-major operands: LBO 16, SBO 1024 (the 64-column
                // half of a tile is a separate base); MN-major ones: LBO = the stride between
                // 64-element halves (or 64-key chunks), SBO 1024.
                constexpr uint32_t kQStage = sizeof(S.q[0]) >> 4, kQHalf = sizeof(S.q[0][0]) >> 4;
                constexpr uint32_t kKHalf = sizeof(S.k[0]) >> 4, kPChunk = sizeof(S.p[0]) >> 4;
                const uint32_t dq_q = (uint32_t)smem_desc_sw128(smem_u32(S.q[0][0]), 16, 1024);       // Q, K-major
                const uint32_t dq_do = (uint32_t)smem_desc_sw128(smem_u32(S.dout[0][0]), 16, 1024);   // dO, K-major
                const uint32_t dq_k = (uint32_t)smem_desc_sw128(smem_u32(S.k[0]), 16, 1024);          // K, K-major
                const uint32_t dq_v = (uint32_t)smem_desc_sw128(smem_u32(S.v[0]), 16, 1024);          // V, K-major
                const uint32_t dt_q = (uint32_t)smem_desc_sw128(smem_u32(S.q[0][0]), 16384, 1024);    // Q^T
                const uint32_t dt_do = (uint32_t)smem_desc_sw128(smem_u32(S.dout[0][0]), 16384, 1024); // dO^T
                const uint32_t dt_p = (uint32_t)smem_desc_sw128(smem_u32(S.p[0]), 16384, 1024);       // P (keys x rows)
                const uint32_t dt_ds = (uint32_t)smem_desc_sw128(smem_u32(S.ds[0]), 16384, 1024);     // dS (keys x rows)
                const uint32_t dk_ds = (uint32_t)smem_desc_sw128(smem_u32(S.ds[0]), 16, 1024);        // dS, K-major
                const uint32_t dk_kmn = (uint32_t)smem_desc_sw128(smem_u32(S.k[0]), BS * 128, 1024);  // K, MN-major
                auto sdp = [&](int i, bool newkv) -> bool {
                    if (newkv) {
                        if (!wait(&S.kv_full, kv_loads & 1, 54)) return false;
                        ++kv_loads;
                    }
                    const int s = i % NTS, stg = i % NQ;
                    if (!wait(&S.tmem_empty[s], ((i / NTS) & 1) ^ 1, 55)) return false;
                    if (!wait(&S.q_full[stg], (i / NQ) & 1, 56)) return false;
                    tc_fence_after();
                    const uint32_t tS = tmem + s * kSlotCols, tdP = tS + BS;
                    const uint32_t aq = dq_q + (uint32_t)stg * kQStage, ad = dq_do + (uint32_t)stg * kQStage;
    #pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        const uint32_t oa = (uint32_t)((ks >> 2) * kQHalf + (ks & 3) * 2);
                        const uint32_t ob = (uint32_t)((ks >> 2) * kKHalf + (ks & 3) * 2);
                        mma_ss_e(tS, aq + oa, dq_k + ob, kIdescS, ks > 0 ? 1u : 0u, elected);
                    }
    #pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        const uint32_t oa = (uint32_t)((ks >> 2) * kQHalf + (ks & 3) * 2);
                        const uint32_t ob = (uint32_t)((ks >> 2) * kKHalf + (ks & 3) * 2);
                        mma_ss_e(tdP, ad + oa, dq_v + ob, kIdescS, ks > 0 ? 1u : 0u, elected);
                    }
                    mma_commit_e(&S.sdp_full[s], elected);
                    return true;
                };
                auto rest = [&](int i, bool first, bool last, int k, bool release_kv) -> bool {
                    const int s = i % NTS, stg = i % NQ;
                    if (!wait(&S.pds_full, i & 1, 57)) return false;
                    if (first && !wait(&S.acc_empty, (k & 1) ^ 1, 58)) return false;
                    tc_fence_after();
                    const uint32_t aq = dt_q + (uint32_t)stg * kQStage, ad = dt_do + (uint32_t)stg * kQStage;
    #pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {   // K = 128 rows, 16 per step (2048 bytes)
                        const uint32_t off = (uint32_t)ks * 128u;
                        const uint32_t acc = (first && ks == 0) ? 0u : 1u;
                        mma_ss_e(tmem + kColDV, ad + off, dt_p + off, kIdescT, acc, elected);
                        mma_ss_e(tmem + kColDK, aq + off, dt_ds + off, kIdescT, acc, elected);
                    }
                    mma_commit_e(&S.q_empty[stg], elected);   // the stage is free once dV / dK have read it
    #pragma unroll
                    for (int ks = 0; ks < BS / 16; ++ks)   // K = BS keys
                        mma_ss_e(tmem + s * kSlotCols,
                                 dk_ds + (uint32_t)((ks >> 2) * kPChunk + (ks & 3) * 2),
                                 dk_kmn + (uint32_t)ks * 128u, kIdescQ, ks > 0 ? 1u : 0u, elected);
                    mma_commit_e(&S.dq_full[s], elected);
                    mma_commit_e(&S.pds_empty, elected);
                    if (last) {
                        mma_commit_e(&S.acc_full, elected);
                        if (release_kv) mma_commit_e(&S.kv_empty, elected);
                    }
                    return true;
                };
                // Tiles in order, S/dP running at most one tile ahead of the products (two
                // TMEM slots, two Q/dO stages).  The issuer serves whichever is ready first:
                // the products of the oldest tile whose S/dP is done (preferred: they release
                // its Q/dO stage for the gather two tiles on) or S/dP of the next tile.  A
                // fixed order would make each stage's release wait for the next tile's gather.
                // S/dP of a tile that needs a new K/V block waits until every product of the
                // previous block is issued (a single K/V buffer).
                int fk = 0, ftt = 0, fi = 0;                 // next S/dP: unit, tile in unit, index
                int4 fu = ld_unit(0), fu1 = ld_unit(1);
                int fb = ld_bucket(0), fb1 = ld_bucket(1);
                int ri = 0;                                  // next products: tile index
                // pending tiles' flags, even / odd tile index: unit << 3 | release K/V << 2 |
                // last of unit << 1 | first of unit (registers, no local-memory array)
                int pend0 = 0, pend1 = 0;
                long long idle_since = clock64();
                const long long wait_budget =
                    st->wait_budget > 0 ? st->wait_budget : kWaitBudgetCycles;
                while (ok && (fk < nk || ri < fi)) {
                    bool go_r = false, go_s = false;
                    const int pend = (ri & 1) ? pend1 : pend0;
                    const bool newkv = ftt == 0 && fb != prev_bucket;
                    if (lane == 0) {   // one lane polls (32 lanes on one barrier serialise)
                        if (ri < fi)
                            go_r = mbar_test(&S.pds_full, ri & 1) &&
                                   (!(pend & 1) || mbar_test(&S.acc_empty, ((pend >> 3) & 1) ^ 1));
                        if (!go_r && fk < nk && fi - ri <= 1)
                            go_s = (!newkv || ri == fi) &&
                                   mbar_test(&S.q_full[fi % NQ], (fi / NQ) & 1) &&
                                   mbar_test(&S.tmem_empty[fi % NTS], ((fi / NTS) & 1) ^ 1) &&
                                   (!newkv || mbar_test(&S.kv_full, kv_loads & 1));
                    }
                    go_r = __shfl_sync(0xffffffffu, go_r, 0);
                    go_s = __shfl_sync(0xffffffffu, go_s, 0);
                    if (go_r) {
                        ok = rest(ri, pend & 1, (pend >> 1) & 1, pend >> 3, (pend >> 2) & 1);
                        ++ri;
                        idle_since = clock64();
                    } else if (go_s) {
                        const int ntl = fu.w & 255;
                        const bool lst = ftt == ntl - 1;
                        const int info = (fk << 3) | ((lst && (fk + 1 >= nk || fb1 != fb)) << 2) |
                                         (lst << 1) | (ftt == 0);
                        if (fi & 1) pend1 = info; else pend0 = info;
                        ok = sdp(fi, newkv);
                        if (newkv) prev_bucket = fb;
                        ++fi;
                        if (++ftt == ntl) {
                            ftt = 0;
                            ++fk;
                            fu = fu1; fb = fb1;
                            fu1 = ld_unit(fk + 1); fb1 = ld_bucket(fk + 1);
                        }
                        idle_since = clock64();
                    } else if (__shfl_sync(0xffffffffu, *abort_flag, 0)) {
                        ok = false;
                    } else if (__shfl_sync(0xffffffffu, clock64() - idle_since > wait_budget, 0)) {
                        if (lane == 0) record_error(st, NSA_ERR_TIMEOUT, 56, blockIdx.x);
                        *abort_flag = 1;
                        ok = false;
                    }
                }
                mma_commit_e(&S.drain, elected);
                mbar_wait(&S.drain, 0, st, 59);
            }
        }
    } else {
        reg_alloc<kRegsWg>();
        // ------------------------------------------------- P / dS and the epilogues
        // Both warpgroups work on every tile, warpgroup wg on half of its columns: keys
        // [wg BS/2, (wg + 1) BS/2) of P / dS and of the unit's dV / dK, columns
        // [64 wg, 64 wg + 64) of dQ.  Row r = TMEM lane (= d for dV^T / dK^T).  With two
        // TMEM slots the dQ epilogue of tile i - 1 runs after P / dS of tile i is stored,
        // so that the products of tile i can follow those of tile i - 1 at once.
        constexpr int kKeysWg = BS / 2;
        constexpr bool kDefer = NSLOT == 2;
        const int wg = (warp - 4) >> 2;
        const int r = (warp & 3) * 32 + lane;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        uint8_t* const dqb = static_cast<uint8_t*>(p.part_dq);
        const uint32_t sb = smem_u32(S.dqs[warp - 4]);
        const float2 sc2 = make_float2(p.scale, p.scale);
        // dQ partial of tile j (row r, this warpgroup's 64 columns); then, after the
        // unit's last tile, dV and scale*dK of its block as fp32 [2][BS][128]
        auto epilogue = [&](int j, long long prow, bool unit_last, int k) -> bool {
            const int s = j % NTS;
            if (!wait(&S.dq_full[s], (j / NTS) & 1, 63)) return false;
            tc_fence_after();
            const uint32_t tq = tmem + s * kSlotCols + lane_off;
            // per 32-column quarter: scale, bf16, stage the warp's 32 rows (16-byte pieces
            // XOR-swizzled so that both phases are conflict-free), then write 8 rows x 64
            // contiguous bytes per warp instruction.  The TMEM slot is released as soon as
            // the warpgroup's last quarter is read.
#pragma unroll 1
            for (int h = 0; h < 2; ++h) {
                const int qtr = 2 * wg + h;
                float o[32];
                tmem_ld32_sync(tq + qtr * 32, o);
                if (h == 1) {
                    tc_fence_before();
                    mbar_arrive(&S.tmem_empty[s]);
                }
#pragma unroll
                for (int pc = 0; pc < 4; ++pc) {
                    uint32_t u[4];
#pragma unroll
                    for (int q2 = 0; q2 < 4; ++q2) {
                        const float2 z = mul2(make_float2(o[pc * 8 + 2 * q2], o[pc * 8 + 2 * q2 + 1]), sc2);
                        u[q2] = pack_bf16x2(z.x, z.y);
                    }
                    st_shared_v4(sb + lane * 64 + ((pc ^ ((lane >> 1) & 3)) << 4), u[0], u[1], u[2], u[3]);
                }
                __syncwarp();
#pragma unroll
                for (int it = 0; it < 4; ++it) {
                    const int rr = it * 8 + (lane >> 2), pc = lane & 3;
                    const long long gr = __shfl_sync(0xffffffffu, prow, rr);
                    uint4 v;
                    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                                 : "r"(sb + rr * 64 + ((pc ^ ((rr >> 1) & 3)) << 4))
                                 : "memory");
                    if (gr >= 0)
                        *reinterpret_cast<uint4*>(dqb + gr * (kHeadDim * 2) + qtr * 64 + pc * 16) = v;
                }
                __syncwarp();
            }
            if (unit_last) {
                if (!wait(&S.acc_full, k & 1, 64)) return false;
                tc_fence_after();
                float* dvp = p.part_dkdv + (size_t)unit_of(k) * 2 * BS * kHeadDim;
                float* dkp = dvp + (size_t)BS * kHeadDim;
#pragma unroll 1
                for (int c32 = wg * (kKeysWg / 32); c32 < (wg + 1) * (kKeysWg / 32); ++c32) {
                    float xv[32], xk[32];
                    tmem_ld32_sync(tmem + kColDV + lane_off + c32 * 32, xv);
                    tmem_ld32_sync(tmem + kColDK + lane_off + c32 * 32, xk);
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const int key = c32 * 32 + c;
                        dvp[(size_t)key * kHeadDim + r] = xv[c];
                        dkp[(size_t)key * kHeadDim + r] = xk[c] * p.scale;
                    }
                }
                tc_fence_before();
                mbar_arrive(&S.acc_empty);
            }
            return true;
        };
        int4 u0 = ld_unit(0), u1 = ld_unit(1);
        int i = 0;
        bool ok = true;
        long long prev_prow = -1;
        bool prev_last = false;
        int prev_k = 0;
        for (int k = 0; k < nk && ok; ++k) {
            const int4 d = u0;
            u0 = u1; u1 = ld_unit(k + 2);
            const int ntl = d.w & 255;
            for (int tt = 0; tt < ntl && ok; ++tt, ++i) {
                const int stg = i % NQ, s = i % NTS;
                if (!(ok = wait(&S.meta_full[stg], (i / NQ) & 1, 60))) break;
                const int4 m = S.meta[stg][r];
                const float lse2 = S.rlse[stg][r], delta = S.rdelta[stg][r];
                mbar_arrive(&S.meta_empty[stg]);
                const int my_lim = m.w;                   // keys my_lo .. my_lim visible
                const int my_lo = p.swin > 0 ? my_lim - p.swin + 1 : 0;
                const long long prow = m.x < 0 ? -1ll : ((long long)m.x * p.hq + m.y) * p.topk + m.z;
                if (!(ok = wait(&S.sdp_full[s], (i / NTS) & 1, 61))) break;
                tc_fence_after();
                // P and dS of this row over the warpgroup's keys, into registers while the
                // products of the previous tile may still read the P / dS tile
                const uint32_t tS = tmem + s * kSlotCols + lane_off + wg * kKeysWg, tdP = tS + BS;
                uint32_t pk[kKeysWg / 2], dk[kKeysWg / 2];
                {
                    float sv[kKeysWg], dp[kKeysWg];
                    if constexpr (kKeysWg == 32) {
                        tmem_ld32_sync(tS, sv);
                        tmem_ld32_sync(tdP, dp);
                    } else {
                        tmem_ld64_sync(tS, sv);
                        tmem_ld64_sync(tdP, dp);
                    }
                    const float2 c2 = make_float2(p.scale_log2, p.scale_log2);
                    const float2 nl2 = make_float2(-lse2, -lse2), nd2 = make_float2(-delta, -delta);
                    auto p_ds = [&](const bool masked) {
#pragma unroll
                        for (int c = 0; c < kKeysWg; c += 2) {
                            const int key = wg * kKeysWg + c;
                            float2 x = fma2(make_float2(sv[c], sv[c + 1]), c2, nl2);
                            if (masked) {
                                x.x = (key <= my_lim && key >= my_lo) ? ex2_approx(x.x) : 0.f;
                                x.y = (key + 1 <= my_lim && key + 1 >= my_lo) ? ex2_approx(x.y) : 0.f;
                            } else {
                                x.x = ex2_approx(x.x);
                                x.y = ex2_approx(x.y);
                            }
                            const float2 ds = mul2(x, add2(make_float2(dp[c], dp[c + 1]), nd2));
                            pk[c / 2] = pack2<F16>(x.x, x.y);    // P, dS in the operands' type
                            dk[c / 2] = pack2<F16>(ds.x, ds.y);
                        }
                    };
                    // warps whose rows all see every key of this warpgroup's half skip the
                    // mask (padding rows have my_lim = -1 and always take the masked form)
                    if (__all_sync(0xffffffffu, my_lo <= wg * kKeysWg && my_lim >= (wg + 1) * kKeysWg - 1))
                        p_ds(false);
                    else
                        p_ds(true);
                }
                tc_fence_before();
                if (!(ok = wait(&S.pds_empty, (i & 1) ^ 1, 62))) break;
#pragma unroll
                for (int pc = 0; pc < kKeysWg / 8; ++pc) {   // 16-byte pieces of 8 keys
                    const int gp = wg * (kKeysWg / 8) + pc;
                    const int c64 = gp >> 3, pp = gp & 7;
                    st_shared_v4(smem_u32(S.p[c64]) + sw128_offset(r, pp), pk[pc * 4], pk[pc * 4 + 1],
                                 pk[pc * 4 + 2], pk[pc * 4 + 3]);
                    st_shared_v4(smem_u32(S.ds[c64]) + sw128_offset(r, pp), dk[pc * 4], dk[pc * 4 + 1],
                                 dk[pc * 4 + 2], dk[pc * 4 + 3]);
                }
                fence_async_smem();
                mbar_arrive(&S.pds_full);
                const bool last = tt == ntl - 1;
                if constexpr (kDefer) {
                    if (i > 0 && !(ok = epilogue(i - 1, prev_prow, prev_last, prev_k))) break;
                    prev_prow = prow;
                    prev_last = last;
                    prev_k = k;
                } else {
                    if (!(ok = epilogue(i, prow, last, k))) break;
                }
            }
        }
        if (kDefer && ok && i > 0) epilogue(i - 1, prev_prow, prev_last, prev_k);
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace

template <int BS, int NQ, int NSLOT, int F16>
static void launch_bwd_variant(const BwdPlan& p, const CUtensorMap* kmap, const CUtensorMap* vmap,
                               const CUtensorMap* qmap, const CUtensorMap* domap,
                               cudaStream_t stream) {
    constexpr size_t smem = bwd_smem_bytes<BS, NQ, NSLOT>();
    cudaFuncSetAttribute(k_bwd_tiles<BS, NQ, NSLOT, F16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    k_bwd_tiles<BS, NQ, NSLOT, F16><<<p.num_sms, kThreads, smem, stream>>>(p, *kmap, *vmap, *qmap,
                                                                          *domap);
}

cudaError_t launch_bwd_tiles(const BwdPlan& p, const CUtensorMap* kmap, const CUtensorMap* vmap,
                             const CUtensorMap* qmap, const CUtensorMap* domap,
                             cudaStream_t stream) {
    if (p.bs == 64) {
        if (p.f16) launch_bwd_variant<64, 2, 2, 1>(p, kmap, vmap, qmap, domap, stream);
        else launch_bwd_variant<64, 2, 2, 0>(p, kmap, vmap, qmap, domap, stream);
    } else {
        if (p.f16) launch_bwd_variant<128, 1, 1, 1>(p, kmap, vmap, qmap, domap, stream);
        else launch_bwd_variant<128, 1, 1, 0>(p, kmap, vmap, qmap, domap, stream);
    }
    return cudaGetLastError();
}

}  // namespace nsa
