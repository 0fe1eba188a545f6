// fwd.cu -- forward tile kernel of selected-block attention (KV-block major).
//
// A tile is (KV head g, KV block B, up to 128 gathered query rows), a row being
// (token, query head) for a token whose index row selected B; the G query heads of a
// token are adjacent rows, so a group of any size fills the 128-row tensor-core tile
// (the loop swap of the FSA pages: "FSA: Efficient Implementation of Native Sparse
// Attention" blog, second paragraph).  Per tile:
//
//   S   = Q K_B^T                  tcgen05.mma (Q, K from shared memory) -> TMEM
//   P   = exp2(c S - c m), causal mask on the diagonal block (and, under a sliding
//         window, on the block where the window starts), l = sum P; P is written as
//         bf16 back into the S columns of TMEM
//   O_B = P V_B                    tcgen05.mma with A = P read from TMEM
//   partial: O_B * 2^-e / lr as fp16 (lr the sum of the rounded P values O_B used),
//         lse_B = m + log l (l the fp32 sum), and the factor f that brings the stored
//         row back to the block's convex combination of V_B's rows.  e is the block's V
//         exponent (k_vblock_exp): 0 unless max |V_B| > 2^14, so the convex combination
//         always fits fp16 after the 2^-e.
//
// A tile covers the consecutive entries [e0, e0 + ntok) of the sorted index list
// (invert.cu), so its partial rows (entry * G + head offset) are one contiguous
// range: the epilogue stages them in shared memory and writes whole 128-byte lines.
// The merge (merge.cu) finds a (token, head, slot)'s partial through the position map
// of the inversion.
//
// Tiles come in (g, token window, B) order; one persistent CTA per SM takes chunks of
// kChunk consecutive tiles round-robin (consecutive tiles of one (g, window, B) list
// share K_B / V_B).  Each CTA is warp-specialised and pipelined:
//
//   warps 0-3, 18, 19  Q loaders: coalesced cp.async gather (two 256-byte rows per warp
//                      instruction) into the 128B-swizzled Q tile, kNQ stages
//   warp 16            TMA producer: K_B and V_B (128B swizzle) into NKV stages
//   warp 17            MMA issuer (one elected lane of a warp-uniform loop): S(i+1) is
//                      issued before PV(i)
//   warps 4-7          softmax of even tiles  } TMEM slot 0 / 1: S (P)
//   warps 8-11         softmax of odd tiles   }
//   warps 12-15        epilogue of every tile: O from TMEM, scale, fp16, store
//
// The softmax hands each row's scale 2^-e / l to the epilogue in shared memory
// (double-buffered per slot, with its own barrier).  Producer/consumer hand-offs are
// mbarriers; every wait is bounded (nsa_common.cuh).
#include <math_constants.h>

#include "nsa_common.cuh"
#include "nsa_kernels.h"

namespace nsa {
namespace {

// Warp roles (five warpgroups; warp % 4 = TMEM lane quadrant):
//   warpgroup 0 (warps 0-3)    Q loaders 0-3
//   warpgroups 1, 2 (4-11)     softmax of even / odd tiles
//   warpgroup 3 (12-15)        epilogue
//   warpgroup 4 (16-19)        TMA producer (16), MMA issuer (17), Q loaders 4-5 (18, 19)
// The gather's throughput grows with the number of warps issuing cp.async, so six
// warps load Q.  Registers are rebalanced with setmaxnreg: the launch gives every
// thread 96; warpgroups 0 and 4 drop to 56, the softmax warpgroups rise to 136
// (2 x 128 x 56 + 128 x 96 + 2 x 128 x 136 = 640 x 96).
constexpr int kThreads = 640;
constexpr int kLoaderWarps = 6;
constexpr int kLoaderThreads = kLoaderWarps * 32;
constexpr int kRowsPerLoader = (kTileRows + kLoaderWarps - 1) / kLoaderWarps;   // 22
static_assert(kRowsPerLoader <= 32, "one row per loader lane");
constexpr int kTmaWarp = 16, kMmaWarp = 17;
constexpr int kRegsLow = 56, kRegsSoftmax = 136;

template <int N>
__device__ __forceinline__ void reg_dealloc() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void reg_alloc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
constexpr int kWgThreads = 128;
constexpr int kChunk = 4;      // consecutive tiles per scheduling chunk
// Per head dimension D = 64 NH (NH 64-column halves):
//   kNQ   Q stages (S(i) completing frees stage i % kNQ: q_empty); two for D = 256,
//         whose 64 KB Q tiles leave room for one K / V stage only
//   kNSt  epilogue staging halves per warp (reused every kNSt halves)
template <int NH>
struct FwdCfg {
    static constexpr int kNQ = NH == 4 ? 2 : 3;
    static constexpr int kNSt = NH == 4 ? 1 : 2;
};
// Row-scale buffers: softmax(i + kNSc) may run once PV(i + kNSc - 2) is issued, which
// waits for the epilogue of tile i + kNSc - 2 - NO; kNSc >= NO + 2 keeps it behind the
// epilogue's read of sc[i % kNSc].
constexpr int kNSc = 8;

template <int BS, int NKV, int NH>
struct alignas(1024) FwdSmem {
    static constexpr int kNQ = FwdCfg<NH>::kNQ;
    uint8_t q[kNQ][NH][kTileRows * 128];      // Q tile per stage: [64-column half][row]
    uint8_t kv[NKV][2][NH][BS * 128];         // [stage][K, V][64-column half][key]
    uint8_t stage[4][FwdCfg<NH>::kNSt][32 * 128];   // epilogue staging: [warp][half buffer]
    float sc[kNSc][kTileRows];                // row scale 2^-e / l of tile i in sc[i % kNSc]
    uint64_t q_full[kNQ], q_empty[kNQ];
    uint64_t kv_full[NKV], kv_empty[NKV];
    uint64_t s_full[2], p_full[2];
    uint64_t o_full[3], o_free[3];            // O accumulator buffers (1 to 3 of them)
    uint64_t pv_done[2];                      // PV of S slot s done (one O buffer only)
    uint64_t l_full[kNSc];                    // sc[i % kNSc] written
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
    int ntiles;
};

template <int BS, int NKV, int NH>
constexpr size_t fwd_smem_bytes() {
    return sizeof(FwdSmem<BS, NKV, NH>) + 1024;
}

__device__ __forceinline__ void cp_async_wait_one_pending() {
    asm volatile("cp.async.wait_group 1;" ::: "memory");
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

template <int BS, int NKV, int NH, int F16>
__global__ void __launch_bounds__(kThreads, 1)
    k_fwd_tiles(const FwdPlan p, const __grid_constant__ CUtensorMap kmap,
                const __grid_constant__ CUtensorMap vmap, const __grid_constant__ CUtensorMap omap8,
                const __grid_constant__ CUtensorMap omap32) {
    constexpr int kNQ = FwdCfg<NH>::kNQ, kNSt = FwdCfg<NH>::kNSt;
    constexpr int D = 64 * NH;                // head dimension
    extern __shared__ uint8_t smem_raw[];
    FwdSmem<BS, NKV, NH>& S = *reinterpret_cast<FwdSmem<BS, NKV, NH>*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    DevStatus* st = p.st;
    // TMEM columns: S of slot s (and P, bf16, in its first BS/2 columns) at s * BS;
    // O accumulator buffer b at 2 * BS + b * D.
    constexpr int NO = NH == 4 ? 1 : ((BS == 64 || NH == 1) ? 3 : 2);
    constexpr int kColO = 2 * BS;
    static_assert(kColO + NO * D <= 512, "TMEM budget");

    if (tid == 0) {
        S.abort_flag = (*reinterpret_cast<volatile int*>(&st->code) != 0);
        S.ntiles = *reinterpret_cast<volatile int*>(&st->ntiles_fwd);
        for (int i = 0; i < kNQ; ++i) {
            mbar_init(&S.q_full[i], kLoaderThreads);
            mbar_init(&S.q_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.s_full[i], 1);
            mbar_init(&S.p_full[i], kWgThreads);
        }
        for (int i = 0; i < NO; ++i) {
            mbar_init(&S.o_full[i], 1);
            mbar_init(&S.o_free[i], kWgThreads);
        }
        for (int i = 0; i < 2; ++i) mbar_init(&S.pv_done[i], 1);
        for (int i = 0; i < kNSc; ++i) mbar_init(&S.l_full[i], kWgThreads);
        for (int i = 0; i < NKV; ++i) {
            mbar_init(&S.kv_full[i], 1);
            mbar_init(&S.kv_empty[i], 1);
        }
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
    // This CTA's tiles: chunks blockIdx.x, blockIdx.x + gridDim.x, ... of kChunk
    // consecutive tiles; only the globally last chunk can be short, and it is the
    // last chunk of its CTA, so tiles 0 .. n-1 of the sequence all exist.
    const int ntiles = S.abort_flag ? 0 : S.ntiles;
    const int nch = (ntiles + kChunk - 1) / kChunk;
    const int bid = (int)blockIdx.x, grid = (int)gridDim.x;
    const int mych = bid < nch ? (nch - 1 - bid) / grid + 1 : 0;
    int n = mych * kChunk;
    if (mych > 0 && bid + (mych - 1) * grid == nch - 1) n -= nch * kChunk - ntiles;
    auto tile_of = [&](int i) { return ((i / kChunk) * grid + bid) * kChunk + (i % kChunk); };
    auto ld_desc = [&](int i) {
        return i < n ? __ldg(p.tile_desc + tile_of(i)) : make_int4(0, 0, 0, -1);
    };
    volatile int* abort_flag = &S.abort_flag;
    auto wait = [&](uint64_t* bar, uint32_t parity, int where) -> bool {
        if (*abort_flag) return false;
        if (!mbar_wait(bar, parity, st, where)) {
            *abort_flag = 1;
            return false;
        }
        return true;
    };
    // a warp leaves its loop together: every wait of a warp-collective role is voted
    auto wait_w = [&](uint64_t* bar, uint32_t parity, int where) -> bool {
        return __all_sync(0xffffffffu, wait(bar, parity, where));
    };

    const int wgrp = warp >> 2;
    const int li = wgrp == 0 ? warp : (warp >= 18 ? warp - 14 : -1);   // loader index

    if (wgrp == 0 || wgrp == 4) {
        reg_dealloc<kRegsLow>();
        if (li >= 0) {
            // ---------------------------------------------------------------- Q loaders
            // Loader w fills the tile rows [R w, min(R w + R, 128)), R = kRowsPerLoader.
            // Lane l computes the source address of row R w + l from the index entry (token)
            // and the row (head); in copy step k the loader moves rows R w + 2k and
            // R w + 2k + 1, lane l taking the 16-byte chunk l % 16 of row R w + 2k + l / 16
            // (a 512-byte coalesced read).  The copies of tile i are published one tile
            // later (wait for the older cp.async group, fence for the tensor core's async
            // proxy, arrive on q_full), so two tiles' gathers are in flight.
            const int w = li;
            const int nr_w = min(kRowsPerLoader, kTileRows - kRowsPerLoader * w);   // rows of this loader
            const uint8_t* qb = static_cast<const uint8_t*>(p.q);
            const int rA = kRowsPerLoader * w + lane;
            auto ld_ent = [&](const int4& d, int r) -> uint32_t {
                return (lane < nr_w && r < (d.z & 255)) ? __ldg(p.entries + d.y + r / p.G) : 0u;
            };
            auto row_addr = [&](const int4& d, int r, uint32_t ent) -> unsigned long long {
                const int g = d.z >> 8;
                return reinterpret_cast<unsigned long long>(
                    qb + ((size_t)(ent >> 6) * p.hq + g * p.G + r % p.G) * (D * 2));
            };
            // test-only fault injection (NSA_TEST_SKIP_ARRIVE): loader 0 of CTA 0 withholds
            // its arrival on the first tile's Q barrier; its copies still complete, and no
            // MMA reads the stage, so the MMA issuer's bounded wait expires with nothing
            // in flight behind it
            auto skip_arrive = [&](int tile) {
                return p.test_skip_arrive && blockIdx.x == 0 && w == 0 && tile == 0;
            };
            int4 d0 = ld_desc(0), d1 = ld_desc(1);
            uint32_t ea = ld_ent(d0, rA);
            int published = 0, issued = 0;
            // a row is 2 D bytes = kCpr 16-byte chunks; one warp instruction copies kRpi rows
            constexpr int kCpr = 8 * NH, kRpi = 32 / kCpr;
            const int c = lane % kCpr;
            const uint32_t dst_c = (uint32_t)(c >> 3) * (kTileRows * 128);
            for (int i = 0; i < n; ++i) {
                const int4 d = d0;
                const unsigned long long addrA = row_addr(d, rA, ea);
                if (kChecks) {   // the gathered row must lie inside q
                    const bool row_in = !(lane < nr_w && rA < (d.z & 255)) ||
                                        ((int)(ea >> 6) < p.T && (int)(ea & 63u) < p.topk &&
                                         (d.z >> 8) < p.hkv);
                    if (!__all_sync(0xffffffffu, check_ok(row_in, st, 140, i))) {
                        *abort_flag = 1;
                        break;
                    }
                }
                d0 = d1;
                d1 = ld_desc(i + 2);
                ea = ld_ent(d0, rA);           // next tile's entries, used one iteration later
                const int nrows = d.z & 255;
                const int stg = i % kNQ;
                // stage i % kNQ is free once S(i - kNQ), which read it, has completed
                if (!wait_w(&S.q_empty[stg], ((i / kNQ) & 1) ^ 1, 30)) break;
                const uint32_t q0 = smem_u32(S.q[stg][0]) + dst_c;
    #pragma unroll 4
                for (int k = 0; k < (kRowsPerLoader + kRpi - 1) / kRpi; ++k) {
                    const int rw = kRpi * k + lane / kCpr;       // row within the loader's rows
                    const unsigned long long a = __shfl_sync(0xffffffffu, addrA, rw & 31) + c * 16;
                    const int row = kRowsPerLoader * w + rw;
                    if (rw < nr_w && row < nrows)
                        cp_async_16(q0 + sw128_offset(row, c & 7), reinterpret_cast<const void*>(a));
                }
                cp_async_commit();
                issued = i + 1;
                if (i > 0) {
                    cp_async_wait_one_pending();
                    fence_async_smem();
                    if (!skip_arrive(i - 1)) mbar_arrive(&S.q_full[(i - 1) % kNQ]);
                    published = i;
                }
            }
            cp_async_wait_all();   // nothing may still be in flight when the CTA exits
            if (issued == n && published == n - 1 && n > 0) {
                fence_async_smem();
                if (!skip_arrive(n - 1)) mbar_arrive(&S.q_full[(n - 1) % kNQ]);
            }
        } else if (warp == kTmaWarp) {
            // ------------------------------------------------------------- K/V producer
            if (lane == 0) {
                prefetch_tmap(&kmap);
                prefetch_tmap(&vmap);
                int prev = -1, uses = 0;
                int last_parity[NKV];
                bool loaded[NKV];
                for (int s = 0; s < NKV; ++s) { last_parity[s] = 0; loaded[s] = false; }
                int4 d0 = ld_desc(0), d1 = ld_desc(1), d2 = ld_desc(2);
                for (int i = 0; i < n; ++i) {
                    const int4 d = d0;
                    d0 = d1; d1 = d2; d2 = ld_desc(i + 3);
                    if (d.w == prev) continue;
                    prev = d.w;
                    if (!check_ok(d.x >= 0 && d.x < p.T && (d.z >> 8) < p.hkv, st, 141, i)) {
                        *abort_flag = 1;
                        break;
                    }
                    const int stg = uses % NKV;
                    if (!wait(&S.kv_empty[stg], ((uses / NKV) & 1) ^ 1, 32)) break;
                    const int g = d.z >> 8;
                    mbar_arrive_expect_tx(&S.kv_full[stg], 2u * NH * BS * 128u);
    #pragma unroll
                    for (int h = 0; h < NH; ++h) {
                        tma_load_3d(S.kv[stg][0][h], &kmap, &S.kv_full[stg], 64 * h, g, d.x);
                        tma_load_3d(S.kv[stg][1][h], &vmap, &S.kv_full[stg], 64 * h, g, d.x);
                    }
                    last_parity[stg] = (uses / NKV) & 1;
                    loaded[stg] = true;
                    ++uses;
                }
                if (*abort_flag)   // let copies still in flight land before the CTA exits
                    for (int s = 0; s < NKV; ++s)
                        if (loaded[s]) mbar_wait(&S.kv_full[s], last_parity[s], st, 40);
            }
        } else if (warp == kMmaWarp) {
            // -------------------------------------------------------------- MMA issuer
            // The whole warp runs the issue loop (warp-uniform state); one elected lane
            // executes the tcgen05 instructions.
            {
                const uint32_t elected = elect_one();
                constexpr uint32_t kIdescS = idesc_f16kind_f32(F16, 128, BS, false, false);
                constexpr uint32_t kIdescO = idesc_f16kind_f32(F16, 128, D, false, true);
                int kv_uses = 0, prev_bucket = -1, cur = 0;
                int kvs_of[2] = {0, 0};
                // S(i) = Q K^T into slot i & 1.  The slot's previous S / P (tile i - 2) was
                // last read by PV(i - 2), which was issued earlier: tcgen05.mma of one thread
                // run in issue order.
                // Shared-memory descriptors are computed once; an MMA step only adds the
                // byte offset / 16 to the start-address field (addresses stay < 2^18 bytes,
                // so the 14-bit field never carries).  This keeps the issuing thread's
                // instruction count per MMA small: it shares its SMSP with busy warps.
                constexpr uint32_t kQStage = sizeof(S.q[0]) >> 4, kQHalf = sizeof(S.q[0][0]) >> 4;
                constexpr uint32_t kKvStage = sizeof(S.kv[0]) >> 4, kKvHalf = sizeof(S.kv[0][0][0]) >> 4;
                const uint32_t q_desc0 = (uint32_t)smem_desc_sw128(smem_u32(S.q[0][0]), 16, 1024);
                const uint32_t k_desc0 = (uint32_t)smem_desc_sw128(smem_u32(S.kv[0][0][0]), 16, 1024);
                const uint32_t v_desc0 = (uint32_t)smem_desc_sw128(smem_u32(S.kv[0][1][0]), BS * 128, 1024);
                // S(i) = Q K^T into slot i & 1, whose previous P (tile i - 2) PV(i - 2) reads
                // (see the wait below).  q_empty tells the loaders that the Q stage i % kNQ
                // is free again.
                auto issue_s = [&](int i, int bucket) -> bool {
                    if (bucket != prev_bucket) {
                        cur = kv_uses % NKV;
                        if (!wait(&S.kv_full[cur], (kv_uses / NKV) & 1, 33)) return false;
                        ++kv_uses;
                        prev_bucket = bucket;
                    }
                    const int slot = i & 1, stg = i % kNQ;
                    kvs_of[slot] = cur;
                    if (!wait(&S.q_full[stg], (i / kNQ) & 1, 35)) return false;
                    // S(i) overwrites the TMEM slot from which PV(i - 2) reads P(i - 2) as its
                    // A operand: S(i) waits until PV(i - 2) has completed, so that no write of
                    // it can overtake those reads.  With two or three O buffers PV(i - 1) and
                    // PV(i - 2) arrive on different o_full barriers; with one, PV(i - 1) may
                    // already be done when S(i) comes after it, and waiting on the shared
                    // barrier's parity would alias, so each S slot has its own pv_done.
                    if constexpr (NO == 1) {
                        if (i >= 2 && !wait(&S.pv_done[slot], ((i >> 1) - 1) & 1, 42)) return false;
                    } else {
                        if (i >= 2 && !wait(&S.o_full[(i - 2) % NO], ((i - 2) / NO) & 1, 42)) return false;
                    }
                    tc_fence_after();
                    const uint32_t tS = tmem + slot * BS;
                    const uint32_t a0 = q_desc0 + (uint32_t)stg * kQStage;
                    const uint32_t b0 = k_desc0 + (uint32_t)cur * kKvStage;
    #pragma unroll
                    for (int ks = 0; ks < 4 * NH; ++ks) {     // K = D, 16 per step
                        const uint32_t off = (uint32_t)((ks >> 2) * kQHalf + (ks & 3) * 2);
                        const uint32_t offk = (uint32_t)((ks >> 2) * kKvHalf + (ks & 3) * 2);
                        mma_ss_e(tS, a0 + off, b0 + offk, kIdescS, ks > 0 ? 1u : 0u, elected);
                    }
                    mma_commit_e(&S.s_full[slot], elected);
                    mma_commit_e(&S.q_empty[stg], elected);
                    return true;
                };
                // O(i) = P(i) V into buffer i % NO once the softmax wrote P(i) and the
                // epilogue of tile i - NO has read the buffer's previous O.
                auto issue_pv = [&](int i, bool release_kv) -> bool {
                    const int slot = i & 1, ob = i % NO;
                    if (!wait(&S.p_full[slot], (i >> 1) & 1, 36)) return false;
                    if (!wait(&S.o_free[ob], ((i / NO) & 1) ^ 1, 34)) return false;
                    tc_fence_after();
                    const uint32_t tS = tmem + slot * BS, tO = tmem + kColO + ob * D;
                    const int kvs = kvs_of[slot];
                    const uint32_t b0 = v_desc0 + (uint32_t)kvs * kKvStage;
    #pragma unroll
                    for (int ks = 0; ks < BS / 16; ++ks)    // 16 keys = 2048 bytes per step
                        mma_ts_e(tO, tS + (uint32_t)ks * 8u, b0 + (uint32_t)ks * 128u, kIdescO,
                                 ks > 0 ? 1u : 0u, elected);
                    mma_commit_e(&S.o_full[ob], elected);
                    if constexpr (NO == 1) mma_commit_e(&S.pv_done[slot], elected);
                    if (release_kv) mma_commit_e(&S.kv_empty[kvs], elected);
                    return true;
                };
                int4 dc = ld_desc(0), dn = ld_desc(1), dnn = ld_desc(2);
                bool ok = n > 0 && issue_s(0, dc.w);
                for (int i = 0; i < n && ok; ++i) {
                    const bool more = i + 1 < n;
                    const bool same = more && dn.w == dc.w;
                    // S(i+1) goes ahead of PV(i) unless it needs the only K/V stage
                    const bool ahead = more && (NKV > 1 || same);
                    if (ahead && !(ok = issue_s(i + 1, dn.w))) break;
                    if (!(ok = issue_pv(i, !same))) break;
                    if (more && !ahead && !(ok = issue_s(i + 1, dn.w))) break;
                    dc = dn; dn = dnn; dnn = ld_desc(i + 3);
                }
                // every MMA issued above has finished once this commit arrives
                mma_commit_e(&S.drain, elected);
                mbar_wait(&S.drain, 0, st, 41);
            }
        }
    } else if (wgrp == 1 || wgrp == 2) {
        reg_alloc<kRegsSoftmax>();
        // ------------------------------------------------------------------ softmax
        // Thread = tile row = TMEM lane.  Non-diagonal tiles (every row sees the whole
        // block) skip the causal mask; the test is warp-uniform.
        const int wg = (warp - 4) >> 2;                  // 0: even tiles, 1: odd tiles
        const int quad = warp & 3;                       // TMEM lanes 32*quad ..
        const int r = quad * 32 + lane;
        const uint32_t tS = tmem + wg * BS + ((uint32_t)(quad * 32) << 16);
        const float c = p.scale_log2;
        const float kLn2 = 0.69314718055994531f;
        auto ld_row = [&](const int4& d, int i) -> uint32_t {
            return (i < n && r < (d.z & 255)) ? __ldg(p.entries + d.y + r / p.G) : 0u;
        };
        auto ld_vexp = [&](const int4& d, int i) -> int { return i < n ? __ldg(p.vexp + d.w) : 0; };
        // scores of keys past the causal limit or before the sliding window -> -inf
        // (diagonal and window-edge tiles only)
        auto mask64 = [&](float* v, int lo, int lim, int base) {
#pragma unroll
            for (int k = 0; k < 64; ++k)
                if (base + k > lim || base + k < lo) v[k] = -CUDART_INF_F;
        };
        auto row_max64 = [&](const float* v) -> float {
            float a = -CUDART_INF_F, b = -CUDART_INF_F;
#pragma unroll
            for (int k = 0; k < 64; k += 4) {
                a = fmax3(a, v[k], v[k + 1]);
                b = fmax3(b, v[k + 2], v[k + 3]);
            }
            return fmaxf(a, b);
        };
        // v[k] <- 2^(c v[k] - c m) over 64 scores (a masked -inf gives 0); l += sum
        auto exp_chunk = [&](float* v, float mc, float2& l2) {
            const float2 c2 = make_float2(c, c), nmc2 = make_float2(-mc, -mc);
#pragma unroll
            for (int k2 = 0; k2 < 32; ++k2) {
                float2 x = fma2(make_float2(v[2 * k2], v[2 * k2 + 1]), c2, nmc2);
                x.x = ex2_approx(x.x);
                x.y = ex2_approx(x.y);
                l2 = add2(l2, x);
                v[2 * k2] = x.x;
                v[2 * k2 + 1] = x.y;
            }
        };
        // 64 values times s as packed bf16 pairs; ls += the packed (rounded) values, the
        // weights the P V product will actually use
        auto pack_chunk = [&](const float* v, float s, uint32_t* pk, float2& ls) {
            const float2 s2 = make_float2(s, s);
#pragma unroll
            for (int k2 = 0; k2 < 32; ++k2) {
                const float2 x = mul2(make_float2(v[2 * k2], v[2 * k2 + 1]), s2);
                pk[k2] = pack2<F16>(x.x, x.y);   // P in the type of V (one MMA, one type)
                ls = add2(ls, unpack2<F16>(pk[k2]));
            }
        };
        // descriptors two tiles ahead, entries and exponents one tile ahead, so that no
        // dependent global load sits on the path from S(i) to P(i)
        int4 dn = ld_desc(wg), dnn = ld_desc(wg + 2);
        uint32_t en = ld_row(dn, wg);
        int vn = ld_vexp(dn, wg);
        for (int i = wg; i < n; i += 2) {
            const int4 d = dn;
            const uint32_t ent = en;
            const int ve = vn;
            dn = dnn;
            dnn = ld_desc(i + 4);
            en = ld_row(dn, i + 2);
            vn = ld_vexp(dn, i + 2);
            const uint32_t ph = (i >> 1) & 1;
            const bool valid = r < (d.z & 255);
            // keys lo .. lim of the block are visible to this row (causal on the diagonal,
            // lo > 0 where the sliding window starts inside the block)
            const int lim = valid ? (int)(ent >> 6) - d.x : -1;
            const int lo = p.swin > 0 ? lim - p.swin + 1 : 0;
            const bool nomask = __all_sync(0xffffffffu, !valid || (lim >= BS - 1 && lo <= 0));
            if (!wait_w(&S.s_full[wg], ph, 38)) break;
            tc_fence_after();
            float sv[64];
            tmem_ld64_sync(tS, sv);
            if (!nomask) mask64(sv, lo, lim, 0);
            float mx = row_max64(sv);
            if constexpr (BS == 128) {
                tmem_ld64_sync(tS + 64, sv);
                if (!nomask) mask64(sv, lo, lim, 64);
                mx = fmaxf(mx, row_max64(sv));
            }
            if (!valid) mx = 0.f;                      // every valid row has lo <= lim
            const float mc = mx * c;
            // l (fp32 sum of P) gives the block's LSE; the partial O is normalised by lr,
            // the sum of the rounded P values the product uses, so that its weights sum to
            // one exactly (a plain 1 / l would leave a bias of up to 2^-9 |V| on rows
            // where one key dominates).
            float2 l2 = make_float2(0.f, 0.f), lr2 = make_float2(0.f, 0.f);
            float l, f;                                // f: partial O x f = the block's O
            uint32_t pk[32];
            if constexpr (BS == 64) {
                // P pre-scaled by 2^-e / l: the epilogue only converts O
                exp_chunk(sv, mc, l2);
                l = l2.x + l2.y;
                pack_chunk(sv, valid ? ldexpf(1.f / l, -ve) : 0.f, pk, lr2);
                tmem_st32_sync(tS, pk);
                f = 1.f / (lr2.x + lr2.y);
            } else {
#pragma unroll
                for (int c64 = 0; c64 < 2; ++c64) {    // scores of this 64-key chunk again
                    tmem_ld64_sync(tS + c64 * 64, sv);
                    if (!nomask) mask64(sv, lo, lim, c64 * 64);
                    exp_chunk(sv, mc, l2);
                    pack_chunk(sv, 1.f, pk, lr2);
                    tmem_st32_sync(tS + c64 * 32, pk);
                }
                l = l2.x + l2.y;
                f = ldexpf(1.f, ve);
            }
            tc_fence_before();
            mbar_arrive(&S.p_full[wg]);
            if constexpr (BS != 64) {                  // the epilogue applies 2^-e / lr
                S.sc[i % kNSc][r] = valid ? ldexpf(1.f / (lr2.x + lr2.y), -ve) : 0.f;
                mbar_arrive(&S.l_full[i % kNSc]);
            }
            if (valid)
                p.part_meta[(size_t)tile_of(i) * kTileRows + r] =
                    make_float2((mc + __log2f(l)) * kLn2, f);
        }
    } else {
        // ----------------------------------------------------------------- epilogue
        // O * (2^-e / l) as fp16, per 64-column half: each thread writes its row into
        // the warp's staging buffer in the 128-byte-swizzled layout, then one lane
        // stores the warp's valid rows, rounded up to 8, by TMA into the tile's own
        // 128-row partial slot (rows past the list only land in the slot's padding).
        const int quad = warp & 3;
        const int ew = warp - 12;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        int4 dn = ld_desc(0);
        for (int i = 0; i < n; ++i) {
            const int4 d = dn;
            dn = ld_desc(i + 1);
            const int ob = i % NO;
            if (!wait_w(&S.o_full[ob], (i / NO) & 1, 39)) break;
            float sc = 1.f;
            if constexpr (BS != 64) {
                if (!wait_w(&S.l_full[i % kNSc], (i / kNSc) & 1, 43)) break;
                sc = S.sc[i % kNSc][quad * 32 + lane];
            }
            tc_fence_after();
            const float2 sc2 = make_float2(sc, sc);
            const int valid = min(32, max(0, (d.z & 255) - quad * 32));
            const int nbox = (valid + 7) >> 3;
            const int prow0 = tile_of(i) * kTileRows + quad * 32;   // warp's first row
            const uint32_t tO = tmem + kColO + ob * D + lane_off;
#pragma unroll
            for (int h = 0; h < NH; ++h) {
                float x[64];
                tmem_ld64_sync(tO + h * 64, x);
                if (h == NH - 1) {            // the buffer's O has been read: release it
                    tc_fence_before();
                    mbar_arrive(&S.o_free[ob]);
                }
                // staging buffers in turn over the halves of consecutive tiles; the TMA
                // store that last read this one (kNSt halves ago) is done
                const int hb = (i * NH + h) % kNSt;
                if (lane == 0) bulk_wait_read<kNSt - 1>();
                __syncwarp();
                const uint32_t sb = smem_u32(S.stage[ew][hb]);
#pragma unroll
                for (int pc = 0; pc < 8; ++pc) {
                    const float* y = x + pc * 8;
                    uint32_t u[4];
#pragma unroll
                    for (int q2 = 0; q2 < 4; ++q2) {
                        float2 z = make_float2(y[2 * q2], y[2 * q2 + 1]);
                        if constexpr (BS != 64) z = mul2(z, sc2);
                        u[q2] = pack_f16x2(z.x, z.y);
                    }
                    st_shared_v4(sb + lane * 128 + ((pc ^ (lane & 7)) << 4),
                                 make_uint4(u[0], u[1], u[2], u[3]));
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0 && nbox > 0) {
                    if (nbox == 4) {
                        tma_store_2d(&omap32, S.stage[ew][hb], h * 64, prow0);
                    } else {
                        for (int b = 0; b < nbox; ++b)
                            tma_store_2d(&omap8, S.stage[ew][hb] + b * 1024, h * 64, prow0 + b * 8);
                    }
                    bulk_commit();
                }
            }
        }
        if (lane == 0) bulk_wait<0>();   // every store performed before the CTA exits
    }

    // ---- teardown: every role has left its loop (all waits are bounded) and the MMA
    //      issuer has drained its tensor-core work
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

// Per (KV head g, global block B): e = 0 unless max |V_B| > 2^14, then the exponent
// that brings it under 2^15 (fp16 partials of O / l stay finite).  One CTA of 256
// threads per (B, g) reads the block as 16-byte chunks: d / 8 threads per key row,
// 256 / (d / 8) rows per pass, the loads of four passes in flight together.
__global__ void __launch_bounds__(256) k_vblock_exp(const __nv_bfloat16* v, const int32_t* cu,
                                                    int nseq, int hkv, int d, int bs,
                                                    const int32_t* blkoff, const DevStatus* st,
                                                    int32_t* vexp) {
    __shared__ float wmax[8];
    const int B = blockIdx.x, g = blockIdx.y;
    const int nbtot = st->nblocks_total;
    if (st->code != 0 || B >= nbtot) return;
    const int s = upper_index(blkoff, nseq, B);
    const int key0 = __ldg(cu + s) + (B - __ldg(blkoff + s)) * bs;
    const int kend = min(key0 + bs, __ldg(cu + s + 1));
    const int cpr = d >> 3;                       // 16-byte chunks per key row
    const int rpp = (int)blockDim.x / cpr;        // key rows per pass
    const int r = (int)threadIdx.x / cpr, c = (int)threadIdx.x - r * cpr;
    const uint4* base = reinterpret_cast<const uint4*>(v + (size_t)g * d) + c;
    const size_t row_stride = (size_t)hkv * d / 8;   // in 16-byte chunks
    float m = 0.f;
#pragma unroll 4
    for (int key = key0 + r; key < kend; key += rpp) {
        const uint4 x = __ldg(base + (size_t)key * row_stride);
        const uint32_t w4[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int k2 = 0; k2 < 4; ++k2) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[k2]));
            m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
    }
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, wmax[w]);
        m = fmaxf(m, wmax[0]);
        vexp[g * nbtot + B] = m > 16384.f ? min(ilogbf(m) - 14, 120) : 0;
    }
}

}  // namespace

cudaError_t launch_vblock_exp(const FwdPlan& p, const void* v, int nb_stride, int32_t* vexp,
                              cudaStream_t stream) {
    if (p.T > 0 && nb_stride > 0) {
        if (p.f16)   // |V| <= 65504 already fits the fp16 partials: every exponent is 0
            return cudaMemsetAsync(vexp, 0, sizeof(int32_t) * (size_t)p.hkv * nb_stride, stream);
        k_vblock_exp<<<dim3((unsigned)nb_stride, (unsigned)p.hkv), 256, 0, stream>>>(
            static_cast<const __nv_bfloat16*>(v), p.cu, p.nseq, p.hkv, p.d, p.bs, p.blkoff, p.st,
            vexp);
    }
    return cudaGetLastError();
}

template <int BS, int NKV, int NH, int F16>
static void launch_fwd_variant(const FwdPlan& p, const CUtensorMap* kmap, const CUtensorMap* vmap,
                               const CUtensorMap* omap, cudaStream_t stream) {
    constexpr size_t smem = fwd_smem_bytes<BS, NKV, NH>();
    static_assert(smem <= 232448, "shared memory per CTA");
    cudaFuncSetAttribute(k_fwd_tiles<BS, NKV, NH, F16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    k_fwd_tiles<BS, NKV, NH, F16><<<p.num_sms, kThreads, smem, stream>>>(p, *kmap, *vmap, omap[0],
                                                                          omap[1]);
}

template <int NH, int F16>
static void launch_fwd_nh(const FwdPlan& p, const CUtensorMap* kmap, const CUtensorMap* vmap,
                          const CUtensorMap* omap, cudaStream_t stream) {
    if (p.bs == 64) launch_fwd_variant<64, NH == 4 ? 1 : 2, NH, F16>(p, kmap, vmap, omap, stream);
    else if constexpr (NH != 4) launch_fwd_variant<128, 1, NH, F16>(p, kmap, vmap, omap, stream);
}

cudaError_t launch_fwd_tiles(const FwdPlan& p, const CUtensorMap* kmap, const CUtensorMap* vmap,
                             const CUtensorMap* omap, cudaStream_t stream) {
    if (p.d == 256 && p.bs != 64) return cudaErrorInvalidValue;   // no shared memory for it
    switch (p.d) {
        case 64:
            if (p.f16) launch_fwd_nh<1, 1>(p, kmap, vmap, omap, stream);
            else launch_fwd_nh<1, 0>(p, kmap, vmap, omap, stream);
            break;
        case 128:
            if (p.f16) launch_fwd_nh<2, 1>(p, kmap, vmap, omap, stream);
            else launch_fwd_nh<2, 0>(p, kmap, vmap, omap, stream);
            break;
        case 256:
            if (p.f16) launch_fwd_nh<4, 1>(p, kmap, vmap, omap, stream);
            else launch_fwd_nh<4, 0>(p, kmap, vmap, omap, stream);
            break;
        default:
            return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace nsa
