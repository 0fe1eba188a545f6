// dense.cu -- forward pass over the init and local blocks, with the merge folded in.
//
// Every token's index row holds its init block (0) and its local blocks (qb - 1, qb)
// ("Relaxed-System-Lab/Flash-Sparse-Attention" project page, Quick start:
// init_blocks 1, local_blocks 2).  All 128 / G consecutive tokens of a tile share
// their query block (or, at block 64 with group 1, two neighbouring ones), so these
// blocks are shared by every row of a tile: they are computed here query-major, as
// dense tensor-core tiles with a contiguous Q box (no gather, no partial), and the
// KV-block-major tile kernel (fwd.cu) handles only the other selected blocks.  In
// each (KV head, block) list of the inversion the entries of these blocks are the
// tokens of query blocks B and B + 1 (or every token for B = 0), a prefix of the
// token-sorted list, which the forward's tile split skips (invert.cu).
//
// The same kernel then merges, per (token, query head) row, its result over these
// blocks with the KV-major partials of the row's other blocks and writes O and the
// LSE: the reduction and online-softmax steps of the project page's key-features
// table, with no atomics and no separate merge pass.
//
// A tile is (sequence s, KV head g, tokens i0 .. i0 + 128/G - 1 of s) x the G query
// heads of g, rows token-major (one 3D TMA box of Q).  Its candidate blocks are 0 and
// qb_lo - 1 .. qb_hi (2 to 4 blocks); a row keeps the candidates that its own index
// row selects among {0, qb - 1, qb} (set semantics), masked causally (and by the
// sliding window).
//
//   S_c = Q K_c^T for every candidate c     tcgen05.mma -> TMEM columns c * BS
//   one softmax over all candidates          thread = row: max, P = 2^(cS - cm),
//                                            l = sum P; P as 16-bit into S's columns
//   O_d = sum_c P_c V_c                      tcgen05.mma (A = P from TMEM) -> TMEM
//   fold                                     O = (w_d O_d / l + sum_j w_j o_j) / Lambda
//                                            over the row's KV-major partials j
//
// Warps: 0 TMA producer (Q box; K then V of every candidate through a ring of block
// slots), 1 MMA issuer (one elected lane of a warp-uniform loop), 4-7 softmax and
// the O_d hand-off (TMEM -> shared memory, fp32), 8-15 the fold (one warp per row,
// lane = four columns; each warp keeps two rows' partial loads in flight, and issues
// the next tile's first loads before that tile's O_d is ready).  The fold reads the
// partials from HBM and is the kernel's bound; the tensor-core work of a tile runs
// under the fold of the previous one.
#include <math_constants.h>

#include "nsa_common.cuh"
#include "nsa_kernels.h"

namespace nsa {
namespace {

constexpr int kDThreads = 512;
constexpr int kFoldWarp0 = 8;
constexpr int kFoldWarps = 8;
constexpr int kColO = 384;                 // TMEM: S / P of the candidates below, O_d here
constexpr int kWgThreads128 = 128;         // threads of the softmax warpgroup

template <int BS>
struct DenseCfg {
    static constexpr int kMaxCand = BS == 64 ? 4 : 3;
    static constexpr int kSlots = BS == 64 ? 6 : 3;            // K / V block ring
    static constexpr int kSlotBytes = 2 * BS * 128;             // two 64-column halves
};

template <int BS>
struct alignas(1024) DenseSmem {
    uint8_t q[2][kTileRows * 128];                               // Q tile: [half][row]
    uint8_t kv[DenseCfg<BS>::kSlots][2][BS * 128];               // ring: [slot][half][key]
    float od[kTileRows * kHeadDim];                              // O_d / l, fp32, swizzled
    float od_lse[kTileRows];                                     // LSE over these blocks
    uint64_t q_full, q_empty;
    uint64_t kv_full[DenseCfg<BS>::kSlots], kv_empty[DenseCfg<BS>::kSlots];
    uint64_t s_full, p_full, o_full, o_free;
    uint64_t od_full, od_empty;
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};

// float4 chunk c (0..31) of row r of the O_d buffer: chunks permuted by the row so that
// a warp writing one chunk of 32 rows (thread = row) and a warp reading one row (lane =
// chunk) are both free of bank conflicts.
__device__ __forceinline__ int od_index(int r, int c) { return r * kHeadDim + ((c ^ (r & 31)) << 2); }

template <int N>
__device__ __forceinline__ void reg_dealloc_d() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void reg_alloc_d() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

struct DTile {
    int s, g, i0, L, tok0, ncand;
    int cand[4];
};

__device__ __forceinline__ DTile dense_tile(const DensePlan& p, int ti) {
    DTile t;
    t.g = ti % p.hkv;
    const int u = ti / p.hkv;
    t.s = upper_index(p.dtile_off, p.nseq, u);
    t.i0 = (u - __ldg(p.dtile_off + t.s)) * p.tpt;
    const int c0 = __ldg(p.cu + t.s);
    t.L = __ldg(p.cu + t.s + 1) - c0;
    t.tok0 = c0 + t.i0;
    const int qlo = t.i0 / p.bs;
    const int qhi = (min(t.i0 + p.tpt, t.L) - 1) / p.bs;
    // 0, then max(qlo - 1, 1) .. qhi (at most three blocks: qhi <= qlo + 1)
    const int b1 = max(qlo - 1, 1);
    t.ncand = 1 + max(qhi - b1 + 1, 0);
#pragma unroll
    for (int k = 0; k < 4; ++k) t.cand[k] = k == 0 ? 0 : (k < t.ncand ? b1 + k - 1 : -1);
    return t;
}

// -------------------------------------------------------------------------- fold
constexpr int kFoldFirst = 16;   // slots whose partial loads go out ahead of the merge

struct FoldRow {
    int t, h;                // token, query head (h < 0: no row)
    unsigned r0, r1;         // partial rows of this lane's slots (lane, lane + 32)
    float2 m0, m1;           // their (lse, exponent)
    uint2 u[kFoldFirst];     // this lane's four columns of the first slots' partials
};

template <int BS, int F16, int KS>
__device__ __forceinline__ void fold_rows(const DensePlan& p, const float* od, const float* od_lse,
                                          uint64_t* od_full, uint64_t* od_empty, int fw, int lane,
                                          int bid, int grid, int ntiles, volatile int* abort_flag,
                                          DevStatus* st) {
    constexpr bool kTopk32 = KS <= 32;
    constexpr int kRows = kTileRows / kFoldWarps;   // 16 rows per warp and tile
    constexpr unsigned kNone = 0xFFFFFFFFu;
    const unsigned nrows_part = (unsigned)(*reinterpret_cast<volatile int*>(&st->ntiles_fwd)) *
                                (unsigned)kTileRows;
    const uint2* po_base = reinterpret_cast<const uint2*>(p.part_o) + lane;

    // index step 1 of a tile: the block number of this lane's slot(s) of each row
    auto idx_blocks = [&](const DTile& t, int (&b0)[kRows], int (&b1)[kRows]) {
#pragma unroll
        for (int k = 0; k < kRows; ++k) {
            const int tokr = (fw + kFoldWarps * k) / p.G;
            const bool valid = t.i0 + tokr < t.L;
            const size_t base = ((size_t)(t.tok0 + tokr) * p.hkv + t.g) * p.topk;
            b0[k] = (valid && lane < p.topk) ? __ldg(p.bidx + base + lane) : -1;
            b1[k] = (!kTopk32 && valid && lane + 32 < p.topk) ? __ldg(p.bidx + base + lane + 32) : -1;
        }
    };
    // index step 2: the partial row of each slot merged here (kNone for the others)
    auto idx_rows = [&](const DTile& t, const int (&b0)[kRows], const int (&b1)[kRows],
                        unsigned (&r0)[kRows], unsigned (&r1)[kRows]) {
#pragma unroll
        for (int k = 0; k < kRows; ++k) {
            const int r = fw + kFoldWarps * k;
            const int tokr = r / p.G;
            const int i = t.i0 + tokr;
            const int qb = i / BS;
            const size_t base = ((size_t)(t.tok0 + tokr) * p.hkv + t.g) * p.topk;
            const unsigned hoff = (unsigned)(r - tokr * p.G);
            auto row_of = [&](int b, int j) -> unsigned {
                if (b <= 0 || b >= qb - 1 || !block_valid(b, qb, i, BS, p.swin)) return kNone;
                const unsigned pr = (unsigned)__ldg(p.posmap + base + j) * (unsigned)p.G + hoff;
                return pr < nrows_part ? pr : kNone;
            };
            r0[k] = row_of(b0[k], lane);
            r1[k] = kTopk32 ? kNone : row_of(b1[k], lane + 32);
        }
    };
    auto ld_part = [&](unsigned r0, unsigned r1, int j) -> uint2 {
        const unsigned rj = __shfl_sync(0xFFFFFFFFu, j < 32 ? r0 : r1, j & 31);
        return (j < p.topk && rj != kNone) ? __ldg(po_base + (size_t)rj * (kHeadDim / 4))
                                           : make_uint2(0u, 0u);
    };
    auto load_row = [&](FoldRow& R, const DTile& t, int k, unsigned r0, unsigned r1) {
        const int r = fw + kFoldWarps * k;
        const int tokr = r / p.G;
        R.t = t.tok0 + tokr;
        R.h = (t.i0 + tokr < t.L) ? t.g * p.G + (r - tokr * p.G) : -1;
        R.r0 = r0;
        R.r1 = r1;
        R.m0 = r0 != kNone ? __ldg(p.part_meta + r0) : make_float2(-CUDART_INF_F, 0.f);
        R.m1 = r1 != kNone ? __ldg(p.part_meta + r1) : make_float2(-CUDART_INF_F, 0.f);
#pragma unroll
        for (int j = 0; j < kFoldFirst; ++j) R.u[j] = ld_part(r0, r1, j);
    };
    auto finish_row = [&](const FoldRow& R, int k) {
        if (R.h < 0) return;
        const int r = fw + kFoldWarps * k;
        const float ld = od_lse[r];
        const float4 o4 = *reinterpret_cast<const float4*>(&od[od_index(r, lane)]);
        float M = fmaxf(R.m0.x, R.m1.x);
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xFFFFFFFFu, M, o));
        M = fmaxf(M, ld);
        uint2* outp = reinterpret_cast<uint2*>(static_cast<uint8_t*>(p.out) +
                                               ((size_t)R.t * p.hq + R.h) * (kHeadDim * 2)) + lane;
        if (M == -CUDART_INF_F) {      // nothing selected: O = 0, LSE = -inf
            *outp = make_uint2(0u, 0u);
            if (lane == 0 && p.lse) p.lse[(size_t)R.h * p.T + R.t] = -CUDART_INF_F;
            return;
        }
        const float w0 = R.m0.x == -CUDART_INF_F ? 0.f : __expf(R.m0.x - M);
        const float w1 = R.m1.x == -CUDART_INF_F ? 0.f : __expf(R.m1.x - M);
        float lam = w0 + w1;
        for (int o = 16; o > 0; o >>= 1) lam += __shfl_xor_sync(0xFFFFFFFFu, lam, o);
        const float wd = ld == -CUDART_INF_F ? 0.f : __expf(ld - M);
        lam += wd;
        const float s0 = ldexpf(w0, (int)R.m0.y), s1 = ldexpf(w1, (int)R.m1.y);   // weight x 2^e
        float acc[4] = {wd * o4.x, wd * o4.y, wd * o4.z, wd * o4.w};
        auto add = [&](const uint2& u, int j) {
            const float wj = __shfl_sync(0xFFFFFFFFu, j < 32 ? s0 : s1, j & 31);
            const float2 a = unpack_f16x2(u.x), b = unpack_f16x2(u.y);
            acc[0] = fmaf(wj, a.x, acc[0]);
            acc[1] = fmaf(wj, a.y, acc[1]);
            acc[2] = fmaf(wj, b.x, acc[2]);
            acc[3] = fmaf(wj, b.y, acc[3]);
        };
#pragma unroll
        for (int j = 0; j < kFoldFirst; ++j) add(R.u[j], j);
#pragma unroll
        for (int j0 = kFoldFirst; j0 < KS; j0 += 16) {   // larger topk: 16 slots at a time
            uint2 v[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = ld_part(R.r0, R.r1, j0 + j);
#pragma unroll
            for (int j = 0; j < 16; ++j) add(v[j], j0 + j);
        }
        const float inv = 1.f / lam;
        *outp = make_uint2(pack2<F16>(acc[0] * inv, acc[1] * inv), pack2<F16>(acc[2] * inv, acc[3] * inv));
        if (lane == 0 && p.lse) p.lse[(size_t)R.h * p.T + R.t] = M + __logf(lam);
    };

    if (bid >= ntiles) return;
    DTile t = dense_tile(p, bid);
    int bb0[kRows], bb1[kRows];
    unsigned r0[kRows], r1[kRows];
    idx_blocks(t, bb0, bb1);
    idx_rows(t, bb0, bb1, r0, r1);
    FoldRow A, B;
    load_row(A, t, 0, r0[0], r1[0]);
    int n = 0;
    for (int ti = bid; ti < ntiles; ti += grid, ++n) {
        const bool more = ti + grid < ntiles;
        DTile tn = t;
        if (more) {
            tn = dense_tile(p, ti + grid);
            idx_blocks(tn, bb0, bb1);           // the next tile's index, step 1
        }
        unsigned n0[kRows], n1[kRows];
        bool ready = false;
#pragma unroll
        for (int k = 0; k < kRows; ++k) {
            if (k == kRows / 2 && more) idx_rows(tn, bb0, bb1, n0, n1);   // step 2
            // the next row's loads: this tile's row k + 1, or the next tile's row 0
            if (k + 1 < kRows) load_row(B, t, k + 1, r0[k + 1], r1[k + 1]);
            else if (more) load_row(B, tn, 0, n0[0], n1[0]);
            if (!ready) {
                if (!__all_sync(0xffffffffu, !*abort_flag && mbar_wait(od_full, n & 1, st, 134))) {
                    *abort_flag = 1;
                    return;
                }
                ready = true;
            }
            finish_row(A, k);
            A = B;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(od_empty);
        if (more) {
#pragma unroll
            for (int k = 0; k < kRows; ++k) {
                r0[k] = n0[k];
                r1[k] = n1[k];
            }
        }
        t = tn;
    }
}

template <int BS, int F16, int KS>
__global__ void __launch_bounds__(kDThreads, 1)
    k_fwd_dense(const DensePlan p, const __grid_constant__ CUtensorMap qmap,
                const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap) {
    using Cfg = DenseCfg<BS>;
    constexpr int NS = Cfg::kSlots;
    static_assert(Cfg::kMaxCand * BS <= kColO, "TMEM budget");
    extern __shared__ uint8_t smem_raw[];
    DenseSmem<BS>& S = *reinterpret_cast<DenseSmem<BS>*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    DevStatus* st = p.st;
    if (tid == 0) {
        S.abort_flag = (*reinterpret_cast<volatile int*>(&st->code) != 0);
        mbar_init(&S.q_full, 1);
        mbar_init(&S.q_empty, 1);
        for (int i = 0; i < NS; ++i) {
            mbar_init(&S.kv_full[i], 1);
            mbar_init(&S.kv_empty[i], 1);
        }
        mbar_init(&S.s_full, 1);
        mbar_init(&S.p_full, kWgThreads128);
        mbar_init(&S.o_full, 1);
        mbar_init(&S.o_free, kWgThreads128);
        mbar_init(&S.od_full, kWgThreads128);
        mbar_init(&S.od_empty, kFoldWarps);
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
    const int ntiles = S.abort_flag ? 0 : __ldg(p.dtile_off + p.nseq) * p.hkv;
    const int bid = (int)blockIdx.x, grid = (int)gridDim.x;
    volatile int* abort_flag = &S.abort_flag;
    auto wait = [&](uint64_t* bar, uint32_t parity, int where) -> bool {
        if (*abort_flag) return false;
        if (!mbar_wait(bar, parity, st, where)) {
            *abort_flag = 1;
            return false;
        }
        return true;
    };
    auto wait_w = [&](uint64_t* bar, uint32_t parity, int where) -> bool {
        return __all_sync(0xffffffffu, wait(bar, parity, where));
    };

    // Registers: the launch gives every thread 128; the producer / MMA warpgroup drops
    // to 48, the softmax warpgroup keeps 128 and the fold warpgroups rise to 168
    // (128 x 48 + 128 x 128 + 256 x 168 = 512 x 128).
    if (warp < 4) {
      reg_dealloc_d<48>();
      if (warp == 0) {
        // ----------------------------------------------------------------- producer
        if (lane == 0) {
            prefetch_tmap(&qmap);
            prefetch_tmap(&kmap);
            prefetch_tmap(&vmap);
            int n = 0, u = 0;
            int qpar = -1, slot_par[NS];
            for (int i = 0; i < NS; ++i) slot_par[i] = -1;
            for (int ti = bid; ti < ntiles; ti += grid, ++n) {
                const DTile t = dense_tile(p, ti);
                if (!wait(&S.q_empty, (n & 1) ^ 1, 120)) break;
                mbar_arrive_expect_tx(&S.q_full, 2u * kTileRows * 128u);
                tma_load_3d(S.q[0], &qmap, &S.q_full, 0, t.g * p.G, t.tok0);
                tma_load_3d(S.q[1], &qmap, &S.q_full, 64, t.g * p.G, t.tok0);
                qpar = n & 1;
                const int key_base = t.tok0 - t.i0;          // first token of the sequence
                if (!check_ok(t.tok0 < p.T && t.g < p.hkv, st, 144, ti)) {
                    *abort_flag = 1;
                    break;
                }
                bool ok = true;
                for (int kvsel = 0; kvsel < 2 && ok; ++kvsel)   // K of every candidate, then V
                    for (int c = 0; c < t.ncand; ++c, ++u) {
                        const int sl = u % NS;
                        if (!(ok = wait(&S.kv_empty[sl], ((u / NS) & 1) ^ 1, 121))) break;
                        mbar_arrive_expect_tx(&S.kv_full[sl], (uint32_t)Cfg::kSlotBytes);
                        const CUtensorMap* m = kvsel == 0 ? &kmap : &vmap;
                        const int key0 = key_base + t.cand[c] * BS;
                        tma_load_3d(S.kv[sl][0], m, &S.kv_full[sl], 0, t.g, key0);
                        tma_load_3d(S.kv[sl][1], m, &S.kv_full[sl], 64, t.g, key0);
                        slot_par[sl] = (u / NS) & 1;
                    }
                if (!ok) break;
            }
            if (*abort_flag) {   // let copies still in flight land before the CTA exits
                if (qpar >= 0) mbar_wait(&S.q_full, qpar, st, 122);
                for (int i = 0; i < NS; ++i)
                    if (slot_par[i] >= 0) mbar_wait(&S.kv_full[i], slot_par[i], st, 123);
            }
        }
    } else if (warp == 1) {
        // --------------------------------------------------------------- MMA issuer
        const uint32_t elected = elect_one();
        constexpr uint32_t kIdescS = idesc_f16kind_f32(F16, 128, BS, false, false);
        constexpr uint32_t kIdescO = idesc_f16kind_f32(F16, 128, 128, false, true);
        constexpr uint32_t kQHalf = sizeof(S.q[0]) >> 4;
        constexpr uint32_t kSlot = sizeof(S.kv[0]) >> 4, kSlotHalf = sizeof(S.kv[0][0]) >> 4;
        const uint32_t q_desc0 = (uint32_t)smem_desc_sw128(smem_u32(S.q[0]), 16, 1024);
        const uint32_t k_desc0 = (uint32_t)smem_desc_sw128(smem_u32(S.kv[0][0]), 16, 1024);
        const uint32_t v_desc0 = (uint32_t)smem_desc_sw128(smem_u32(S.kv[0][0]), BS * 128, 1024);
        int n = 0, u = 0;
        bool ok = true;
        for (int ti = bid; ti < ntiles && ok; ti += grid, ++n) {
            const DTile t = dense_tile(p, ti);
            if (!(ok = wait(&S.q_full, n & 1, 124))) break;
            // S of this tile overwrites the P columns that PV of the previous tile read
            if (n > 0 && !(ok = wait(&S.o_full, (n - 1) & 1, 125))) break;
            tc_fence_after();
            for (int c = 0; c < t.ncand && ok; ++c, ++u) {
                const int sl = u % NS;
                if (!(ok = wait(&S.kv_full[sl], (u / NS) & 1, 126))) break;
                tc_fence_after();
                const uint32_t b0 = k_desc0 + (uint32_t)sl * kSlot;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t off = (uint32_t)((ks >> 2) * kQHalf + (ks & 3) * 2);
                    const uint32_t offk = (uint32_t)((ks >> 2) * kSlotHalf + (ks & 3) * 2);
                    mma_ss_e(tmem + (uint32_t)(c * BS), q_desc0 + off, b0 + offk, kIdescS,
                             ks > 0 ? 1u : 0u, elected);
                }
                mma_commit_e(&S.kv_empty[sl], elected);
            }
            if (!ok) break;
            mma_commit_e(&S.s_full, elected);
            mma_commit_e(&S.q_empty, elected);
            if (!(ok = wait(&S.p_full, n & 1, 127))) break;
            // O_d accumulates where the previous tile's O_d was: read out by now?
            if (!(ok = wait(&S.o_free, (n & 1) ^ 1, 128))) break;
            tc_fence_after();
            for (int c = 0; c < t.ncand && ok; ++c, ++u) {
                const int sl = u % NS;
                if (!(ok = wait(&S.kv_full[sl], (u / NS) & 1, 129))) break;
                tc_fence_after();
                const uint32_t b0 = v_desc0 + (uint32_t)sl * kSlot;
#pragma unroll
                for (int ks = 0; ks < BS / 16; ++ks)
                    mma_ts_e(tmem + kColO, tmem + (uint32_t)(c * BS + ks * 8), b0 + (uint32_t)ks * 128u,
                             kIdescO, (c > 0 || ks > 0) ? 1u : 0u, elected);
                mma_commit_e(&S.kv_empty[sl], elected);
            }
            if (!ok) break;
            mma_commit_e(&S.o_full, elected);
        }
        // every tcgen05 operation issued above has finished once this commit arrives
        mma_commit_e(&S.drain, elected);
        mbar_wait(&S.drain, 0, st, 130);
      }
    } else if (warp < 8) {
        // ------------------------------------------- softmax and the O_d hand-off
        const int quad = warp & 3, r = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const float c = p.scale_log2;
        const float kLn2 = 0.69314718055994531f;
        const int tokr = r / p.G;
        int n = 0;
        for (int ti = bid; ti < ntiles; ti += grid, ++n) {
            const DTile t = dense_tile(p, ti);
            const int i = t.i0 + tokr;                   // local position of this row
            const bool valid = i < t.L;
            const int qb = valid ? i / BS : -1;
            // which candidates this row keeps: its own index row, among {0, qb - 1, qb}
            unsigned keep = 0;
            if (valid) {
                const int32_t* bi = p.bidx + ((size_t)(t.tok0 + tokr) * p.hkv + t.g) * p.topk;
                for (int j = 0; j < p.topk; ++j) {
                    const int b = __ldg(bi + j);
                    if ((b == 0 || b == qb || b == qb - 1) && block_valid(b, qb, i, BS, p.swin))
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            if (k < t.ncand && t.cand[k] == b) keep |= 1u << k;
                }
            }
            if (!wait_w(&S.s_full, n & 1, 131)) break;
            tc_fence_after();
            // visible keys of candidate k: kk in [lo_k, lim_k] of the block
            auto bounds = [&](int k, int& lo, int& lim) {
                lim = ((keep >> k) & 1u) ? i - t.cand[k] * BS : -1;
                lo = p.swin > 0 ? lim - p.swin + 1 : 0;
            };
            float mx = -CUDART_INF_F;
#pragma unroll
            for (int k = 0; k < Cfg::kMaxCand; ++k) {
                if (k >= t.ncand) break;
                int lo, lim;
                bounds(k, lo, lim);
#pragma unroll
                for (int h64 = 0; h64 < BS / 64; ++h64) {
                    float sv[64];
                    tmem_ld64_sync(tmem + lane_off + (uint32_t)(k * BS + h64 * 64), sv);
#pragma unroll
                    for (int kk = 0; kk < 64; ++kk) {
                        const int key = h64 * 64 + kk;
                        if (key <= lim && key >= lo) mx = fmaxf(mx, sv[kk]);
                    }
                }
            }
            const bool any = mx != -CUDART_INF_F;
            const float mc = any ? mx * c : 0.f;
            float2 l2 = make_float2(0.f, 0.f);
#pragma unroll
            for (int k = 0; k < Cfg::kMaxCand; ++k) {
                if (k >= t.ncand) break;
                int lo, lim;
                bounds(k, lo, lim);
#pragma unroll
                for (int h64 = 0; h64 < BS / 64; ++h64) {
                    float sv[64];
                    tmem_ld64_sync(tmem + lane_off + (uint32_t)(k * BS + h64 * 64), sv);
                    uint32_t pk[32];
#pragma unroll
                    for (int k2 = 0; k2 < 32; ++k2) {
                        const int key = h64 * 64 + 2 * k2;
                        float2 x = fma2(make_float2(sv[2 * k2], sv[2 * k2 + 1]), make_float2(c, c),
                                        make_float2(-mc, -mc));
                        x.x = (key <= lim && key >= lo) ? ex2_approx(x.x) : 0.f;
                        x.y = (key + 1 <= lim && key + 1 >= lo) ? ex2_approx(x.y) : 0.f;
                        l2 = add2(l2, x);
                        pk[k2] = pack2<F16>(x.x, x.y);
                    }
                    tmem_st32_sync(tmem + lane_off + (uint32_t)(k * BS + h64 * 32), pk);
                }
            }
            tc_fence_before();
            mbar_arrive(&S.p_full);
            const float l = l2.x + l2.y;
            const float inv_l = l > 0.f ? 1.f / l : 0.f;
            const float lse_d = l > 0.f ? (mc + __log2f(l)) * kLn2 : -CUDART_INF_F;
            // O_d of this tile: TMEM -> registers -> the shared buffer (once the fold of the
            // previous tile has read it)
            if (!wait_w(&S.o_full, n & 1, 132)) break;
            tc_fence_after();
            if (!wait_w(&S.od_empty, (n & 1) ^ 1, 133)) break;
#pragma unroll
            for (int h64 = 0; h64 < 2; ++h64) {
                float x[64];
                tmem_ld64_sync(tmem + lane_off + (uint32_t)(kColO + h64 * 64), x);
#pragma unroll
                for (int c4 = 0; c4 < 16; ++c4) {
                    const float4 y = make_float4(x[4 * c4] * inv_l, x[4 * c4 + 1] * inv_l,
                                                 x[4 * c4 + 2] * inv_l, x[4 * c4 + 3] * inv_l);
                    *reinterpret_cast<float4*>(&S.od[od_index(r, h64 * 16 + c4)]) = y;
                }
            }
            S.od_lse[r] = lse_d;
            tc_fence_before();
            mbar_arrive(&S.o_free);
            mbar_arrive(&S.od_full);
        }
    } else {
        reg_alloc_d<168>();
        // ------------------------------------------------------------------- fold
        // Row r = fw + 8 k (k = 0 .. 15) of a tile is handled by fold warp fw; lane j owns
        // slot j (and j + 32) of the row.  A slot is merged from the KV-major partials if
        // its block is valid and not one of this kernel's blocks; its partial row is
        // posmap * G + head offset.  The index work of a tile (block numbers, then their
        // positions: two dependent loads) is done one tile ahead, spread over the rows of
        // the current tile, so that a row costs one memory latency (its partials and their
        // (lse, exponent)), and two rows' partial loads are in flight at a time.
        fold_rows<BS, F16, KS>(p, S.od, S.od_lse, &S.od_full, &S.od_empty, warp - kFoldWarp0,
                               lane, bid, grid, ntiles, abort_flag, st);
    }

    // ---- teardown: every role has left its loop (all waits are bounded) and the MMA
    //      issuer has drained its tensor-core work
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

template <int BS, int F16, int KS>
void launch_dense_variant(const DensePlan& p, const CUtensorMap* qmap, const CUtensorMap* kmap,
                          const CUtensorMap* vmap, cudaStream_t stream) {
    constexpr size_t smem = sizeof(DenseSmem<BS>) + 1024;
    cudaFuncSetAttribute(k_fwd_dense<BS, F16, KS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    k_fwd_dense<BS, F16, KS><<<p.num_sms, kDThreads, smem, stream>>>(p, *qmap, *kmap, *vmap);
}

template <int BS, int F16>
void launch_dense_ks(const DensePlan& p, const CUtensorMap* qmap, const CUtensorMap* kmap,
                     const CUtensorMap* vmap, cudaStream_t stream) {
    if (p.topk <= 16) launch_dense_variant<BS, F16, 16>(p, qmap, kmap, vmap, stream);
    else if (p.topk <= 32) launch_dense_variant<BS, F16, 32>(p, qmap, kmap, vmap, stream);
    else launch_dense_variant<BS, F16, 64>(p, qmap, kmap, vmap, stream);
}

}  // namespace

cudaError_t launch_fwd_dense(const DensePlan& p, const CUtensorMap* qmap, const CUtensorMap* kmap,
                             const CUtensorMap* vmap, cudaStream_t stream) {
    if (p.bs == 64) {
        if (p.f16) launch_dense_ks<64, 1>(p, qmap, kmap, vmap, stream);
        else launch_dense_ks<64, 0>(p, qmap, kmap, vmap, stream);
    } else {
        if (p.f16) launch_dense_ks<128, 1>(p, qmap, kmap, vmap, stream);
        else launch_dense_ks<128, 0>(p, qmap, kmap, vmap, stream);
    }
    return cudaGetLastError();
}

}  // namespace nsa
