// fwd.cu -- forward tile kernel of selected-block attention (KV-block major).
//
// A tile is (KV head g, KV block B, up to 128 gathered query rows), a row being
// (token, query head) for a token whose index row selected B; the G query heads of a
// token are adjacent rows, so a group of any size fills the 128-row tensor-core tile
// (the loop swap of the FSA pages: "FSA: Efficient Implementation of Native Sparse
// Attention" blog, second paragraph).  Per tile:
//
//   S   = Q K_B^T                  tcgen05.mma, fp32 accumulator in TMEM
//   P   = exp(scale S - m), causal mask on the diagonal block, l = sum P
//   O_B = P V_B                    tcgen05.mma (P staged in shared memory)
//   partial: O_B / l as fp16 with a power-of-two row exponent, lse_B = m + log l,
//   stored per (token, head, slot) for the log-sum-exp merge in merge.cu.
//
// Tiles are ordered (g, token window, B) and dealt round-robin to one persistent CTA
// per SM, so at any time all SMs gather query rows of one window (a few MB, L2
// resident).  Each CTA is warp-specialised and pipelined:
//
//   warps 0-1   loaders: row metadata, cp.async gather of the Q rows (2 Q stages)
//   warp 2      TMA producer: K_B and V_B (128B swizzle) into NKV stages
//   warp 3      MMA issuer (one thread): S(i+1) is issued before PV(i)
//   warps 4-7   softmax + epilogue of even tiles   } TMEM slots 0 / 1:
//   warps 8-11  softmax + epilogue of odd tiles    } S and O accumulators each
//
// Producer/consumer hand-offs are mbarriers; every wait is bounded (nsa_common.cuh).
#include <math_constants.h>

#include "nsa_common.cuh"
#include "nsa_kernels.h"

namespace nsa {
namespace {

constexpr int kThreads = 384;
constexpr int kLoaderThreads = 64;
constexpr int kSoftmaxThreads = 128;

template <int BS, int NKV>
struct alignas(1024) FwdSmem {
    uint8_t q[2][2][kTileRows * 128];         // Q rows: [stage][64-column half]
    uint8_t kv[NKV][2][2][BS * 128];          // [stage][K, V][half]
    uint8_t p[2][BS / 64][kTileRows * 128];   // P bf16 [row][key] per TMEM slot
    int4 meta[2][kTileRows];                  // (token or -1, head, slot, causal limit)
    int tile_bucket[2];                       // bucket of the tile in each Q stage
    uint64_t q_full[2], q_empty[2], meta_full[2], meta_empty[2];
    uint64_t kv_full[NKV], kv_empty[NKV];
    uint64_t s_full[2], p_full[2], o_full[2], tmem_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
    int loader_stop;
    int ntiles;
};

template <int BS, int NKV>
constexpr size_t fwd_smem_bytes() {
    return sizeof(FwdSmem<BS, NKV>) + 1024;
}

// Tile descriptor (built by k_tile_desc): first key of the block, first entry of the
// tile, rows | g << 8, and the block's bucket id g * NB + B (identifies K_B / V_B).
struct Tile {
    int key0, e0, nrows, g, bucket;
};

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ void cp_async_wait_one_pending() {
    asm volatile("cp.async.wait_group 1;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

template <int BS, int NKV>
__global__ void __launch_bounds__(kThreads, 1)
    k_fwd_tiles(const FwdPlan p, const __grid_constant__ CUtensorMap kmap,
                const __grid_constant__ CUtensorMap vmap) {
    extern __shared__ uint8_t smem_raw[];
    FwdSmem<BS, NKV>& S = *reinterpret_cast<FwdSmem<BS, NKV>*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    DevStatus* st = p.st;

    if (tid == 0) {
        S.abort_flag = (*reinterpret_cast<volatile int*>(&st->code) != 0);
        S.loader_stop = 0;
        S.ntiles = *reinterpret_cast<volatile int*>(&st->ntiles_fwd);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.q_full[i], kLoaderThreads);
            mbar_init(&S.q_empty[i], 1);
            mbar_init(&S.meta_full[i], kLoaderThreads);
            mbar_init(&S.meta_empty[i], kSoftmaxThreads);
            mbar_init(&S.s_full[i], 1);
            mbar_init(&S.p_full[i], kSoftmaxThreads);
            mbar_init(&S.o_full[i], 1);
            mbar_init(&S.tmem_empty[i], kSoftmaxThreads);
        }
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
    const int ntiles = S.ntiles;
    const int n = (!S.abort_flag && (int)blockIdx.x < ntiles)
                      ? (ntiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1
                      : 0;
    auto tile_of = [&](int i) { return (int)blockIdx.x + i * (int)gridDim.x; };
    volatile int* abort_flag = &S.abort_flag;
    auto wait = [&](uint64_t* bar, uint32_t parity, int where) -> bool {
        if (*abort_flag) return false;
        if (!mbar_wait(bar, parity, st, where)) {
            *abort_flag = 1;
            return false;
        }
        return true;
    };

    if (warp < 2) {
        // ------------------------------------------------------------------ loaders
        // The 64 loader threads share each tile's row metadata through shared memory
        // (named barrier 1).  The copies of tile i are published one tile later: wait
        // for the older cp.async group, make it visible to the tensor core's (async)
        // proxy, then arrive on q_full.  Tile descriptors are prefetched four tiles
        // ahead and the next tile's index entries one tile ahead.
        const int lt = tid;                       // 0 .. 63
        const __nv_bfloat16* q = reinterpret_cast<const __nv_bfloat16*>(p.q);
        volatile int* stop = &S.loader_stop;
        auto ld_desc = [&](int i) {
            return i < n ? __ldg(p.tile_desc + tile_of(i)) : make_int4(0, 0, 0, -1);
        };
        int4 d0 = ld_desc(0), d1 = ld_desc(1), d2 = ld_desc(2), d3 = ld_desc(3);
        auto ld_ent = [&](const int4& d, int r) -> uint32_t {
            return r < (d.z & 255) ? __ldg(p.entries + d.y + r / p.G) : 0u;
        };
        uint32_t ent0 = n > 0 ? ld_ent(d0, 2 * lt) : 0u, ent1 = n > 0 ? ld_ent(d0, 2 * lt + 1) : 0u;
        int done = 0;
        for (int i = 0; i < n; ++i) {
            const Tile ti{d0.x, d0.y, d0.z & 255, d0.z >> 8, d0.w};
            d0 = d1; d1 = d2; d2 = d3; d3 = ld_desc(i + 4);
            const int slot = i & 1;
            const uint32_t ph_empty = ((i >> 1) & 1) ^ 1;
            const bool ok = wait(&S.meta_empty[slot], ph_empty, 30) &&
                            wait(&S.q_empty[slot], ph_empty, 31);
            if (!ok) *stop = 1;
            if (ok) {
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {   // metadata of rows 2*lt and 2*lt + 1
                    const int r = 2 * lt + rr;
                    const uint32_t ent = rr ? ent1 : ent0;
                    int4 m = make_int4(-1, 0, 0, 0);
                    if (r < ti.nrows) {
                        m.x = (int)(ent >> 6);
                        m.y = ti.g * p.G + r % p.G;
                        m.z = (int)(ent & 63u);
                        m.w = m.x - ti.key0;
                    }
                    S.meta[slot][r] = m;
                }
                if (lt == 0) S.tile_bucket[slot] = ti.bucket;
            }
            if (i + 1 < n) {                      // next tile's index entries
                ent0 = ld_ent(d0, 2 * lt);
                ent1 = ld_ent(d0, 2 * lt + 1);
            }
            named_bar_sync(1, kLoaderThreads);
            if (*stop) break;                     // read after the barrier: uniform
            mbar_arrive(&S.meta_full[slot]);
            // gather: 2048 16-byte chunks, 32 per thread; a warp instruction covers two
            // 256-byte rows (the G heads of a token are adjacent rows)
            const uint32_t q0 = smem_u32(S.q[slot][0]);
#pragma unroll 4
            for (int k = 0; k < 32; ++k) {
                const int idx = lt + k * kLoaderThreads;
                const int row = idx >> 4, c = idx & 15;
                const int4 m = S.meta[slot][row];
                if (m.x >= 0) {
                    const __nv_bfloat16* src = q + ((size_t)m.x * p.hq + m.y) * kHeadDim + c * 8;
                    cp_async_16(q0 + (c >> 3) * (kTileRows * 128) + sw128_offset(row, c & 7), src);
                }
            }
            cp_async_commit();
            if (i > 0) {
                cp_async_wait_one_pending();
                fence_async_smem();
                mbar_arrive(&S.q_full[(i - 1) & 1]);
            }
            done = i + 1;
        }
        cp_async_wait_all();
        fence_async_smem();
        if (done > 0 && done == n) mbar_arrive(&S.q_full[(n - 1) & 1]);
    } else if (warp == 2) {
        // ------------------------------------------------------------- K/V producer
        if (lane == 0) {
            prefetch_tmap(&kmap);
            prefetch_tmap(&vmap);
            int prev = -1, uses = 0;
            int last_parity[NKV];
            bool loaded[NKV];
            for (int s = 0; s < NKV; ++s) { last_parity[s] = 0; loaded[s] = false; }
            auto ld_desc = [&](int i) { return i < n ? __ldg(p.tile_desc + tile_of(i)) : make_int4(0, 0, 0, -1); };
            int4 d0 = ld_desc(0), d1 = ld_desc(1), d2 = ld_desc(2), d3 = ld_desc(3);
            for (int i = 0; i < n; ++i) {
                const Tile ti{d0.x, d0.y, d0.z & 255, d0.z >> 8, d0.w};
                d0 = d1; d1 = d2; d2 = d3; d3 = ld_desc(i + 4);
                if (ti.bucket == prev) continue;
                prev = ti.bucket;
                const int stg = uses % NKV;
                if (!wait(&S.kv_empty[stg], ((uses / NKV) & 1) ^ 1, 32)) break;
                mbar_arrive_expect_tx(&S.kv_full[stg], 4u * BS * 128u);
                tma_load_3d(S.kv[stg][0][0], &kmap, &S.kv_full[stg], 0, ti.g, ti.key0);
                tma_load_3d(S.kv[stg][0][1], &kmap, &S.kv_full[stg], 64, ti.g, ti.key0);
                tma_load_3d(S.kv[stg][1][0], &vmap, &S.kv_full[stg], 0, ti.g, ti.key0);
                tma_load_3d(S.kv[stg][1][1], &vmap, &S.kv_full[stg], 64, ti.g, ti.key0);
                last_parity[stg] = (uses / NKV) & 1;
                loaded[stg] = true;
                ++uses;
            }
            if (*abort_flag)   // let copies still in flight land before the CTA exits
                for (int s = 0; s < NKV; ++s)
                    if (loaded[s]) mbar_wait(&S.kv_full[s], last_parity[s], st, 40);
        }
    } else if (warp == 3) {
        // -------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdescS = idesc_bf16_f32(128, BS, false, false);
            constexpr uint32_t kIdescO = idesc_bf16_f32(128, 128, false, true);
            int kv_uses = 0, prev_bucket = -1, cur = 0;
            int kvs_of[2] = {0, 0};
            // Waits for tile i's Q rows, learns its block from the loaders' record and
            // switches K/V stage when the block changes; returns the bucket or -2.
            auto acquire = [&](int i) -> int {
                const int slot = i & 1;
                if (!wait(&S.q_full[slot], (i >> 1) & 1, 35)) return -2;
                const int bucket = *reinterpret_cast<volatile int*>(&S.tile_bucket[slot]);
                return bucket;
            };
            auto issue_s = [&](int i, int bucket) -> bool {
                if (bucket != prev_bucket) {
                    cur = kv_uses % NKV;
                    if (!wait(&S.kv_full[cur], (kv_uses / NKV) & 1, 33)) return false;
                    ++kv_uses;
                    prev_bucket = bucket;
                }
                const int slot = i & 1;
                kvs_of[slot] = cur;
                if (!wait(&S.tmem_empty[slot], ((i >> 1) & 1) ^ 1, 34)) return false;
                tc_fence_after();
                const uint32_t tS = tmem + slot * 256;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t off = (uint32_t)(ks & 3) * 32u;
                    const uint64_t a =
                        smem_desc_sw128(smem_u32(S.q[slot][ks >> 2]) + off, 16, 1024);
                    const uint64_t b =
                        smem_desc_sw128(smem_u32(S.kv[cur][0][ks >> 2]) + off, 16, 1024);
                    mma_bf16_ss(tS, a, b, kIdescS, ks > 0 ? 1u : 0u);
                }
                mma_commit(&S.s_full[slot]);
                mma_commit(&S.q_empty[slot]);
                return true;
            };
            if (n > 0) {
                int bucket_cur = acquire(0);
                bool ok = bucket_cur != -2 && issue_s(0, bucket_cur);
                for (int i = 0; i < n && ok; ++i) {
                    const int slot = i & 1;
                    // with two K/V stages S(i+1) goes ahead of PV(i)
                    int bucket_next = -1;
                    bool issued_next = false;
                    if (NKV > 1 && i + 1 < n) {
                        bucket_next = acquire(i + 1);
                        if (bucket_next == -2 || !(ok = issue_s(i + 1, bucket_next))) { ok = false; break; }
                        issued_next = true;
                    }
                    if (!(ok = wait(&S.p_full[slot], (i >> 1) & 1, 36))) break;
                    tc_fence_after();
                    const uint32_t tO = tmem + slot * 256 + 128;
                    const int kvs = kvs_of[slot];
#pragma unroll
                    for (int ks = 0; ks < BS / 16; ++ks) {
                        const uint64_t a = smem_desc_sw128(
                            smem_u32(S.p[slot][ks >> 2]) + (uint32_t)(ks & 3) * 32u, 16, 1024);
                        const uint64_t b = smem_desc_sw128(
                            smem_u32(S.kv[kvs][1][0]) + (uint32_t)ks * 2048u, BS * 128, 1024);
                        mma_bf16_ss(tO, a, b, kIdescO, ks > 0 ? 1u : 0u);
                    }
                    mma_commit(&S.o_full[slot]);
                    if (!issued_next && i + 1 < n) {
                        bucket_next = acquire(i + 1);
                        if (bucket_next == -2) { ok = false; break; }
                    }
                    if (bucket_next != bucket_cur) mma_commit(&S.kv_empty[kvs]);
                    if (!issued_next && i + 1 < n && !(ok = issue_s(i + 1, bucket_next))) break;
                    bucket_cur = bucket_next;
                }
            }
            // every MMA issued above has finished once this commit arrives
            mma_commit(&S.drain);
            mbar_wait(&S.drain, 0, st, 41);
        }
    } else {
        // ---------------------------------------------------- softmax + epilogue
        const int wg = (warp - 4) >> 2;                  // 0: even tiles, 1: odd tiles
        const int r = (warp & 3) * 32 + lane;            // row = TMEM lane
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + wg * 256 + lane_off;
        const uint32_t tO = tS + 128;
        const float kLn2 = 0.69314718055994531f;
        for (int i = wg; i < n; i += 2) {
            const uint32_t ph = (i >> 1) & 1;
            if (!wait(&S.meta_full[wg], ph, 37)) break;
            const int4 m4 = S.meta[wg][r];
            mbar_arrive(&S.meta_empty[wg]);
            const int my_t = m4.x, my_h = m4.y, my_j = m4.z, my_lim = m4.w;
            if (!wait(&S.s_full[wg], ph, 38)) break;
            tc_fence_after();
            // scores of this row: all BS columns in one batch of TMEM loads
            float sv[BS];
#pragma unroll
            for (int c32 = 0; c32 < BS / 32; ++c32) tmem_ld32(tS + c32 * 32, sv + c32 * 32);
            tmem_wait_ld();
            float mx = -CUDART_INF_F;
#pragma unroll
            for (int c = 0; c < BS; ++c) {
                sv[c] = (c <= my_lim) ? sv[c] * p.scale_log2 : -CUDART_INF_F;
                mx = fmaxf(mx, sv[c]);
            }
            if (my_t < 0) mx = 0.f;
            // P = exp2(s - m) as bf16 into the slot's P tile, l = sum P
            float l = 0.f;
#pragma unroll
            for (int pc = 0; pc < BS / 8; ++pc) {
                float x[8];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    x[c] = exp2f(sv[pc * 8 + c] - mx);
                    l += x[c];
                }
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                                 smem_u32(S.p[wg][pc >> 3]) + sw128_offset(r, pc & 7)),
                             "r"(pack_bf16x2(x[0], x[1])), "r"(pack_bf16x2(x[2], x[3])),
                             "r"(pack_bf16x2(x[4], x[5])), "r"(pack_bf16x2(x[6], x[7]))
                             : "memory");
            }
            fence_async_smem();
            mbar_arrive(&S.p_full[wg]);
            if (!wait(&S.o_full[wg], ph, 39)) break;
            tc_fence_after();
            // epilogue: O_B / l as fp16 with exponent e (0 unless max |O_B / l| > 2^14);
            // the whole 128-column row in one batch of TMEM loads
            float o[128];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(tO + c * 32, o + c * 32);
            tmem_wait_ld();
            const float inv_l = 1.f / l;
            float omax = 0.f;
#pragma unroll
            for (int k = 0; k < 128; ++k) omax = fmaxf(omax, fabsf(o[k]));
            omax *= inv_l;
            const int e = omax > 16384.f ? ilogbf(omax) - 14 : 0;
            const float sc = ldexpf(inv_l, -e);
            const size_t prow = ((size_t)(my_t < 0 ? 0 : my_t) * p.hq + my_h) * p.topk + my_j;
            if (my_t >= 0) {
                uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__half*>(p.part_o) + prow * kHeadDim);
#pragma unroll
                for (int q8 = 0; q8 < 16; ++q8) {
                    const float* x = o + q8 * 8;
                    uint4 w;
                    w.x = pack_f16x2(x[0] * sc, x[1] * sc);
                    w.y = pack_f16x2(x[2] * sc, x[3] * sc);
                    w.z = pack_f16x2(x[4] * sc, x[5] * sc);
                    w.w = pack_f16x2(x[6] * sc, x[7] * sc);
                    dst[q8] = w;
                }
            }
            if (my_t >= 0) p.part_meta[prow] = make_float2((mx + __log2f(l)) * kLn2, (float)e);
            tc_fence_before();
            mbar_arrive(&S.tmem_empty[wg]);
        }
    }

    // ---- teardown: every role has left its loop (all waits are bounded) and the MMA
    //      issuer has drained its tensor-core work
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace

cudaError_t launch_fwd_tiles(const FwdPlan& p, const CUtensorMap* kmap, const CUtensorMap* vmap,
                             cudaStream_t stream) {
    if (p.bs == 64) {
        constexpr size_t smem = fwd_smem_bytes<64, 2>();
        cudaFuncSetAttribute(k_fwd_tiles<64, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
        k_fwd_tiles<64, 2><<<p.num_sms, kThreads, smem, stream>>>(p, *kmap, *vmap);
    } else {
        constexpr size_t smem = fwd_smem_bytes<128, 1>();
        cudaFuncSetAttribute(k_fwd_tiles<128, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
        k_fwd_tiles<128, 1><<<p.num_sms, kThreads, smem, stream>>>(p, *kmap, *vmap);
    }
    return cudaGetLastError();
}

}  // namespace nsa
