// bwd.cu -- backward tile kernel of selected-block attention (KV-block major).
//
// The full loss-backward named in the key-features table of the
// "Relaxed-System-Lab/Flash-Sparse-Attention" project page, organised like the
// forward: a work unit is up to `chunk_tiles` consecutive 128-row tiles of one
// (KV head, KV block) list.  Per tile (rows = gathered (token, head) pairs):
//
//   S  = Q K^T,  dP = dO V^T                    tcgen05.mma -> TMEM
//   P  = exp(scale S - LSE) (causal on the diagonal block),  dS = P (dP - D)
//   dV^T += dO^T P,  dK^T += Q^T dS              accumulate in TMEM over the unit
//   dQ_part = scale * dS K                       per (row, slot), bf16
//
// At the end of a unit dV and scale*dK of its block are written as fp32 partials;
// k_dkdv_reduce sums the units of each block in order and k_dq_merge sums the dQ
// partials of each row over its slots.  No atomics anywhere: the result is
// deterministic.
#include <math_constants.h>

#include "nsa_common.cuh"
#include "nsa_kernels.h"

namespace nsa {
namespace {

constexpr int kBwdThreads = 128;

template <int BS>
struct alignas(1024) BwdSmem {
    uint8_t q[2][kTileRows * 128];
    uint8_t dout[2][kTileRows * 128];
    uint8_t k[2][BS * 128];
    uint8_t v[2][BS * 128];
    uint8_t p[BS / 64][kTileRows * 128];
    uint8_t ds[BS / 64][kTileRows * 128];
    uint64_t bar_kv;
    uint64_t bar_mma;
    uint32_t tmem_base;
    int abort_flag;
    int nunits;
    int row_tok[kTileRows];
    int row_head[kTileRows];
};

template <int BS>
constexpr size_t bwd_smem_bytes() {
    return sizeof(BwdSmem<BS>) + 1024;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

template <int BS>
__global__ void __launch_bounds__(kBwdThreads, 1)
    k_bwd_tiles(const BwdPlan p, const __grid_constant__ CUtensorMap kmap,
                const __grid_constant__ CUtensorMap vmap) {
    extern __shared__ uint8_t smem_raw[];
    BwdSmem<BS>& S = *reinterpret_cast<BwdSmem<BS>*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    DevStatus* st = p.st;

    if (tid == 0) {
        S.abort_flag = (*reinterpret_cast<volatile int*>(&st->code) != 0);
        S.nunits = *reinterpret_cast<volatile int*>(&st->nchunks);
        mbar_init(&S.bar_kv, 1);
        mbar_init(&S.bar_mma, 1);
        fence_barrier_init();
        prefetch_tmap(&kmap);
        prefetch_tmap(&vmap);
    }
    if (warp == 0) {
        tmem_alloc(&S.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;
    const uint32_t tS = tmem;          // S, later dQ: columns [0, 128)
    const uint32_t tdP = tmem + 128;   // dP
    const uint32_t tdV = tmem + 256;   // dV^T  (lane = head-dim index, column = key)
    const uint32_t tdK = tmem + 384;   // dK^T
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;

    const int nbtot = __ldg(p.blkoff + p.nseq);
    const int nbk = p.hkv * nbtot;
    const int nunits = S.nunits;
    const long long ub = (long long)nunits * blockIdx.x / gridDim.x;
    const long long ue = (long long)nunits * (blockIdx.x + 1) / gridDim.x;
    const int tpt = kTileRows / p.G;
    constexpr uint32_t kIdescS = idesc_bf16_f32(128, BS, false, false);    // S, dP
    constexpr uint32_t kIdescT = idesc_bf16_f32(128, BS, true, true);      // dV^T, dK^T
    constexpr uint32_t kIdescQ = idesc_bf16_f32(128, 128, false, true);    // dQ
    const float kLog2e = 1.4426950408889634f;

    uint32_t kv_phase = 0, mma_phase = 0;
    bool kv_unwaited = false, mma_unwaited = false;
    int cached_bucket = -1;

    for (long long unit = ub; unit < ue && !S.abort_flag; ++unit) {
        const int bucket = upper_index(p.chunk_off, nbk, (int)unit);
        const int g = bucket / nbtot;
        const int gb = bucket - g * nbtot;
        const int s = upper_index(p.blkoff, p.nseq, gb);
        const int b = gb - __ldg(p.blkoff + s);
        const int seq0 = __ldg(p.cu + s);
        const int key0 = seq0 + b * BS;
        const int tile_lo = __ldg(p.tile_off + bucket) +
                            ((int)unit - __ldg(p.chunk_off + bucket)) * p.chunk_tiles;
        const int tile_hi = min(tile_lo + p.chunk_tiles, __ldg(p.tile_off + bucket + 1));
        const int ent_lo = __ldg(p.offsets + bucket);
        const int ent_hi = __ldg(p.offsets + bucket + 1);

        for (int tile = tile_lo; tile < tile_hi; ++tile) {
            const bool first = tile == tile_lo;
            const int e0 = ent_lo + (tile - __ldg(p.tile_off + bucket)) * tpt;
            const int e1 = min(e0 + tpt, ent_hi);
            const int nrows = (e1 - e0) * p.G;

            int my_t = -1, my_h = 0, my_j = 0, my_lim = -1;
            float my_lse2 = 0.f, my_delta = 0.f;
            if (tid < nrows) {
                const uint32_t ent = __ldg(p.entries + e0 + tid / p.G);
                my_t = (int)(ent >> 6);
                my_j = (int)(ent & 63u);
                my_h = g * p.G + tid % p.G;
                my_lim = (my_t - seq0) - b * BS;
                my_lse2 = __ldg(p.lse + (size_t)my_h * p.T + my_t) * kLog2e;
                my_delta = __ldg(p.delta + (size_t)my_h * p.T + my_t);
            }
            S.row_tok[tid] = my_t;
            S.row_head[tid] = my_h;
            __syncthreads();

            if (first && bucket != cached_bucket && tid == 0) {
                mbar_arrive_expect_tx(&S.bar_kv, 4u * BS * 128u);
                tma_load_3d(S.k[0], &kmap, &S.bar_kv, 0, g, key0);
                tma_load_3d(S.k[1], &kmap, &S.bar_kv, 64, g, key0);
                tma_load_3d(S.v[0], &vmap, &S.bar_kv, 0, g, key0);
                tma_load_3d(S.v[1], &vmap, &S.bar_kv, 64, g, key0);
                kv_unwaited = true;
            }
            cached_bucket = bucket;

            // gather Q and dO rows; rows past the list are zero so that they add
            // nothing to the dV / dK sums over rows
            {
                const __nv_bfloat16* q = reinterpret_cast<const __nv_bfloat16*>(p.q);
                const __nv_bfloat16* dO = reinterpret_cast<const __nv_bfloat16*>(p.dout);
                const uint32_t q0 = smem_u32(S.q[0]), q1 = smem_u32(S.q[1]);
                const uint32_t d0 = smem_u32(S.dout[0]), d1 = smem_u32(S.dout[1]);
#pragma unroll 4
                for (int it = 0; it < 32; ++it) {
                    const int idx = tid + it * kBwdThreads;     // 0 .. 4095
                    const int which = idx >> 11;                // 0: Q, 1: dO
                    const int row = (idx >> 4) & 127, c = idx & 15;
                    const int t = S.row_tok[row];
                    const uint32_t dst = (which ? (c < 8 ? d0 : d1) : (c < 8 ? q0 : q1)) +
                                         sw128_offset(row, c & 7);
                    if (t >= 0) {
                        const __nv_bfloat16* src = (which ? dO : q) +
                                                   ((size_t)t * p.hq + S.row_head[row]) * kHeadDim + c * 8;
                        cp_async_16(dst, src);
                    } else {
                        st_shared_v4(dst, 0u, 0u, 0u, 0u);
                    }
                }
                cp_async_commit();
                cp_async_wait_all();
                fence_async_smem();
            }
            __syncthreads();

            // S = Q K^T and dP = dO V^T
            if (tid == 0) {
                bool ok = true;
                if (kv_unwaited) {
                    ok = mbar_wait(&S.bar_kv, kv_phase, st, 20);
                    if (ok) { kv_phase ^= 1; kv_unwaited = false; }
                }
                if (ok) {
                    tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        const uint32_t off = (uint32_t)(ks & 3) * 32u;
                        mma_bf16_ss(tS, smem_desc_sw128(smem_u32(S.q[ks >> 2]) + off, 16, 1024),
                                    smem_desc_sw128(smem_u32(S.k[ks >> 2]) + off, 16, 1024),
                                    kIdescS, ks > 0 ? 1u : 0u);
                    }
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        const uint32_t off = (uint32_t)(ks & 3) * 32u;
                        mma_bf16_ss(tdP, smem_desc_sw128(smem_u32(S.dout[ks >> 2]) + off, 16, 1024),
                                    smem_desc_sw128(smem_u32(S.v[ks >> 2]) + off, 16, 1024),
                                    kIdescS, ks > 0 ? 1u : 0u);
                    }
                    mma_commit(&S.bar_mma);
                    mma_unwaited = true;
                } else {
                    S.abort_flag = 1;
                }
            }
            __syncthreads();
            if (S.abort_flag) break;
            {
                const bool ok = mbar_wait(&S.bar_mma, mma_phase, st, 21);
                if (!ok) S.abort_flag = 1;
                mma_phase ^= 1;
                if (tid == 0 && ok) mma_unwaited = false;
            }
            tc_fence_after();

            // P and dS of this thread's row, 32 columns at a time
#pragma unroll
            for (int c32 = 0; c32 < BS / 32; ++c32) {
                float sv[32], dp[32];
                tmem_ld32(tS + lane_off + c32 * 32, sv);
                tmem_ld32(tdP + lane_off + c32 * 32, dp);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const int key = c32 * 32 + c;
                    const float pr = (key <= my_lim) ? exp2f(sv[c] * p.scale_log2 - my_lse2) : 0.f;
                    sv[c] = pr;
                    dp[c] = pr * (dp[c] - my_delta);
                }
                const int chunk = c32 >> 1;
                const uint32_t pb = smem_u32(S.p[chunk]);
                const uint32_t db = smem_u32(S.ds[chunk]);
#pragma unroll
                for (int pc4 = 0; pc4 < 4; ++pc4) {
                    const int pc = (c32 & 1) * 4 + pc4;
                    const float* x = sv + pc4 * 8;
                    const float* y = dp + pc4 * 8;
                    st_shared_v4(pb + sw128_offset(tid, pc), pack_bf16x2(x[0], x[1]),
                                 pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                                 pack_bf16x2(x[6], x[7]));
                    st_shared_v4(db + sw128_offset(tid, pc), pack_bf16x2(y[0], y[1]),
                                 pack_bf16x2(y[2], y[3]), pack_bf16x2(y[4], y[5]),
                                 pack_bf16x2(y[6], y[7]));
                }
            }
            fence_async_smem();
            tc_fence_before();
            __syncthreads();
            if (S.abort_flag) break;

            // dV^T += dO^T P,  dK^T += Q^T dS,  dQ = dS K
            if (tid == 0) {
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {     // K = 128 rows, 16 per step
                    const uint32_t off = (uint32_t)ks * 2048u;
                    const uint32_t acc = (first && ks == 0) ? 0u : 1u;
                    mma_bf16_ss(tdV, smem_desc_sw128(smem_u32(S.dout[0]) + off, 16384, 1024),
                                smem_desc_sw128(smem_u32(S.p[0]) + off, 16384, 1024), kIdescT, acc);
                    mma_bf16_ss(tdK, smem_desc_sw128(smem_u32(S.q[0]) + off, 16384, 1024),
                                smem_desc_sw128(smem_u32(S.ds[0]) + off, 16384, 1024), kIdescT, acc);
                }
#pragma unroll
                for (int ks = 0; ks < BS / 16; ++ks) {   // K = BS keys
                    mma_bf16_ss(tS,
                                smem_desc_sw128(smem_u32(S.ds[ks >> 2]) + (uint32_t)(ks & 3) * 32u, 16, 1024),
                                smem_desc_sw128(smem_u32(S.k[0]) + (uint32_t)ks * 2048u, BS * 128, 1024),
                                kIdescQ, ks > 0 ? 1u : 0u);
                }
                mma_commit(&S.bar_mma);
                mma_unwaited = true;
            }
            {
                const bool ok = mbar_wait(&S.bar_mma, mma_phase, st, 22);
                if (!ok) S.abort_flag = 1;
                mma_phase ^= 1;
                if (tid == 0 && ok) mma_unwaited = false;
            }
            tc_fence_after();

            // dQ partial of this row and slot
            {
                const size_t prow = ((size_t)(my_t < 0 ? 0 : my_t) * p.hq + my_h) * p.topk + my_j;
                uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.part_dq) +
                                                      prow * kHeadDim);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float o[32];
                    tmem_ld32(tS + lane_off + c * 32, o);
                    tmem_wait_ld();
                    if (my_t >= 0) {
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            const float* x = o + q4 * 8;
                            uint4 w;
                            w.x = pack_bf16x2(x[0] * p.scale, x[1] * p.scale);
                            w.y = pack_bf16x2(x[2] * p.scale, x[3] * p.scale);
                            w.z = pack_bf16x2(x[4] * p.scale, x[5] * p.scale);
                            w.w = pack_bf16x2(x[6] * p.scale, x[7] * p.scale);
                            dst[c * 4 + q4] = w;
                        }
                    }
                }
            }
            tc_fence_before();
            __syncthreads();
        }
        if (S.abort_flag) break;

        // unit epilogue: dV and scale*dK of this block as fp32 partials [2][BS][128]
        {
            float* dvp = p.part_dkdv + (size_t)unit * 2 * BS * kHeadDim;
            float* dkp = dvp + (size_t)BS * kHeadDim;
#pragma unroll
            for (int c32 = 0; c32 < BS / 32; ++c32) {
                float xv[32], xk[32];
                tmem_ld32(tdV + lane_off + c32 * 32, xv);
                tmem_ld32(tdK + lane_off + c32 * 32, xk);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const int key = c32 * 32 + c;
                    dvp[(size_t)key * kHeadDim + tid] = xv[c];
                    dkp[(size_t)key * kHeadDim + tid] = xk[c] * p.scale;
                }
            }
        }
        tc_fence_before();
        __syncthreads();
    }

    if (tid == 0 && S.abort_flag) {
        if (kv_unwaited) mbar_wait(&S.bar_kv, kv_phase, st, 23);
        if (mma_unwaited) mbar_wait(&S.bar_mma, mma_phase, st, 24);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace

cudaError_t launch_bwd_tiles(const BwdPlan& p, const CUtensorMap* kmap, const CUtensorMap* vmap,
                             cudaStream_t stream) {
    if (p.bs == 64) {
        constexpr size_t smem = bwd_smem_bytes<64>();
        cudaFuncSetAttribute(k_bwd_tiles<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k_bwd_tiles<64><<<p.num_sms, kBwdThreads, smem, stream>>>(p, *kmap, *vmap);
    } else {
        constexpr size_t smem = bwd_smem_bytes<128>();
        cudaFuncSetAttribute(k_bwd_tiles<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k_bwd_tiles<128><<<p.num_sms, kBwdThreads, smem, stream>>>(p, *kmap, *vmap);
    }
    return cudaGetLastError();
}

}  // namespace nsa
