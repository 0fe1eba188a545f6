// fwd.cu -- forward tile kernel of selected-block attention (KV-block major).
//
// One work unit ("tile") is (KV head g, KV block B, up to 128 gathered query rows),
// where a row is (token, query head) for a token whose index row selected B; the G
// query heads of a token are adjacent rows, so a group of any size fills the
// 128-row tensor-core tile (the loop swap of the FSA pages: "FSA: Efficient
// Implementation of Native Sparse Attention" blog, second paragraph).  Per tile:
//
//   K_B, V_B  --TMA (128B swizzle)-->  shared memory   (skipped when B repeats)
//   Q rows    --cp.async gather----->  shared memory   (same swizzled layout)
//   S   = Q K_B^T                      tcgen05.mma, fp32 accumulator in TMEM
//   P   = exp(scale * S - m), causal mask on the diagonal block, l = sum P
//   O_B = P V_B                        tcgen05.mma (P from shared memory)
//   partial (O_B / l as fp16 with a power-of-two exponent, lse_B = m + log l)
//   stored per (token, head, slot)
//
// The log-sum-exp merge of the partials over a row's slots (no atomics) is in
// merge.cu.  Persistent CTAs take contiguous tile ranges, so consecutive tiles of
// one CTA usually share B and K_B/V_B stay in shared memory.
#include <math_constants.h>

#include "nsa_common.cuh"
#include "nsa_kernels.h"

namespace nsa {
namespace {

constexpr int kFwdThreads = 128;

template <int BS>
struct alignas(1024) FwdSmem {
    uint8_t q[2][kTileRows * 128];         // Q rows, two 64-column halves (K-major)
    uint8_t k[2][BS * 128];                // K block, two halves (K-major)
    uint8_t v[2][BS * 128];                // V block, two halves (MN-major view)
    uint8_t p[BS / 64][kTileRows * 128];   // P bf16 [row][key] in 64-key chunks
    uint64_t bar_kv;
    uint64_t bar_mma;
    uint32_t tmem_base;
    int abort_flag;
    int ntiles;
    int row_tok[kTileRows];
    int row_head[kTileRows];
    int row_slot[kTileRows];
    int row_lim[kTileRows];
};

template <int BS>
constexpr size_t fwd_smem_bytes() {
    return sizeof(FwdSmem<BS>) + 1024;   // + alignment slack
}

template <int BS>
__global__ void __launch_bounds__(kFwdThreads, 1)
    k_fwd_tiles(const FwdPlan p, const __grid_constant__ CUtensorMap kmap,
                const __grid_constant__ CUtensorMap vmap) {
    extern __shared__ uint8_t smem_raw[];
    FwdSmem<BS>& S = *reinterpret_cast<FwdSmem<BS>*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    DevStatus* st = p.st;

    if (tid == 0) {
        S.abort_flag = (*reinterpret_cast<volatile int*>(&st->code) != 0);
        S.ntiles = *reinterpret_cast<volatile int*>(&st->ntiles);
        mbar_init(&S.bar_kv, 1);
        mbar_init(&S.bar_mma, 1);
        fence_barrier_init();
        prefetch_tmap(&kmap);
        prefetch_tmap(&vmap);
    }
    if (warp == 0) {
        tmem_alloc(&S.tmem_base, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;
    const uint32_t tS = tmem;            // columns [0, BS)
    const uint32_t tO = tmem + 128;      // columns [128, 256)
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;

    const int nbtot = __ldg(p.blkoff + p.nseq);
    const int nbk = p.hkv * nbtot;
    const int ntiles = S.ntiles;
    const long long tb = (long long)ntiles * blockIdx.x / gridDim.x;
    const long long te = (long long)ntiles * (blockIdx.x + 1) / gridDim.x;
    const int tpt = kTileRows / p.G;
    constexpr uint32_t kIdescS = idesc_bf16_f32(128, BS, false, false);
    constexpr uint32_t kIdescO = idesc_bf16_f32(128, 128, false, true);
    const float kLn2 = 0.69314718055994531f;

    uint32_t kv_phase = 0, mma_phase = 0;
    bool kv_unwaited = false, mma_unwaited = false;   // meaningful in thread 0 only
    int cached_bucket = -1;

    for (long long tile = tb; tile < te && !S.abort_flag; ++tile) {
        // ---- decode the tile: bucket, entry range, block position
        const int bucket = upper_index(p.tile_off, nbk, (int)tile);
        const int g = bucket / nbtot;
        const int gb = bucket - g * nbtot;
        const int s = upper_index(p.blkoff, p.nseq, gb);
        const int b = gb - __ldg(p.blkoff + s);
        const int seq0 = __ldg(p.cu + s);
        const int key0 = seq0 + b * BS;
        const int e0 = __ldg(p.offsets + bucket) + ((int)tile - __ldg(p.tile_off + bucket)) * tpt;
        const int e1 = min(e0 + tpt, __ldg(p.offsets + bucket + 1));
        const int nrows = (e1 - e0) * p.G;

        // ---- row metadata (thread == row)
        int my_t = -1, my_h = 0, my_j = 0, my_lim = 0;
        if (tid < nrows) {
            const uint32_t ent = __ldg(p.entries + e0 + tid / p.G);
            my_t = (int)(ent >> 6);
            my_j = (int)(ent & 63u);
            my_h = g * p.G + tid % p.G;
            my_lim = (my_t - seq0) - b * BS;     // allowed key offsets c <= my_lim
        }
        S.row_tok[tid] = my_t;
        S.row_head[tid] = my_h;
        __syncthreads();

        // ---- K/V block by TMA (only when the block changes)
        const bool load_kv = bucket != cached_bucket;
        if (load_kv && tid == 0) {
            mbar_arrive_expect_tx(&S.bar_kv, 4u * BS * 128u);
            tma_load_3d(S.k[0], &kmap, &S.bar_kv, 0, g, key0);
            tma_load_3d(S.k[1], &kmap, &S.bar_kv, 64, g, key0);
            tma_load_3d(S.v[0], &vmap, &S.bar_kv, 0, g, key0);
            tma_load_3d(S.v[1], &vmap, &S.bar_kv, 64, g, key0);
            kv_unwaited = true;
        }
        cached_bucket = bucket;

        // ---- gather the Q rows (16-byte chunks, 16 chunks per 256-byte row)
        {
            const uint32_t qs0 = smem_u32(S.q[0]);
            const uint32_t qs1 = smem_u32(S.q[1]);
            const __nv_bfloat16* q = reinterpret_cast<const __nv_bfloat16*>(p.q);
#pragma unroll
            for (int it = 0; it < 16; ++it) {
                const int idx = tid + it * kFwdThreads;
                const int row = idx >> 4, c = idx & 15;
                const int t = S.row_tok[row];
                if (t >= 0) {
                    const __nv_bfloat16* src =
                        q + ((size_t)t * p.hq + S.row_head[row]) * kHeadDim + c * 8;
                    cp_async_16((c < 8 ? qs0 : qs1) + sw128_offset(row, c & 7), src);
                }
            }
            cp_async_commit();
            cp_async_wait_all();
            fence_async_smem();
        }
        __syncthreads();

        // ---- S = Q K^T
        if (tid == 0) {
            bool ok = true;
            if (kv_unwaited) {
                ok = mbar_wait(&S.bar_kv, kv_phase, st, 10);
                if (ok) { kv_phase ^= 1; kv_unwaited = false; }
            }
            if (ok) {
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t off = (uint32_t)(ks & 3) * 32u;
                    const uint64_t a = smem_desc_sw128(smem_u32(S.q[ks >> 2]) + off, 16, 1024);
                    const uint64_t bd = smem_desc_sw128(smem_u32(S.k[ks >> 2]) + off, 16, 1024);
                    mma_bf16_ss(tS, a, bd, kIdescS, ks > 0 ? 1u : 0u);
                }
                mma_commit(&S.bar_mma);
                mma_unwaited = true;
            } else {
                S.abort_flag = 1;
            }
        }
        __syncthreads();
        if (S.abort_flag) break;
        if (!mbar_wait(&S.bar_mma, mma_phase, st, 11)) S.abort_flag = 1;
        mma_phase ^= 1;
        if (tid == 0) mma_unwaited = false;
        tc_fence_after();

        // ---- softmax of this thread's row; P (bf16) to shared memory
        float sv[BS];
#pragma unroll
        for (int c = 0; c < BS / 32; ++c) tmem_ld32(tS + lane_off + c * 32, sv + c * 32);
        tmem_wait_ld();
        float m = -CUDART_INF_F;
#pragma unroll
        for (int c = 0; c < BS; ++c) {
            float x = sv[c] * p.scale_log2;
            x = (c <= my_lim) ? x : -CUDART_INF_F;
            sv[c] = x;
            m = fmaxf(m, x);
        }
        if (my_t < 0) m = 0.f;              // unused row: keep the arithmetic finite
        float l = 0.f;
#pragma unroll
        for (int c = 0; c < BS; ++c) {
            const float e = exp2f(sv[c] - m);
            sv[c] = e;
            l += e;
        }
#pragma unroll
        for (int chunk = 0; chunk < BS / 64; ++chunk) {
            const uint32_t base = smem_u32(S.p[chunk]);
#pragma unroll
            for (int pc = 0; pc < 8; ++pc) {
                const float* x = sv + chunk * 64 + pc * 8;
                const uint32_t w0 = pack_bf16x2(x[0], x[1]), w1 = pack_bf16x2(x[2], x[3]);
                const uint32_t w2 = pack_bf16x2(x[4], x[5]), w3 = pack_bf16x2(x[6], x[7]);
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                                 base + sw128_offset(tid, pc)),
                             "r"(w0), "r"(w1), "r"(w2), "r"(w3)
                             : "memory");
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (S.abort_flag) break;

        // ---- O_B = P V_B
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < BS / 16; ++ks) {
                const uint64_t a = smem_desc_sw128(
                    smem_u32(S.p[ks >> 2]) + (uint32_t)(ks & 3) * 32u, 16, 1024);
                const uint64_t bd =
                    smem_desc_sw128(smem_u32(S.v[0]) + (uint32_t)ks * 2048u, BS * 128, 1024);
                mma_bf16_ss(tO, a, bd, kIdescO, ks > 0 ? 1u : 0u);
            }
            mma_commit(&S.bar_mma);
            mma_unwaited = true;
        }
        if (!mbar_wait(&S.bar_mma, mma_phase, st, 12)) S.abort_flag = 1;
        mma_phase ^= 1;
        if (tid == 0) mma_unwaited = false;
        tc_fence_after();

        // ---- epilogue: normalised partial O as fp16 with a power-of-two row exponent
        //      (e = 0 unless max|O_B / l| > 2^14), plus lse_B = m + log l
        {
            float o[128];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(tO + lane_off + c * 32, o + c * 32);
            tmem_wait_ld();
            if (my_t >= 0) {
                const float inv_l = 1.f / l;
                float mx = 0.f;
#pragma unroll
                for (int c = 0; c < 128; ++c) mx = fmaxf(mx, fabsf(o[c]));
                mx *= inv_l;
                const int e = mx > 16384.f ? ilogbf(mx) - 14 : 0;
                const float sc = ldexpf(inv_l, -e);
                const size_t prow = ((size_t)my_t * p.hq + my_h) * p.topk + my_j;
                uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__half*>(p.part_o) +
                                                      prow * kHeadDim);
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
                p.part_meta[prow] = make_float2((m + __log2f(l)) * kLn2, (float)e);
            }
        }
        tc_fence_before();
        __syncthreads();
    }

    // ---- teardown: drain what is still in flight (bounded), free TMEM
    if (tid == 0 && S.abort_flag) {
        if (kv_unwaited) mbar_wait(&S.bar_kv, kv_phase, st, 13);
        if (mma_unwaited) mbar_wait(&S.bar_mma, mma_phase, st, 14);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

}  // namespace

cudaError_t launch_fwd_tiles(const FwdPlan& p, const CUtensorMap* kmap, const CUtensorMap* vmap,
                             cudaStream_t stream) {
    // Two CTAs per SM (256 TMEM columns each) for bs = 64, one for bs = 128.
    if (p.bs == 64) {
        constexpr size_t smem = fwd_smem_bytes<64>();
        cudaFuncSetAttribute(k_fwd_tiles<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
        k_fwd_tiles<64><<<2 * p.num_sms, kFwdThreads, smem, stream>>>(p, *kmap, *vmap);
    } else {
        constexpr size_t smem = fwd_smem_bytes<128>();
        cudaFuncSetAttribute(k_fwd_tiles<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
        k_fwd_tiles<128><<<p.num_sms, kFwdThreads, smem, stream>>>(p, *kmap, *vmap);
    }
    return cudaGetLastError();
}

}  // namespace nsa
