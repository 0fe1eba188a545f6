// fwd.cu -- forward tile kernel of selected-block attention (KV-block major).
//
// A tile is (KV head g, KV block B, up to 128 gathered query rows), a row being
// (token, query head) for a token whose index row selected B; the G query heads of a
// token are adjacent rows, so a group of any size fills the 128-row tensor-core tile
// (the loop swap of the FSA pages: "FSA: Efficient Implementation of Native Sparse
// Attention" blog, second paragraph).  Per tile:
//
//   S   = Q K_B^T                  tcgen05.mma (Q, K from shared memory) -> TMEM
//   P   = exp2(c S - c m), causal mask on the diagonal block, l = sum P, written
//         as bf16 back into the S columns of TMEM
//   O_B = P V_B                    tcgen05.mma with A = P read from TMEM
//   partial: O_B / l as fp16 with a power-of-two row exponent, lse_B = m + log l.
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
//   warps 0-1   Q loaders: coalesced cp.async gather (two 256-byte rows per warp
//               instruction) into the 128B-swizzled Q tile, kNQ stages
//   warp 2      TMA producer: K_B and V_B (128B swizzle) into NKV stages
//   warp 3      MMA issuer (one thread): S(i+1) is issued before PV(i)
//   warps 4-7   softmax + epilogue of even tiles   } TMEM slots 0 / 1: S (P) and
//   warps 8-11  softmax + epilogue of odd tiles    } O accumulators each
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
constexpr int kNQ = 2;         // Q stages
constexpr int kChunk = 2;      // consecutive tiles per scheduling chunk

template <int BS, int NKV>
struct alignas(1024) FwdSmem {
    uint8_t q[kNQ][2][kTileRows * 128];       // Q tile per stage: [64-column half][row]
    uint8_t kv[NKV][2][2][BS * 128];          // [stage][K, V][64-column half][key]
    uint8_t stage[8][32 * 128];               // epilogue staging, 4 KB per softmax warp
    uint64_t q_full[kNQ], q_empty[kNQ];
    uint64_t kv_full[NKV], kv_empty[NKV];
    uint64_t s_full[2], p_full[2], o_full[2], o_free[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
    int ntiles;
};

template <int BS, int NKV>
constexpr size_t fwd_smem_bytes() {
    return sizeof(FwdSmem<BS, NKV>) + 1024;
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
    // TMEM columns of slot s: S (and P, bf16, in its first BS/2 columns) at
    // s * kSlot, the O accumulator at s * kSlot + BS.
    constexpr int kSlot = BS + kHeadDim;
    static_assert(2 * kSlot <= 512, "TMEM budget");

    if (tid == 0) {
        S.abort_flag = (*reinterpret_cast<volatile int*>(&st->code) != 0);
        S.ntiles = *reinterpret_cast<volatile int*>(&st->ntiles_fwd);
        for (int i = 0; i < kNQ; ++i) {
            mbar_init(&S.q_full[i], kLoaderThreads);
            mbar_init(&S.q_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.s_full[i], 1);
            mbar_init(&S.p_full[i], kSoftmaxThreads);
            mbar_init(&S.o_full[i], 1);
            mbar_init(&S.o_free[i], kSoftmaxThreads);
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

    if (warp < 2) {
        // ---------------------------------------------------------------- Q loaders
        // Warp w fills tile rows [64w, 64w + 64).  Lane l computes the source address of
        // rows 64w + l and 64w + 32 + l (token from the index entry, head from the row);
        // in copy step k the warp moves rows 64w + 2k and 64w + 2k + 1, lane l taking the
        // 16-byte chunk l % 16 of row 64w + 2k + l / 16 (a 512-byte coalesced read).
        // The copies of tile i are published one tile later (wait for the older
        // cp.async group, fence for the tensor core's async proxy, arrive on q_full),
        // so two tiles' gathers are in flight.  A warp leaves the loop together: every
        // wait is followed by a warp vote.
        const int w = warp;
        const uint8_t* qb = static_cast<const uint8_t*>(p.q);
        const int rA = 64 * w + lane, rB = rA + 32;
        auto ld_ent = [&](const int4& d, int r) -> uint32_t {
            return r < (d.z & 255) ? __ldg(p.entries + d.y + r / p.G) : 0u;
        };
        auto row_addr = [&](const int4& d, int r, uint32_t ent) -> unsigned long long {
            const int g = d.z >> 8;
            return reinterpret_cast<unsigned long long>(
                qb + ((size_t)(ent >> 6) * p.hq + g * p.G + r % p.G) * (kHeadDim * 2));
        };
        int4 d0 = ld_desc(0), d1 = ld_desc(1);
        uint32_t ea = ld_ent(d0, rA), eb = ld_ent(d0, rB);
        int published = 0, issued = 0;
        for (int i = 0; i < n; ++i) {
            const int4 d = d0;
            const unsigned long long addrA = row_addr(d, rA, ea), addrB = row_addr(d, rB, eb);
            d0 = d1;
            d1 = ld_desc(i + 2);
            ea = ld_ent(d0, rA);           // next tile's entries, used one iteration later
            eb = ld_ent(d0, rB);
            const int nrows = d.z & 255;
            const int stg = i % kNQ;
            const bool ok = wait(&S.q_empty[stg], ((i / kNQ) & 1) ^ 1, 30);
            if (!__all_sync(0xffffffffu, ok)) break;
            const uint32_t q0 = smem_u32(S.q[stg][0]);
            const int c = lane & 15;
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                const int rw = 2 * k + (lane >> 4);          // row within the warp's 64
                const unsigned long long a =
                    __shfl_sync(0xffffffffu, k < 16 ? addrA : addrB, rw & 31);
                const int row = 64 * w + rw;
                if (row < nrows)
                    cp_async_16(q0 + (c >> 3) * (kTileRows * 128) + sw128_offset(row, c & 7),
                                reinterpret_cast<const void*>(a + c * 16));
            }
            cp_async_commit();
            issued = i + 1;
            if (i > 0) {
                cp_async_wait_one_pending();
                fence_async_smem();
                mbar_arrive(&S.q_full[(i - 1) % kNQ]);
                published = i;
            }
        }
        cp_async_wait_all();   // nothing may still be in flight when the CTA exits
        if (issued == n && published == n - 1 && n > 0) {
            fence_async_smem();
            mbar_arrive(&S.q_full[(n - 1) % kNQ]);
        }
    } else if (warp == 2) {
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
                const int stg = uses % NKV;
                if (!wait(&S.kv_empty[stg], ((uses / NKV) & 1) ^ 1, 32)) break;
                const int g = d.z >> 8;
                mbar_arrive_expect_tx(&S.kv_full[stg], 4u * BS * 128u);
                tma_load_3d(S.kv[stg][0][0], &kmap, &S.kv_full[stg], 0, g, d.x);
                tma_load_3d(S.kv[stg][0][1], &kmap, &S.kv_full[stg], 64, g, d.x);
                tma_load_3d(S.kv[stg][1][0], &vmap, &S.kv_full[stg], 0, g, d.x);
                tma_load_3d(S.kv[stg][1][1], &vmap, &S.kv_full[stg], 64, g, d.x);
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
            // S(i) = Q K^T into slot i & 1.  The slot's previous S / P (tile i - 2) was
            // last read by PV(i - 2), which was issued earlier: tcgen05.mma of one thread
            // run in issue order.
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
                tc_fence_after();
                const uint32_t tS = tmem + slot * kSlot;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t off = (uint32_t)(ks & 3) * 32u;
                    const uint64_t a = smem_desc_sw128(smem_u32(S.q[stg][ks >> 2]) + off, 16, 1024);
                    const uint64_t b =
                        smem_desc_sw128(smem_u32(S.kv[cur][0][ks >> 2]) + off, 16, 1024);
                    mma_bf16_ss(tS, a, b, kIdescS, ks > 0 ? 1u : 0u);
                }
                mma_commit(&S.s_full[slot]);
                mma_commit(&S.q_empty[stg]);
                return true;
            };
            // O(i) = P(i) V into slot i & 1 once the softmax wrote P(i) and the epilogue
            // of tile i - 2 has read the slot's previous O.
            auto issue_pv = [&](int i, bool release_kv) -> bool {
                const int slot = i & 1;
                if (!wait(&S.p_full[slot], (i >> 1) & 1, 36)) return false;
                if (!wait(&S.o_free[slot], ((i >> 1) & 1) ^ 1, 34)) return false;
                tc_fence_after();
                const uint32_t tS = tmem + slot * kSlot, tO = tS + BS;
                const int kvs = kvs_of[slot];
#pragma unroll
                for (int ks = 0; ks < BS / 16; ++ks) {
                    const uint64_t b = smem_desc_sw128(
                        smem_u32(S.kv[kvs][1][0]) + (uint32_t)ks * 2048u, BS * 128, 1024);
                    mma_bf16_ts(tO, tS + (uint32_t)ks * 8u, b, kIdescO, ks > 0 ? 1u : 0u);
                }
                mma_commit(&S.o_full[slot]);
                if (release_kv) mma_commit(&S.kv_empty[kvs]);
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
            mma_commit(&S.drain);
            mbar_wait(&S.drain, 0, st, 41);
        }
    } else {
        // ---------------------------------------------------- softmax + epilogue
        const int wg = (warp - 4) >> 2;                  // 0: even tiles, 1: odd tiles
        const int quad = warp & 3;                       // TMEM lanes 32*quad ..
        const int r = quad * 32 + lane;                  // tile row = TMEM lane
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const uint32_t tS = tmem + wg * kSlot + lane_off;
        const uint32_t tO = tS + BS;
        const uint32_t stg_base = smem_u32(S.stage[warp - 4]);
        const float c = p.scale_log2;
        const float kLn2 = 0.69314718055994531f;
        uint8_t* const part_o = static_cast<uint8_t*>(p.part_o);
        int4 dn = ld_desc(wg);
        uint32_t en = (wg < n && r < (dn.z & 255)) ? __ldg(p.entries + dn.y + r / p.G) : 0u;
        for (int i = wg; i < n; i += 2) {
            const int4 d = dn;
            const uint32_t ent = en;
            dn = ld_desc(i + 2);
            en = (i + 2 < n && r < (dn.z & 255)) ? __ldg(p.entries + dn.y + r / p.G) : 0u;
            const uint32_t ph = (i >> 1) & 1;
            const int nrows = d.z & 255;
            const bool valid = r < nrows;
            // keys 0 .. lim of the block are visible to this row (causal on the diagonal)
            const int lim = valid ? (int)(ent >> 6) - d.x : -1;
            if (!__all_sync(0xffffffffu, wait(&S.s_full[wg], ph, 38))) break;
            tc_fence_after();
            float sv[BS];
#pragma unroll
            for (int c32 = 0; c32 < BS / 32; ++c32) tmem_ld32(tS + c32 * 32, sv + c32 * 32);
            tmem_wait_ld();
            float mx = -CUDART_INF_F;
#pragma unroll
            for (int k = 0; k < BS; ++k) mx = fmaxf(mx, k <= lim ? sv[k] : -CUDART_INF_F);
            if (lim < 0) mx = 0.f;
            const float mc = mx * c;
            // P = 2^(c s - c m) as bf16 over the S columns, l = sum of P (fp32)
            float l = 0.f;
#pragma unroll
            for (int c64 = 0; c64 < BS / 64; ++c64) {
                uint32_t pk[32];
#pragma unroll
                for (int k2 = 0; k2 < 32; ++k2) {
                    const int k = c64 * 64 + 2 * k2;
                    const float x0 = k <= lim ? ex2_approx(fmaf(sv[k], c, -mc)) : 0.f;
                    const float x1 = k + 1 <= lim ? ex2_approx(fmaf(sv[k + 1], c, -mc)) : 0.f;
                    l += x0 + x1;
                    pk[k2] = pack_bf16x2(x0, x1);
                }
                tmem_st32(tS + c64 * 32, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&S.p_full[wg]);
            if (!__all_sync(0xffffffffu, wait(&S.o_full[wg], ph, 39))) break;
            tc_fence_after();
            // epilogue pass 1: the row's max |O| picks the exponent e (0 unless
            // max |O_B / l| > 2^14), so that O_B / l * 2^-e fits fp16
            float om = 0.f;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float x[64];
                tmem_ld32(tO + h * 64, x);
                tmem_ld32(tO + h * 64 + 32, x + 32);
                tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 64; ++k) om = fmaxf(om, fabsf(x[k]));
            }
            const float inv_l = valid ? 1.f / l : 0.f;
            const float omax = om * inv_l;
            const int e = omax > 16384.f ? ilogbf(omax) - 14 : 0;
            const float sc = ldexpf(inv_l, -e);
            const size_t row0 = (size_t)d.y * p.G + (size_t)quad * 32;   // warp's first partial row
            // pass 2, per 64-column half: scale, fp16, stage (16-byte pieces XOR-swizzled
            // by row), then write 4 rows x 128 contiguous bytes per warp instruction
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float x[64];
                tmem_ld32(tO + h * 64, x);
                tmem_ld32(tO + h * 64 + 32, x + 32);
                tmem_wait_ld();
                if (h == 1) {                 // the slot's O has been read: release it
                    tc_fence_before();
                    mbar_arrive(&S.o_free[wg]);
                }
#pragma unroll
                for (int pc = 0; pc < 8; ++pc) {
                    const float* y = x + pc * 8;
                    uint4 v;
                    v.x = pack_f16x2(y[0] * sc, y[1] * sc);
                    v.y = pack_f16x2(y[2] * sc, y[3] * sc);
                    v.z = pack_f16x2(y[4] * sc, y[5] * sc);
                    v.w = pack_f16x2(y[6] * sc, y[7] * sc);
                    st_shared_v4(stg_base + lane * 128 + ((pc ^ (lane & 7)) << 4), v);
                }
                __syncwarp();
#pragma unroll
                for (int it = 0; it < 8; ++it) {
                    const int rr = it * 4 + (lane >> 3), pc = lane & 7;
                    const uint4 v = ld_shared_v4(stg_base + rr * 128 + ((pc ^ (rr & 7)) << 4));
                    if (quad * 32 + rr < nrows)
                        *reinterpret_cast<uint4*>(part_o + (row0 + rr) * (kHeadDim * 2) + h * 128 +
                                                  pc * 16) = v;
                }
                __syncwarp();
            }
            if (valid)
                p.part_meta[row0 + lane] = make_float2((mc + __log2f(l)) * kLn2, (float)e);
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
        constexpr size_t smem = fwd_smem_bytes<64, 3>();
        cudaFuncSetAttribute(k_fwd_tiles<64, 3>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
        k_fwd_tiles<64, 3><<<p.num_sms, kThreads, smem, stream>>>(p, *kmap, *vmap);
    } else {
        constexpr size_t smem = fwd_smem_bytes<128, 1>();
        cudaFuncSetAttribute(k_fwd_tiles<128, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
        k_fwd_tiles<128, 1><<<p.num_sms, kThreads, smem, stream>>>(p, *kmap, *vmap);
    }
    return cudaGetLastError();
}

}  // namespace nsa
