// merge.cu -- the memory-bound passes around the tensor-core kernels.
//
//  k_merge         forward: per (token, query head) the log-sum-exp merge of the
//                  per-block partials, O = sum_j e^{lse_j - LSE} o_j and
//                  LSE = log sum_j e^{lse_j}; one warp per row, no atomics (the
//                  reduction / online-softmax kernels of the key-features table on
//                  the "Relaxed-System-Lab/Flash-Sparse-Attention" project page).
//  k_bwd_delta     backward preprocess D = rowsum(dO * O) (fp32, [hq, T]).
//  k_dq_merge      backward: dQ = sum over the row's slots of the dQ partials.
//  k_dkdv_reduce   backward: dK, dV of every key = sum over the backward work
//                  units of its (KV head, block), in unit order (deterministic).
#include <math_constants.h>

#include "nsa_common.cuh"
#include "nsa_kernels.h"

namespace nsa {
namespace {

constexpr int kWarpsPerBlock = 8;

__device__ __forceinline__ float warp_max(float x) {
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xFFFFFFFFu, x, o));
    return x;
}
__device__ __forceinline__ float warp_sum(float x) {
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xFFFFFFFFu, x, o);
    return x;
}

// The 2 NH fp16 values of a partial or output row (d = 64 NH) that one lane owns: lane
// l holds columns [2 NH l, 2 NH l + 2 NH), loaded and stored as one vector.
template <int NH> struct LaneVecT;
template <> struct LaneVecT<1> { using type = uint32_t; };
template <> struct LaneVecT<2> { using type = uint2; };
template <> struct LaneVecT<4> { using type = uint4; };

template <typename V> __device__ __forceinline__ uint32_t vget(const V& v, int q);
template <> __device__ __forceinline__ uint32_t vget<uint32_t>(const uint32_t& v, int) { return v; }
template <> __device__ __forceinline__ uint32_t vget<uint2>(const uint2& v, int q) { return q ? v.y : v.x; }
template <> __device__ __forceinline__ uint32_t vget<uint4>(const uint4& v, int q) {
    return q == 0 ? v.x : q == 1 ? v.y : q == 2 ? v.z : v.w;
}
template <typename V> __device__ __forceinline__ V vzero();
template <> __device__ __forceinline__ uint32_t vzero<uint32_t>() { return 0u; }
template <> __device__ __forceinline__ uint2 vzero<uint2>() { return make_uint2(0u, 0u); }
template <> __device__ __forceinline__ uint4 vzero<uint4>() { return make_uint4(0u, 0u, 0u, 0u); }

// One warp per (token, query head) row.  Lane j (and j + 32) owns slot j: a slot whose
// block is valid has its partial at row posmap * G + head offset of the forward tiles.
// The block numbers and positions come in one round of requests, then the valid slots'
// (lse_j, factor_j) and partial rows (2 NH columns per lane) in a second: the row
// costs two dependent memory latencies (d = 256 with topk > 16: further rounds of 16
// partial rows, so that the loads in flight fit the registers).
template <int kS, int NH, int F16>   // slots held by the warp: 16, 32 or 64 (>= topk)
__global__ void __launch_bounds__(kWarpsPerBlock * 32, kS == 16 ? (NH == 4 ? 2 : 5) : 1)
    k_merge(const MergePlan p) {
    using V = typename LaneVecT<NH>::type;
    constexpr bool kTopk32 = kS <= 32;
    constexpr int kChunk = (NH == 4 && kS > 16) ? 16 : kS;   // partial rows in flight per round
    const int lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
    if (row >= (long long)p.T * p.hq) return;
    // after a recorded device error (malformed cu_seqlens, an expired wait) the
    // position map and partials are incomplete: leave the outputs untouched
    if (*reinterpret_cast<const volatile int*>(&p.st->code) != 0) return;
    const int t = (int)(row / p.hq);
    const int h = (int)(row - (long long)t * p.hq);
    const int g = h / p.G;
    const int hoff = h - g * p.G;
    const unsigned nrows_part = (unsigned)p.st->ntiles_fwd * (unsigned)kTileRows;
    const int s = seq_of_token(p.cu, p.nseq, t);
    const int i = t - __ldg(p.cu + s);
    const int qb = i / p.bs;
    const size_t base = ((size_t)t * p.hkv + g) * p.topk;
    // level 1: block number and position of slots lane, lane + 32, loaded together (the
    // position is read whether or not the slot is valid: it is always in bounds)
    auto slot_row = [&](int b, int pos) -> unsigned {
        if (!block_valid(b, qb, i, p.bs, p.swin)) return 0xFFFFFFFFu;
        const unsigned r = (unsigned)pos * (unsigned)p.G + (unsigned)hoff;
        return r < nrows_part ? r : 0xFFFFFFFFu;
    };
    int b0 = -1, b1 = -1, pos0 = 0, pos1 = 0;
    if (lane < p.topk) {
        b0 = __ldg(p.bidx + base + lane);
        pos0 = __ldg(p.posmap + base + lane);
    }
    if (!kTopk32 && lane + 32 < p.topk) {
        b1 = __ldg(p.bidx + base + lane + 32);
        pos1 = __ldg(p.posmap + base + lane + 32);
    }
    const unsigned r0 = slot_row(b0, pos0);
    const unsigned r1 = kTopk32 ? 0xFFFFFFFFu : slot_row(b1, pos1);
    // level 2: the (lse, factor) of this lane's slots and every valid partial row
    float2 m0 = make_float2(-CUDART_INF_F, 0.f), m1 = m0;
    if (r0 != 0xFFFFFFFFu) m0 = __ldg(p.part_meta + r0);
    if (r1 != 0xFFFFFFFFu) m1 = __ldg(p.part_meta + r1);
    const V* po = reinterpret_cast<const V*>(p.part_o) + lane;
    const int nslot = min(p.topk, kS);
    V u[kChunk];
#pragma unroll
    for (int j = 0; j < kChunk; ++j) {
        const unsigned rj = __shfl_sync(0xFFFFFFFFu, j < 32 ? r0 : r1, j & 31);
        u[j] = (j < nslot && rj != 0xFFFFFFFFu) ? __ldg(po + (size_t)rj * 32) : vzero<V>();
    }
    const float M = warp_max(fmaxf(m0.x, m1.x));
    V* outp = reinterpret_cast<V*>(p.out) + (size_t)row * 32 + lane;
    if (M == -CUDART_INF_F) {          // nothing selected: O = 0, LSE = -inf
        *outp = vzero<V>();
        if (lane == 0 && p.lse) p.lse[(size_t)h * p.T + t] = -CUDART_INF_F;
        return;
    }
    const float w0 = m0.x == -CUDART_INF_F ? 0.f : __expf(m0.x - M);
    const float w1 = m1.x == -CUDART_INF_F ? 0.f : __expf(m1.x - M);
    const float Lam = warp_sum(w0 + w1);
    const float s0 = w0 * m0.y, s1 = w1 * m1.y;   // weight x the partial's factor
    float acc[2 * NH];
#pragma unroll
    for (int q = 0; q < 2 * NH; ++q) acc[q] = 0.f;
    auto add = [&](const V& v, int j) {
        const float wj = __shfl_sync(0xFFFFFFFFu, j < 32 ? s0 : s1, j & 31);
#pragma unroll
        for (int q = 0; q < NH; ++q) {
            const float2 a = unpack_f16x2(vget<V>(v, q));
            acc[2 * q] = fmaf(wj, a.x, acc[2 * q]);
            acc[2 * q + 1] = fmaf(wj, a.y, acc[2 * q + 1]);
        }
    };
#pragma unroll
    for (int j = 0; j < kChunk; ++j) add(u[j], j);
#pragma unroll
    for (int j0 = kChunk; j0 < kS; j0 += kChunk) {    // d = 256, topk > 16: further rounds
#pragma unroll
        for (int j = 0; j < kChunk; ++j) {
            const unsigned rj = __shfl_sync(0xFFFFFFFFu, j0 + j < 32 ? r0 : r1, (j0 + j) & 31);
            u[j] = (j0 + j < nslot && rj != 0xFFFFFFFFu) ? __ldg(po + (size_t)rj * 32) : vzero<V>();
        }
#pragma unroll
        for (int j = 0; j < kChunk; ++j) add(u[j], j0 + j);
    }
    const float inv = 1.f / Lam;
    uint32_t w[NH];
#pragma unroll
    for (int q = 0; q < NH; ++q) w[q] = pack2<F16>(acc[2 * q] * inv, acc[2 * q + 1] * inv);
    if constexpr (NH == 1) *outp = w[0];
    else if constexpr (NH == 2) *outp = make_uint2(w[0], w[1]);
    else *outp = make_uint4(w[0], w[1], w[2], w[3]);
    if (lane == 0 && p.lse) p.lse[(size_t)h * p.T + t] = M + __logf(Lam);
}

// Eight rows per warp, half a warp per row and 16-byte loads: four rows' loads of O and
// dO are in flight per lane before the first reduction (d = 64: the row's 8 chunks on
// lanes 0-7 of the half warp).
constexpr int kDeltaRowsPerWarp = 8;
template <int F16>
__global__ void __launch_bounds__(kWarpsPerBlock * 32) k_bwd_delta(const void* out, const void* dout,
                                                                  float* delta, int T, int hq,
                                                                  int d) {
    const int lane = threadIdx.x & 31, half = lane >> 4, c = lane & 15;
    const long long nrows = (long long)T * hq;
    const long long row0 =
        ((long long)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5)) * kDeltaRowsPerWarp;
    const int cpr = d >> 3;   // 16-byte chunks per row
    uint4 o[kDeltaRowsPerWarp / 2], dv[kDeltaRowsPerWarp / 2];
#pragma unroll
    for (int it = 0; it < kDeltaRowsPerWarp / 2; ++it) {
        const long long row = row0 + 2 * it + half;
        o[it] = dv[it] = make_uint4(0u, 0u, 0u, 0u);
        if (row < nrows && c < cpr) {
            o[it] = __ldg(reinterpret_cast<const uint4*>(out) + row * cpr + c);
            dv[it] = __ldg(reinterpret_cast<const uint4*>(dout) + row * cpr + c);
        }
    }
#pragma unroll
    for (int it = 0; it < kDeltaRowsPerWarp / 2; ++it) {
        const uint32_t ow[4] = {o[it].x, o[it].y, o[it].z, o[it].w};
        const uint32_t dw[4] = {dv[it].x, dv[it].y, dv[it].z, dv[it].w};
        float x = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float2 a = unpack2<F16>(ow[q]), b = unpack2<F16>(dw[q]);
            x = fmaf(a.x, b.x, x);
            x = fmaf(a.y, b.y, x);
        }
        for (int off = 8; off > 0; off >>= 1) x += __shfl_xor_sync(0xFFFFFFFFu, x, off);
        const long long row = row0 + 2 * it + half;
        if (c == 0 && row < nrows) {
            const int t = (int)(row / hq), h = (int)(row - (long long)t * hq);
            delta[(size_t)h * T + t] = x;
        }
    }
}

template <int F16>   // dQ partials are bf16 either way; F16: fp16 output
__global__ void __launch_bounds__(kWarpsPerBlock * 32) k_dq_merge(const BwdPlan p, const int32_t* bidx,
                                                                 void* dq) {
    const int lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
    if (row >= (long long)p.T * p.hq) return;
    if (*reinterpret_cast<const volatile int*>(&p.st->code) != 0) return;
    const int t = (int)(row / p.hq);
    const int h = (int)(row - (long long)t * p.hq);
    const int g = h / p.G;
    const int s = seq_of_token(p.cu, p.nseq, t);
    const int i = t - __ldg(p.cu + s);
    const int qb = i / p.bs;
    const int32_t* bi = bidx + ((size_t)t * p.hkv + g) * p.topk;
    const uint2* pd = reinterpret_cast<const uint2*>(reinterpret_cast<const __nv_bfloat16*>(p.part_dq) +
                                                     (size_t)row * p.topk * kHeadDim) + lane;
    const int b0 = lane < p.topk ? __ldg(bi + lane) : -1;
    const int b1 = lane + 32 < p.topk ? __ldg(bi + lane + 32) : -1;
    const unsigned v0 = __ballot_sync(0xFFFFFFFFu, block_valid(b0, qb, i, p.bs, p.swin));
    const unsigned v1 = __ballot_sync(0xFFFFFFFFu, block_valid(b1, qb, i, p.bs, p.swin));
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < p.topk; ++j) {
        const bool ok = j < 32 ? ((v0 >> j) & 1u) : ((v1 >> (j - 32)) & 1u);
        if (!ok) continue;
        const uint2 u = __ldg(pd + (size_t)j * (kHeadDim / 4));
        const float2 a = unpack_bf16x2(u.x), b = unpack_bf16x2(u.y);
        acc[0] += a.x;
        acc[1] += a.y;
        acc[2] += b.x;
        acc[3] += b.y;
    }
    // d = 64: the partials' columns 64..127 are zero and not stored
    if (lane * 4 < p.d) {
        uint2* o = reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(dq) + (size_t)row * p.d) + lane;
        *o = make_uint2(pack2<F16>(acc[0], acc[1]), pack2<F16>(acc[2], acc[3]));
    }
}

// One warp per (key token, KV head); each lane owns 4 of the 128 columns.
template <int F16>
__global__ void __launch_bounds__(kWarpsPerBlock * 32) k_dkdv_reduce(const BwdPlan p, void* dk, void* dv) {
    const int lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
    if (row >= (long long)p.T * p.hkv) return;
    // after a recorded device error the unit lists may not belong to this call
    if (*reinterpret_cast<const volatile int*>(&p.st->code) != 0) return;
    const int t = (int)(row / p.hkv);
    const int g = (int)(row - (long long)t * p.hkv);
    const int s = seq_of_token(p.cu, p.nseq, t);
    const int i = t - __ldg(p.cu + s);
    const int b = i / p.bs;
    const int r = i - b * p.bs;
    const int nbtot = __ldg(p.blkoff + p.nseq);
    const int bucket = g * nbtot + __ldg(p.blkoff + s) + b;
    const int c0 = __ldg(p.chunk_off + bucket), c1 = __ldg(p.chunk_off + bucket + 1);
    float4 av = make_float4(0.f, 0.f, 0.f, 0.f), ak = av;
    for (int c = c0; c < c1; ++c) {
        const float* base = p.part_dkdv + ((size_t)c * 2 * p.bs + r) * kHeadDim;
        const float4 x = __ldg(reinterpret_cast<const float4*>(base) + lane);
        const float4 y = __ldg(reinterpret_cast<const float4*>(base + (size_t)p.bs * kHeadDim) + lane);
        av.x += x.x; av.y += x.y; av.z += x.z; av.w += x.w;
        ak.x += y.x; ak.y += y.y; ak.z += y.z; ak.w += y.w;
    }
    if (lane * 4 >= p.d) return;   // d = 64: the partials' columns 64..127 are zero
    uint2* ov = reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(dv) + (size_t)row * p.d) + lane;
    uint2* ok = reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(dk) + (size_t)row * p.d) + lane;
    *ov = make_uint2(pack2<F16>(av.x, av.y), pack2<F16>(av.z, av.w));
    *ok = make_uint2(pack2<F16>(ak.x, ak.y), pack2<F16>(ak.z, ak.w));
}

inline unsigned blocks_for(long long rows) {
    return (unsigned)((rows + kWarpsPerBlock - 1) / kWarpsPerBlock);
}

}  // namespace

template <int NH, int F16>
static void launch_merge_nh(const MergePlan& p, unsigned nb, cudaStream_t stream) {
    const unsigned nt = kWarpsPerBlock * 32;
    if (p.topk <= 16) k_merge<16, NH, F16><<<nb, nt, 0, stream>>>(p);
    else if (p.topk <= 32) k_merge<32, NH, F16><<<nb, nt, 0, stream>>>(p);
    else k_merge<64, NH, F16><<<nb, nt, 0, stream>>>(p);
}

cudaError_t launch_merge(const MergePlan& p, cudaStream_t stream) {
    const unsigned nb = blocks_for((long long)p.T * p.hq);
    switch (p.d) {
        case 64: if (p.f16) launch_merge_nh<1, 1>(p, nb, stream); else launch_merge_nh<1, 0>(p, nb, stream); break;
        case 128: if (p.f16) launch_merge_nh<2, 1>(p, nb, stream); else launch_merge_nh<2, 0>(p, nb, stream); break;
        case 256: if (p.f16) launch_merge_nh<4, 1>(p, nb, stream); else launch_merge_nh<4, 0>(p, nb, stream); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_bwd_preprocess(const void* out, const void* dout, float* delta, int T, int hq,
                                  int d, int f16, cudaStream_t stream) {
    const long long rows = (long long)T * hq;
    const long long per_block = (long long)kWarpsPerBlock * kDeltaRowsPerWarp;
    const unsigned nb = (unsigned)((rows + per_block - 1) / per_block);
    if (rows > 0) {
        if (f16) k_bwd_delta<1><<<nb, kWarpsPerBlock * 32, 0, stream>>>(out, dout, delta, T, hq, d);
        else k_bwd_delta<0><<<nb, kWarpsPerBlock * 32, 0, stream>>>(out, dout, delta, T, hq, d);
    }
    return cudaGetLastError();
}

cudaError_t launch_bwd_dq_merge(const BwdPlan& p, const int32_t* bidx, void* dq, cudaStream_t stream) {
    const unsigned nb = blocks_for((long long)p.T * p.hq);
    if (p.f16) k_dq_merge<1><<<nb, kWarpsPerBlock * 32, 0, stream>>>(p, bidx, dq);
    else k_dq_merge<0><<<nb, kWarpsPerBlock * 32, 0, stream>>>(p, bidx, dq);
    return cudaGetLastError();
}

cudaError_t launch_bwd_dkdv_reduce(const BwdPlan& p, void* dk, void* dv, cudaStream_t stream) {
    const unsigned nb = blocks_for((long long)p.T * p.hkv);
    if (p.f16) k_dkdv_reduce<1><<<nb, kWarpsPerBlock * 32, 0, stream>>>(p, dk, dv);
    else k_dkdv_reduce<0><<<nb, kWarpsPerBlock * 32, 0, stream>>>(p, dk, dv);
    return cudaGetLastError();
}

}  // namespace nsa
