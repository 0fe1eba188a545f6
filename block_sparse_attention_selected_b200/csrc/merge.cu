// merge.cu -- the memory-bound passes around the backward's tensor-core kernel (the
// forward's merge is folded into dense.cu).
//
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

// Eight rows per warp, half a warp per row and 16-byte loads: four rows' loads of O and
// dO are in flight per lane before the first reduction.
constexpr int kDeltaRowsPerWarp = 8;
template <int F16>
__global__ void __launch_bounds__(kWarpsPerBlock * 32) k_bwd_delta(const void* out, const void* dout,
                                                                  float* delta, int T, int hq) {
    const int lane = threadIdx.x & 31, half = lane >> 4, c = lane & 15;
    const long long nrows = (long long)T * hq;
    const long long row0 =
        ((long long)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5)) * kDeltaRowsPerWarp;
    uint4 o[kDeltaRowsPerWarp / 2], d[kDeltaRowsPerWarp / 2];
#pragma unroll
    for (int it = 0; it < kDeltaRowsPerWarp / 2; ++it) {
        const long long row = row0 + 2 * it + half;
        o[it] = d[it] = make_uint4(0u, 0u, 0u, 0u);
        if (row < nrows) {
            o[it] = __ldg(reinterpret_cast<const uint4*>(out) + row * (kHeadDim / 8) + c);
            d[it] = __ldg(reinterpret_cast<const uint4*>(dout) + row * (kHeadDim / 8) + c);
        }
    }
#pragma unroll
    for (int it = 0; it < kDeltaRowsPerWarp / 2; ++it) {
        const uint32_t ow[4] = {o[it].x, o[it].y, o[it].z, o[it].w};
        const uint32_t dw[4] = {d[it].x, d[it].y, d[it].z, d[it].w};
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
    uint2* o = reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(dq) + (size_t)row * kHeadDim) + lane;
    *o = make_uint2(pack2<F16>(acc[0], acc[1]), pack2<F16>(acc[2], acc[3]));
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
    uint2* ov = reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(dv) + (size_t)row * kHeadDim) + lane;
    uint2* ok = reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(dk) + (size_t)row * kHeadDim) + lane;
    *ov = make_uint2(pack2<F16>(av.x, av.y), pack2<F16>(av.z, av.w));
    *ok = make_uint2(pack2<F16>(ak.x, ak.y), pack2<F16>(ak.z, ak.w));
}

inline unsigned blocks_for(long long rows) {
    return (unsigned)((rows + kWarpsPerBlock - 1) / kWarpsPerBlock);
}

}  // namespace

cudaError_t launch_bwd_preprocess(const void* out, const void* dout, float* delta, int T, int hq,
                                  int f16, cudaStream_t stream) {
    const long long rows = (long long)T * hq;
    const long long per_block = (long long)kWarpsPerBlock * kDeltaRowsPerWarp;
    const unsigned nb = (unsigned)((rows + per_block - 1) / per_block);
    if (rows > 0) {
        if (f16) k_bwd_delta<1><<<nb, kWarpsPerBlock * 32, 0, stream>>>(out, dout, delta, T, hq);
        else k_bwd_delta<0><<<nb, kWarpsPerBlock * 32, 0, stream>>>(out, dout, delta, T, hq);
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
