// select.cu -- kernels of the block-selection step that produces block_idx.
//
// The step ahead of the selected attention in NSA: keys and values are compressed
// per sequence (block c covers tokens [c * stride, c * stride + kernel_size); the
// quick start of the "Relaxed-System-Lab/Flash-Sparse-Attention" project page sets
// kernel_size 32, kernel_stride 16), the compressed attention scores every selection
// block, and each (token, KV head) row keeps its initial and local blocks plus the
// best scored others (init_blocks 1, local_blocks 2, topk 16 there).  The pages print
// no formula; the compressed key and value are the means of the covered rows, and the
// top-k orders by score with ties to the lower block.
//
//   k_cmp_offsets   cu_cmp[s] = compressed blocks of the sequences before s
//   k_compress_kv   one warp per (compressed block, KV head): mean of kernel_size rows
//                   of K and of V (lane = four columns, 256-byte coalesced rows)
//   k_select_topk   one warp per (token, KV head): forced blocks, then repeated warp
//                   arg-max over the remaining causal blocks' scores held in registers
#include <math_constants.h>

#include "nsa_common.cuh"
#include "nsa_kernels.h"

namespace nsa {
namespace {

constexpr int kSelWarps = 8;   // warps per block of the per-row kernels

// Single block: exclusive prefix sum of the per-sequence compressed block counts.
__global__ void __launch_bounds__(1024) k_cmp_offsets(const int32_t* cu, int nseq, int ksize,
                                                      int stride, int32_t* cu_cmp) {
    __shared__ int warp_tot[32];
    __shared__ int carry_s;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    if (threadIdx.x == 0) carry_s = 0;
    __syncthreads();
    for (int base = 0; base < nseq; base += blockDim.x) {
        const int s = base + threadIdx.x;
        int n = 0;
        if (s < nseq) {
            const int L = __ldg(cu + s + 1) - __ldg(cu + s);
            n = L < ksize ? 0 : (L - ksize) / stride + 1;
        }
        int x = n;                                   // inclusive scan within the warp
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) warp_tot[w] = x;
        __syncthreads();
        if (w == 0) {
            int t = lane < (int)(blockDim.x >> 5) ? warp_tot[lane] : 0;
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, t, o);
                if (lane >= o) t += y;
            }
            warp_tot[lane] = t;                      // inclusive over warps
        }
        __syncthreads();
        const int carry = carry_s;
        const int before = carry + (w > 0 ? warp_tot[w - 1] : 0) + x - n;
        if (s < nseq) cu_cmp[s] = before;
        __syncthreads();
        if (threadIdx.x == blockDim.x - 1) carry_s = carry + warp_tot[(blockDim.x >> 5) - 1];
        __syncthreads();
    }
    if (threadIdx.x == 0) cu_cmp[nseq] = carry_s;
}

template <int F16>
__global__ void __launch_bounds__(kSelWarps * 32) k_compress_kv(const void* k, const void* v,
                                                               const int32_t* cu, int nseq,
                                                               int hkv, int ksize, int stride,
                                                               long long npairs,
                                                               const int32_t* cu_cmp, void* kc,
                                                               void* vc) {
    const int lane = threadIdx.x & 31;
    const long long w = (long long)blockIdx.x * kSelWarps + (threadIdx.x >> 5);
    if (w >= npairs) return;
    const int c = (int)(w / hkv), g = (int)(w - (long long)c * hkv);
    if (c >= __ldg(cu_cmp + nseq)) return;          // past the last compressed block
    const int s = upper_index(cu_cmp, nseq, c);
    const int t0 = __ldg(cu + s) + (c - __ldg(cu_cmp + s)) * stride;
    const uint2* kp = reinterpret_cast<const uint2*>(k) + ((size_t)t0 * hkv + g) * (kHeadDim / 4) + lane;
    const uint2* vp = reinterpret_cast<const uint2*>(v) + ((size_t)t0 * hkv + g) * (kHeadDim / 4) + lane;
    const size_t row = (size_t)hkv * (kHeadDim / 4);
    float ak[4] = {0.f, 0.f, 0.f, 0.f}, av[4] = {0.f, 0.f, 0.f, 0.f};
    for (int r = 0; r < ksize; ++r) {
        const uint2 a = __ldg(kp + r * row), b = __ldg(vp + r * row);
        const float2 a0 = unpack2<F16>(a.x), a1 = unpack2<F16>(a.y);
        const float2 b0 = unpack2<F16>(b.x), b1 = unpack2<F16>(b.y);
        ak[0] += a0.x; ak[1] += a0.y; ak[2] += a1.x; ak[3] += a1.y;
        av[0] += b0.x; av[1] += b0.y; av[2] += b1.x; av[3] += b1.y;
    }
    const float inv = 1.f / (float)ksize;
    uint2* ko = reinterpret_cast<uint2*>(kc) + ((size_t)c * hkv + g) * (kHeadDim / 4) + lane;
    uint2* vo = reinterpret_cast<uint2*>(vc) + ((size_t)c * hkv + g) * (kHeadDim / 4) + lane;
    *ko = make_uint2(pack2<F16>(ak[0] * inv, ak[1] * inv), pack2<F16>(ak[2] * inv, ak[3] * inv));
    *vo = make_uint2(pack2<F16>(av[0] * inv, av[1] * inv), pack2<F16>(av[2] * inv, av[3] * inv));
}

// (score, block) order of the top-k: higher score first, the lower block on ties
__device__ __forceinline__ bool better(float a, int ia, float b, int ib) {
    return a > b || (a == b && ia < ib);
}

// J = candidate blocks per lane (nb_stride <= 32 J)
template <int J>
__global__ void __launch_bounds__(kSelWarps * 32) k_select_topk(const float* scores,
                                                               const int32_t* cu, int nseq, int T,
                                                               int hkv, int nb_stride, int bs,
                                                               int topk, int init_blocks,
                                                               int local_blocks, int32_t* bidx,
                                                               DevStatus* st) {
    const int lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * kSelWarps + (threadIdx.x >> 5);
    if (row >= (long long)T * hkv) return;
    const int t = (int)(row / hkv);
    const int s = seq_of_token(cu, nseq, t);
    const int i = t - __ldg(cu + s);
    const int qb = i / bs;
    int32_t* out = bidx + (size_t)row * topk;
    if (qb >= nb_stride) {                          // the score rows are too short
        for (int j = lane; j < topk; j += 32) out[j] = -1;
        if (lane == 0) record_error(st, NSA_ERR_INVALID_ARG, 90, t);
        return;
    }
    // forced blocks: 0 .. init_blocks - 1, then qb, qb - 1, .. (local_blocks of them),
    // within [0, qb], each once, at most topk
    auto forced_at = [&](int n) -> int {           // n-th forced block, or -1
        int m = 0;
        for (int b = 0; b < init_blocks && b <= qb; ++b)
            if (m++ == n) return b;
        for (int b = qb; b > qb - local_blocks && b >= 0; --b) {
            if (b < init_blocks) continue;          // already among the initial blocks
            if (m++ == n) return b;
        }
        return -1;
    };
    int nforced = 0;
    while (nforced < topk && forced_at(nforced) >= 0) ++nforced;
    auto is_forced = [&](int b) {
        return b < init_blocks || (b > qb - local_blocks && b <= qb);
    };
    // lane l holds blocks l, l + 32, ...; excluded ones (forced, future) are -inf
    const float* sr = scores + (size_t)row * nb_stride;
    float v[J];
#pragma unroll
    for (int j = 0; j < J; ++j) {
        const int b = lane + 32 * j;
        v[j] = (b <= qb && !is_forced(b)) ? __ldg(sr + b) : -CUDART_INF_F;
    }
    // this lane's best remaining candidate
    auto local_best = [&](float& bv, int& bb) {
        bv = -CUDART_INF_F;
        bb = 0x7fffffff;
#pragma unroll
        for (int j = 0; j < J; ++j) {
            const int b = lane + 32 * j;
            if (v[j] != -CUDART_INF_F && better(v[j], b, bv, bb)) { bv = v[j]; bb = b; }
        }
    };
    float bv;
    int bb;
    local_best(bv, bb);
    const int nrest = min(topk - nforced, (qb + 1) - nforced);
    // forced slots and padding here; the chosen slots only by lane 0 below (no slot is
    // stored by two lanes)
    for (int j = lane; j < topk; j += 32) {
        if (j < nforced) out[j] = forced_at(j);
        else if (j >= nforced + nrest) out[j] = -1;
    }
    for (int n = 0; n < nrest; ++n) {
        float wv = bv;
        int wb = bb;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, wv, o);
            const int ob = __shfl_xor_sync(0xffffffffu, wb, o);
            if (better(ov, ob, wv, wb)) { wv = ov; wb = ob; }
        }
        if (lane == 0) out[nforced + n] = wb;
        if ((wb & 31) == lane) {                    // the winner drops it and rescans
#pragma unroll
            for (int j = 0; j < J; ++j)
                if (lane + 32 * j == wb) v[j] = -CUDART_INF_F;
            local_best(bv, bb);
        }
    }
}

}  // namespace

cudaError_t launch_compress_kv(const void* k, const void* v, const int32_t* cu, int nseq, int T,
                               int hkv, int ksize, int stride, int f16, int32_t* cu_cmp, void* kc,
                               void* vc, cudaStream_t stream) {
    k_cmp_offsets<<<1, 1024, 0, stream>>>(cu, nseq, ksize, stride, cu_cmp);
    const long long npairs = (long long)(T / stride) * hkv;   // bound on (block, head) pairs
    if (npairs > 0) {
        const unsigned grid = (unsigned)((npairs + kSelWarps - 1) / kSelWarps);
        if (f16)
            k_compress_kv<1><<<grid, kSelWarps * 32, 0, stream>>>(k, v, cu, nseq, hkv, ksize, stride,
                                                                  npairs, cu_cmp, kc, vc);
        else
            k_compress_kv<0><<<grid, kSelWarps * 32, 0, stream>>>(k, v, cu, nseq, hkv, ksize, stride,
                                                                  npairs, cu_cmp, kc, vc);
    }
    return cudaGetLastError();
}

cudaError_t launch_select_topk(const float* scores, const int32_t* cu, int nseq, int T, int hkv,
                               int nb_stride, int bs, int topk, int init_blocks, int local_blocks,
                               int32_t* bidx, DevStatus* st, cudaStream_t stream) {
    const long long rows = (long long)T * hkv;
    if (rows == 0) return cudaGetLastError();
    const unsigned grid = (unsigned)((rows + kSelWarps - 1) / kSelWarps);
#define NSA_TOPK_LAUNCH(J)                                                                     \
    k_select_topk<J><<<grid, kSelWarps * 32, 0, stream>>>(scores, cu, nseq, T, hkv, nb_stride, \
                                                          bs, topk, init_blocks, local_blocks,  \
                                                          bidx, st)
    if (nb_stride <= 32) NSA_TOPK_LAUNCH(1);
    else if (nb_stride <= 128) NSA_TOPK_LAUNCH(4);
    else if (nb_stride <= 512) NSA_TOPK_LAUNCH(16);
    else NSA_TOPK_LAUNCH(32);
#undef NSA_TOPK_LAUNCH
    return cudaGetLastError();
}

}  // namespace nsa
