// nsa_common.cuh -- device helpers shared by the selected-attention kernels.
//
// Hand-written sm_100a PTX wrappers: mbarriers with bounded waits, TMA tile loads,
// tcgen05 (TMEM allocation, MMA issue/commit, TMEM loads) and the shared-memory
// matrix descriptors of the 5th-generation tensor cores.  Every spin-wait in the
// library goes through mbar_wait(), which gives up after a fixed cycle budget,
// records NSA_ERR_TIMEOUT in the device status word and returns false.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/nsa_sel.h"

namespace nsa {

constexpr int kHeadDim = 128;        // head dimension supported by the kernels
constexpr int kTileRows = 128;       // MMA M: (token, head) rows per tile
constexpr int kMaxTopk = 64;         // entry = token * 64 + slot
constexpr int kMaxGroup = 128;       // query heads per KV head (a divisor of the 128-row tile)

// Device status word layout (int32 slots at the start of the workspace).
struct DevStatus {
    int code;          // first error code recorded (nsa_status_t), 0 = none
    int where;         // kernel-specific location tag of the first error
    int aux0, aux1;    // extra detail (e.g. tile index)
    int nblocks_total; // sum over sequences of ceil(L_s / block_size)
    int ntiles;        // number of 128-row tiles of the last inversion
    int nchunks;       // number of backward work units of the last inversion
    int nentries;      // number of valid (token, KV head, slot) entries
    long long bad_range, bad_dup;   // validation counters
    int ntiles_fwd;    // number of forward tiles in window order
    int pad0;
    unsigned long long index_tag;   // identifies the inputs of the inversion held here
    long long wait_budget;          // cycles a bounded wait may spin (0: kWaitBudgetCycles)
    int pad[46];
};
static_assert(sizeof(DevStatus) == 256, "status block is 256 bytes");

__device__ __forceinline__ void record_error(DevStatus* st, int code, int where, int a0 = 0,
                                             int a1 = 0) {
    if (atomicCAS(&st->code, 0, code) == 0) {
        st->where = where;
        st->aux0 = a0;
        st->aux1 = a1;
    }
}

// Bounds-checking build (compiled with -DNSA_SEL_CHECKS, libnsa_sel_checks.so): every
// gathered row and every K/V block coordinate taken from the index inversion is checked
// before its copy is issued.  A failed check records NSA_ERR_BAD_INDEX (with the
// kernel's location tag) in the status block and the CTA stops early, like an expired
// wait: the copy is not issued and nothing traps.
#ifdef NSA_SEL_CHECKS
constexpr bool kChecks = true;
#else
constexpr bool kChecks = false;
#endif

__device__ __forceinline__ bool check_ok(bool cond, DevStatus* st, int where, int a0 = 0) {
    if (!kChecks || cond) return true;
    record_error(st, NSA_ERR_BAD_INDEX, where, a0, (int)blockIdx.x);
    return false;
}

// ------------------------------------------------------------------ small utilities

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ int seq_of_token(const int32_t* cu, int nseq, int t) {
    int lo = 0, hi = nseq - 1;        // last s with cu[s] <= t
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (__ldg(cu + mid) <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Largest i in [0, n) with a[i] <= x (a ascending, a[0] <= x).
__device__ __forceinline__ int upper_index(const int32_t* a, int n, int x) {
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (a[mid] <= x) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// ---------------------------------------------------------------------- mbarriers

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Non-blocking test of the phase with the given parity (for a thread that polls
// several barriers and serves whichever completes first).
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase with the given parity.  By default about one second of
// SM clock at most (the call's status block may set a shorter budget: the test-only
// NSA_TEST_SHORT_WAITS option); on expiry records NSA_ERR_TIMEOUT and returns false.
constexpr long long kWaitBudgetCycles = 2000000000LL;

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, DevStatus* st,
                                          int where) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long start = clock64();
    const long long set = st->wait_budget;
    const long long budget = set > 0 ? set : kWaitBudgetCycles;
    // a compact loop: this function is inlined at every wait of the warp-specialised
    // kernels, whose code must stay small enough for the instruction caches
#pragma unroll 1
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - start > budget) {
            record_error(st, NSA_ERR_TIMEOUT, where, blockIdx.x);
            return false;
        }
    }
    return true;
}

// ---------------------------------------------------------------------------- TMA

__device__ __forceinline__ void tma_load_3d(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

// Four rows of a 2D tensor map (box: 64 columns x 1 row) at arbitrary row coordinates
// r0..r3, column c0, into four consecutive 128-byte rows of shared memory, with the
// map's swizzle applied from the destination address (so a 4-row group may start at any
// 512-byte offset of a 128B-swizzled tile).  Rows outside the tensor read as zero.
__device__ __forceinline__ void tma_gather4(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int r0, int r1, int r2, int r3) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(r0), "r"(r1),
        "r"(r2), "r"(r3)
        : "memory");
}

// TMA tile store shared -> global (bulk-group completion); x must be a multiple of 16
// bytes, neither coordinate negative.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* smem_src, int c0,
                                             int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(smem_u32(smem_src)), "r"(c0), "r"(c1)
        : "memory");
}
__device__ __forceinline__ void bulk_commit() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until at most N bulk groups of this thread still read their shared-memory source.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Wait until at most N bulk groups of this thread are incomplete (writes performed).
template <int N>
__device__ __forceinline__ void bulk_wait() {
    asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ------------------------------------------------------------------------ cp.async

__device__ __forceinline__ void cp_async_16(uint32_t smem_dst, const void* gsrc) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_dst), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Make generic-proxy shared-memory writes visible to the async proxy (tensor core reads).
__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------------- tcgen05

__device__ __forceinline__ void tmem_alloc(uint32_t* smem_slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(smem_slot)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// tcgen05.mma of kind::f16 (A and B both bf16 or both fp16, as the instruction
// descriptor says; fp32 accumulate in TMEM), issued warp-uniformly: the issuing warp
// runs its whole loop with every lane (so that descriptors and loop state stay
// warp-uniform) and one elected lane executes the tcgen05 instructions.  A single
// issuing lane inside a divergent branch was measured to lose most of its issue slots
// to busy warps on the same SM sub-partition (about 150 instead of 50 cycles per
// M=128, N=64 MMA).  Shared-memory operands come as the low 32 bits of SW128
// descriptors whose stride byte offset is 1024 (start address and LBO); the high word
// (SBO, descriptor version, swizzle mode) is then a constant, which saves a register
// per descriptor in the issuer.
constexpr uint32_t kSw128Sbo1024DescHi = (1024u >> 4) | (1u << 14) | (2u << 29);
__device__ __forceinline__ uint32_t elect_one() {
    uint32_t e;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "elect.sync _|p, 0xffffffff;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(e));
    return e;
}
// D[tmem] (+)= A[smem] * B[smem]^T
__device__ __forceinline__ void mma_ss_e(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo,
                                         uint32_t idesc, uint32_t accumulate, uint32_t elected) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t.reg .b64 da, db;\n\t"
        "setp.ne.b32 e, %5, 0;\n\t"
        "mov.b64 da, {%1, %6};\n\t"
        "mov.b64 db, {%2, %6};\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_lo), "r"(b_lo), "r"(idesc), "r"(accumulate), "r"(elected),
        "r"(kSw128Sbo1024DescHi)
        : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]^T: the A operand (M rows x K, two 16-bit values per
// 32-bit column, row = TMEM lane) is read from tensor memory.
__device__ __forceinline__ void mma_ts_e(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo,
                                         uint32_t idesc, uint32_t accumulate, uint32_t elected) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t.reg .b64 db;\n\t"
        "setp.ne.b32 e, %5, 0;\n\t"
        "mov.b64 db, {%2, %6};\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], db, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "r"(b_lo), "r"(idesc), "r"(accumulate), "r"(elected),
        "r"(kSw128Sbo1024DescHi)
        : "memory");
}
// Arrive on an mbarrier once all tcgen05 ops the elected lane issued before have finished.
__device__ __forceinline__ void mma_commit_e(uint64_t* bar, uint32_t elected) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "setp.ne.b32 e, %1, 0;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
            smem_u32(bar)),
        "r"(elected)
        : "memory");
}

// Store 32 consecutive 32-bit columns of this thread's TMEM lane (32x32b shape) and wait
// for the store: source registers of tcgen05.st may be read asynchronously, so the wait
// is in the same asm statement (the compiler cannot reuse them before it).
__device__ __forceinline__ void tmem_st32_sync(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "{\n\t"
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n\t"
        "tcgen05.wait::st.sync.aligned;\n\t}"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

// 2^x on the special-function unit (the PTX ex2.approx instruction; flushes
// subnormal results to zero, 2^-inf = 0).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Packed pairs of fp32 (Blackwell f32x2 arithmetic: one instruction, two lanes).
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;"
        : "=l"(d)
        : "l"(*reinterpret_cast<uint64_t*>(&a)), "l"(*reinterpret_cast<uint64_t*>(&b)),
          "l"(*reinterpret_cast<uint64_t*>(&c)));
    return *reinterpret_cast<float2*>(&d);
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;"
        : "=l"(d)
        : "l"(*reinterpret_cast<uint64_t*>(&a)), "l"(*reinterpret_cast<uint64_t*>(&b)));
    return *reinterpret_cast<float2*>(&d);
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;"
        : "=l"(d)
        : "l"(*reinterpret_cast<uint64_t*>(&a)), "l"(*reinterpret_cast<uint64_t*>(&b)));
    return *reinterpret_cast<float2*>(&d);
}
// max of three fp32 values in one instruction
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// TMEM loads fused with their wait.  The destination registers of tcgen05.ld are
// written asynchronously and are valid only after tcgen05.wait::ld; with the load and
// the wait in separate asm statements the compiler may copy or spill the registers in
// between (it sees them as defined by the load) and use stale values.  Keeping both in
// one asm statement makes the values defined only after the wait.
__device__ __forceinline__ void tmem_ld32_sync(uint32_t taddr, float* v) {
    uint32_t* r = reinterpret_cast<uint32_t*>(v);
    asm volatile(
        "{\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;\n\t}"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

// 64 consecutive fp32 columns of this thread's TMEM lane, waited for.
__device__ __forceinline__ void tmem_ld64_sync(uint32_t taddr, float* v) {
    uint32_t* r = reinterpret_cast<uint32_t*>(v);
    asm volatile(
        "{\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];\n\t"
        "tcgen05.wait::ld.sync.aligned;\n\t}"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
        : "r"(taddr)
        : "memory");
}

// Shared-memory matrix descriptor (sm_100 format): start address, leading and stride
// byte offsets (16-byte units), version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo_bytes,
                                                    uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;          // descriptor version for sm_100
    d |= (uint64_t)2 << 61;          // SWIZZLE_128B
    return d;
}

// Instruction descriptor for kind::f16 with fp32 D and A, B both bf16 (f16 = false) or
// both fp16 (f16 = true): the two operands of one MMA always have the same type.
__host__ __device__ constexpr uint32_t idesc_f16kind_f32(bool f16, int M, int N, bool a_mn_major,
                                                         bool b_mn_major) {
    return (1u << 4)                      // D format: f32
           | ((f16 ? 0u : 1u) << 7)       // A format: f16 0, bf16 1
           | ((f16 ? 0u : 1u) << 10)      // B format: the same
           | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}


// Byte offset of the 16-byte chunk `c16` (0..7) of row `r` inside a K-major tile whose
// rows are 128 bytes, stored as 8-row x 128-byte atoms with the 128-byte swizzle.
__device__ __forceinline__ uint32_t sw128_offset(int r, int c16) {
    return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((c16 ^ (r & 7)) << 4));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float2 unpack_f16x2(uint32_t u) {
    __half2 v = *reinterpret_cast<__half2*>(&u);
    return __half22float2(v);
}

__device__ __forceinline__ float2 unpack_bf16x2(uint32_t u) {
    __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&u);
    return __bfloat1622float2(v);
}

// The 16-bit element type of the attention tensors: bf16 (F16 = 0) or fp16 (F16 = 1).
template <int F16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    return F16 ? pack_f16x2(lo, hi) : pack_bf16x2(lo, hi);
}
template <int F16>
__device__ __forceinline__ float2 unpack2(uint32_t u) {
    return F16 ? unpack_f16x2(u) : unpack_bf16x2(u);
}

// Entry validity shared by every kernel.  Slot value b of the token at local position
// i (query block qb = i / bs) contributes keys iff 0 <= b <= qb (-1 pads; future and
// out-of-range blocks drop) and, under a sliding window of swin > 0 keys, the block's
// last key (b + 1) bs - 1 lies in the window (i - swin, i]; a valid entry therefore
// always keeps at least one visible key.
__device__ __forceinline__ bool block_valid(int b, int qb, int i, int bs, int swin) {
    return b >= 0 && b <= qb && (swin <= 0 || i - (b + 1) * bs < swin - 1);
}

}  // namespace nsa
