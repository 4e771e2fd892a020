// rrs_device.cuh -- sm_100a device helpers shared by the RRS kernels:
// bounded mbarrier waits, tcgen05 (TMEM / UMMA) wrappers, shared-memory
// descriptors and the workspace error word.  Inline PTX written for this
// library from the PTX ISA's descriptions of these instructions.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>

namespace rrs {

// ---------------------------------------------------------------- errors ---
// Error word layout in the caller's workspace (uint32 at offset 0):
// bit 0: a GEMM wait gave up; bit 1: a prep wait gave up; bit 2: the
// fault-injection kernel gave up (expected); bits 8..15: role code of the first
// thread that gave up.
enum : uint32_t {
    kErrGemmTimeout = 1u,
    kErrPrepTimeout = 2u,
    kErrProbeTimeout = 4u,
};

// Default wait limit for every spin in the kernels: one second.
constexpr uint64_t kWaitLimitNs = 1000ull * 1000ull * 1000ull;

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier ---
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Tests phase completion; if the phase is still open the warp is suspended
// (issuing nothing) until it completes or about `hint_ns` pass, so waiting
// warps do not steal issue slots from working warps on the same scheduler.
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity, uint32_t hint_ns = 20000u) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Non-blocking test of phase completion.
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait until the phase with the given parity of `bar` has completed.  Gives
// up after `limit_ns`, or as soon as another thread of the CTA has raised
// *abort; on giving up it records `err_bit` in the workspace error word, raises
// *abort and returns false.  SPIN polls without suspending (lowest hand-off
// latency, for the few single-thread and producer roles); otherwise the warp
// sleeps in try_wait between polls.
template <bool SPIN = false>
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  volatile int* abort, uint32_t* err,
                                                  uint32_t err_bit, uint64_t limit_ns) {
    if (SPIN ? mbar_test_wait(bar, parity) : mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (SPIN ? mbar_test_wait(bar, parity) : mbar_try_wait(bar, parity)) return true;
        if ((it & (SPIN ? 1023u : 3u)) == 0) {
            if (*abort) return false;
            if (globaltimer_ns() - t0 > limit_ns) {
                if (err) atomicOr(err, err_bit);
                *abort = 1;
                return false;
            }
        }
    }
}

// ------------------------------------------------------------------ proxies ---
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------ tcgen05 ---
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(dst_smem)), "r"(ncols) : "memory");
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
// Make `bar` track completion of every tcgen05 operation this thread issued so far.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_u32(bar)) : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, int8 x int8 -> int32, one CTA.
__device__ __forceinline__ void umma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                        uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}\n"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Instruction descriptor for kind::i8: D s32, A s8, B s8, both K-major,
// M = 128, N = n (multiple of 16, <= 256).
__host__ __device__ constexpr uint32_t idesc_i8(int m, int n) {
    return (2u << 4)                               // D format: s32
           | (1u << 7)                             // A format: s8
           | (1u << 10)                            // B format: s8
           | ((uint32_t)(n >> 3) << 17)            // N / 8
           | ((uint32_t)(m >> 4) << 24);           // M / 16
}

// Shared-memory matrix descriptor for a K-major operand stored as 8-row x
// 128-byte atoms with the 128-byte swizzle (16-byte chunk c of row r at chunk
// c ^ (r & 7)), atoms 1024 bytes apart along M/N.  The atom base must be
// 1024-byte aligned; advancing `saddr` by 32 bytes selects the next K = 32
// slice inside the atom.
__device__ __forceinline__ uint64_t sdesc_k_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);      // start address
    d |= (uint64_t)1 << 16;                        // leading byte offset (unused here): 16 B
    d |= (uint64_t)(1024u >> 4) << 32;             // stride byte offset: 1024 B between 8-row atoms
    d |= (uint64_t)1 << 46;                        // descriptor version for sm_100
    d |= (uint64_t)2 << 61;                        // 128-byte swizzle
    return d;
}

__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ------------------------------------------------------------------ cp.async ---
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)),
                 "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Named barrier over `nthreads` threads (a multiple of 32).
__device__ __forceinline__ void named_bar(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Grid-wide barrier for a cooperative launch: sense reversal on two words
// (arrival count, generation).  The last CTA to arrive resets the count and
// advances the generation; the others wait for the generation to change, at
// most limit_ns, then record a timeout in the error word and report failure.
__device__ __forceinline__ bool grid_barrier(uint32_t* gbar, uint32_t* err, uint64_t limit_ns) {
    __shared__ int ok_s;
    __syncthreads();
    if (threadIdx.x == 0) {
        int ok = 1;
        volatile uint32_t* vgen = gbar + 1;
        const uint32_t gen = *vgen;
        __threadfence();
        const uint32_t old = atomicAdd(gbar, 1u);
        if (old == gridDim.x - 1) {
            atomicExch(gbar, 0u);
            __threadfence();
            atomicAdd(gbar + 1, 1u);
        } else {
            const uint64_t t0 = globaltimer_ns();
            uint32_t it = 0;
            while (*vgen == gen) {
                if ((++it & 63u) == 0 && globaltimer_ns() - t0 > limit_ns) {
                    atomicOr(err, kErrPrepTimeout);
                    ok = 0;
                    break;
                }
                __nanosleep(64);
            }
        }
        __threadfence();
        ok_s = ok;
    }
    __syncthreads();
    return ok_s != 0;
}

// Division a / b for b > 0 by Markstein's method (P. Markstein, "Computation of
// elementary functions on the IBM RISC System/6000 processor", IBM J. Res.
// Dev. 34(1), 1990): with y = RN(1/b) and q0 = RN(a*y), the residual
// r = a - b*q0 is exact (one fma) and RN(q0 + r*y) is the correctly rounded
// quotient RN(a/b), barring underflow/overflow of the intermediates, which the
// value ranges here exclude (|a| <= b, |a| >= 2^-40 or a == 0).  It is checked
// against the IEEE division in the GPU tests.
__device__ __forceinline__ float2 div_markstein(float2 a, float2 nb, float2 y) {
    const float2 q0 = __fmul2_rn(a, y);
    const float2 r = __ffma2_rn(q0, nb, a);
    return __ffma2_rn(r, y, q0);
}
__device__ __forceinline__ float div_markstein(float a, float nb, float y) {
    const float q0 = __fmul_rn(a, y);
    const float r = __fmaf_rn(q0, nb, a);
    return __fmaf_rn(r, y, q0);
}

// Programmatic dependent launch: the dependent kernel waits here until the
// kernel before it in the stream has completed and its memory operations are
// visible (a no-op when it was not launched as a dependent); the primary kernel
// lets its dependents start launching early.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dependents_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// The gated-MLP activation of one output: silu(g) * u with silu(g) = g / (1 +
// exp(-g)) in fp32, saturated to +-65504 (the fp16 range the next layer's
// activation path takes); the caller rounds it to fp16.  One definition for the
// element-wise step and the GEMM epilogue that fuses it, so both give the same bits.
__device__ __forceinline__ float silu_mul(float g, float u) {
    const float sg = __fdiv_rn(g, __fadd_rn(1.0f, expf(-g)));
    const float h = __fmul_rn(sg, u);
    return fminf(fmaxf(h, -65504.0f), 65504.0f);
}

}  // namespace rrs
