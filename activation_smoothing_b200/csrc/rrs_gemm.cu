// rrs_gemm.cu -- group-scaled W4A4 GEMM of Rotated Runtime Smooth on the
// sm_100a tensor cores.
//
//   P_g[t][n] = sum_{k in group g} qX[t][k] * qW[n][k]          (exact int32)
//   Y[t][n]   = (sum_g s_g * P_g[t][n]) * scale_t[t] * scale_w[n]
//
// The smoothing scale s_g is shared by every element of group g, so it cannot
// be folded into the integer operands; it is applied group-wise to exact
// integer partial sums, which is the hardware-aligned scheme the rebuttal page
// describes ("Novelty": reorder, then a group-wise smoothing scale).
//
// Kernel structure (one CTA per 128 x BN output tile, 13 warps):
//   warps 0-7   epilogue: per group, tcgen05.ld the int32 partial from TMEM,
//               convert exactly, acc += s_g * P_g in fp32 registers; at the
//               end Y = acc * scale_t * scale_w.
//   warps 8-11  producers: load packed INT4 rows of qX / qW, unpack to INT8
//               (sign-correct by placing each nibble in the high half of a
//               byte, i.e. 16 * q), store into the 128-byte-swizzled K-major
//               shared-memory layout the MMA reads.
//   warp 12     TMEM allocation and, on one thread, tcgen05.mma.kind::i8
//               (M = 128, N = BN, K = 32 per instruction, 4 per 128-wide K
//               block) into a double-buffered TMEM accumulator, one buffer per
//               group.
// The products are 256 * qX * qW; the partial is shifted right by 8 (exact)
// before the fp32 conversion.
#include <cuda_runtime.h>

#include <cstdint>

#include "rrs_device.cuh"
#include "rrs_internal.h"

namespace rrs {

namespace gemm {

constexpr int BM = 128;
constexpr int BK = 128;                 // K elements per pipeline stage
constexpr int NSTAGE = 4;
constexpr int EPI_WARPS = 8;
constexpr int PROD_WARPS = 4;
constexpr int MMA_WARP = EPI_WARPS + PROD_WARPS;
constexpr int NTHREADS = (MMA_WARP + 1) * 32;
constexpr int MAX_GROUPS = 256;         // K / G with K <= 32768, G >= 128

template <int BN>
struct Smem {
    static constexpr int A_BYTES = BM * BK;         // int8
    static constexpr int B_BYTES = BN * BK;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int BAR_OFF = NSTAGE * STAGE_BYTES;
    static constexpr int TOTAL = BAR_OFF + 1024 + MAX_GROUPS * 4 + 1024;   // + alignment slack
};

struct Args {
    const uint8_t* qX;
    const uint8_t* qW;
    const float* s;
    const float* scale_t;
    const float* scale_w;
    int M, N, K, G;
    float* Y;
    int32_t* P;
    uint32_t* err;
    uint64_t limit_ns;
};

// Byte offset of 16-byte logical chunk `lc` of operand row `row` inside a
// K-major, 128-byte-swizzled tile (8-row atoms of 1024 bytes).
__device__ __forceinline__ uint32_t sw128_off(int row, int lc) {
    return (uint32_t)((row >> 3) * 1024 + (row & 7) * 128 + ((lc ^ (row & 7)) << 4));
}

// 8 packed INT4 codes (reading R9: even k in the low nibble) -> 8 int8 bytes
// holding 16 * q, in k order.
__device__ __forceinline__ void unpack8(uint32_t w, uint32_t& o0, uint32_t& o1) {
    const uint32_t lo = (w << 4) & 0xF0F0F0F0u;   // k = 0, 2, 4, 6 of this word, x16
    const uint32_t hi = w & 0xF0F0F0F0u;          // k = 1, 3, 5, 7, x16
    o0 = __byte_perm(lo, hi, 0x5140);             // k 0..3
    o1 = __byte_perm(lo, hi, 0x7362);             // k 4..7
}

__device__ __forceinline__ void store_unpacked(uint8_t* tile, int row, int pc, uint4 v) {
    uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
    unpack8(v.x, a0, a1);
    unpack8(v.y, a2, a3);
    unpack8(v.z, b0, b1);
    unpack8(v.w, b2, b3);
    *reinterpret_cast<uint4*>(tile + sw128_off(row, 2 * pc)) = make_uint4(a0, a1, a2, a3);
    *reinterpret_cast<uint4*>(tile + sw128_off(row, 2 * pc + 1)) = make_uint4(b0, b1, b2, b3);
}

template <int BN, bool DEBUG_P>
__global__ void __launch_bounds__(NTHREADS, 1) gemm_kernel(Args g) {
    using S = Smem<BN>;
    extern __shared__ __align__(1024) unsigned char smem_dyn[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::BAR_OFF);
    uint64_t* empty = full + NSTAGE;
    uint64_t* tfull = empty + NSTAGE;
    uint64_t* tempty = tfull + 2;
    uint64_t* done = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
    float* s_sm = reinterpret_cast<float*>(smem + S::BAR_OFF + 1024);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int m0 = blockIdx.y * BM;
    const int n0 = blockIdx.x * BN;
    const int K = g.K;
    const int KB = K / BK;
    const int NG = K / g.G;
    const int kb_per_group = g.G / BK;
    volatile int* abortv = abort_flag;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NSTAGE; ++i) {
            mbar_init(&full[i], PROD_WARPS * 32);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], EPI_WARPS);
        }
        mbar_init(done, 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (!DEBUG_P) {
        for (int i = threadIdx.x; i < NG; i += blockDim.x) s_sm[i] = g.s[i];
    }
    if (warp == MMA_WARP) {
        tmem_alloc(tmem_slot, 2 * BN);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp >= EPI_WARPS && warp < MMA_WARP) {
        // ------------------------------------------------------ producers
        const int p = threadIdx.x - EPI_WARPS * 32;
        const int pc = p & 3;
        const int rsub = p >> 2;
        const size_t ldk = (size_t)(K / 2);
        for (int kb = 0; kb < KB; ++kb) {
            const int slot = kb % NSTAGE;
            const uint32_t ph = (uint32_t)(kb / NSTAGE) & 1u;
            uint4 ra[BM / 32];
            uint4 rb[BN / 32];
#pragma unroll
            for (int i = 0; i < BM / 32; ++i) {
                const int grow = m0 + rsub + 32 * i;
                ra[i] = grow < g.M ? __ldg(reinterpret_cast<const uint4*>(
                                         g.qX + (size_t)grow * ldk + (size_t)kb * 64 + pc * 16))
                                   : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int i = 0; i < BN / 32; ++i) {
                const int grow = n0 + rsub + 32 * i;
                rb[i] = grow < g.N ? __ldg(reinterpret_cast<const uint4*>(
                                         g.qW + (size_t)grow * ldk + (size_t)kb * 64 + pc * 16))
                                   : make_uint4(0, 0, 0, 0);
            }
            if (!mbar_wait_bounded(&empty[slot], ph ^ 1u, abortv, g.err, kErrGemmTimeout, g.limit_ns))
                break;
            uint8_t* at = smem + slot * S::STAGE_BYTES;
            uint8_t* bt = at + S::A_BYTES;
#pragma unroll
            for (int i = 0; i < BM / 32; ++i) store_unpacked(at, rsub + 32 * i, pc, ra[i]);
#pragma unroll
            for (int i = 0; i < BN / 32; ++i) store_unpacked(bt, rsub + 32 * i, pc, rb[i]);
            fence_proxy_async_smem();
            mbar_arrive(&full[slot]);
        }
    } else if (warp == MMA_WARP) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_i8(BM, BN);
            bool ok = true;
            for (int kb = 0; kb < KB && ok; ++kb) {
                const int slot = kb % NSTAGE;
                const uint32_t ph = (uint32_t)(kb / NSTAGE) & 1u;
                const int gi = kb / kb_per_group;
                const bool first = (kb % kb_per_group) == 0;
                const bool last = (kb % kb_per_group) == kb_per_group - 1;
                const int buf = gi & 1;
                if (first) {
                    ok = mbar_wait_bounded(&tempty[buf], (((uint32_t)gi >> 1) & 1u) ^ 1u, abortv,
                                           g.err, kErrGemmTimeout, g.limit_ns);
                    if (!ok) break;
                }
                ok = mbar_wait_bounded(&full[slot], ph, abortv, g.err, kErrGemmTimeout, g.limit_ns);
                if (!ok) break;
                tc_fence_after();
                const uint32_t a_base = smem_u32(smem + slot * S::STAGE_BYTES);
                const uint32_t b_base = a_base + S::A_BYTES;
                const uint32_t d = tmem + (uint32_t)(buf * BN);
#pragma unroll
                for (int k = 0; k < BK / 32; ++k) {
                    umma_i8(d, sdesc_k_sw128(a_base + 32 * k), sdesc_k_sw128(b_base + 32 * k), idesc,
                            (first && k == 0) ? 0u : 1u);
                }
                tc_commit(&empty[slot]);
                if (last) tc_commit(&tfull[buf]);
            }
            // Wait for every issued MMA before TMEM can be released.
            tc_commit(done);
            volatile int dummy_abort = 0;
            mbar_wait_bounded(done, 0, &dummy_abort, g.err, kErrGemmTimeout, g.limit_ns);
        }
    } else {
        // ------------------------------------------------------ epilogue
        const int quarter = warp & 3;
        const int colhalf = warp >> 2;
        const int row = m0 + 32 * quarter + lane;
        const int col0 = n0 + 64 * colhalf;
        float acc[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) acc[i] = 0.0f;
        bool ok = true;
        for (int gi = 0; gi < NG; ++gi) {
            const int buf = gi & 1;
            ok = mbar_wait_bounded(&tfull[buf], ((uint32_t)gi >> 1) & 1u, abortv, g.err,
                                   kErrGemmTimeout, g.limit_ns);
            if (!ok) break;
            tc_fence_after();
            const uint32_t taddr = tmem + ((uint32_t)(32 * quarter) << 16) + (uint32_t)(buf * BN + 64 * colhalf);
            const float sg = DEBUG_P ? 0.0f : s_sm[gi];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t r[32];
                tmem_ld32(taddr + 32 * h, r);
                tmem_ld_wait();
                if (h == 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&tempty[buf]);
                }
                if (DEBUG_P) {
                    if (row < g.M) {
                        int32_t* dst = g.P + ((size_t)gi * g.M + row) * g.N;
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            const int col = col0 + 32 * h + i;
                            if (col < g.N) dst[col] = ((int32_t)r[i]) >> 8;
                        }
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const float pf = (float)(((int32_t)r[i]) >> 8);
                        acc[32 * h + i] = __fmaf_rn(sg, pf, acc[32 * h + i]);
                    }
                }
            }
        }
        if (!DEBUG_P && ok && row < g.M) {
            const float st = g.scale_t[row];
            float* yrow = g.Y + (size_t)row * g.N;
            const bool vec = ((g.N & 3) == 0);
#pragma unroll
            for (int i = 0; i < 64; i += 4) {
                const int col = col0 + i;
                if (vec && col + 3 < g.N) {
                    const float4 sw = __ldg(reinterpret_cast<const float4*>(g.scale_w + col));
                    float4 y;
                    y.x = __fmul_rn(__fmul_rn(acc[i], st), sw.x);
                    y.y = __fmul_rn(__fmul_rn(acc[i + 1], st), sw.y);
                    y.z = __fmul_rn(__fmul_rn(acc[i + 2], st), sw.z);
                    y.w = __fmul_rn(__fmul_rn(acc[i + 3], st), sw.w);
                    *reinterpret_cast<float4*>(yrow + col) = y;
                } else {
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        if (col + u < g.N)
                            yrow[col + u] = __fmul_rn(__fmul_rn(acc[i + u], st), g.scale_w[col + u]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem, 2 * BN);
    }
}

__global__ void wait_probe_kernel(uint64_t limit_ns, uint32_t* err) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        mbar_fence_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        volatile int* ab = &abort_flag;
        // Phase 0 of a fresh barrier never completes: nothing arrives on it.
        mbar_wait_bounded(&bar, 0, ab, err, kErrProbeTimeout, limit_ns);
    }
}

}  // namespace gemm

cudaError_t launch_gemm(const GemmLaunch& gl, cudaStream_t stream) {
    constexpr int BN = 128;
    using S = gemm::Smem<BN>;
    gemm::Args a;
    a.qX = gl.qX;
    a.qW = gl.qW;
    a.s = gl.s;
    a.scale_t = gl.scale_t;
    a.scale_w = gl.scale_w;
    a.M = gl.M;
    a.N = gl.N;
    a.K = gl.K;
    a.G = gl.G;
    a.Y = gl.Y;
    a.P = gl.P;
    a.err = gl.err;
    a.limit_ns = kWaitLimitNs;
    dim3 grid((gl.N + BN - 1) / BN, (gl.M + gemm::BM - 1) / gemm::BM);
    const int smem = S::TOTAL;
    if (gl.P) {
        auto kern = gemm::gemm_kernel<BN, true>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        kern<<<grid, gemm::NTHREADS, smem, stream>>>(a);
    } else {
        auto kern = gemm::gemm_kernel<BN, false>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        kern<<<grid, gemm::NTHREADS, smem, stream>>>(a);
    }
    return cudaGetLastError();
}

cudaError_t launch_wait_probe(uint64_t limit_ns, uint32_t* err, cudaStream_t stream) {
    gemm::wait_probe_kernel<<<1, 32, 0, stream>>>(limit_ns, err);
    return cudaGetLastError();
}

}  // namespace rrs
