// rrs_gemm.cu -- group-scaled W4A4 GEMM of Rotated Runtime Smooth on the
// sm_100a tensor cores.
//
//   P_g[t][n] = sum_{k in group g} qX[t][k] * qW[n][k]          (exact int32)
//   Y[t][n]   = (sum_g s_g * P_g[t][n]) * scale_t[t] * scale_w[n]
//
// The smoothing scale s_g is shared by all elements of group g and is a
// runtime float, so it cannot be folded into the integer operands; it is
// applied group-wise to exact integer partial sums -- the hardware-aligned
// scheme the rebuttal page describes ("Novelty": reorder, then a group-wise
// smoothing scale).
//
// Persistent kernel, one CTA per SM, 128 x 192 output tiles, 16 warps:
//   warp 0       TMA, one thread driving two independent streams: packed INT4
//                weight tiles (192 rows x 64 bytes) and int8 activation tiles
//                (128 rows x 128 k, 128-byte swizzle) per k-block
//   warp 1       tcgen05.mma.kind::i8 (M=128, N=192, K=32, 4 per k-block) into
//                a double-buffered TMEM accumulator, one buffer per group
//   warps 2-3    TMEM allocation (warp 2, 512 columns), then unpack the weight
//                tile to int8 (16 * q, sign-correct without extension) in the
//                128-byte-swizzled K-major layout
//   warps 4-15   epilogue, 64 accumulator columns per thread: per group, read
//                the int32 partial from TMEM, convert it exactly,
//                acc += s_g * P_g (fp32, packed f32x2); per tile,
//                Y = acc * scale_t * scale_w
//
// Exact promotion: the weight operand holds 16 q, so a group's int32 sum is
// 16 * P_g with |16 P_g| <= 16 * 64 * 4096 = 2^22 for groups of up to 4096 k;
// its int32 -> fp32 conversion is then exact.
//
// Longer groups are promoted in blocks of up to 4096 k that divide the group
// (promotion_block).  Weights expanded to one code per byte take the fp8
// kernel of rrs_gemm_f8.cu instead.
//
// k order: inside each 32-wide k chunk both operands store the codes in the
// order 0,2,4,6,1,3,5,7, 8,10,... (what a nibble mask produces); the integer
// sum over the chunk does not depend on the order.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "rrs_device.cuh"
#include "rrs_internal.h"

namespace rrs {
namespace gemm {

constexpr int BM = 128;
constexpr int BN = 192;
constexpr int TMEM_BUF = 256;                 // column stride of the two TMEM buffers
constexpr int BK = 128;
constexpr int NS = 4;                         // MMA stages (A int8 + B int8)
constexpr int NP = 5;                         // packed-weight stages
constexpr int A_BYTES = BM * BK;              // 16 KB
constexpr int B8_BYTES = BN * BK;             // 24 KB
constexpr int BP_BYTES = BN * BK / 2;         // 12 KB
constexpr int OFF_A = 0;
constexpr int OFF_B8 = OFF_A + NS * A_BYTES;
constexpr int OFF_BP = OFF_B8 + NS * B8_BYTES;
constexpr int OFF_BAR = OFF_BP + NP * BP_BYTES;
constexpr int OFF_S = OFF_BAR + 1024;
constexpr int MAX_PB = 4096;                  // longest promoted block of k (|16 P| <= 2^22 stays exact)
constexpr int MAX_NPB = 32768 / 128;          // promotion blocks per tile (K <= 32768)
constexpr int SMEM = OFF_S + MAX_NPB * 4 + 1024;
constexpr int NTHREADS = 512;
constexpr int UNPACK_WARPS = 2;
constexpr int EPI_WARPS = 12;

struct Args {
    const float* s;
    const float* scale_t;
    const float* scale_w;
    int M, N, K, G, PB;
    float* Y;
    int32_t* P;          // debug partials [K/G, M, N] or null
    uint32_t* err;
    uint64_t limit_ns;
    int S;               // k splits per tile (1: none); each work item is (tile, split)
    float* part;         // S > 1: [S, M, N] fp32 partial sums (x 1/16), reduced by splitk_reduce_kernel
    bool ybf16;          // Y is bf16 [M, N] (the fp32 result rounded to nearest even)
};

__device__ __forceinline__ uint32_t sw128_off(int row, int lc) {
    return (uint32_t)((row >> 3) * 1024 + (row & 7) * 128 + ((lc ^ (row & 7)) << 4));
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}


// Epilogue warps (4 .. 15): per promotion block, read the int32 partial
// sums of this warp's 32 rows x 64 columns from TMEM, promote them exactly to
// fp32 and accumulate s_g * P_g; at the end of a tile apply scale_t * scale_w
// and store Y (or, in debug mode, store the exact per-group partials).
template <bool DEBUG_P, bool SPLIT, bool YBF16>
__device__ __forceinline__ void epilogue_role(const Args& g, uint32_t tmem, uint64_t* tfull, uint64_t* tempty,
                                              const float* s_sm, volatile int* abortv, int warp, int lane,
                                              int nwork, int nmb, int NPBS) {
    // ------------------------------------------------------------ epilogue
    const int GS = SPLIT ? g.S : 1;               // k splits per tile
    const int quarter = warp & 3;
    const int cgrp = (warp - 4) >> 2;             // 0..2: 64-column slice of the tile
    const uint32_t lane_base = tmem + ((uint32_t)(32 * quarter) << 16);
    const int col0 = 64 * cgrp;
    if (lane == 0) {                      // both accumulator buffers start free
        mbar_arrive(&tempty[0]);
        mbar_arrive(&tempty[1]);
    }
    const float2 sixteenth = make_float2(0.0625f, 0.0625f);
    uint32_t gc = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < nwork && ok; w += gridDim.x) {
        const int tile = w / GS;
        const int sp = w % GS;
        const int pb0 = sp * NPBS;                    // first promotion block of this k split
        const int m0 = (tile % nmb) * BM;
        const int n0 = (tile / nmb) * BN;
        float2 acc[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) acc[i] = make_float2(0.0f, 0.0f);
        const int row = m0 + 32 * quarter + lane;
        for (int pb = pb0; pb < pb0 + NPBS; ++pb, ++gc) {
            const int buf = gc & 1;
            if (!(ok = mbar_wait_bounded(&tfull[buf], (gc >> 1) & 1u, abortv, g.err, kErrGemmTimeout,
                                         g.limit_ns)))
                break;
            tc_fence_after();
            const float sg = DEBUG_P ? 0.0f : s_sm[pb];
            const float2 s2 = make_float2(sg, sg);
#pragma unroll
            for (int c = 0; c < 4; c += 2) {
                uint32_t r[16], r2[16];
                tmem_ld16(lane_base + buf * TMEM_BUF + col0 + 16 * c, r);
                tmem_ld16(lane_base + buf * TMEM_BUF + col0 + 16 * c + 16, r2);
                tmem_ld_wait();
                if (c == 2) {
                    // all of this warp's columns are in registers: release the buffer
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&tempty[buf]);
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const uint32_t* rr = i < 8 ? r : r2;
                    const int ii = i & 7;
                    // |16 P| <= 2^22: the int32 -> fp32 conversion is exact
                    const float2 p16 = make_float2(__int2float_rn((int)rr[2 * ii]), __int2float_rn((int)rr[2 * ii + 1]));
                    if (DEBUG_P) acc[8 * c + i] = __ffma2_rn(p16, sixteenth, acc[8 * c + i]);  // exact ints
                    else acc[8 * c + i] = __ffma2_rn(s2, p16, acc[8 * c + i]);
                }
            }
            if (DEBUG_P && ((pb + 1) * g.PB) % g.G == 0) {
                const int gi = ((pb + 1) * g.PB) / g.G - 1;
                if (row < g.M) {
                    int32_t* dst = g.P + ((size_t)gi * g.M + row) * g.N;
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int col = n0 + col0 + 2 * i;
                        if (col < g.N) dst[col] = (int32_t)acc[i].x;
                        if (col + 1 < g.N) dst[col + 1] = (int32_t)acc[i].y;
                    }
                }
#pragma unroll
                for (int i = 0; i < 32; ++i) acc[i] = make_float2(0.0f, 0.0f);
            }
        }
        if (!DEBUG_P && ok) {
            // lane l holds scale_w of columns col0 + 2l, 2l + 1; broadcast by shuffles
            const int cl = n0 + col0 + 2 * lane;
            const float2 swl = make_float2(cl < g.N ? g.scale_w[cl] : 0.0f, cl + 1 < g.N ? g.scale_w[cl + 1] : 0.0f);
            const float st = row < g.M ? g.scale_t[row] : 0.0f;
            const float2 st2 = make_float2(st, st);
            // one k split of several: its partial sum (x 1/16) goes to the workspace and
            // splitk_reduce_kernel adds the splits in order and applies the scales
            const bool split = SPLIT && GS > 1;
            float* ybase = split ? g.part + (size_t)sp * g.M * g.N : g.Y;
            float* yrow = ybase + (size_t)row * g.N;
            // Each lane owns one row, so a warp's store touches 32 rows.  Whole
            // 32-byte sectors per lane (8 columns, one 256-bit store) keep the
            // L2 from merging partial sectors; ragged edges, N % 8 != 0 and a Y
            // not 32-byte aligned fall back to scalar stores.
            const bool v8 = (g.N & 7) == 0 && (reinterpret_cast<uintptr_t>(ybase) & 31u) == 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                float2 y[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int i = 4 * j + q;
                    const float2 sw = make_float2(__shfl_sync(0xffffffffu, swl.x, i),
                                                  __shfl_sync(0xffffffffu, swl.y, i));
                    y[q] = split ? __fmul2_rn(acc[i], sixteenth)
                                 : __fmul2_rn(__fmul2_rn(__fmul2_rn(acc[i], sixteenth), st2), sw);
                }
                const int col = n0 + col0 + 8 * j;
                if (YBF16 && row < g.M && !split) {
                    // bf16 output: 8 columns = one 16-byte store
                    __nv_bfloat16* brow = reinterpret_cast<__nv_bfloat16*>(g.Y) + (size_t)row * g.N;
                    if ((g.N & 7) == 0 && col + 7 < g.N) {
                        uint32_t u[4];
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const __nv_bfloat162 b = __float22bfloat162_rn(y[q]);
                            u[q] = *reinterpret_cast<const uint32_t*>(&b);
                        }
                        *reinterpret_cast<uint4*>(brow + col) = make_uint4(u[0], u[1], u[2], u[3]);
                    } else {
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            if (col + 2 * q < g.N) brow[col + 2 * q] = __float2bfloat16_rn(y[q].x);
                            if (col + 2 * q + 1 < g.N) brow[col + 2 * q + 1] = __float2bfloat16_rn(y[q].y);
                        }
                    }
                } else if (row < g.M) {
                    if (v8 && col + 7 < g.N) {
                        asm volatile("st.global.v8.f32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
                                     ::"l"(yrow + col), "f"(y[0].x), "f"(y[0].y), "f"(y[1].x), "f"(y[1].y),
                                       "f"(y[2].x), "f"(y[2].y), "f"(y[3].x), "f"(y[3].y)
                                     : "memory");
                    } else {
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            if (col + 2 * q < g.N) yrow[col + 2 * q] = y[q].x;
                            if (col + 2 * q + 1 < g.N) yrow[col + 2 * q + 1] = y[q].y;
                        }
                    }
                }
            }
        }
    }
}

template <bool DEBUG_P, bool SPLIT, bool YBF16>
__global__ void __launch_bounds__(NTHREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, Args g) {
    extern __shared__ __align__(1024) unsigned char smem_dyn[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    uint64_t* afull = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
    uint64_t* bfull = afull + NS;
    uint64_t* mempty = bfull + NS;
    uint64_t* pfull = mempty + NS;
    uint64_t* pempty = pfull + NP;
    uint64_t* tfull = pempty + NP;
    uint64_t* tempty = tfull + 2;
    uint64_t* done = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
    float* s_sm = reinterpret_cast<float*>(smem + OFF_S);
    volatile int* abortv = abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int K = g.K;
    const int KB = K / BK;
    const int NPB = K / g.PB;          // promotion blocks per tile
    const int kb_per_pb = g.PB / BK;
    const int GS = SPLIT ? g.S : 1;    // k splits per tile
    const int KBS = KB / GS;          // k-blocks per work item (the host makes S divide NPB)
    const int nmb = (g.M + BM - 1) / BM;
    const int nnb = (g.N + BN - 1) / BN;
    const int ntiles = nmb * nnb;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NS; ++i) {
            mbar_init(&afull[i], 1);
            mbar_init(&bfull[i], UNPACK_WARPS);
            mbar_init(&mempty[i], 1);
        }
        for (int i = 0; i < NP; ++i) {
            mbar_init(&pfull[i], 1);
            mbar_init(&pempty[i], UNPACK_WARPS);
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
        for (int i = threadIdx.x; i < NPB; i += blockDim.x) s_sm[i] = g.s[(i * g.PB) / g.G];
    }
    if (warp == 2) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp < 4) {
        if (warp == 0 && lane == 0) {
            // -------------------------------------------------------- TMA
            // One thread, two independent streams: packed weight tiles (bounded
            // only by the unpack freeing a slot) and activation tiles (bounded by
            // the MMA freeing a stage).  Neither waits behind the other.
            const int nwork = ntiles * GS;
            const uint32_t my_items = blockIdx.x < (unsigned)nwork ? (nwork - 1 - blockIdx.x) / gridDim.x + 1 : 0;
            const uint32_t total = my_items * KBS;
            uint32_t itB = 0, itA = 0;
            // position of each stream: work item, its tile and first k-block, k-block within it
            int wB = blockIdx.x, wA = blockIdx.x;
            int tileB = wB / GS, tileA = wA / GS;
            int kb0B = (wB % GS) * KBS, kb0A = (wA % GS) * KBS;
            int kkB = 0, kkA = 0;
            uint64_t t0 = 0;
            uint32_t idle = 0;
            bool ok = true;
            while (itB < total || itA < total) {
                bool progress = false;
                if (itB < total && mbar_test_wait(&pempty[itB % NP], ((itB / NP) & 1u) ^ 1u)) {
                    const int ps = itB % NP;
                    arrive_expect_tx(&pfull[ps], BP_BYTES);
                    tma_load_2d(smem + OFF_BP + ps * BP_BYTES, &tmB, (kb0B + kkB) * (BK / 2), (tileB / nmb) * BN,
                                &pfull[ps]);
                    if (++kkB == KBS) {
                        kkB = 0;
                        wB += gridDim.x;
                        tileB = wB / GS;
                        kb0B = (wB % GS) * KBS;
                    }
                    ++itB;
                    progress = true;
                }
                if (itA < total && mbar_test_wait(&mempty[itA % NS], ((itA / NS) & 1u) ^ 1u)) {
                    const int ms = itA % NS;
                    arrive_expect_tx(&afull[ms], A_BYTES);
                    tma_load_2d(smem + OFF_A + ms * A_BYTES, &tmA, (kb0A + kkA) * BK, (tileA % nmb) * BM, &afull[ms]);
                    if (++kkA == KBS) {
                        kkA = 0;
                        wA += gridDim.x;
                        tileA = wA / GS;
                        kb0A = (wA % GS) * KBS;
                    }
                    ++itA;
                    progress = true;
                }
                if (progress) {
                    idle = 0;
                    continue;
                }
                // bounded wait: give up after the limit or when another role gave up
                if (idle++ == 0) t0 = globaltimer_ns();
                if ((idle & 1023u) == 0) {
                    if (*abortv) { ok = false; break; }
                    if (globaltimer_ns() - t0 > g.limit_ns) {
                        atomicOr(g.err, kErrGemmTimeout);
                        *abortv = 1;
                        ok = false;
                        break;
                    }
                }
            }
            if (!ok) {
                // let every copy already issued land before the CTA exits
                volatile int no_abort = 0;
                for (uint32_t j = itB > NP ? itB - NP : 0; j < itB; ++j)
                    mbar_wait_bounded<true>(&pfull[j % NP], (j / NP) & 1u, &no_abort, nullptr, 0, g.limit_ns);
                for (uint32_t j = itA > NS ? itA - NS : 0; j < itA; ++j)
                    mbar_wait_bounded<true>(&afull[j % NS], (j / NS) & 1u, &no_abort, nullptr, 0, g.limit_ns);
            }
        } else if (warp == 1 && lane == 0) {
            // -------------------------------------------------------- MMA
            constexpr uint32_t idesc = idesc_i8(BM, BN);
            uint32_t it = 0, gc = 0;
            bool ok = true;
            for (int w = blockIdx.x; w < ntiles * GS && ok; w += gridDim.x) {
                for (int kb = 0; kb < KBS; ++kb, ++it) {
                    const bool first = (kb % kb_per_pb) == 0;
                    const bool last = (kb % kb_per_pb) == kb_per_pb - 1;
                    const int buf = gc & 1;
                    if (first && !(ok = mbar_wait_bounded<true>(&tempty[buf], (gc >> 1) & 1u, abortv, g.err,
                                                         kErrGemmTimeout, g.limit_ns)))
                        break;
                    const int ms = it % NS;
                    const uint32_t mph = (it / NS) & 1u;
                    if (!(ok = mbar_wait_bounded<true>(&afull[ms], mph, abortv, g.err, kErrGemmTimeout, g.limit_ns))) break;
                    if (!(ok = mbar_wait_bounded<true>(&bfull[ms], mph, abortv, g.err, kErrGemmTimeout, g.limit_ns))) break;
                    tc_fence_after();
                    const uint32_t a_base = smem_u32(smem + OFF_A + ms * A_BYTES);
                    const uint32_t b_base = smem_u32(smem + OFF_B8 + ms * B8_BYTES);
                    const uint32_t d = tmem + (uint32_t)(buf * TMEM_BUF);
#pragma unroll
                    for (int k = 0; k < BK / 32; ++k)
                        umma_i8(d, sdesc_k_sw128(a_base + 32 * k), sdesc_k_sw128(b_base + 32 * k), idesc,
                                (first && k == 0) ? 0u : 1u);
                    tc_commit(&mempty[ms]);
                    if (last) {
                        tc_commit(&tfull[buf]);
                        ++gc;
                    }
                }
            }
            tc_commit(done);
            volatile int no_abort = 0;
            mbar_wait_bounded(done, 0, &no_abort, g.err, kErrGemmTimeout, g.limit_ns);
        } else if (warp >= 2) {
            // -------------------------------------------------------- unpack
            const int p = threadIdx.x - 64;            // 0..63
            const int pc = p & 3;
            const int r0 = p >> 2;                     // 0..15
            uint32_t it = 0;
            bool ok = true;
            for (int w = blockIdx.x; w < ntiles * GS && ok; w += gridDim.x) {
                for (int kb = 0; kb < KBS; ++kb, ++it) {
                    const int ps = it % NP;
                    const uint32_t pph = (it / NP) & 1u;
                    const int ms = it % NS;
                    const uint32_t mph = (it / NS) & 1u;
                    if (!(ok = mbar_wait_bounded<true>(&pfull[ps], pph, abortv, g.err, kErrGemmTimeout, g.limit_ns))) break;
                    if (!(ok = mbar_wait_bounded<true>(&mempty[ms], mph ^ 1u, abortv, g.err, kErrGemmTimeout, g.limit_ns)))
                        break;
                    const unsigned char* src = smem + OFF_BP + ps * BP_BYTES;
                    unsigned char* dst = smem + OFF_B8 + ms * B8_BYTES;
                    // All loads first, then all stores: the compiler cannot move a
                    // shared load above a shared store it cannot prove disjoint.
                    uint4 v[BN / 16];
#pragma unroll
                    for (int j = 0; j < BN / 16; ++j)
                        v[j] = *reinterpret_cast<const uint4*>(src + (r0 + 16 * j) * 64 + pc * 16);
#pragma unroll
                    for (int j = 0; j < BN / 16; ++j) {
                        const int row = r0 + 16 * j;
                        // low nibbles (even k) and high nibbles (odd k), each as 16 * q
                        const uint4 o0 = make_uint4((v[j].x << 4) & 0xF0F0F0F0u, v[j].x & 0xF0F0F0F0u,
                                                    (v[j].y << 4) & 0xF0F0F0F0u, v[j].y & 0xF0F0F0F0u);
                        const uint4 o1 = make_uint4((v[j].z << 4) & 0xF0F0F0F0u, v[j].z & 0xF0F0F0F0u,
                                                    (v[j].w << 4) & 0xF0F0F0F0u, v[j].w & 0xF0F0F0F0u);
                        *reinterpret_cast<uint4*>(dst + sw128_off(row, 2 * pc)) = o0;
                        *reinterpret_cast<uint4*>(dst + sw128_off(row, 2 * pc + 1)) = o1;
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive(&bfull[ms]);
                        mbar_arrive(&pempty[ps]);
                    }
                }
            }
        }
    } else {
        epilogue_role<DEBUG_P, SPLIT, YBF16>(g, tmem, tfull, tempty, s_sm, abortv, warp, lane, ntiles * GS, nmb, NPB / GS);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// Y = (sum over splits of the partial sums, in split order) * scale_t * scale_w.
// The partials already carry the factor 1/16, so the products are applied in
// the order of the unsplit epilogue.
__global__ void splitk_reduce_kernel(const float* part, int S, int M, int N, const float* scale_t,
                                     const float* scale_w, float* Y, bool ybf16) {
    const size_t total = (size_t)M * N;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
        float a = part[i];
        for (int sp = 1; sp < S; ++sp) a = __fadd_rn(a, part[(size_t)sp * total + i]);
        const int m = (int)(i / (size_t)N);
        const int n = (int)(i % (size_t)N);
        const float y = __fmul_rn(__fmul_rn(a, scale_t[m]), scale_w[n]);
        if (ybf16) reinterpret_cast<__nv_bfloat16*>(Y)[i] = __float2bfloat16_rn(y);
        else Y[i] = y;
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

// ------------------------------------------------------------------ host ---

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

static bool make_map_u8(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                        uint32_t box_outer, CUtensorMapSwizzle swz) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {inner};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t es[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace gemm

int promotion_block(int G) {
    int pb = G < gemm::MAX_PB ? G : gemm::MAX_PB;
    pb -= pb % 128;
    while (pb > 128 && G % pb != 0) pb -= 128;
    return pb;
}

cudaError_t launch_gemm(const GemmLaunch& gl, cudaStream_t stream) {
    using namespace gemm;
    CUtensorMap tmA, tmB;
    if (!make_map_u8(&tmA, gl.qX8, (uint64_t)gl.K, (uint64_t)gl.M, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (!make_map_u8(&tmB, gl.qW, (uint64_t)gl.K / 2, (uint64_t)gl.N, BK / 2, BN, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    Args a;
    a.s = gl.s;
    a.scale_t = gl.scale_t;
    a.scale_w = gl.scale_w;
    a.M = gl.M;
    a.N = gl.N;
    a.K = gl.K;
    a.G = gl.G;
    a.PB = promotion_block(gl.G);
    a.Y = gl.Y;
    a.P = gl.P;
    a.err = gl.err;
    a.limit_ns = kWaitLimitNs;
    const int nsm = device_sm_count();
    const int ntiles = ((gl.M + BM - 1) / BM) * ((gl.N + BN - 1) / BN);
    // Few tiles (decode token counts): split k over whole promotion blocks so that
    // every SM streams weights, if the workspace has room for the partial sums.
    int S = 1;
    if (gl.P == nullptr && gl.part != nullptr && gl.M <= kSplitRoomMaxM && ntiles < nsm) {
        const int npb = gl.K / a.PB;
        for (int c = 2; c <= kSplitRoom; ++c)
            if (npb % c == 0 && (long)ntiles * c <= 4L * nsm && (size_t)c * gl.M * gl.N * 4 <= gl.part_bytes) S = c;
    }
    a.S = S;
    a.part = S > 1 ? gl.part : nullptr;
    a.ybf16 = gl.y_bf16;
    const int nwork = ntiles * S;
    const int grid = nwork < nsm ? nwork : nsm;
    cudaError_t e;
    // (with split k the bf16 rounding happens in splitk_reduce_kernel)
    if (gl.P) {
        auto kern = gemm_kernel<true, false, false>;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
        if (e != cudaSuccess) return e;
        kern<<<grid, NTHREADS, SMEM, stream>>>(tmA, tmB, a);
    } else {
        auto kern = S > 1    ? gemm_kernel<false, true, false>
                    : a.ybf16 ? gemm_kernel<false, false, true>
                              : gemm_kernel<false, false, false>;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
        if (e != cudaSuccess) return e;
        kern<<<grid, NTHREADS, SMEM, stream>>>(tmA, tmB, a);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess || S == 1) return e;
    const size_t total = (size_t)gl.M * gl.N;
    size_t blocks = (total + 255) / 256;
    if (blocks > (size_t)nsm * 8) blocks = (size_t)nsm * 8;
    splitk_reduce_kernel<<<(unsigned)blocks, 256, 0, stream>>>(gl.part, S, gl.M, gl.N, gl.scale_t, gl.scale_w, gl.Y,
                                                               gl.y_bf16);
    return cudaGetLastError();
}

cudaError_t launch_wait_probe(uint64_t limit_ns, uint32_t* err, cudaStream_t stream) {
    gemm::wait_probe_kernel<<<1, 32, 0, stream>>>(limit_ns, err);
    return cudaGetLastError();
}

}  // namespace rrs
