// rrs_gemm_f8.cu -- group-scaled W4A4 GEMM of Rotated Runtime Smooth on the
// sm_100a tensor cores, with both INT4 operands held as fp8 (e4m3) codes.
//
//   P_g[t][n] = sum_{k in group g} qX[t][k] * qW[n][k]          (exact)
//   Y[t][n]   = (sum_g s_g * P_g[t][n]) * scale_t[t] * scale_w[n]
//
// Every INT4 code q in [-8, 7] is an e4m3 number exactly, every product of two
// codes is an integer of magnitude <= 64, and the fp32 accumulator of
// tcgen05.mma.kind::f8f6f4 holds the group sum exactly (|P_g| <= 64 * 4096 =
// 2^18 for promotion blocks of up to 4096 k; checked bit for bit against the
// int8 kind by the debug-partials tests).  The accumulator therefore leaves
// TMEM already as the fp32 value of the exact integer P_g, and the group
// promotion acc += s_g * P_g is one fused multiply-add per element: no
// int32 -> fp32 conversion on the epilogue's critical path.  This is the
// group-wise, hardware-aligned smoothing scale of the rebuttal page
// ("Novelty"), applied to exact partial sums in fp32.
//
// Persistent kernel, one CTA per SM, BM x BN output tiles (BM = 128, BN = 128
// or 256), 11 warps:
//   warps 0-1    TMA producers: stage i is loaded by warp i % 2 (lanes 2i and
//                2i + 1: the activation tile and the weight tile, one barrier)
//   warp 2       TMEM allocation (512 columns) and the MMA thread:
//                tcgen05.mma.kind::f8f6f4 (M=128, N=BN, K=32, 4 per k-block)
//                into 512 / BN rotating TMEM accumulator buffers, one per
//                promotion block
//   warps 3-10   epilogue: warp w reads TMEM lane quarter w % 4 and one half
//                of the tile's columns; per promotion block it loads the
//                fp32 partial sums and accumulates s_g * P_g in registers; per
//                tile it applies scale_t * scale_w and stores Y
//
// Operands: A = activation codes e4m3 [M, K] (the workspace operand written by
// the activation kernels or by the expand kernel), B = weight codes e4m3
// [N, K] (rrs_expand_weights), both in natural k order, loaded by TMA as
// 128-row x 128-byte boxes in the 128-byte swizzled K-major layout that the
// MMA descriptors read.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "rrs_device.cuh"
#include "rrs_internal.h"

namespace rrs {
namespace f8 {

constexpr int BM = 128;
constexpr int BK = 128;
constexpr int A_BYTES = BM * BK;             // 16 KB
constexpr int NTHREADS = 352;                // 11 warps
constexpr int NPROD = 2;                     // producer warps
constexpr int MMA_WARP = 2;
constexpr int EPI_WARP0 = 3;
constexpr int EPI_WARPS = 8;
constexpr int MAX_NPB = 32768 / 128;         // promotion blocks per tile (K <= 32768)

template <int BN>
struct Cfg {
    static constexpr int NBUF = 512 / BN;                 // TMEM accumulator buffers
    static constexpr int B_BYTES = BN * BK;
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int NST = (BN == 256) ? 4 : 6;       // 192 KB of stages either way
    static constexpr int OFF_B = NST * A_BYTES;
    static constexpr int OFF_BAR = OFF_B + NST * B_BYTES;
    static constexpr int OFF_S = OFF_BAR + 1024;
    static constexpr int SMEM = OFF_S + MAX_NPB * 4 + 1024;   // + alignment slack
    static constexpr int CW = BN / 2;                      // columns per epilogue warp
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
    static_assert(OFF_B % 1024 == 0 && B_BYTES % 1024 == 0, "swizzled tiles need 1024-byte alignment");
    static_assert(2 * NST <= 32, "two lanes per stage");
};

struct Args {
    const float* s;
    const float* scale_t;
    const float* scale_w;
    int M, N, K, G, PB;
    void* Y;
    int32_t* P;          // debug partials [K/G, M, N] or null
    uint32_t* err;
    uint64_t limit_ns;
};

// D[tmem] (+)= A[smem] * B[smem]^T, e4m3 x e4m3 -> fp32, one CTA.
__device__ __forceinline__ void umma_f8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Instruction descriptor for kind::f8f6f4: D f32, A e4m3, B e4m3, both K-major.
__host__ __device__ constexpr uint32_t idesc_f8(int m, int n) {
    return (1u << 4)                                 // D format: f32
           | (0u << 7) | (0u << 10)                  // A, B format: e4m3
           | ((uint32_t)(n >> 3) << 17)              // N / 8
           | ((uint32_t)(m >> 4) << 24);             // M / 16
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// Brings a tile into L2 ahead of its load (no shared memory, no completion):
// the weight k-blocks are first touched by several CTAs at once, and without it
// each of them waits out the same DRAM miss inside the load's round trip.
__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap* map, int x, int y) {
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global [%0, {%1, %2}];"
                 ::"l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y) : "memory");
}
__device__ __forceinline__ void tma_prefetch_3d(const CUtensorMap* map, int x, int y, int z) {
    asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global [%0, {%1, %2, %3}];"
                 ::"l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z) : "memory");
}
constexpr int PF_STAGES = 8;   // how many stages ahead the weight tiles are prefetched into L2

__device__ __forceinline__ void arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

// Output of a tile row, YMODE: 0 fp32 Y, 1 bf16 Y (the fp32 value rounded to
// nearest even), 2 the gated-MLP activation H = fp16(silu(y[2f]) * y[2f+1]) of
// an interleaved gate/up projection (H is [M, N/2]; silu_mul as rrs_silu_mul).
enum : int { kYF32 = 0, kYBF16 = 1, kYSiluMul = 2 };

// y[row][colbase + c] = acc_c * scale_t[row] * scale_w[colbase + c] for this
// lane's row and CW columns, stored as YMODE says.  Every lane of the warp runs
// the shuffles; rows past M skip only their stores.  Lane l holds scale_w of two
// columns of each 64-column chunk and shuffles broadcast them.  Each lane owns
// one row: whole 32-byte sectors per lane (one 256-bit store) keep L2 from
// merging partial sectors; ragged edges and misaligned outputs take scalar stores.
template <int CW, int YMODE>
__device__ __forceinline__ void store_tile(const Args& g, const float2 (&acc)[CW / 2], int row, int colbase,
                                           int lane) {
    const bool rv = row < g.M;
    const float st = rv ? g.scale_t[row] : 0.0f;
    const float2 st2 = make_float2(st, st);
    const bool v8 = (g.N & 7) == 0 && (reinterpret_cast<uintptr_t>(g.Y) & 31u) == 0;
#pragma unroll
    for (int ch = 0; ch < CW / 64; ++ch) {
        const int cl = colbase + 64 * ch + 2 * lane;
        const float2 swl = make_float2(cl < g.N ? g.scale_w[cl] : 0.0f, cl + 1 < g.N ? g.scale_w[cl + 1] : 0.0f);
        if (YMODE == kYSiluMul) {
            // 32 columns -> 16 halves = one 32-byte store per lane
            const int NH = g.N / 2;
            const bool hv = (NH & 15) == 0 && (reinterpret_cast<uintptr_t>(g.Y) & 31u) == 0;
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                uint32_t hw[8];
#pragma unroll
                for (int q = 0; q < 16; q += 2) {
                    float hq[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int i = 16 * jj + q + e;
                        const float2 sw = make_float2(__shfl_sync(0xffffffffu, swl.x, i),
                                                      __shfl_sync(0xffffffffu, swl.y, i));
                        const float2 y = __fmul2_rn(__fmul2_rn(acc[32 * ch + i], st2), sw);
                        hq[e] = silu_mul(y.x, y.y);
                    }
                    const __half2 h2 = __floats2half2_rn(hq[0], hq[1]);
                    hw[q / 2] = *reinterpret_cast<const uint32_t*>(&h2);
                }
                const int f0 = (colbase + 64 * ch + 32 * jj) / 2;
                if (!rv) continue;
                __half* hrow = reinterpret_cast<__half*>(g.Y) + (size_t)row * NH;
                if (hv && f0 + 15 < NH) {
                    asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
                                 ::"l"(hrow + f0), "r"(hw[0]), "r"(hw[1]), "r"(hw[2]), "r"(hw[3]),
                                   "r"(hw[4]), "r"(hw[5]), "r"(hw[6]), "r"(hw[7])
                                 : "memory");
                } else {
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const __half2 h2 = *reinterpret_cast<const __half2*>(&hw[q]);
                        if (f0 + 2 * q < NH) hrow[f0 + 2 * q] = __low2half(h2);
                        if (f0 + 2 * q + 1 < NH) hrow[f0 + 2 * q + 1] = __high2half(h2);
                    }
                }
            }
            continue;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            float2 y[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int i = 4 * j + q;
                const float2 sw = make_float2(__shfl_sync(0xffffffffu, swl.x, i), __shfl_sync(0xffffffffu, swl.y, i));
                y[q] = __fmul2_rn(__fmul2_rn(acc[32 * ch + i], st2), sw);
            }
            const int col = colbase + 64 * ch + 8 * j;
            if (!rv) continue;
            if (YMODE == kYBF16) {
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
            } else {
                float* yrow = reinterpret_cast<float*>(g.Y) + (size_t)row * g.N;
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

// Epilogue warps: per promotion block, read this warp's 32 rows x CW columns of
// fp32 partial sums from TMEM and accumulate s_g * P_g; per tile apply
// scale_t * scale_w and store Y (debug: store the exact per-group partials).
template <int BN, bool DEBUG_P, int YMODE>
__device__ __forceinline__ void epilogue(const Args& g, uint32_t tmem, uint64_t* tfull, uint64_t* tempty,
                                         const float* s_sm, volatile int* abortv, int warp, int lane, int ntiles,
                                         int nmb, int NPB) {
    using C = Cfg<BN>;
    constexpr int CW = C::CW;
    const int quarter = warp & 3;
    const int half = (warp - EPI_WARP0) >> 2;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * quarter) << 16);
    const int col0 = CW * half;
    if (lane == 0) {
#pragma unroll
        for (int b = 0; b < C::NBUF; ++b) mbar_arrive(&tempty[b]);   // every buffer starts free
    }
    uint32_t gc = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        const int m0 = (tile % nmb) * BM;
        const int n0 = (tile / nmb) * BN;
        const int row = m0 + 32 * quarter + lane;
        float2 acc[CW / 2];
#pragma unroll
        for (int i = 0; i < CW / 2; ++i) acc[i] = make_float2(0.0f, 0.0f);
        for (int pb = 0; pb < NPB; ++pb, ++gc) {
            const int buf = (int)(gc % C::NBUF);
            if (!(ok = mbar_wait_bounded(&tfull[buf], (gc / C::NBUF) & 1u, abortv, g.err, kErrGemmTimeout,
                                         g.limit_ns)))
                break;
            tc_fence_after();
            const float sg = DEBUG_P ? 1.0f : s_sm[pb];
            const float2 s2 = make_float2(sg, sg);
            const uint32_t src = lane_base + (uint32_t)(buf * BN + col0);
#pragma unroll
            for (int c = 0; c < CW / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(src + 32 * c, r);
                tmem_ld_wait();
                if (c == CW / 32 - 1) {
                    // every column of this warp is in registers: release the buffer
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&tempty[buf]);
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float2 p = make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
                    acc[16 * c + i] = __ffma2_rn(s2, p, acc[16 * c + i]);
                }
            }
            if (DEBUG_P && ((pb + 1) * g.PB) % g.G == 0) {
                const int gi = ((pb + 1) * g.PB) / g.G - 1;
                if (row < g.M) {
                    int32_t* dst = g.P + ((size_t)gi * g.M + row) * g.N;
#pragma unroll
                    for (int i = 0; i < CW / 2; ++i) {
                        const int col = n0 + col0 + 2 * i;
                        if (col < g.N) dst[col] = __float2int_rn(acc[i].x);
                        if (col + 1 < g.N) dst[col + 1] = __float2int_rn(acc[i].y);
                    }
                }
#pragma unroll
                for (int i = 0; i < CW / 2; ++i) acc[i] = make_float2(0.0f, 0.0f);
            }
        }
        if (!DEBUG_P && ok) store_tile<CW, YMODE>(g, acc, row, n0 + col0, lane);
    }
}

template <int BN, bool DEBUG_P, int YMODE>
__global__ void __launch_bounds__(NTHREADS, 1)
    gemm_f8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, Args g) {
    using C = Cfg<BN>;
    extern __shared__ __align__(1024) unsigned char smem_dyn[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* empty = full + C::NST;
    uint64_t* tfull = empty + C::NST;
    uint64_t* tempty = tfull + C::NBUF;
    uint64_t* done = tempty + C::NBUF;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
    float* s_sm = reinterpret_cast<float*>(smem + C::OFF_S);
    volatile int* abortv = abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int KB = g.K / BK;
    const int NPB = g.K / g.PB;
    const int kb_per_pb = g.PB / BK;
    const int nmb = (g.M + BM - 1) / BM;
    const int nnb = (g.N + BN - 1) / BN;
    const int ntiles = nmb * nnb;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::NST; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < C::NBUF; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], EPI_WARPS);
        }
        mbar_init(done, 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == MMA_WARP) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    // launched as a programmatic dependent of the activation kernel: everything
    // above overlapped its end; its outputs (operand, s, scale_t) are read below
    grid_dependency_wait();
    if (!DEBUG_P) {
        for (int i = threadIdx.x; i < NPB; i += blockDim.x) s_sm[i] = g.s[(i * g.PB) / g.G];
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp < NPROD) {
        // -------------------------------------------------------- TMA
        const uint32_t my_tiles = blockIdx.x < (unsigned)ntiles ? (ntiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
        const uint32_t total = my_tiles * KB;
        uint32_t last = 0xFFFFFFFFu;
        bool ok = true;
        for (uint32_t it = warp; it < total; it += NPROD) {
            const int st = (int)(it % C::NST);
            uint32_t free = 1;
            if (lane == 0)
                free = mbar_wait_bounded<true>(&empty[st], ((it / C::NST) & 1u) ^ 1u, abortv, g.err,
                                               kErrGemmTimeout, g.limit_ns) ? 1u : 0u;
            if (!__shfl_sync(0xffffffffu, free, 0)) {
                ok = false;
                break;
            }
            const int tile = blockIdx.x + (int)(it / KB) * gridDim.x;
            const int kb = (int)(it % KB);
            if (lane == 0) arrive_expect_tx(&full[st], C::STAGE);
            __syncwarp();
            // Stage st's two copies are issued by lanes 2st and 2st + 1: the bulk
            // copies of one thread complete one after another, so giving every
            // stage its own threads keeps all stages' copies in flight at once.
            const int la = 2 * st;
            if (lane == la || lane == la + 1) {
                const bool isA = lane == la;
                unsigned char* dst = isA ? smem + st * A_BYTES : smem + C::OFF_B + st * C::B_BYTES;
                const CUtensorMap* map = isA ? &tmA : &tmB;
                const int y = isA ? (tile % nmb) * BM : (tile / nmb) * BN;
                tma_load_2d(dst, map, kb * BK, y, &full[st]);
                const uint32_t ip = it + PF_STAGES;
                if (!isA && ip < total) {
                    const int tp = blockIdx.x + (int)(ip / KB) * gridDim.x;
                    tma_prefetch_2d(&tmB, (int)(ip % KB) * BK, (tp / nmb) * BN);
                }
            }
            __syncwarp();
            last = it;
        }
        if (!ok && lane == 0 && last != 0xFFFFFFFFu) {
            // let this warp's copies land before the CTA exits
            volatile int no_abort = 0;
            mbar_wait_bounded<true>(&full[last % C::NST], (last / C::NST) & 1u, &no_abort, nullptr, 0, g.limit_ns);
        }
    } else if (warp == MMA_WARP) {
        if (lane == 0) {
            // -------------------------------------------------------- MMA
            constexpr uint32_t idesc = idesc_f8(BM, BN);
            uint32_t it = 0, gc = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const bool first = (kb % kb_per_pb) == 0;
                    const bool lastk = (kb % kb_per_pb) == kb_per_pb - 1;
                    const int buf = (int)(gc % C::NBUF);
                    if (first && !(ok = mbar_wait_bounded<true>(&tempty[buf], (gc / C::NBUF) & 1u, abortv, g.err,
                                                                kErrGemmTimeout, g.limit_ns)))
                        break;
                    const int st = (int)(it % C::NST);
                    if (!(ok = mbar_wait_bounded<true>(&full[st], (it / C::NST) & 1u, abortv, g.err, kErrGemmTimeout,
                                                       g.limit_ns)))
                        break;
                    tc_fence_after();
                    const uint32_t a_base = smem_u32(smem + st * A_BYTES);
                    const uint32_t b_base = smem_u32(smem + C::OFF_B + st * C::B_BYTES);
                    const uint32_t d = tmem + (uint32_t)(buf * BN);
#pragma unroll
                    for (int k = 0; k < BK / 32; ++k)
                        umma_f8(d, sdesc_k_sw128(a_base + 32 * k), sdesc_k_sw128(b_base + 32 * k), idesc,
                                (first && k == 0) ? 0u : 1u);
                    tc_commit(&empty[st]);
                    if (lastk) {
                        tc_commit(&tfull[buf]);
                        ++gc;
                    }
                }
            }
            tc_commit(done);
            volatile int no_abort = 0;
            mbar_wait_bounded(done, 0, &no_abort, g.err, kErrGemmTimeout, g.limit_ns);
        }
    } else {
        epilogue<BN, DEBUG_P, YMODE>(g, tmem, tfull, tempty, s_sm, abortv, warp, lane, ntiles, nmb, NPB);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------------
// CTA-pair variant (cta_group::2): a cluster of two CTAs on two SMs computes a
// 256 x 256 tile.  Each CTA loads its own 128 activation rows and its own half
// (128 rows) of the weight tile; one tcgen05.mma.cta_group::2 (M = 256, N = 256,
// K = 32) issued by the even CTA reads the A rows of both CTAs and both halves
// of B, and writes rows 0-127 of the accumulator into the even CTA's TMEM and
// rows 128-255 into the odd CTA's.  Per SM this moves 32 KB per k-block from L2
// for 128 x 256 outputs, against 48 KB for the 128 x 256 single-CTA tile: the
// operand stream from L2, not the tensor pipe, bounds the single-CTA kernel.
//
// Synchronisation (all waits bounded):
//   full[s]   even CTA only: one arrival (its producer, expecting the bytes of
//             both CTAs) + the transaction bytes of all four copies, which
//             both CTAs' producers direct at the even CTA's barrier
//   empty[s]  both CTAs: the MMA thread's commit, multicast to both
//   tfull[b]  both CTAs: the MMA thread's commit, multicast to both
//   tempty[b] even CTA only: 16 arrivals, the epilogue warps of both CTAs
// No load uses cluster multicast; the only multicast is tcgen05.commit's.
namespace pair {
// Tile shape of the pair: 256 rows x PBN columns (PBN = 256, or 128 for narrow N).
template <int PBN>
struct PCfg {
    static constexpr int BN = PBN;                      // tile columns (both CTAs)
    static constexpr int BNH = PBN / 2;                 // weight rows loaded per CTA
    static constexpr int KPS = 2;                       // k-blocks per stage: one 3-D copy per operand carries both
    static constexpr int A_TILE = BM * BK;              // 16 KB: one k-block of activation rows
    static constexpr int B_TILE = BNH * BK;             // one k-block of weight rows
    static constexpr int A_STAGE = KPS * A_TILE;
    static constexpr int B_STAGE = KPS * B_TILE;
    static constexpr int STAGE = A_STAGE + B_STAGE;     // 64 KB (PBN 256) or 48 KB per CTA
    static constexpr int NST = PBN == 256 ? 3 : 4;
    static constexpr int NBUF = 512 / PBN;              // TMEM accumulator buffers of PBN columns
    static constexpr int OFF_B = NST * A_STAGE;
    static constexpr int OFF_BAR = OFF_B + NST * B_STAGE;
    static constexpr int OFF_S = OFF_BAR + 1024;
    static constexpr int SMEM = OFF_S + MAX_NPB * 4 + 1024;
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
    static_assert(2 * NST <= 32, "two lanes per stage");
};

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_id() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_count() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// shared::cluster address of the same shared-memory location in CTA `rank`
__device__ __forceinline__ uint32_t map_to_rank(const void* p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
    return r;
}
// Arrival on a barrier of either CTA of the pair.  CTA-scope release: it orders
// this thread's own earlier operations (the TMEM loads, already waited for and
// fenced with tcgen05.fence::before_thread_sync), not its outstanding global
// stores, which a cluster-scope release would first have to complete.
__device__ __forceinline__ void arrive_remote(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// One copy of KPS consecutive k-blocks of 128 rows: the tensor map views the
// [rows, K] operand as {128 bytes, rows, K / 128} with the k-block stride 128
// bytes, so the box lands as KPS consecutive 16 KB swizzled tiles.
__device__ __forceinline__ void tma_load_3d_pair(void* dst, const CUtensorMap* map, int y, int kb,
                                                 uint32_t bar_cluster) {
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(y), "r"(kb), "r"(bar_cluster)
        : "memory");
}
__device__ __forceinline__ void umma_f8_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive on `bar` in both CTAs of the pair once every tcgen05 operation this
// thread issued so far has completed.
__device__ __forceinline__ void commit_both(uint64_t* bar) {
    const uint16_t mask = 3;
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
                 ::"r"(smem_u32(bar)), "h"(mask) : "memory");
}
}  // namespace pair

template <int PBN, bool DEBUG_P, int YMODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NTHREADS, 1)
    gemm_f8_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, Args g) {
    using namespace pair;
    using C = PCfg<PBN>;
    constexpr int BN = C::BN, BNH = C::BNH, KPS = C::KPS, A_TILE = C::A_TILE, B_TILE = C::B_TILE;
    constexpr int A_STAGE = C::A_STAGE, B_STAGE = C::B_STAGE, STAGE = C::STAGE, NST = C::NST, NBUF = C::NBUF;
    constexpr int OFF_B = C::OFF_B, OFF_BAR = C::OFF_BAR, OFF_S = C::OFF_S;
    extern __shared__ __align__(1024) unsigned char smem_dyn[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
    uint64_t* empty = full + NST;
    uint64_t* tfull = empty + NST;
    uint64_t* tempty = tfull + NBUF;
    uint64_t* done = tempty + NBUF;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
    float* s_sm = reinterpret_cast<float*>(smem + OFF_S);
    volatile int* abortv = abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    const int pid = (int)cluster_id();
    const int npairs = (int)cluster_count();
    const int KB = g.K / BK;
    const int SPT = (KB + KPS - 1) / KPS;                // stages per tile (the last may hold one k-block)
    const int NPB = g.K / g.PB;
    const int kb_per_pb = g.PB / BK;
    const int nmb = (g.M + 2 * BM - 1) / (2 * BM);      // 256-row blocks
    const int nnb = (g.N + BN - 1) / BN;
    const int ntiles = nmb * nnb;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NST; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < NBUF; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], 2 * EPI_WARPS);
        }
        mbar_init(done, 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == MMA_WARP) {
        // both CTAs' warp 2 allocate together: the same columns in both TMEMs
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(512) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    // launched as a programmatic dependent of the activation kernel: everything
    // above overlapped its end; its outputs (operand, s, scale_t) are read below
    grid_dependency_wait();
    if (!DEBUG_P) {
        for (int i = threadIdx.x; i < NPB; i += blockDim.x) s_sm[i] = g.s[(i * g.PB) / g.G];
    }
    tc_fence_before();
    cluster_sync();          // barriers of both CTAs initialised and visible, TMEM allocated, s staged
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp < NPROD) {
        // -------------------------------------------------------- TMA (both CTAs)
        const uint32_t my_tiles = pid < ntiles ? (uint32_t)((ntiles - 1 - pid) / npairs + 1) : 0u;
        const uint32_t total = my_tiles * SPT;
        uint32_t last = 0xFFFFFFFFu;
        bool ok = true;
        for (uint32_t it = warp; it < total; it += NPROD) {
            const int st = (int)(it % NST);
            uint32_t free = 1;
            if (lane == 0)
                free = mbar_wait_bounded<true>(&empty[st], ((it / NST) & 1u) ^ 1u, abortv, g.err, kErrGemmTimeout,
                                               g.limit_ns) ? 1u : 0u;
            if (!__shfl_sync(0xffffffffu, free, 0)) {
                ok = false;
                break;
            }
            const int tile = pid + (int)(it / SPT) * npairs;
            const int kb0 = (int)(it % SPT) * KPS;
            const uint32_t fbar = map_to_rank(&full[st], 0);
            if (lane == 0 && leader) arrive_expect_tx(&full[st], 2 * STAGE);
            __syncwarp();
            const int la = 2 * st;   // one pair of lanes per stage: a thread's copies complete in turn
            if (lane == la || lane == la + 1) {
                const bool isA = lane == la;
                unsigned char* dst = isA ? smem + st * A_STAGE : smem + OFF_B + st * B_STAGE;
                const CUtensorMap* map = isA ? &tmA : &tmB;
                const int y = isA ? (tile % nmb) * 2 * BM + (int)rank * BM : (tile / nmb) * BN + (int)rank * BNH;
                tma_load_3d_pair(dst, map, y, kb0, fbar);
                const uint32_t ip = it + PF_STAGES;
                if (!isA && ip < total) {
                    const int tp = pid + (int)(ip / SPT) * npairs;
                    tma_prefetch_3d(&tmB, 0, (tp / nmb) * BN + (int)rank * BNH, (int)(ip % SPT) * KPS);
                }
            }
            __syncwarp();
            last = it;
        }
        if (!ok && lane == 0 && last != 0xFFFFFFFFu && leader) {
            // let the copies directed at this CTA's barrier land before it exits
            volatile int no_abort = 0;
            mbar_wait_bounded<true>(&full[last % NST], (last / NST) & 1u, &no_abort, nullptr, 0, g.limit_ns);
        }
    } else if (warp == MMA_WARP) {
        if (lane == 0 && leader) {
            // -------------------------------------------------------- MMA (even CTA)
            constexpr uint32_t idesc = idesc_f8(2 * BM, BN);
            uint32_t it = 0, gc = 0;
            bool ok = true;
            for (int tile = pid; tile < ntiles && ok; tile += npairs) {
                for (int sidx = 0; sidx < SPT && ok; ++sidx, ++it) {
                    const int st = (int)(it % NST);
                    if (!(ok = mbar_wait_bounded<true>(&full[st], (it / NST) & 1u, abortv, g.err, kErrGemmTimeout,
                                                       g.limit_ns)))
                        break;
                    tc_fence_after();
                    for (int j = 0; j < KPS; ++j) {
                        const int kb = sidx * KPS + j;
                        if (kb >= KB) break;
                        const bool first = (kb % kb_per_pb) == 0;
                        const bool lastk = (kb % kb_per_pb) == kb_per_pb - 1;
                        const int buf = (int)(gc % NBUF);
                        if (first && !(ok = mbar_wait_bounded<true>(&tempty[buf], (gc / NBUF) & 1u, abortv, g.err,
                                                                    kErrGemmTimeout, g.limit_ns)))
                            break;
                        tc_fence_after();
                        const uint32_t a_base = smem_u32(smem + st * A_STAGE + j * A_TILE);
                        const uint32_t b_base = smem_u32(smem + OFF_B + st * B_STAGE + j * B_TILE);
                        const uint32_t d = tmem + (uint32_t)(buf * BN);
#pragma unroll
                        for (int k = 0; k < BK / 32; ++k)
                            umma_f8_pair(d, sdesc_k_sw128(a_base + 32 * k), sdesc_k_sw128(b_base + 32 * k), idesc,
                                         (first && k == 0) ? 0u : 1u);
                        if (lastk) {
                            commit_both(&tfull[buf]);
                            ++gc;
                        }
                    }
                    if (!ok) break;
                    commit_both(&empty[st]);
                }
            }
            commit_both(done);
            volatile int no_abort = 0;
            mbar_wait_bounded(done, 0, &no_abort, g.err, kErrGemmTimeout, g.limit_ns);
        }
    } else {
        // -------------------------------------------------------- epilogue (both CTAs)
        constexpr int CW = BN / 2;
        const int quarter = warp & 3;
        const int half = (warp - EPI_WARP0) >> 2;
        const uint32_t lane_base = tmem + ((uint32_t)(32 * quarter) << 16);
        const int col0 = CW * half;
        uint32_t tempty_addr[NBUF];
#pragma unroll
        for (int b = 0; b < NBUF; ++b) tempty_addr[b] = map_to_rank(&tempty[b], 0);
        if (lane == 0) {
#pragma unroll
            for (int b = 0; b < NBUF; ++b) arrive_remote(tempty_addr[b]);   // every buffer starts free
        }
        uint32_t gc = 0;
        bool ok = true;
        for (int tile = pid; tile < ntiles && ok; tile += npairs) {
            const int m0 = (tile % nmb) * 2 * BM + (int)rank * BM;
            const int n0 = (tile / nmb) * BN;
            const int row = m0 + 32 * quarter + lane;
            float2 acc[CW / 2];
#pragma unroll
            for (int i = 0; i < CW / 2; ++i) acc[i] = make_float2(0.0f, 0.0f);
            for (int pb = 0; pb < NPB; ++pb, ++gc) {
                const int buf = (int)(gc % NBUF);
                if (!(ok = mbar_wait_bounded(&tfull[buf], (gc / NBUF) & 1u, abortv, g.err, kErrGemmTimeout,
                                             g.limit_ns)))
                    break;
                tc_fence_after();
                const float sg = DEBUG_P ? 1.0f : s_sm[pb];
                const float2 s2 = make_float2(sg, sg);
                const uint32_t src = lane_base + (uint32_t)(buf * BN + col0);
#pragma unroll
                for (int c = 0; c < CW / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld32(src + 32 * c, r);
                    tmem_ld_wait();
                    if (c == CW / 32 - 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) arrive_remote(tempty_addr[buf]);
                    }
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float2 p = make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
                        acc[16 * c + i] = __ffma2_rn(s2, p, acc[16 * c + i]);
                    }
                }
                if (DEBUG_P && ((pb + 1) * g.PB) % g.G == 0) {
                    const int gi = ((pb + 1) * g.PB) / g.G - 1;
                    if (row < g.M) {
                        int32_t* dst = g.P + ((size_t)gi * g.M + row) * g.N;
#pragma unroll
                        for (int i = 0; i < CW / 2; ++i) {
                            const int col = n0 + col0 + 2 * i;
                            if (col < g.N) dst[col] = __float2int_rn(acc[i].x);
                            if (col + 1 < g.N) dst[col + 1] = __float2int_rn(acc[i].y);
                        }
                    }
#pragma unroll
                    for (int i = 0; i < CW / 2; ++i) acc[i] = make_float2(0.0f, 0.0f);
                }
            }
            if (!DEBUG_P && ok) store_tile<CW, YMODE>(g, acc, row, n0 + col0, lane);
        }
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();          // no CTA leaves while its peer may still signal its barriers or use its TMEM
    if (warp == MMA_WARP) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512) : "memory");
    }
}

// A launch that may begin while the previous kernel in the stream finishes
// (programmatic dependent launch); the kernel waits with griddepcontrol.wait
// before it reads what that kernel wrote.  After any other stream operation it
// behaves as a plain launch.
template <typename Kern>
static cudaError_t launch_dependent(Kern kern, dim3 grid, int threads, int smem, cudaStream_t st,
                                   const CUtensorMap& tmA, const CUtensorMap& tmB, const Args& a) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, tmA, tmB, a);
}

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

// 2-D uint8 tensor [outer, inner] with a (box_inner x box_outer) box, 128-byte swizzle.
static bool make_map(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint32_t box_outer) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {inner};
    const cuuint32_t box[2] = {(cuuint32_t)BK, box_outer};
    const cuuint32_t es[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN>
static cudaError_t launch_bn(const GemmF8Launch& gl, const Args& a, int nsm) {
    using C = Cfg<BN>;
    CUtensorMap tmA, tmB;
    if (!make_map(&tmA, gl.A, (uint64_t)gl.K, (uint64_t)gl.M, BM)) return cudaErrorInvalidValue;
    if (!make_map(&tmB, gl.B, (uint64_t)gl.K, (uint64_t)gl.N, BN)) return cudaErrorInvalidValue;
    const int ntiles = ((gl.M + BM - 1) / BM) * ((gl.N + BN - 1) / BN);
    const int grid = ntiles < nsm ? ntiles : nsm;
    const int v = gl.P ? 0 : 1 + gl.ymode;
    auto kern = v == 0 ? gemm_f8_kernel<BN, true, kYF32>
                : v == 1 ? gemm_f8_kernel<BN, false, kYF32>
                : v == 2 ? gemm_f8_kernel<BN, false, kYBF16>
                         : gemm_f8_kernel<BN, false, kYSiluMul>;
    static KernelSetup setup[4];
    int occ = 0;
    cudaError_t e = kernel_setup(reinterpret_cast<const void*>(kern), NTHREADS, C::SMEM, setup[v], &occ);
    if (e != cudaSuccess) return e;
    return launch_dependent(kern, dim3(grid), NTHREADS, C::SMEM, gl.stream, tmA, tmB, a);
}

// 3-D view {128 bytes, rows, K / 128} of a [rows, K] uint8 operand (k-block
// stride 128 bytes) with a {128, box_rows, KPS} box, 128-byte swizzle.
static bool make_map_kblocks(CUtensorMap* map, const void* base, uint64_t K, uint64_t rows, uint32_t box_rows,
                             uint32_t kps) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)BK, rows, K / BK};
    const cuuint64_t strides[2] = {K, (cuuint64_t)BK};
    const cuuint32_t box[3] = {(cuuint32_t)BK, box_rows, kps};
    const cuuint32_t es[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int PBN>
static cudaError_t launch_pair(const GemmF8Launch& gl, const Args& a, int nsm) {
    using namespace pair;
    using C = PCfg<PBN>;
    constexpr int BN = C::BN, BNH = C::BNH, KPS = C::KPS, SMEM = C::SMEM;
    CUtensorMap tmA, tmB;
    if (!make_map_kblocks(&tmA, gl.A, (uint64_t)gl.K, (uint64_t)gl.M, BM, KPS)) return cudaErrorInvalidValue;
    if (!make_map_kblocks(&tmB, gl.B, (uint64_t)gl.K, (uint64_t)gl.N, BNH, KPS)) return cudaErrorInvalidValue;
    const int ntiles = ((gl.M + 2 * BM - 1) / (2 * BM)) * ((gl.N + BN - 1) / BN);
    const int v = gl.P ? 0 : 1 + gl.ymode;
    auto kern = v == 0 ? gemm_f8_pair_kernel<PBN, true, kYF32>
                : v == 1 ? gemm_f8_pair_kernel<PBN, false, kYF32>
                : v == 2 ? gemm_f8_pair_kernel<PBN, false, kYBF16>
                         : gemm_f8_pair_kernel<PBN, false, kYSiluMul>;
    static KernelSetup setup[4];
    static int maxc_cache[4][16] = {};
    int occ = 0;
    cudaError_t e = kernel_setup(reinterpret_cast<const void*>(kern), NTHREADS, SMEM, setup[v], &occ);
    if (e != cudaSuccess) return e;
    // as many CTA pairs as can be resident at once (persistent), at most one per tile
    int dev = 0;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int maxc = dev >= 0 && dev < 16 ? maxc_cache[v][dev] : 0;
    if (maxc == 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(nsm & ~1));
        cfg.blockDim = dim3(NTHREADS);
        cfg.dynamicSmemBytes = SMEM;
        cfg.stream = gl.stream;
        e = cudaOccupancyMaxActiveClusters(&maxc, kern, &cfg);
        if (e != cudaSuccess) return e;
        if (maxc < 1) return cudaErrorInvalidConfiguration;
        if (dev >= 0 && dev < 16) maxc_cache[v][dev] = maxc;
    }
    const int pairs = ntiles < maxc ? ntiles : maxc;
    return launch_dependent(kern, dim3(2 * pairs), NTHREADS, SMEM, gl.stream, tmA, tmB, a);
}

}  // namespace f8

int gemm_f8_pick_bn(int M, int N, int nsm) {
    // 256 x 256 pair tiles (returned as kPickPair256) read the fewest operand bytes
    // per output; take them when there are enough of them to occupy the SMs.  Then
    // 256 x 128 pair tiles (kPickPair128) when they fill three quarters of the SMs.
    // Otherwise one-CTA 256-column tiles, unless 128-column ones fill more SMs.
    const long tp = (long)((M + 255) / 256) * ((N + 255) / 256);
    if (2 * tp >= nsm) return kPickPair256;
    const long tp128 = (long)((M + 255) / 256) * ((N + 127) / 128);
    if (8 * tp128 >= 3 * (long)nsm) return kPickPair128;
    const int nmb = (M + f8::BM - 1) / f8::BM;
    const long t256 = (long)nmb * ((N + 255) / 256);
    const long t128 = (long)nmb * ((N + 127) / 128);
    if (t256 >= nsm) return 256;
    return t128 > t256 ? 128 : 256;
}

cudaError_t launch_gemm_f8(const GemmF8Launch& gl) {
    using namespace f8;
    f8::Args a;
    a.s = gl.s;
    a.scale_t = gl.scale_t;
    a.scale_w = gl.scale_w;
    a.M = gl.M;
    a.N = gl.N;
    a.K = gl.K;
    a.G = gl.G;
    a.PB = gl.PB;
    a.Y = gl.Y;
    a.P = gl.P;
    a.err = gl.err;
    a.limit_ns = kWaitLimitNs;
    const int nsm = device_sm_count();
    const int bn = gl.bn ? gl.bn : gemm_f8_pick_bn(gl.M, gl.N, nsm);
    if (bn == kPickPair256) return f8::launch_pair<256>(gl, a, nsm);
    if (bn == kPickPair128) return f8::launch_pair<128>(gl, a, nsm);
    return bn == 128 ? launch_bn<128>(gl, a, nsm) : launch_bn<256>(gl, a, nsm);
}

}  // namespace rrs
