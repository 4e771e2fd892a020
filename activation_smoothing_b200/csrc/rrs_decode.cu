// rrs_decode.cu -- the whole RRS W4A4 linear layer for few tokens (decode,
// M <= 16) in one cooperative launch.
//
// With M <= 16 tokens the layer reads far more weight bytes (N * K / 2) than
// activation bytes, so its floor is the weight stream from HBM, and two
// launches (activation kernel, then GEMM) leave the stream idle while the
// activations are prepared.  Here one persistent kernel (one CTA per SM) does
// every step of the summary page's "Approach" for the layer, and the weight
// stream starts at once: each CTA first asks L2 to prefetch the weight tiles it
// multiplies first, then
//
//   phase 1  rotation: (token, channel chunk) items spread over the CTAs; the
//            normalised Hadamard transform of each block in shared memory
//            (fp32, stages h = 1, 2, 4, ... with the pair (a + b, a - b), then
//            one multiply by c_n), written as fp32 X_rot to the workspace;
//                                                          -- grid barrier
//   phase 2  runtime smoothing scales: the CTA that owns group g gathers the
//            reordered channels X'[t][j] = X_rot[t][perm[j]] of every token and
//            writes s_g = max |X'|; it also keeps, per token, the largest
//            |X'| / s_g over its groups;                   -- grid barrier
//   phase 3  per-token scales scale_t = amax_t / 7 from those maxima, then the
//            INT4 codes q = clamp(rint((X' / s_g) / scale_t), -8, 7) of the
//            channel chunks this CTA multiplies (into shared memory) and of the
//            groups it owns (to qX);
//   phase 4  the group-scaled contraction over work units of 16 output
//            channels x 1024 input channels.  A warp loads its unit's packed
//            weights straight into registers, turns eight packed codes into two
//            int8x4 words holding 16 * code with one shift and two ANDs (no
//            sign extension needed), and multiplies on the tensor cores with
//            mma.sync m16n8k32 (weights as the 16-row operand, tokens as the
//            8 columns).  Each group's exact sum 256 * P_g is shifted back and
//            promoted, acc += s_g * P_g, in group order.  A unit's sums go to
//            the workspace; the last unit of an output tile to finish adds the
//            chunks in order and applies scale_t * scale_w.
//
// All integer results (codes, s, scale_t) are the same bits the two-launch
// path gives; Y differs from it only in the order of the fp32 sums over chunks.
// The tensor work here is under one percent of the tensor peak: what matters is
// keeping enough weight bytes in flight, which register loads do without a
// shared-memory round trip (a tcgen05 MMA would need the unpacked weights in
// shared memory first).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "rrs_device.cuh"
#include "rrs_internal.h"

namespace rrs {
namespace dec {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int KC = 1024;                  // input channels per work unit
constexpr int kBlocksPerUnit = KC / 128;  // 128-channel MMA blocks per unit
constexpr int kActWords = KC / 8;         // 8-channel words per token row of a staged chunk
constexpr int kActStride = kActWords * 8 + 16;  // bytes per token row: (even, odd) word pairs + pad
constexpr int kMaxSlots = 4;              // code chunks staged per CTA
constexpr int kMaxTokens = 16;
constexpr int kMaxChunk = 8192;           // channels rotated per item
constexpr int kMaxGroups = 256;           // K / G
constexpr int kMaxCtas = 1024;            // rows of the per-token maxima table
constexpr int kPrefetchUnits = 24;        // units per CTA asked of L2 up front

constexpr size_t kSmemBytes = (size_t)kMaxChunk * 4 + (size_t)kMaxSlots * kMaxTokens * kActStride +
                              (size_t)kMaxGroups * 4 + 256;

struct Args {
    const __half* X;
    const int32_t* perm;
    const uint8_t* qW;
    const float* scale_w;
    int M, N, K, G, n;
    float c_n;
    int unit_scales;
    uint8_t* qX;
    float* s;
    float* scale_t;
    void* Y;
    int ybf16;
    float* Xr;      // [M, K] rotated activations
    float* pamax;   // [gridDim.x, 16] per-CTA per-token maxima of |X'| / s
    int* cnt;       // [N / 16] finished units per output tile
    float* part;    // [K / KC, M, N] per-chunk sums
    int L;          // channels per rotation item: max(n, 1024)
    int RT, KCN, U; // output tiles, chunks, units
    uint32_t* gbar;
    uint32_t* err;
    uint64_t limit_ns;
};

__device__ __forceinline__ void mma_s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                       uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Eight packed codes (low nibble = even channel) as int8x4 words of 16 * code:
// the four even channels, then the four odd ones.
__device__ __forceinline__ uint32_t nib_even(uint32_t w) { return (w << 4) & 0xF0F0F0F0u; }
__device__ __forceinline__ uint32_t nib_odd(uint32_t w) { return w & 0xF0F0F0F0u; }

__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// The INT4 code of one smoothed, reordered activation: x = X'[t][j], sd the
// group's divisor (s_g, or 1 where s_g == 0), sc the token's scale.
__device__ __forceinline__ int code_of(float x, float sd, float sc) {
    if (sc == 0.0f) return 0;
    const int q = __float2int_rn(__fdiv_rn(__fdiv_rn(x, sd), sc));
    return q < -8 ? -8 : (q > 7 ? 7 : q);
}

// Block-wide max of non-negative floats; every thread gets the result.
__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    const int warp = threadIdx.x >> 5;
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[warp] = v;
    __syncthreads();
    float m = red[0];
    for (int w = 1; w < kWarps; ++w) m = fmaxf(m, red[w]);
    return m;
}

__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const Args p) {
    extern __shared__ __align__(16) unsigned char smem[];
    float* buf = reinterpret_cast<float*>(smem);                                   // [kMaxChunk]
    uint8_t* act = smem + (size_t)kMaxChunk * 4;                                   // [slots][16][kActStride]
    float* s_sm = reinterpret_cast<float*>(act + (size_t)kMaxSlots * kMaxTokens * kActStride);  // [NG] divisors
    float* red = s_sm + kMaxGroups;                                                // [32]
    float* sc_sm = red + 32;                                                       // [16] scale_t
    uint32_t* pam = reinterpret_cast<uint32_t*>(sc_sm + 16);                       // [16] bits of max |X'|/s

    const int tid = threadIdx.x;
    const int K = p.K, M = p.M, N = p.N, G = p.G;
    const int NG = K / G;
    const int Kh = K / 2;

    // this CTA's work units (chunk-major: u = kc * RT + rt), the chunks they span
    const int u0 = (int)((long long)blockIdx.x * p.U / gridDim.x);
    const int u1 = (int)((long long)(blockIdx.x + 1) * p.U / gridDim.x);
    const int kc_first = u0 / p.RT;

    // ---- phase 0: start the weight stream (L2 prefetch), clear the tile counters
    {
        const int npf = min(u1 - u0, kPrefetchUnits);
        for (int e = tid; e < npf * 16; e += kThreads) {
            const int u = u0 + e / 16;
            const int row = (u % p.RT) * 16 + (e % 16);
            prefetch_l2(p.qW + (size_t)row * Kh + (size_t)(u / p.RT) * (KC / 2), KC / 2);
        }
        for (int i = blockIdx.x * kThreads + tid; i < p.RT; i += gridDim.x * kThreads) p.cnt[i] = 0;
        if (tid < kMaxTokens) pam[tid] = 0u;
    }

    // ---- phase 1: rotation, one (token, chunk of L channels) item at a time
    {
        const int L = p.L;
        const int per_row = K / L;
        for (int item = blockIdx.x; item < M * per_row; item += gridDim.x) {
            const int t = item / per_row;
            const int c0 = (item % per_row) * L;
            const __half* xs = p.X + (size_t)t * K + c0;
            for (int i = tid * 8; i < L; i += kThreads * 8) {
                const uint4 v = *reinterpret_cast<const uint4*>(xs + i);
                const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float2 f = __half22float2(h[q]);
                    buf[i + 2 * q] = f.x;
                    buf[i + 2 * q + 1] = f.y;
                }
            }
            __syncthreads();
            for (int h = 1; h < p.n; h <<= 1) {
                for (int q = tid; q < L / 2; q += kThreads) {
                    const int j = ((q & ~(h - 1)) << 1) | (q & (h - 1));
                    const float a = buf[j], b = buf[j + h];
                    buf[j] = __fadd_rn(a, b);
                    buf[j + h] = __fsub_rn(a, b);
                }
                __syncthreads();
            }
            float* xr = p.Xr + (size_t)t * K + c0;
            for (int i = tid * 4; i < L; i += kThreads * 4) {
                float4 o;
                o.x = __fmul_rn(buf[i], p.c_n);
                o.y = __fmul_rn(buf[i + 1], p.c_n);
                o.z = __fmul_rn(buf[i + 2], p.c_n);
                o.w = __fmul_rn(buf[i + 3], p.c_n);
                *reinterpret_cast<float4*>(xr + i) = o;
            }
            __syncthreads();
        }
    }
    if (!grid_barrier(p.gbar, p.err, p.limit_ns)) return;

    // ---- phase 2: s_g of the groups this CTA owns; per-token max of |X'| / s_g.
    // A thread takes one channel of the group and loads it for every token at once.
    for (int g = blockIdx.x; g < NG; g += gridDim.x) {
        float m = 0.0f;
        for (int jj = tid; jj < G; jj += kThreads) {
            const int src = __ldg(p.perm + g * G + jj);
            float v[kMaxTokens];
#pragma unroll
            for (int t = 0; t < kMaxTokens; ++t) v[t] = t < M ? __ldcg(p.Xr + (size_t)t * K + src) : 0.0f;
#pragma unroll
            for (int t = 0; t < kMaxTokens; ++t) m = fmaxf(m, fabsf(v[t]));
        }
        float sg = block_max(m, red);
        if (p.unit_scales) sg = 1.0f;
        if (tid == 0) p.s[g] = sg;
        const float sd = sg == 0.0f ? 1.0f : sg;
        for (int jj = tid; jj < G; jj += kThreads) {
            const int src = __ldg(p.perm + g * G + jj);
            float v[kMaxTokens];
#pragma unroll
            for (int t = 0; t < kMaxTokens; ++t) v[t] = t < M ? __ldcg(p.Xr + (size_t)t * K + src) : 0.0f;
#pragma unroll
            for (int t = 0; t < kMaxTokens; ++t)
                if (t < M) atomicMax(pam + t, __float_as_uint(__fdiv_rn(fabsf(v[t]), sd)));
        }
    }
    __syncthreads();
    if (tid < kMaxTokens) p.pamax[(size_t)blockIdx.x * kMaxTokens + tid] = __uint_as_float(pam[tid]);
    if (!grid_barrier(p.gbar, p.err, p.limit_ns)) return;

    // ---- phase 3: per-token scales; codes of the staged chunks and of owned groups
    {
        const int warp = tid >> 5, lane = tid & 31;
        if (warp < M) {
            float a = 0.0f;
            for (int c = lane; c < (int)gridDim.x; c += 32) a = fmaxf(a, __ldcg(p.pamax + (size_t)c * kMaxTokens + warp));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
            if (lane == 0) {
                const float sc = __fdiv_rn(a, 7.0f);
                sc_sm[warp] = sc;
                if (blockIdx.x == 0) p.scale_t[warp] = sc;
            }
        }
        for (int g = tid; g < NG; g += kThreads) {
            const float sg = __ldcg(p.s + g);
            s_sm[g] = sg == 0.0f ? 1.0f : sg;
        }
        __syncthreads();
        // Staged chunks, as the tensor cores' column operand: per token and 8-channel
        // word, the codes of the even channels and of the odd ones as int8x4 words of
        // 16 * code.  A thread takes one word and four tokens (all loads at once).
        const int nslot = u1 > u0 ? (u1 - 1) / p.RT - kc_first + 1 : 0;
        const int TOK = M <= 8 ? 8 : 16;
        for (int e = tid; e < nslot * kActWords * 4; e += kThreads) {
            const int wi = e % kActWords;
            const int tq = (e / kActWords) % 4;
            const int sl = e / (kActWords * 4);
            const int j0 = (kc_first + sl) * KC + 8 * wi;
            const int4 pa = __ldg(reinterpret_cast<const int4*>(p.perm + j0));
            const int4 pb = __ldg(reinterpret_cast<const int4*>(p.perm + j0 + 4));
            const int src[8] = {pa.x, pa.y, pa.z, pa.w, pb.x, pb.y, pb.z, pb.w};
            const float sd = s_sm[j0 / G];
            float x[4][8];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int t = tq + 4 * q;
#pragma unroll
                for (int c = 0; c < 8; ++c) x[q][c] = t < M ? __ldcg(p.Xr + (size_t)t * K + src[c]) : 0.0f;
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int t = tq + 4 * q;
                if (t >= TOK) continue;
                uint32_t ev = 0, od = 0;
                if (t < M) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        ev |= ((uint32_t)(code_of(x[q][2 * c], sd, sc_sm[t]) << 4) & 0xF0u) << (8 * c);
                        od |= ((uint32_t)(code_of(x[q][2 * c + 1], sd, sc_sm[t]) << 4) & 0xF0u) << (8 * c);
                    }
                }
                *reinterpret_cast<uint2*>(act + ((size_t)sl * kMaxTokens + t) * kActStride + 8 * wi) = make_uint2(ev, od);
            }
        }
        // packed codes of the owned groups (the layer's qX output)
        for (int g = blockIdx.x; g < NG; g += gridDim.x) {
            for (int e = tid; e < M * (G / 2); e += kThreads) {
                const int t = e / (G / 2);
                const int j = g * G + 2 * (e % (G / 2));
                const float* xr = p.Xr + (size_t)t * K;
                const float sd = s_sm[g];
                const int q0 = code_of(__ldcg(xr + __ldg(p.perm + j)), sd, sc_sm[t]);
                const int q1 = code_of(__ldcg(xr + __ldg(p.perm + j + 1)), sd, sc_sm[t]);
                p.qX[(size_t)t * Kh + j / 2] = (uint8_t)((uint32_t)(q0 & 15) | ((uint32_t)(q1 & 15) << 4));
            }
        }
        __syncthreads();
    }

    // ---- phase 4: group-scaled contraction of the units
    {
        const int warp = tid >> 5, lane = tid & 31;
        const int gq = lane >> 2, tq = lane & 3;
        const int gpb = G / 128;                   // MMA blocks per group (G divides KC)
        const bool two = M > 8;
        for (int u = u0 + warp; u < u1; u += kWarps) {
            const int kc = u / p.RT, rt = u % p.RT;
            {
                // keep the L2 prefetch kPrefetchUnits units ahead of the loads
                const int up = u + kPrefetchUnits;
                if (lane < 16 && up < u1)
                    prefetch_l2(p.qW + (size_t)((up % p.RT) * 16 + lane) * Kh + (size_t)(up / p.RT) * (KC / 2), KC / 2);
            }
            const uint8_t* wr = p.qW + (size_t)(rt * 16 + gq) * Kh + (size_t)kc * (KC / 2) + 16 * tq;
            uint4 wa[kBlocksPerUnit], wb[kBlocksPerUnit];
#pragma unroll
            for (int i = 0; i < kBlocksPerUnit; ++i) {
                wa[i] = __ldcs(reinterpret_cast<const uint4*>(wr + 64 * i));
                wb[i] = __ldcs(reinterpret_cast<const uint4*>(wr + (size_t)8 * Kh + 64 * i));
            }
            const uint8_t* ar = act + ((size_t)(kc - kc_first) * kMaxTokens + gq) * kActStride + 32 * tq;
            float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
            int d0[4] = {0, 0, 0, 0}, d1[4] = {0, 0, 0, 0};
#pragma unroll
            for (int i = 0; i < kBlocksPerUnit; ++i) {
                // this thread's channels of block i: words 16 i + 4 tq + w, w = 0..3
                const uint4 b01 = *reinterpret_cast<const uint4*>(ar + 128 * i);
                const uint4 b23 = *reinterpret_cast<const uint4*>(ar + 128 * i + 16);
                const uint32_t be[4] = {b01.x, b01.z, b23.x, b23.z}, bo[4] = {b01.y, b01.w, b23.y, b23.w};
                const uint32_t wA[4] = {wa[i].x, wa[i].y, wa[i].z, wa[i].w};
                const uint32_t wB[4] = {wb[i].x, wb[i].y, wb[i].z, wb[i].w};
#pragma unroll
                for (int w = 0; w < 4; ++w)
                    mma_s8(d0, nib_even(wA[w]), nib_even(wB[w]), nib_odd(wA[w]), nib_odd(wB[w]), be[w], bo[w]);
                if (two) {
                    const uint8_t* ar1 = ar + (size_t)8 * kActStride;
                    const uint4 c01 = *reinterpret_cast<const uint4*>(ar1 + 128 * i);
                    const uint4 c23 = *reinterpret_cast<const uint4*>(ar1 + 128 * i + 16);
                    const uint32_t ce[4] = {c01.x, c01.z, c23.x, c23.z}, co[4] = {c01.y, c01.w, c23.y, c23.w};
#pragma unroll
                    for (int w = 0; w < 4; ++w)
                        mma_s8(d1, nib_even(wA[w]), nib_even(wB[w]), nib_odd(wA[w]), nib_odd(wB[w]), ce[w], co[w]);
                }
                if ((i + 1) % gpb == 0) {
                    // end of a group: 256 * P_g exactly; promote with s_g
                    const float sg = s_sm[(kc * KC + i * 128) / G];
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        acc0[r] = __fmaf_rn(sg, (float)(d0[r] >> 8), acc0[r]);
                        d0[r] = 0;
                        if (two) {
                            acc1[r] = __fmaf_rn(sg, (float)(d1[r] >> 8), acc1[r]);
                            d1[r] = 0;
                        }
                    }
                }
            }
            // this unit's sums: rows gq, gq + 8 of the tile; tokens 2 tq, 2 tq + 1 (+ 8)
            float* pc = p.part + (size_t)kc * M * N;
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int row = rt * 16 + gq + (r >= 2 ? 8 : 0);
                const int t0 = 2 * tq + (r & 1);
                if (t0 < M) pc[(size_t)t0 * N + row] = acc0[r];
                if (two && t0 + 8 < M) pc[(size_t)(t0 + 8) * N + row] = acc1[r];
            }
            __threadfence();
            __syncwarp();
            int last = 0;
            if (lane == 0) last = atomicAdd(p.cnt + rt, 1) == p.KCN - 1;
            last = __shfl_sync(0xFFFFFFFFu, last, 0);
            if (last) {
                __threadfence();
                for (int e = lane; e < 16 * M; e += 32) {
                    const int row = rt * 16 + (e & 15);
                    const int t = e >> 4;
                    float a = __ldcg(p.part + (size_t)t * N + row);
                    for (int c = 1; c < p.KCN; ++c) a = __fadd_rn(a, __ldcg(p.part + ((size_t)c * M + t) * N + row));
                    const float y = __fmul_rn(__fmul_rn(a, sc_sm[t]), __ldg(p.scale_w + row));
                    if (p.ybf16)
                        reinterpret_cast<__nv_bfloat16*>(p.Y)[(size_t)t * N + row] = __float2bfloat16_rn(y);
                    else
                        reinterpret_cast<float*>(p.Y)[(size_t)t * N + row] = y;
                }
                if (lane == 0) p.cnt[rt] = 0;
            }
        }
    }
}

}  // namespace dec

static int decode_grid() {
    const int g = device_sm_count();
    return g < dec::kMaxCtas ? g : dec::kMaxCtas;
}

bool decode_supported(int M, int N, int K, int G, int n) {
    using namespace dec;
    if (!(M >= 1 && M <= kMaxTokens && N >= 16 && N % 16 == 0 && K % KC == 0 && G >= 128 && G % 128 == 0 &&
          KC % G == 0 && K / G <= kMaxGroups && n <= kMaxChunk))
        return false;
    // every CTA's units (chunk-major) span at most kMaxSlots chunks of staged codes
    const int grid = decode_grid();
    if (grid < 1) return false;
    const long long RT = N / 16, U = RT * (K / KC);
    for (int c = 0; c < grid; ++c) {
        const long long u0 = c * U / grid, u1 = (c + 1) * U / grid;
        if (u1 > u0 && (u1 - 1) / RT - u0 / RT + 1 > kMaxSlots) return false;
    }
    return true;
}

// Workspace bytes after the 256-byte header: X_rot, the per-token maxima table,
// the tile counters and the per-chunk sums, each 256-byte aligned.
static size_t al256(size_t x) { return (x + 255) & ~size_t(255); }
size_t decode_ws_bytes(int M, int N, int K) {
    return al256((size_t)M * K * 4) + al256((size_t)dec::kMaxCtas * dec::kMaxTokens * 4) + al256((size_t)(N / 16) * 4) +
           al256((size_t)(K / dec::KC) * M * N * 4);
}

cudaError_t launch_decode(const DecodeLaunch& dl, cudaStream_t st) {
    using namespace dec;
    static KernelSetup setup;
    int occ = 0;
    cudaError_t e = kernel_setup(reinterpret_cast<const void*>(decode_kernel), kThreads, kSmemBytes, setup, &occ);
    if (e != cudaSuccess) return e;
    if (occ < 1) return cudaErrorInvalidConfiguration;
    const int grid = decode_grid();
    Args a{};
    a.X = reinterpret_cast<const __half*>(dl.X);
    a.perm = dl.perm;
    a.qW = dl.qW;
    a.scale_w = dl.scale_w;
    a.M = dl.M;
    a.N = dl.N;
    a.K = dl.K;
    a.G = dl.G;
    a.n = dl.n;
    a.c_n = dl.c_n;
    a.unit_scales = dl.unit_scales;
    a.qX = dl.qX;
    a.s = dl.s;
    a.scale_t = dl.scale_t;
    a.Y = dl.Y;
    a.ybf16 = dl.ybf16;
    unsigned char* w = static_cast<unsigned char*>(dl.body);
    a.Xr = reinterpret_cast<float*>(w);
    w += al256((size_t)dl.M * dl.K * 4);
    a.pamax = reinterpret_cast<float*>(w);
    w += al256((size_t)kMaxCtas * kMaxTokens * 4);
    a.cnt = reinterpret_cast<int*>(w);
    w += al256((size_t)(dl.N / 16) * 4);
    a.part = reinterpret_cast<float*>(w);
    a.L = dl.n > KC ? dl.n : KC;
    a.RT = dl.N / 16;
    a.KCN = dl.K / KC;
    a.U = a.RT * a.KCN;
    a.gbar = dl.gbar;
    a.err = dl.err;
    a.limit_ns = kWaitLimitNs;
    void* params[] = {&a};
    return cudaLaunchCooperativeKernel(reinterpret_cast<void*>(decode_kernel), dim3(grid), dim3(kThreads), params,
                                       kSmemBytes, st);
}

}  // namespace rrs
