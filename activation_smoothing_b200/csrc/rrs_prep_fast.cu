// rrs_prep_fast.cu -- online activation path for K a multiple of 2048 (every
// LLaMA projection shape): two kernels with an fp32 scratch between them.
//
//   rot_gather_kernel   X (fp16) -> X' = reorder(rotate(X)) (fp32, scratch) and
//                       s[g] = max over tokens and group channels |X'|
//   smooth_quant_kernel X' -> qX (packed INT4), qX8 (int8 GEMM operand), scale_t
//
// The scratch holds X' once (M*K*4 bytes), so the Hadamard transform runs once
// per element; at the LLaMA-3-8B shapes the scratch (33.5 MB) stays in L2.
//
// Work split: a team of T = K/64 threads (a multiple of 32) owns one row; each
// thread holds 64 elements.  Rotation rounds: up to 6 butterfly stages on the
// 64 registers (f32x2 packed add/sub for every stage but the first of a round),
// an exchange through a swizzled fp32 row buffer, the next 6 stages (and a
// third round for n = 8192).
//
// Arithmetic is bit-identical to the library contract: stage order h = 1, 2, 4,
// ... with (a + b, a - b); one multiply by c_n; IEEE division (computed with
// Markstein's correction from a correctly rounded reciprocal, see
// div_markstein); round half to even; clamp to [-8, 7].
#include <cuda_runtime.h>

#include <cstdint>

#include "rrs_device.cuh"
#include "rrs_internal.h"

namespace rrs {
namespace fast {

constexpr int E = 64;        // elements per thread
constexpr int LOGE = 6;
constexpr int CTA = 256;     // threads per CTA when T <= 256

__device__ __forceinline__ int swz(int idx) { return idx ^ (((idx >> LOGE) & 7) << 2); }

__device__ __forceinline__ int opaque(int x) {
    int y;
    asm volatile("mov.b32 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

// Butterfly stages 0..A-1 over v[0..63] (stage k pairs l and l + 2^k).  Stage 0
// combines the two lanes of one float2 (scalar); later stages combine two
// float2 registers lane by lane with packed instructions.  a - b is computed
// as fma(b, -1, a), which is exactly RN(a - b).
template <int A>
__device__ __forceinline__ void stages(float2 (&v)[32]) {
    const float2 neg1 = make_float2(-1.0f, -1.0f);
    if constexpr (A >= 1) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const float x = v[i].x, y = v[i].y;
            v[i].x = __fadd_rn(x, y);
            v[i].y = __fsub_rn(x, y);
        }
    }
#pragma unroll
    for (int k = 1; k < A; ++k) {
        const int h = 1 << (k - 1);   // distance in float2 units
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if (!(i & h)) {
                const float2 a = v[i], b = v[i + h];
                v[i] = __fadd2_rn(a, b);
                v[i + h] = __ffma2_rn(b, neg1, a);
            }
        }
    }
}

// Register l of a round with first active bit B0 and A active bits holds the
// element index rindex(t, l); its swizzled word address is raddr(t, l).
template <int B0, int A>
__device__ __forceinline__ int rindex(int t, int T, int l) {
    const int j = l >> A;
    const int mid = l & ((1 << A) - 1);
    const int q = t + j * T;
    return (((q >> B0) << (B0 + A)) | (q & ((1 << B0) - 1))) | (mid << B0);
}
template <int B0, int A>
__device__ __forceinline__ int raddr(int t, int T, int l) {
    const int j = l >> A;
    const int mid = l & ((1 << A) - 1);
    const int q = t + j * T;
    const int sb = swz(((q >> B0) << (B0 + A)) | (q & ((1 << B0) - 1)));
    if constexpr (B0 == LOGE) return (sb ^ ((mid & 7) << 2)) + (mid << B0);
    else return sb + (mid << B0);
}

template <int B0, int A>
__device__ __forceinline__ void rload(float2 (&v)[32], const float* buf, int t, int T) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        v[i].x = buf[raddr<B0, A>(t, T, 2 * i)];
        v[i].y = buf[raddr<B0, A>(t, T, 2 * i + 1)];
    }
}
template <int B0, int A>
__device__ __forceinline__ void rstore(const float2 (&v)[32], float* buf, int t, int T) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        buf[raddr<B0, A>(t, T, 2 * i)] = v[i].x;
        buf[raddr<B0, A>(t, T, 2 * i + 1)] = v[i].y;
    }
}

struct RotArgs {
    const __half* X;     // [rows, K]
    int rows, K, G;
    float c_n;
    const int32_t* perm; // [K]
    float* xp;           // scratch [rows, K] fp32, thread-interleaved (see xp_offset)
    uint32_t* smax;      // [K/G] fp32 bits, zeroed by the host
};

// Scratch layout of one row: the 64 reordered values of team thread t are 16
// float4 at float4 index i*T + t (i = 0..15), so both the writes here and the
// reads of smooth_quant_kernel are coalesced.
__device__ __forceinline__ size_t xp_row(int r, int K) { return (size_t)r * K; }

template <int L, int MAXT>
__global__ void __launch_bounds__(MAXT) rot_gather_kernel(RotArgs p) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    constexpr int NR = (L <= LOGE) ? 1 : (L <= 2 * LOGE ? 2 : 3);
    constexpr int A1 = L < LOGE ? L : LOGE;
    constexpr int A2 = (L - LOGE) < LOGE ? (L - LOGE) : LOGE;
    constexpr int A3 = L - 2 * LOGE;
    const int K = p.K;
    const int T = K / E;
    const int R = blockDim.x / T;
    const int team = threadIdx.x / T;
    const int t = threadIdx.x % T;
    float* rowbuf = reinterpret_cast<float*>(smem_raw) + (size_t)team * K;
    __half* stage0 = reinterpret_cast<__half*>(reinterpret_cast<float*>(smem_raw) + (size_t)R * K) +
                     (size_t)team * 2 * K;
    const int bar_id = 1 + team;

    // Gather addresses of this thread's outputs j in [64t, 64t + 64) (one group).
    // perm is staged through shared memory: coalesced 16-byte global loads, and
    // 16-byte chunk c stored at c ^ ((c >> 4) & 7) so that each thread's 16
    // chunk reads below are bank-conflict free.
    uint32_t gaddr[32];
    {
        int4* pst = reinterpret_cast<int4*>(smem_raw);
        const int4* pg = reinterpret_cast<const int4*>(p.perm);
        for (int c = threadIdx.x; c < K / 4; c += blockDim.x) pst[c ^ ((c >> 4) & 7)] = pg[c];
        __syncthreads();
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            const int c = t * 16 + m;
            const int4 v = pst[c ^ ((c >> 4) & 7)];
            gaddr[2 * m] = (uint32_t)swz(v.x) | ((uint32_t)swz(v.y) << 16);
            gaddr[2 * m + 1] = (uint32_t)swz(v.z) | ((uint32_t)swz(v.w) << 16);
        }
        __syncthreads();   // the row buffers reuse this space
    }
    float tmax = 0.0f;

    auto issue_row = [&](int r, int sb) {
        const __half* src = p.X + (size_t)r * K;
        __half* dst = stage0 + (size_t)sb * K;
        for (int u = t; u < K / 8; u += T) {
            const int owner = u >> 3;
            const int c = u & 7;
            cp_async16(dst + (size_t)(owner * 8 + (c ^ (owner & 7))) * 8, src + (size_t)u * 8);
        }
    };

    const int stride = gridDim.x * R;
    int r = blockIdx.x * R + team;
    int it = 0;
    if (r < p.rows) issue_row(r, 0);
    cp_async_commit();
    for (; r < p.rows; r += stride, ++it) {
        const int sb = it & 1;
        if (r + stride < p.rows) issue_row(r + stride, sb ^ 1);
        cp_async_commit();
        cp_async_wait<1>();
        named_bar(bar_id, T);
        const int tl = opaque(t);

        float2 v[32];
        {
            const __half* st = stage0 + (size_t)sb * K;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 raw = *reinterpret_cast<const uint4*>(st + (size_t)(tl * 8 + (c ^ (tl & 7))) * 8);
                const __half2* h2 = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
                for (int q = 0; q < 4; ++q) v[c * 4 + q] = __half22float2(h2[q]);
            }
        }
        stages<A1>(v);
        if constexpr (NR >= 2) {
#pragma unroll
            for (int i = 0; i < 32; i += 2)
                *reinterpret_cast<float4*>(rowbuf + swz(tl * E + 2 * i)) =
                    make_float4(v[i].x, v[i].y, v[i + 1].x, v[i + 1].y);
            named_bar(bar_id, T);
            rload<LOGE, A2>(v, rowbuf, tl, T);
            stages<A2>(v);
        }
        if constexpr (NR >= 3) {
            rstore<LOGE, LOGE>(v, rowbuf, tl, T);
            named_bar(bar_id, T);
            rload<2 * LOGE, A3>(v, rowbuf, tl, T);
            stages<A3>(v);
        }
        // X_rot = c_n * v, written in natural (swizzled) order for the gather.
        const float2 c2 = make_float2(p.c_n, p.c_n);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __fmul2_rn(v[i], c2);
        if constexpr (NR == 1) {
#pragma unroll
            for (int i = 0; i < 32; i += 2)
                *reinterpret_cast<float4*>(rowbuf + swz(tl * E + 2 * i)) =
                    make_float4(v[i].x, v[i].y, v[i + 1].x, v[i + 1].y);
        } else if constexpr (NR == 2) {
            rstore<LOGE, A2>(v, rowbuf, tl, T);
        } else {
            rstore<2 * LOGE, A3>(v, rowbuf, tl, T);
        }
        named_bar(bar_id, T);

        // gather X'[j] = X_rot[perm[j]], track the group max, write the scratch
        float4* dst = reinterpret_cast<float4*>(p.xp + xp_row(r, K));
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint32_t g0 = gaddr[2 * i], g1 = gaddr[2 * i + 1];
            float4 o;
            o.x = rowbuf[g0 & 0xFFFFu];
            o.y = rowbuf[g0 >> 16];
            o.z = rowbuf[g1 & 0xFFFFu];
            o.w = rowbuf[g1 >> 16];
            tmax = fmaxf(tmax, fmaxf(fmaxf(fabsf(o.x), fabsf(o.y)), fmaxf(fabsf(o.z), fabsf(o.w))));
            dst[i * T + t] = o;
        }
        named_bar(bar_id, T);   // row buffer and staging free for the next row
    }
    cp_async_wait<0>();

    // group max: G/64 consecutive threads share a group; reduce over aligned
    // power-of-two segments of them, then one atomic per segment.
    if (p.smax) {
        const int gsz = p.G / E;
        const int seg = (gsz & -gsz) < 32 ? (gsz & -gsz) : 32;
        float m = tmax;
        for (int o = seg >> 1; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if ((t % seg) == 0 && m > 0.0f) atomicMax(&p.smax[(t * E) / p.G], __float_as_uint(m));
    }
}

// ---------------------------------------------------------------------------
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

struct QuantArgs {
    const float* xp;     // scratch [rows, K] (thread-interleaved rows)
    int rows, K, G;
    int unit_scales;
    const float* s;      // [K/G]
    uint8_t* qX;         // [rows, K/2]
    int8_t* qX8;         // [rows, K] int8 GEMM operand (k order permuted inside each 32-chunk)
    float* scale_t;      // [rows]
    float* s_unit_out;   // [K/G] written as 1 under unit scales (may be null)
};

// Gathers byte 0 of four words into one word: result byte i = byte 0 of w_i.
__device__ __forceinline__ uint32_t low_bytes(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3) {
    return __byte_perm(__byte_perm(w0, w1, 0x0040), __byte_perm(w2, w3, 0x0040), 0x5410);
}

template <int MAXT>
__global__ void __launch_bounds__(MAXT) smooth_quant_kernel(QuantArgs p) {
    const int K = p.K;
    const int T = K / E;
    const int R = blockDim.x / T;
    const int team = threadIdx.x / T;
    const int t = threadIdx.x % T;
    const int bar_id = 1 + team;
    __shared__ float red[8][16];

    float d = 1.0f;
    if (!p.unit_scales) {
        const float sg = p.s[(t * E) / p.G];
        d = (sg == 0.0f) ? 1.0f : sg;
    } else if (p.s_unit_out && blockIdx.x == 0) {
        for (int g = threadIdx.x; g < K / p.G; g += blockDim.x) p.s_unit_out[g] = 1.0f;
    }
    const float yd = __frcp_rn(d);
    const float2 nd2 = make_float2(-d, -d), yd2 = make_float2(yd, yd);
    constexpr float kMagic = 12582912.0f;   // 1.5 * 2^23: adding it rounds to an integer, half to even
    const float2 magic2 = make_float2(kMagic, kMagic);

    const int stride = gridDim.x * R;
    for (int r = blockIdx.x * R + team; r < p.rows; r += stride) {
        const float4* src = reinterpret_cast<const float4*>(p.xp + (size_t)r * K);
        float2 x[32];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float4 f = __ldcs(src + i * T + t);
            x[2 * i] = make_float2(f.x, f.y);
            x[2 * i + 1] = make_float2(f.z, f.w);
        }
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if (!p.unit_scales) x[i] = div_markstein(x[i], nd2, yd2);
            amax = fmaxf(amax, fmaxf(fabsf(x[i].x), fabsf(x[i].y)));
        }
        float tmx = amax;   // this thread's max |x~|
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        if ((t & 31) == 0) red[team][t >> 5] = amax;
        named_bar(bar_id, T);
        amax = red[team][0];
        for (int w = 1; w < T / 32; ++w) amax = fmaxf(amax, red[team][w]);
        const float scale = __fdiv_rn(amax, 7.0f);

        uint32_t pk[8], q8[16];
        if (scale == 0.0f) {
#pragma unroll
            for (int i = 0; i < 8; ++i) pk[i] = 0u;
#pragma unroll
            for (int i = 0; i < 16; ++i) q8[i] = 0u;
        } else {
            const float ys = __frcp_rn(scale);
            const float2 ns2 = make_float2(-scale, -scale), ys2 = make_float2(ys, ys);
            // |x~| / scale <= 7 up to rounding; clamp only if this thread can exceed it.
            const bool clamp = __fdiv_rn(tmx, scale) >= 7.5f;
#pragma unroll
            for (int w = 0; w < 8; ++w) {   // 8 elements (4 float2) per packed word
                uint32_t b[8];
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    float2 z = div_markstein(x[4 * w + h], ns2, ys2);
                    if (clamp) {
                        z.x = fminf(fmaxf(z.x, -8.0f), 7.0f);
                        z.y = fminf(fmaxf(z.y, -8.0f), 7.0f);
                    }
                    z = __fadd2_rn(z, magic2);   // low bits: the rounded code, two's complement
                    b[2 * h] = __float_as_uint(z.x);
                    b[2 * h + 1] = __float_as_uint(z.y);
                }
                const uint32_t lo = low_bytes(b[0], b[2], b[4], b[6]);   // codes of k = 0, 2, 4, 6
                const uint32_t hi = low_bytes(b[1], b[3], b[5], b[7]);   // codes of k = 1, 3, 5, 7
                pk[w] = (lo & 0x0F0F0F0Fu) | ((hi << 4) & 0xF0F0F0F0u);
                q8[2 * w] = lo;
                q8[2 * w + 1] = hi;
            }
        }
        uint4* dq = reinterpret_cast<uint4*>(p.qX + (size_t)r * (K / 2) + (size_t)t * 32);
        dq[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        dq[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        uint4* d8 = reinterpret_cast<uint4*>(p.qX8 + (size_t)r * K + (size_t)t * 64);
#pragma unroll
        for (int i = 0; i < 4; ++i) d8[i] = make_uint4(q8[4 * i], q8[4 * i + 1], q8[4 * i + 2], q8[4 * i + 3]);
        if (t == 0) p.scale_t[r] = scale;
        named_bar(bar_id, T);   // red[] reused by the next row
    }
}

// Packed INT4 rows -> int8 GEMM operand rows (same k order as smooth_quant_kernel).
__global__ void expand_kernel(const uint8_t* qX, int8_t* qX8, size_t nwords) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < nwords; i += (size_t)gridDim.x * blockDim.x) {
        const uint32_t w = reinterpret_cast<const uint32_t*>(qX)[i];
        uint32_t lo = w & 0x0F0F0F0Fu;
        uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;
        lo |= (lo & 0x08080808u) * 0x1Eu;   // sign-extend each nibble to its byte
        hi |= (hi & 0x08080808u) * 0x1Eu;
        reinterpret_cast<uint2*>(qX8)[i] = make_uint2(lo, hi);
    }
}

// Packed INT4 weight rows -> int8 operand rows holding 16 q (the nibble in
// the high half of each byte), in the k order of expand_kernel.  The GEMM's
// epilogue expects the factor 16 on the weight side.
__global__ void expand_weights_kernel(const uint8_t* qW, int8_t* qW8, size_t nwords) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < nwords; i += (size_t)gridDim.x * blockDim.x) {
        const uint32_t w = reinterpret_cast<const uint32_t*>(qW)[i];
        reinterpret_cast<uint2*>(qW8)[i] = make_uint2((w << 4) & 0xF0F0F0F0u, w & 0xF0F0F0F0u);
    }
}

// Self-test of div_markstein against the IEEE division, elementwise.
__global__ void divide_check_kernel(const float* a, const float* b, int n, float* q_fast, float* q_ieee) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        const float bb = b[i];
        const float y = __frcp_rn(bb);
        const float2 q = div_markstein(make_float2(a[i], a[i]), make_float2(-bb, -bb), make_float2(y, y));
        q_fast[i] = q.x;
        q_ieee[i] = __fdiv_rn(a[i], bb);
    }
}

template <int L>
static cudaError_t launch_rot(const RotArgs& a, int threads, int R, size_t smem, int nsm, cudaStream_t st) {
    auto kern = threads <= CTA ? rot_gather_kernel<L, CTA> : rot_gather_kernel<L, 512>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int grid = (a.rows + R - 1) / R;
    if (grid > nsm) grid = nsm;
    kern<<<grid, threads, smem, st>>>(a);
    return cudaGetLastError();
}

}  // namespace fast

bool prep_fast_supported(int K, int n) {
    return K % 2048 == 0 && K / 64 <= 512 && n >= 1 && n <= 8192;
}

size_t prep_fast_scratch_bytes(int M, int K) { return (size_t)M * K * 4; }

cudaError_t launch_prep_fast(const PrepFastLaunch& pl, cudaStream_t st) {
    using namespace fast;
    const int K = pl.K;
    const int T = K / E;
    int R = T <= CTA ? CTA / T : 1;
    const int threads = T * R;
    const size_t smem = (size_t)R * K * 4 + (size_t)R * 2 * K * 2;
    int L = 0;
    while ((1 << L) < pl.n) ++L;
    int dev = 0, nsm = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);

    cudaError_t e;
    if (!pl.unit_scales) {
        e = cudaMemsetAsync(pl.s, 0, sizeof(float) * (size_t)(K / pl.G), st);
        if (e != cudaSuccess) return e;
    }
    RotArgs ra;
    ra.X = reinterpret_cast<const __half*>(pl.X);
    ra.rows = pl.rows;
    ra.K = K;
    ra.G = pl.G;
    ra.c_n = pl.c_n;
    ra.perm = pl.perm;
    ra.xp = pl.scratch;
    ra.smax = pl.unit_scales ? nullptr : reinterpret_cast<uint32_t*>(pl.s);
    switch (L) {
#define RRS_ROT_CASE(LL) \
    case LL: e = launch_rot<LL>(ra, threads, R, smem, nsm, st); break;
        RRS_ROT_CASE(0) RRS_ROT_CASE(1) RRS_ROT_CASE(2) RRS_ROT_CASE(3) RRS_ROT_CASE(4)
        RRS_ROT_CASE(5) RRS_ROT_CASE(6) RRS_ROT_CASE(7) RRS_ROT_CASE(8) RRS_ROT_CASE(9)
        RRS_ROT_CASE(10) RRS_ROT_CASE(11) RRS_ROT_CASE(12) RRS_ROT_CASE(13)
#undef RRS_ROT_CASE
        default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;

    QuantArgs qa;
    qa.xp = pl.scratch;
    qa.rows = pl.rows;
    qa.K = K;
    qa.G = pl.G;
    qa.unit_scales = pl.unit_scales;
    qa.s = pl.s;
    qa.qX = pl.qX;
    qa.qX8 = pl.qX8;
    qa.scale_t = pl.scale_t;
    qa.s_unit_out = pl.unit_scales ? pl.s : nullptr;
    int grid = (pl.rows + R - 1) / R;
    if (grid > 4 * nsm) grid = 4 * nsm;
    if (threads <= CTA) smooth_quant_kernel<CTA><<<grid, threads, 0, st>>>(qa);
    else smooth_quant_kernel<512><<<grid, threads, 0, st>>>(qa);
    return cudaGetLastError();
}

cudaError_t launch_divide_check(const float* a, const float* b, int n, float* q_fast, float* q_ieee,
                                cudaStream_t st) {
    int blocks = (n + 255) / 256;
    if (blocks > 4096) blocks = 4096;
    if (blocks < 1) blocks = 1;
    fast::divide_check_kernel<<<blocks, 256, 0, st>>>(a, b, n, q_fast, q_ieee);
    return cudaGetLastError();
}

cudaError_t launch_expand(const uint8_t* qX, int8_t* qX8, int M, int K, cudaStream_t st) {
    const size_t nwords = (size_t)M * K / 8;
    int dev = 0, nsm = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    size_t blocks = (nwords + 255) / 256;
    if (blocks > (size_t)nsm * 8) blocks = (size_t)nsm * 8;
    fast::expand_kernel<<<(unsigned)blocks, 256, 0, st>>>(qX, qX8, nwords);
    return cudaGetLastError();
}

cudaError_t launch_expand_weights(const uint8_t* qW, int8_t* qW8, int N, int K, cudaStream_t st) {
    const size_t nwords = (size_t)N * K / 8;
    int dev = 0, nsm = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    size_t blocks = (nwords + 255) / 256;
    if (blocks > (size_t)nsm * 8) blocks = (size_t)nsm * 8;
    fast::expand_weights_kernel<<<(unsigned)blocks, 256, 0, st>>>(qW, qW8, nwords);
    return cudaGetLastError();
}

}  // namespace rrs
