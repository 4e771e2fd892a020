// rrs_act.cuh -- the activation kernel of the online path for K a multiple of
// 2048 (included by the files that instantiate it for each Hadamard size; the
// design is described in rrs_prep_fast.cu).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "rrs_device.cuh"
#include "rrs_internal.h"

namespace rrs {
namespace fast {

constexpr int E = 64;        // elements per thread
constexpr int LOGE = 6;
// Threads per CTA when T <= CTA: as many row teams as fit in 320 threads.  At
// K = 4096 that is 5 teams (2048 rows on 148 SMs: at most 3 rows per team and
// phase instead of 4 with 256 threads); 320 threads leave 204 registers each, and
// 5 row buffers with 3 staging slots fit in shared memory.
constexpr int CTA = 320;
constexpr int BIG = 512;     // threads per CTA of the forms for T > CTA (one row team)

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


// ---------------------------------------------------------------------------


// Gathers byte 0 of four words into one word: result byte i = byte 0 of w_i.
__device__ __forceinline__ uint32_t low_bytes(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3) {
    return __byte_perm(__byte_perm(w0, w1, 0x0040), __byte_perm(w2, w3, 0x0040), 0x5410);
}

// One 32-byte store (a whole L2 sector); the address must be 32-byte aligned.
__device__ __forceinline__ void st_v8(void* dst, uint32_t a, uint32_t b, uint32_t c, uint32_t d, uint32_t e,
                                      uint32_t f, uint32_t g, uint32_t h) {
    asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(dst), "r"(a), "r"(b), "r"(c), "r"(d),
                 "r"(e), "r"(f), "r"(g), "r"(h)
                 : "memory");
}

// Two codes (integers in [-8, 7], exact in e4m3) -> two e4m3 bytes: lo in
// the low byte, hi in the high byte.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
    unsigned short r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}



struct ActArgs {
    const __half* X;     // [rows, K]
    int rows, K, G, NG;
    float c_n;
    const int32_t* perm; // [K]
    int phase;           // bit 0: phase A (group maxima -> s), bit 1: phase B (quantise with s)
    int unit_scales;     // s := 1 (no phase A)
    float* s;            // [NG]: written by phase A (CTA 0), read when phase B runs alone
    uint8_t* qX;         // [rows, K/2]
    uint8_t* a8;         // GEMM operand [rows, K]: int8 codes in the packed kernel's k order, or
                         // e4m3 codes in natural k order (the kernel's E4M3 form)
    float* scale_t;      // [rows]
    float* partial;      // [gridDim.x, NG] per-CTA group maxima
    uint32_t* gbar;      // grid barrier state: arrival count, generation (zero-filled before first use)
    uint32_t* err;       // workspace error word
    uint64_t limit_ns;
    int nst;             // fp16 staging slots per team (2..4): rows in flight ahead of the one being rotated
};

// Rows of one CTA for a given K (T = K/64 threads per row).
__host__ __device__ constexpr int act_rows_per_cta(int K) { return (K / E) <= CTA ? CTA / (K / E) : 1; }
// Shared memory: R fp32 row buffers, R x nst fp16 staging rows, 256 words of
// group maxima / scales, R x 16 floats of row-max partials.
__host__ __device__ constexpr size_t act_smem_bytes(int K, int nst = 2) {
    return (size_t)act_rows_per_cta(K) * K * 4 + (size_t)nst * act_rows_per_cta(K) * K * 2 + 1024 +
           (size_t)act_rows_per_cta(K) * 64;
}
constexpr size_t kActSmemLimit = 227 * 1024;
// Most staging slots (2..4) that fit in shared memory.
inline int act_stages(int K) {
    int nst = 4;
    while (nst > 2 && act_smem_bytes(K, nst) > kActSmemLimit) --nst;
    return nst;
}

// Waits until at most `pending` of this thread's cp.async groups are in flight.
__device__ __forceinline__ void cp_async_wait_dyn(int pending) {
    if (pending >= 3) cp_async_wait<3>();
    else if (pending == 2) cp_async_wait<2>();
    else if (pending == 1) cp_async_wait<1>();
    else cp_async_wait<0>();
}


// Loads the staged fp16 row into v and runs every butterfly stage of the
// block Hadamard transform (no scaling).  On return v holds the elements in
// the layout of the last round (see store_natural); the row buffer holds
// intermediate values that only this thread's own positions will overwrite.
template <int L>
__device__ __forceinline__ void rotate_row(float2 (&v)[32], float* rowbuf, const __half* st, int tl, int T,
                                           int bar_id) {
    constexpr int NR = (L <= LOGE) ? 1 : (L <= 2 * LOGE ? 2 : 3);
    constexpr int A1 = L < LOGE ? L : LOGE;
    constexpr int A2 = (L - LOGE) < LOGE ? (L - LOGE) : LOGE;
    constexpr int A3 = L - 2 * LOGE;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint4 raw = *reinterpret_cast<const uint4*>(st + (size_t)(tl * 8 + (c ^ (tl & 7))) * 8);
        const __half2* h2 = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
        for (int q = 0; q < 4; ++q) v[c * 4 + q] = __half22float2(h2[q]);
    }
    stages<A1>(v);
    if constexpr (NR >= 2) {
#pragma unroll
        for (int i = 0; i < 32; i += 2)
            *reinterpret_cast<float4*>(rowbuf + swz(tl * E + 2 * i)) = make_float4(v[i].x, v[i].y, v[i + 1].x, v[i + 1].y);
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
}

// Writes v (in the last round's layout) to the row buffer in natural order,
// swizzled: element i at rowbuf[swz(i)].
template <int L>
__device__ __forceinline__ void store_natural(const float2 (&v)[32], float* rowbuf, int tl, int T) {
    constexpr int NR = (L <= LOGE) ? 1 : (L <= 2 * LOGE ? 2 : 3);
    constexpr int A2 = (L - LOGE) < LOGE ? (L - LOGE) : LOGE;
    constexpr int A3 = L - 2 * LOGE;
    if constexpr (NR == 1) {
#pragma unroll
        for (int i = 0; i < 32; i += 2)
            *reinterpret_cast<float4*>(rowbuf + swz(tl * E + 2 * i)) = make_float4(v[i].x, v[i].y, v[i + 1].x, v[i + 1].y);
    } else if constexpr (NR == 2) {
        rstore<LOGE, A2>(v, rowbuf, tl, T);
    } else {
        rstore<2 * LOGE, A3>(v, rowbuf, tl, T);
    }
}

template <int L, int MAXT, bool KEEP, bool E4M3>
__global__ void __launch_bounds__(MAXT) act_kernel(ActArgs p) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int K = p.K;
    const int T = K / E;
    const int R = blockDim.x / T;
    const int team = threadIdx.x / T;
    const int t = threadIdx.x % T;
    float* rowbufs = reinterpret_cast<float*>(smem_raw);
    float* rowbuf = rowbufs + (size_t)team * K;
    const int nst = p.nst;
    __half* stages0 = reinterpret_cast<__half*>(rowbufs + (size_t)R * K);
    __half* stage0 = stages0 + (size_t)team * nst * K;
    uint32_t* gsm = reinterpret_cast<uint32_t*>(stages0 + (size_t)R * nst * K);   // [256] group max bits, then s
    float* red = reinterpret_cast<float*>(gsm + 256) + team * 16;
    float* s_sm = reinterpret_cast<float*>(gsm);
    const int bar_id = 1 + team;
    const int stride = gridDim.x * R;
    const int r0 = blockIdx.x * R + team;
    // KEEP (every team owns at most one row, both phases run): phase B reuses the
    // rotated row that phase A leaves in the team's row buffer instead of loading
    // and rotating it again.  The host picks it, so each form is its own smaller kernel.
    constexpr bool keep = KEEP;
    const float2 c2 = make_float2(p.c_n, p.c_n);

    auto issue_row = [&](int r, int sb) {
        const __half* src = p.X + (size_t)r * K;
        __half* dst = stage0 + (size_t)sb * K;
        for (int u = t; u < K / 8; u += T) {
            const int owner = u >> 3;
            const int c = u & 7;
            cp_async16(dst + (size_t)(owner * 8 + (c ^ (owner & 7))) * 8, src + (size_t)u * 8);
        }
    };
    // X_rot of the staged row into the row buffer, natural order (c_n applied);
    // a barrier makes it visible to the team.
    auto rotate_into_rowbuf = [&](int sb) {
        const int tl = opaque(t);
        float2 v[32];
        rotate_row<L>(v, rowbuf, stage0 + (size_t)sb * K, tl, T, bar_id);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __fmul2_rn(v[i], c2);   // X_rot = c_n * v
        store_natural<L>(v, rowbuf, tl, T);
        named_bar(bar_id, T);
    };

    // The first nst - 1 rows of a pass in flight, one cp.async group each (empty
    // groups past the last row keep the group count uniform).
    auto prologue = [&]() {
        for (int q = 0; q < nst - 1; ++q) {
            const int r = r0 + q * stride;
            if (r < p.rows) issue_row(r, q);
            cp_async_commit();
        }
    };
    // Before rotating the it-th row of a pass: put row it + nst - 1 in flight and
    // wait for row it.
    auto advance = [&](int r, int it_) {
        const int rn = r + (nst - 1) * stride;
        if (rn < p.rows) issue_row(rn, (it_ + nst - 1) % nst);
        cp_async_commit();
        cp_async_wait_dyn(nst - 1);
        named_bar(bar_id, T);
    };

    // first rows in flight while the gather addresses are built
    int it = 0;
    const bool run_a = (p.phase & 1) != 0;
    if (run_a || !keep) prologue();
    for (int g = threadIdx.x; g < 256; g += blockDim.x) gsm[g] = 0u;

    // Gather addresses of this thread's outputs j in [64t, 64t + 64) (one group).
    // perm is staged through shared memory (`pst`, K int32): 16-byte global loads,
    // four in flight, and 16-byte chunk c stored at c ^ ((c >> 4) & 7) so that each
    // thread's 16 chunk reads below are bank-conflict free.
    uint32_t gaddr[32];
    auto build_gaddr = [&](int4* pst) {
        const int4* pg = reinterpret_cast<const int4*>(p.perm);
        for (int c0 = 0; c0 < K / 4; c0 += 4 * (int)blockDim.x) {
            int4 v[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int c = c0 + q * (int)blockDim.x + (int)threadIdx.x;
                if (c < K / 4) v[q] = __ldg(pg + c);
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int c = c0 + q * (int)blockDim.x + (int)threadIdx.x;
                if (c < K / 4) pst[c ^ ((c >> 4) & 7)] = v[q];
            }
        }
        __syncthreads();
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            const int c = t * 16 + q;
            const int4 v = pst[c ^ ((c >> 4) & 7)];
            gaddr[2 * q] = (uint32_t)swz(v.x) | ((uint32_t)swz(v.y) << 16);
            gaddr[2 * q + 1] = (uint32_t)swz(v.z) | ((uint32_t)swz(v.w) << 16);
        }
        __syncthreads();   // the staging space is reused
    };
    // Phase A without kept rows takes its maxima per channel (no gather per row),
    // and builds the gather addresses afterwards in the staging space.
    const bool colmax = run_a && !keep;
    if (!colmax) build_gaddr(reinterpret_cast<int4*>(rowbufs));
    auto gather = [&](float2 (&x)[32]) {
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            const uint32_t g0 = gaddr[2 * q], g1 = gaddr[2 * q + 1];
            x[2 * q] = make_float2(rowbuf[g0 & 0xFFFFu], rowbuf[g0 >> 16]);
            x[2 * q + 1] = make_float2(rowbuf[g1 & 0xFFFFu], rowbuf[g1 >> 16]);
        }
    };

    if (run_a) {
        // ------------------------------------------------------------- phase A
        // Per row: rotate, reorder (gather), and keep the largest |X'| of this
        // thread's outputs, all of which lie in one group (64 | G).
        float gmx = 0.0f;
        if (keep) {
            // one row per team: rotate into the row buffer (kept for phase B), gather
            for (int r = r0; r < p.rows; r += stride, ++it) {
                advance(r, it);
                rotate_into_rowbuf(it % nst);
                float2 x[32];
                gather(x);
#pragma unroll
                for (int i = 0; i < 32; ++i) gmx = fmaxf(gmx, fmaxf(fabsf(x[i].x), fabsf(x[i].y)));
            }
            cp_async_wait<0>();
        } else {
            // Per row only the rotation; each register keeps the largest |v| of its
            // channel over this thread's rows (v the unscaled transform: fl(c_n |v|)
            // is monotone in |v|, so scaling the maximum once gives the same bits).
            float2 cm[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) cm[i] = make_float2(0.0f, 0.0f);
            for (int r = r0; r < p.rows; r += stride, ++it) {
                advance(r, it);
                const int tl = opaque(t);
                float2 v[32];
                rotate_row<L>(v, rowbuf, stage0 + (size_t)(it % nst) * K, tl, T, bar_id);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    cm[i].x = fmaxf(cm[i].x, fabsf(v[i].x));
                    cm[i].y = fmaxf(cm[i].y, fabsf(v[i].y));
                }
                named_bar(bar_id, T);   // row buffer and staging free for the next row
            }
            cp_async_wait<0>();
            __syncthreads();
            // channel maxima in natural order (swizzled) in every team's buffer, then
            // the CTA's maxima in team 0's buffer (same swizzle: combine position-wise)
            store_natural<L>(cm, rowbuf, opaque(t), T);
            __syncthreads();
            if (R > 1) {
                for (int c = threadIdx.x; c < K; c += blockDim.x) {
                    float m = rowbufs[c];
                    for (int q = 1; q < R; ++q) m = fmaxf(m, rowbufs[(size_t)q * K + c]);
                    rowbufs[c] = m;
                }
                __syncthreads();
            }
            build_gaddr(reinterpret_cast<int4*>(stages0));
            if (team == 0) {
                float2 x[32];
                gather(x);
#pragma unroll
                for (int i = 0; i < 32; ++i) gmx = fmaxf(gmx, fmaxf(x[i].x, x[i].y));
                gmx = __fmul_rn(gmx, p.c_n);
            }
            if (p.phase & 2) {
                // phase B's first rows in flight across the grid barrier
                __syncthreads();
                prologue();
            }
        }
        // threads of one group are consecutive (G / 64 of them): shuffle-reduce
        // within aligned power-of-two segments, one shared atomic per segment
        {
            const int gsz = p.G / E;
            const int seg = (gsz & -gsz) < 32 ? (gsz & -gsz) : 32;
            for (int o = seg >> 1; o > 0; o >>= 1) gmx = fmaxf(gmx, __shfl_xor_sync(0xffffffffu, gmx, o));
            if ((t % seg) == 0 && gmx > 0.0f) atomicMax(&gsm[(t * E) / p.G], __float_as_uint(gmx));
        }
        __syncthreads();
        for (int g = threadIdx.x; g < p.NG; g += blockDim.x) {
            p.partial[(size_t)blockIdx.x * p.NG + g] = __uint_as_float(gsm[g]);
            gsm[g] = 0u;
        }
        if (!grid_barrier(p.gbar, p.err, p.limit_ns)) return;
        // s[g] = max over the CTAs' rows of the table: thread i takes group i % NG and every
        // slices-th CTA from i / NG, eight independent loads at a time, then a shared max
        {
            const int slices = (int)blockDim.x >= p.NG ? (int)blockDim.x / p.NG : 1;
            const int g = threadIdx.x % p.NG;
            const int sl = threadIdx.x / p.NG;
            if (sl < slices) {
                float mx[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) mx[q] = 0.0f;
                int b = sl;
                for (; b + 7 * slices < (int)gridDim.x; b += 8 * slices) {
#pragma unroll
                    for (int q = 0; q < 8; ++q) mx[q] = fmaxf(mx[q], __ldcg(p.partial + (size_t)(b + q * slices) * p.NG + g));
                }
                for (; b < (int)gridDim.x; b += slices) mx[0] = fmaxf(mx[0], __ldcg(p.partial + (size_t)b * p.NG + g));
                float m = mx[0];
#pragma unroll
                for (int q = 1; q < 8; ++q) m = fmaxf(m, mx[q]);
                if (m > 0.0f) atomicMax(&gsm[g], __float_as_uint(m));
            }
            __syncthreads();
            if (blockIdx.x == 0)
                for (int g2 = threadIdx.x; g2 < p.NG; g2 += blockDim.x) p.s[g2] = s_sm[g2];
        }
    } else {
        for (int g = threadIdx.x; g < p.NG; g += blockDim.x) {
            const float v = p.unit_scales ? 1.0f : p.s[g];
            s_sm[g] = v;
            if (p.unit_scales && blockIdx.x == 0) p.s[g] = 1.0f;
        }
    }
    if (!(p.phase & 2)) return;
    __syncthreads();
    // the GEMM that reads this kernel's outputs may start launching (it waits for
    // this kernel's completion before reading them)
    grid_dependents_launch();

    // --------------------------------------------------------------- phase B
    it = 0;
    float d = s_sm[(t * E) / p.G];
    if (d == 0.0f) d = 1.0f;
    const float yd = __frcp_rn(d);
    const float2 nd2 = make_float2(-d, -d), yd2 = make_float2(yd, yd);
    constexpr float kMagic = 12582912.0f;   // 1.5 * 2^23: adding it rounds to an integer, half to even
    const float2 magic2 = make_float2(kMagic, kMagic);
    const bool divide = !p.unit_scales;
    const bool v8_out = ((reinterpret_cast<uintptr_t>(p.qX) | reinterpret_cast<uintptr_t>(p.a8)) & 31u) == 0;

    for (int r = r0; r < p.rows; r += stride, ++it) {
        if (!keep) {
            advance(r, it);
            rotate_into_rowbuf(it % nst);
        }
        // gather X'[j] = X_rot[perm[j]], smooth, per-thread max
        float2 x[32];
        gather(x);
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if (divide) x[i] = div_markstein(x[i], nd2, yd2);
            amax = fmaxf(amax, fmaxf(fabsf(x[i].x), fabsf(x[i].y)));
        }
        const float tmx = amax;   // this thread's max |x~|
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        if ((t & 31) == 0) red[t >> 5] = amax;
        named_bar(bar_id, T);     // also: every thread of the team has gathered from the row buffer
        amax = red[0];
        for (int w = 1; w < T / 32; ++w) amax = fmaxf(amax, red[w]);
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
                uint32_t e8[4];
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
                    if (E4M3) {
                        const float2 cv = __fadd2_rn(z, make_float2(-kMagic, -kMagic));   // the code as an exact float
                        e8[h] = e4m3x2(cv.x, cv.y);
                    }
                }
                const uint32_t lo = low_bytes(b[0], b[2], b[4], b[6]);   // codes of k = 0, 2, 4, 6
                const uint32_t hi = low_bytes(b[1], b[3], b[5], b[7]);   // codes of k = 1, 3, 5, 7
                pk[w] = (lo & 0x0F0F0F0Fu) | ((hi << 4) & 0xF0F0F0F0u);
                if (E4M3) {
                    q8[2 * w] = e8[0] | (e8[1] << 16);
                    q8[2 * w + 1] = e8[2] | (e8[3] << 16);
                } else {
                    q8[2 * w] = lo;
                    q8[2 * w + 1] = hi;
                }
            }
        }
        // whole 32-byte sectors per store where the bases allow it (K / 2 and the
        // thread offsets are multiples of 32)
        unsigned char* dqp = p.qX + (size_t)r * (K / 2) + (size_t)t * 32;
        unsigned char* d8p = p.a8 + (size_t)r * K + (size_t)t * 64;
        if (v8_out) {
            st_v8(dqp, pk[0], pk[1], pk[2], pk[3], pk[4], pk[5], pk[6], pk[7]);
            st_v8(d8p, q8[0], q8[1], q8[2], q8[3], q8[4], q8[5], q8[6], q8[7]);
            st_v8(d8p + 32, q8[8], q8[9], q8[10], q8[11], q8[12], q8[13], q8[14], q8[15]);
        } else {
            uint4* dq = reinterpret_cast<uint4*>(dqp);
            dq[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            dq[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            uint4* d8 = reinterpret_cast<uint4*>(d8p);
#pragma unroll
            for (int i = 0; i < 4; ++i) d8[i] = make_uint4(q8[4 * i], q8[4 * i + 1], q8[4 * i + 2], q8[4 * i + 3]);
        }
        if (t == 0) p.scale_t[r] = scale;
    }
    cp_async_wait<0>();
}

// The launch for Hadamard size 2^L: picks the kernel form (threads, KEEP, E4M3).
template <int L>
cudaError_t launch_act(const ActArgs& a, bool e4m3, int threads, size_t smem, int grid_cap, cudaStream_t st) {
    const int nsm = device_sm_count();
    const int R = threads / (a.K / E);
    int grid = (a.rows + R - 1) / R;
    const bool big = threads > CTA;
    if (threads > BIG) return cudaErrorInvalidConfiguration;
    // occupancy is 1 CTA per SM for every form (shared memory); checked below
    if (grid > nsm) grid = nsm;
    if (grid > grid_cap) grid = grid_cap;
    const bool keep = (a.phase & 3) == 3 && grid * R >= a.rows;
    const int form = (big ? 4 : 0) + (keep ? 2 : 0) + (e4m3 ? 1 : 0);
    using K_t = void (*)(ActArgs);
    static const K_t kerns[8] = {
        act_kernel<L, CTA, false, false>, act_kernel<L, CTA, false, true>,
        act_kernel<L, CTA, true, false>, act_kernel<L, CTA, true, true>,
        act_kernel<L, BIG, false, false>, act_kernel<L, BIG, false, true>,
        act_kernel<L, BIG, true, false>, act_kernel<L, BIG, true, true>};
    static KernelSetup setup[8];
    const K_t kern = kerns[form];
    int occ = 0;
    cudaError_t e = kernel_setup(reinterpret_cast<const void*>(kern), threads, smem, setup[form], &occ);
    if (e != cudaSuccess) return e;
    if (occ < 1) return cudaErrorInvalidConfiguration;
    if (grid > occ * nsm) grid = occ * nsm;
    if (!(a.phase & 1)) {
        // quantisation alone (given scales): no grid-wide barrier, a plain launch
        kern<<<grid, threads, smem, st>>>(a);
        return cudaGetLastError();
    }
    ActArgs args = a;
    void* params[] = {&args};
    // all CTAs must be resident together: the phases meet at a grid-wide barrier
    return cudaLaunchCooperativeKernel(reinterpret_cast<void*>(kern), dim3(grid), dim3(threads), params, smem, st);
}

}  // namespace fast
}  // namespace rrs
