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
//   phase 1  rotation: (token, channel chunk) items spread over teams of the
//            CTAs; the normalised Hadamard transform of each block (fp32, stages
//            h = 1, 2, 4, ... with the pair (a + b, a - b), then one multiply by
//            c_n) in rounds of four stages on sixteen registers per thread with
//            shared-memory exchanges between rounds; X_rot goes to the
//            workspace, and each item's largest |X_rot| per group of the reorder
//            (every channel's group comes from inverting the reorder index once
//            per CTA) to a table;                           -- grid barrier
//   phase 2  every CTA reads the table: m[t][g] = max |X'| of token t in group
//            g, so s_g = max_t m[t][g] and, division being monotone, the
//            per-token maximum after smoothing is max_g m[t][g] / s_g, whence
//            scale_t = amax_t / 7; then the INT4 codes
//            q = clamp(rint((X' / s_g) / scale_t), -8, 7) of the channel chunks
//            this CTA multiplies (into shared memory) and of the groups it owns
//            (to qX);
//   phase 3  the group-scaled contraction over work units of 16 output
//            channels x 1024 input channels.  A warp loads its unit's packed
//            weights straight into registers (the next unit's halves in flight
//            while it multiplies this one), turns eight packed codes into two
//            int8x4 words holding 16 * code with one shift and two ANDs (no
//            sign extension needed), and multiplies on the tensor cores with
//            mma.sync m16n8k32 (weights as the 16-row operand, tokens as the
//            8 columns).  Each group's exact sum 256 * P_g is shifted back and
//            promoted, acc += s_g * P_g, in group order; a unit's sums go to
//            the workspace;                                 -- grid barrier
//   phase 4  every thread of the grid takes outputs: the chunk sums added in
//            chunk order, times scale_t * scale_w.
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
constexpr int KC = 1024;                      // input channels per work unit
constexpr int kBlocksPerUnit = KC / 128;      // 128-channel MMA blocks per unit
constexpr int kHalfBlocks = kBlocksPerUnit / 2;
constexpr int kActWords = KC / 8;             // 8-channel words per token row of a staged chunk
constexpr int kActStride = kActWords * 8 + 16;  // bytes per token row: (even, odd) word pairs + pad
constexpr int kMaxSlots = 4;                  // code chunks staged per CTA
constexpr int kMaxTokens = 16;
constexpr int kEl = 16;                       // elements per thread in the rotation
constexpr int kMaxChunk = kEl * kThreads;     // channels rotated by one CTA at a time
constexpr int kMinChunk = 1024;
constexpr int kMaxGroups = 256;               // K / G (group ids fit a byte)
constexpr int kMaxK = 32768;
constexpr int kMaxCtas = 1024;
constexpr int kPrefetchUnits = 24;            // units per CTA asked of L2 up front

// shared memory: rotation buffers | group of each channel | staged codes |
// per-team group maxima | divisors, token scales, reduction scratch
constexpr int kPadChunk = kMaxChunk + kMaxChunk / 32;   // rotation buffers, one pad word per 32
constexpr size_t kOffGrp = (size_t)kPadChunk * 4;
constexpr size_t kOffAct = kOffGrp + kMaxK;
constexpr size_t kOffGmx = kOffAct + (size_t)kMaxSlots * kMaxTokens * kActStride;
constexpr size_t kOffPerm = kOffGmx + (size_t)kWarps * kMaxGroups * 4;
constexpr int kMaxOwned = 2;                  // groups per CTA whose packed codes it writes
constexpr int kMaxG = KC;
constexpr size_t kOffS = kOffPerm + (size_t)(kMaxSlots * KC + kMaxOwned * kMaxG) * 4;
constexpr size_t kSmemBytes = kOffS + (size_t)(2 * kMaxGroups + 2 * kMaxTokens) * 4;

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
    float* gtab;    // [M, K / L, NG] largest |X_rot| of each rotation item per group
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
// group's divisor (s_g, or 1 where s_g == 0) with yd = RN(1/sd), sc the token's
// scale with ysc = RN(1/sc).  Both divisions are the correctly rounded quotients
// (Markstein's correction, as in the activation kernel); round half to even.
__device__ __forceinline__ int code_of(float x, float sd, float yd, float sc, float ysc) {
    if (sc == 0.0f) return 0;
    const float z = div_markstein(div_markstein(x, -sd, yd), -sc, ysc);
    const int q = __float2int_rn(z);
    return q < -8 ? -8 : (q > 7 ? 7 : q);
}

// dst[0..count) = src[0..count) (count a multiple of 4, both 16-byte aligned):
// 16-byte loads, eight in flight per thread.
__device__ __forceinline__ void copy_i32(int* dst, const int32_t* src, int count) {
    const int4* s4 = reinterpret_cast<const int4*>(src);
    int4* d4 = reinterpret_cast<int4*>(dst);
    const int n4 = count / 4;
    for (int b = threadIdx.x; b < n4; b += blockDim.x * 8) {
        int4 v[8];
#pragma unroll
        for (int q = 0; q < 8; ++q)
            if (b + q * (int)blockDim.x < n4) v[q] = __ldg(s4 + b + q * blockDim.x);
#pragma unroll
        for (int q = 0; q < 8; ++q)
            if (b + q * (int)blockDim.x < n4) d4[b + q * blockDim.x] = v[q];
    }
}

// Element r (0..15) of a thread in a rotation round that covers index bits
// [b0, b0 + nb) of an item of 2^lgL channels: the round's bits come from r's low
// nb bits, every other bit from (thread, r's high bits).
__device__ __forceinline__ int rot_index(int b0, int nb, int tt, int r) {
    const int lo = r & ((1 << nb) - 1);
    const int other = (tt << (4 - nb)) | (r >> nb);
    return ((other >> b0) << (b0 + nb)) | (lo << b0) | (other & ((1 << b0) - 1));
}

// Buffer position of element i: one pad word after every 32, so that the
// power-of-two strides of the rounds fall on different banks.
__device__ __forceinline__ int padi(int i) { return i + (i >> 5); }

// The thread's sixteen elements to / from the buffer in a round's layout; a
// full round (nb = 4) holds elements base + r * 2^b0.
__device__ __forceinline__ void store_round(float* tb, const float (&v)[kEl], int b0, int nb, int tt) {
    if (nb == 4) {
        const int base = ((tt >> b0) << (b0 + 4)) | (tt & ((1 << b0) - 1));
#pragma unroll
        for (int r = 0; r < kEl; ++r) tb[padi(base + (r << b0))] = v[r];
    } else {
#pragma unroll
        for (int r = 0; r < kEl; ++r) tb[padi(rot_index(b0, nb, tt, r))] = v[r];
    }
}
__device__ __forceinline__ void load_round(const float* tb, float (&v)[kEl], int b0, int nb, int tt) {
    if (nb == 4) {
        const int base = ((tt >> b0) << (b0 + 4)) | (tt & ((1 << b0) - 1));
#pragma unroll
        for (int r = 0; r < kEl; ++r) v[r] = tb[padi(base + (r << b0))];
    } else {
#pragma unroll
        for (int r = 0; r < kEl; ++r) v[r] = tb[padi(rot_index(b0, nb, tt, r))];
    }
}

// The butterfly stages of one round on the thread's sixteen elements: stage k
// pairs r and r + 2^k (index bit b0 + k), lower index first.
__device__ __forceinline__ void rot_stages(float (&v)[kEl], int nb) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        if (k < nb) {
#pragma unroll
            for (int r = 0; r < kEl; ++r) {
                if (!(r & (1 << k))) {
                    const float a = v[r], b = v[r + (1 << k)];
                    v[r] = __fadd_rn(a, b);
                    v[r + (1 << k)] = __fsub_rn(a, b);
                }
            }
        }
    }
}

// TWO: more than 8 tokens (a second 8-column MMA tile); a separate form keeps
// the one-token kernel smaller (its code runs once per launch, fetched cold).
template <bool TWO>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const Args p) {
    extern __shared__ __align__(16) unsigned char smem[];
    float* xbuf = reinterpret_cast<float*>(smem);                       // [kPadChunk]
    uint8_t* grp = smem + kOffGrp;                                      // [K] group of each channel
    uint8_t* act = smem + kOffAct;                                      // [slots][16][kActStride]
    uint32_t* gmx = reinterpret_cast<uint32_t*>(smem + kOffGmx);        // [warps][kMaxGroups]
    int* pslot = reinterpret_cast<int*>(smem + kOffPerm);               // perm of the staged chunks
    int* pown = pslot + kMaxSlots * KC;                                 // perm of the owned groups
    float* s_sm = reinterpret_cast<float*>(smem + kOffS);               // [NG] divisors
    float* ys_sm = s_sm + kMaxGroups;                                   // [NG] their reciprocals
    float* sc_sm = ys_sm + kMaxGroups;                                  // [16] scale_t
    float* ysc_sm = sc_sm + kMaxTokens;                                 // [16] their reciprocals

    const int tid = threadIdx.x;
    const int K = p.K, M = p.M, N = p.N, G = p.G;
    const int NG = K / G;
    const int Kh = K / 2;
    const int L = p.L;
    const int per_row = K / L;

    // this CTA's work units (chunk-major: u = kc * RT + rt), the chunks they span
    const int u0 = (int)((long long)blockIdx.x * p.U / gridDim.x);
    const int u1 = (int)((long long)(blockIdx.x + 1) * p.U / gridDim.x);
    const int kc_first = u0 / p.RT;

    // ---- phase 0: start the weight stream (L2 prefetch) and invert the reorder: channel perm[j] of the rotated row lies in group j / G
    {
        // the activation rows of this CTA's first rotation items, then weights
        {
            const int L0 = L, T0 = L0 / kEl, R0 = kThreads / T0;
            const int it0 = blockIdx.x * R0 + tid;
            if (tid < R0 && it0 < M * per_row)
                prefetch_l2(p.X + (size_t)(it0 / per_row) * K + (size_t)(it0 % per_row) * L0, (uint32_t)L0 * 2);
        }
        const int npf = min(u1 - u0, kPrefetchUnits);
        for (int e = tid; e < npf * 16; e += kThreads) {
            const int u = u0 + e / 16;
            const int row = (u % p.RT) * 16 + (e % 16);
            prefetch_l2(p.qW + (size_t)row * Kh + (size_t)(u / p.RT) * (KC / 2), KC / 2);
        }
        const int4* p4 = reinterpret_cast<const int4*>(p.perm);
        for (int b = tid; b < K / 4; b += kThreads * 8) {
            int4 v[8];
#pragma unroll
            for (int q = 0; q < 8; ++q)
                if (b + q * kThreads < K / 4) v[q] = __ldg(p4 + b + q * kThreads);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int c4 = b + q * kThreads;
                if (c4 < K / 4) {
                    const int vv[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
                    for (int w = 0; w < 4; ++w)
                        if ((unsigned)vv[w] < (unsigned)K) grp[vv[w]] = (uint8_t)((4 * c4 + w) / G);
                }
            }
        }
        // the reorder index of the chunks this CTA multiplies and of the groups it owns
        const int nslot = u1 > u0 ? (u1 - 1) / p.RT - kc_first + 1 : 0;
        copy_i32(pslot, p.perm + (size_t)kc_first * KC, nslot * KC);
        for (int k = 0; k < kMaxOwned && (int)blockIdx.x + k * (int)gridDim.x < NG; ++k)
            copy_i32(pown + k * G, p.perm + (size_t)(blockIdx.x + k * gridDim.x) * G, G);
        __syncthreads();
    }

    // ---- phase 1: rotation of (token, chunk of L channels) items by teams of L/16 threads
    {
        const int T = L / kEl;
        const int R = kThreads / T;
        const int team = tid / T, tt = tid % T;
        float* tb = xbuf + (size_t)team * (L + L / 32);
        const int wpt = T / 32;                                  // warps per team
        uint32_t* wg = gmx + (size_t)(tid >> 5) * kMaxGroups;    // this warp's group maxima
        const int lgL = 31 - __clz(L);
        const int lgn = 31 - __clz(p.n);
        const int rounds = (lgn + 3) / 4;
        const int items = M * per_row;
        for (int item = blockIdx.x * R + team; item - team < items; item += gridDim.x * R) {
            // (every team of the CTA runs the same number of iterations; a team past
            // the last item only keeps its barriers)
            const bool live = item < items;
            const int t = live ? item / per_row : 0;
            const int chunk = live ? item % per_row : 0;
            for (int g = tid & 31; g < NG; g += 32) wg[g] = 0u;
            float v[kEl];
            if (live) {
                const __half* xs = p.X + (size_t)t * K + (size_t)chunk * L + tt * kEl;
                const uint4 h0 = *reinterpret_cast<const uint4*>(xs);
                const uint4 h1 = *reinterpret_cast<const uint4*>(xs + 8);
                const __half2* a = reinterpret_cast<const __half2*>(&h0);
                const __half2* b = reinterpret_cast<const __half2*>(&h1);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float2 fa = __half22float2(a[q]), fb = __half22float2(b[q]);
                    v[2 * q] = fa.x;
                    v[2 * q + 1] = fa.y;
                    v[8 + 2 * q] = fb.x;
                    v[8 + 2 * q + 1] = fb.y;
                }
            } else {
#pragma unroll
                for (int r = 0; r < kEl; ++r) v[r] = 0.0f;
            }
            // rounds of up to four stages; between rounds the elements move through
            // the team's buffer to the next round's layout
            int b0 = 0, nb = 4;
            for (int rd = 0; rd < rounds; ++rd) {
                const int nb_r = min(4, lgn - 4 * rd);
                if (rd > 0) {
                    store_round(tb, v, b0, nb, tt);
                    named_bar(1 + team, T);
                    b0 = 4 * rd;
                    nb = nb_r;
                    load_round(tb, v, b0, nb, tt);
                    named_bar(1 + team, T);
                } else {
                    nb = 4;   // the loaded layout: sixteen consecutive channels
                }
                // round rd's stages cover bits [4 rd, 4 rd + nb_r)
                rot_stages(v, nb_r);
            }
            // X_rot = c_n * v, natural order through the buffer
#pragma unroll
            for (int r = 0; r < kEl; ++r) v[r] = __fmul_rn(v[r], p.c_n);
            store_round(tb, v, b0, nb, tt);
            named_bar(1 + team, T);
            if (live) {
                float* xr = p.Xr + (size_t)t * K + (size_t)chunk * L;
                const uint8_t* gc = grp + (size_t)chunk * L;
                for (int c = tt * 4; c < L; c += T * 4) {
                    const int pc = padi(c);   // c .. c + 3 lie in one 32-word run
                    const float4 x4 = make_float4(tb[pc], tb[pc + 1], tb[pc + 2], tb[pc + 3]);
                    *reinterpret_cast<float4*>(xr + c) = x4;
                    atomicMax(wg + gc[c], __float_as_uint(fabsf(x4.x)));
                    atomicMax(wg + gc[c + 1], __float_as_uint(fabsf(x4.y)));
                    atomicMax(wg + gc[c + 2], __float_as_uint(fabsf(x4.z)));
                    atomicMax(wg + gc[c + 3], __float_as_uint(fabsf(x4.w)));
                }
            }
            named_bar(1 + team, T);
            if (live) {
                // the team's maxima: the largest over its warps' private copies
                float* gt = p.gtab + ((size_t)t * per_row + chunk) * NG;
                const uint32_t* w0 = gmx + (size_t)(team * wpt) * kMaxGroups;
                for (int g = tt; g < NG; g += T) {
                    uint32_t m = w0[g];
                    for (int w = 1; w < wpt; ++w) m = max(m, w0[(size_t)w * kMaxGroups + g]);
                    gt[g] = __uint_as_float(m);
                }
            }
            named_bar(1 + team, T);
        }
    }
    if (!grid_barrier(p.gbar, p.err, p.limit_ns)) return;

    // ---- phase 2: m[t][g] = max |X'| of token t over group g (every CTA); s_g =
    // max_t m[t][g]; amax_t = max_g m[t][g] / s_g (RN division is monotone);
    // scale_t = amax_t / 7; then the codes this CTA needs
    {
        float* mt = xbuf;   // [M][NG]
        for (int e = tid; e < M * NG; e += kThreads) {
            const int t = e / NG, g = e % NG;
            const float* gp = p.gtab + (size_t)t * per_row * NG + g;
            float m = 0.0f;
            int c = 0;
            for (; c + 8 <= per_row; c += 8) {
                float w[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) w[q] = __ldcg(gp + (size_t)(c + q) * NG);
#pragma unroll
                for (int q = 0; q < 8; ++q) m = fmaxf(m, w[q]);
            }
            for (; c < per_row; ++c) m = fmaxf(m, __ldcg(gp + (size_t)c * NG));
            mt[e] = m;
        }
        __syncthreads();
        for (int g = tid; g < NG; g += kThreads) {
            float sg = 0.0f;
            for (int t = 0; t < M; ++t) sg = fmaxf(sg, mt[t * NG + g]);
            if (p.unit_scales) sg = 1.0f;
            const float sd = sg == 0.0f ? 1.0f : sg;
            s_sm[g] = sd;
            ys_sm[g] = __frcp_rn(sd);
            if (blockIdx.x == 0) p.s[g] = sg;
        }
        __syncthreads();
        const int warp = tid >> 5, lane = tid & 31;
        if (warp < M) {
            float a = 0.0f;
            for (int g = lane; g < NG; g += 32) a = fmaxf(a, __fdiv_rn(mt[warp * NG + g], s_sm[g]));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
            if (lane == 0) {
                const float sc = __fdiv_rn(a, 7.0f);
                sc_sm[warp] = sc;
                ysc_sm[warp] = sc == 0.0f ? 0.0f : __frcp_rn(sc);
                if (blockIdx.x == 0) p.scale_t[warp] = sc;
            }
        }
        __syncthreads();
        // Staged chunks, as the tensor cores' column operand: per token and 8-channel
        // word, the codes of the even channels and of the odd ones as int8x4 words of
        // 16 * code.  A thread takes one word and four tokens (all loads at once).
        const int nslot = u1 > u0 ? (u1 - 1) / p.RT - kc_first + 1 : 0;
        constexpr int TOK = TWO ? 16 : 8;
        constexpr int NQ = TOK / 4;                // token subsets per staged word
        for (int e = tid; e < nslot * kActWords * 4; e += kThreads) {
            const int wi = e % kActWords;
            const int tq = (e / kActWords) % 4;
            const int sl = e / (kActWords * 4);
            const int j0 = (kc_first + sl) * KC + 8 * wi;
            const int4 pa = *reinterpret_cast<const int4*>(pslot + sl * KC + 8 * wi);
            const int4 pb = *reinterpret_cast<const int4*>(pslot + sl * KC + 8 * wi + 4);
            const int src[8] = {pa.x, pa.y, pa.z, pa.w, pb.x, pb.y, pb.z, pb.w};
            const float sd = s_sm[j0 / G], yd = ys_sm[j0 / G];
            float x[NQ][8];
#pragma unroll
            for (int q = 0; q < NQ; ++q) {
                const int t = tq + 4 * q;
#pragma unroll
                for (int c = 0; c < 8; ++c) x[q][c] = t < M ? __ldcg(p.Xr + (size_t)t * K + src[c]) : 0.0f;
            }
#pragma unroll
            for (int q = 0; q < NQ; ++q) {
                const int t = tq + 4 * q;
                uint32_t ev = 0, od = 0;
                if (t < M) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        ev |= ((uint32_t)(code_of(x[q][2 * c], sd, yd, sc_sm[t], ysc_sm[t]) << 4) & 0xF0u) << (8 * c);
                        od |= ((uint32_t)(code_of(x[q][2 * c + 1], sd, yd, sc_sm[t], ysc_sm[t]) << 4) & 0xF0u) << (8 * c);
                    }
                }
                *reinterpret_cast<uint2*>(act + ((size_t)sl * kMaxTokens + t) * kActStride + 8 * wi) = make_uint2(ev, od);
            }
        }
        // packed codes of this CTA's share of the groups (the layer's qX output)
        for (int k = 0; k < kMaxOwned && (int)blockIdx.x + k * (int)gridDim.x < NG; ++k) {
            const int g = blockIdx.x + k * gridDim.x;
            for (int e = tid; e < M * (G / 2); e += kThreads) {
                const int t = e / (G / 2);
                const int jj = 2 * (e % (G / 2));
                const float* xr = p.Xr + (size_t)t * K;
                const float sd = s_sm[g], yd = ys_sm[g];
                const int q0 = code_of(__ldcg(xr + pown[k * G + jj]), sd, yd, sc_sm[t], ysc_sm[t]);
                const int q1 = code_of(__ldcg(xr + pown[k * G + jj + 1]), sd, yd, sc_sm[t], ysc_sm[t]);
                p.qX[(size_t)t * Kh + (g * G + jj) / 2] = (uint8_t)((uint32_t)(q0 & 15) | ((uint32_t)(q1 & 15) << 4));
            }
        }
        __syncthreads();
    }

    // ---- phase 3: group-scaled contraction of the units
    {
        const int warp = tid >> 5, lane = tid & 31;
        const int gq = lane >> 2, tq = lane & 3;
        const int gpb = G / 128;                   // MMA blocks per group (G divides KC)
        constexpr bool two = TWO;
        // A unit's weights in two register halves (blocks 0-3, 4-7): rows gq (a) and
        // gq + 8 (b) of the tile.  The next unit's halves are loaded as soon as this
        // unit's are used.
        uint4 a0[kHalfBlocks], b0[kHalfBlocks], a1[kHalfBlocks], b1[kHalfBlocks];
        auto load_half = [&](int uu, int h, uint4 (&A)[kHalfBlocks], uint4 (&B)[kHalfBlocks]) {
            const uint8_t* wr = p.qW + (size_t)((uu % p.RT) * 16 + gq) * Kh + (size_t)(uu / p.RT) * (KC / 2) +
                                16 * tq + 64 * kHalfBlocks * h;
#pragma unroll
            for (int i = 0; i < kHalfBlocks; ++i) {
                A[i] = __ldcs(reinterpret_cast<const uint4*>(wr + 64 * i));
                B[i] = __ldcs(reinterpret_cast<const uint4*>(wr + (size_t)8 * Kh + 64 * i));
            }
        };
        int u = u0 + warp;
        if (u < u1) {
            load_half(u, 0, a0, b0);
            load_half(u, 1, a1, b1);
        }
        for (; u < u1; u += kWarps) {
            const int kc = u / p.RT, rt = u % p.RT;
            const int un = u + kWarps;
            {
                // keep the L2 prefetch kPrefetchUnits units ahead of the loads
                const int up = u + kPrefetchUnits;
                if (lane < 16 && up < u1)
                    prefetch_l2(p.qW + (size_t)((up % p.RT) * 16 + lane) * Kh + (size_t)(up / p.RT) * (KC / 2), KC / 2);
            }
            const uint8_t* ar = act + ((size_t)(kc - kc_first) * kMaxTokens + gq) * kActStride + 32 * tq;
            float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
            int d0[4] = {0, 0, 0, 0}, d1[4] = {0, 0, 0, 0};
            auto mma_half = [&](int h, const uint4 (&A)[kHalfBlocks], const uint4 (&B)[kHalfBlocks]) {
#pragma unroll
                for (int i = 0; i < kHalfBlocks; ++i) {
                    const int blk = kHalfBlocks * h + i;
                    // this thread's channels of block blk: words 16 blk + 4 tq + w, w = 0..3
                    const uint4 x01 = *reinterpret_cast<const uint4*>(ar + 128 * blk);
                    const uint4 x23 = *reinterpret_cast<const uint4*>(ar + 128 * blk + 16);
                    const uint32_t be[4] = {x01.x, x01.z, x23.x, x23.z}, bo[4] = {x01.y, x01.w, x23.y, x23.w};
                    const uint32_t wA[4] = {A[i].x, A[i].y, A[i].z, A[i].w};
                    const uint32_t wB[4] = {B[i].x, B[i].y, B[i].z, B[i].w};
#pragma unroll
                    for (int w = 0; w < 4; ++w)
                        mma_s8(d0, nib_even(wA[w]), nib_even(wB[w]), nib_odd(wA[w]), nib_odd(wB[w]), be[w], bo[w]);
                    if (two) {
                        const uint8_t* ar1 = ar + (size_t)8 * kActStride;
                        const uint4 y01 = *reinterpret_cast<const uint4*>(ar1 + 128 * blk);
                        const uint4 y23 = *reinterpret_cast<const uint4*>(ar1 + 128 * blk + 16);
                        const uint32_t ce[4] = {y01.x, y01.z, y23.x, y23.z}, co[4] = {y01.y, y01.w, y23.y, y23.w};
#pragma unroll
                        for (int w = 0; w < 4; ++w)
                            mma_s8(d1, nib_even(wA[w]), nib_even(wB[w]), nib_odd(wA[w]), nib_odd(wB[w]), ce[w], co[w]);
                    }
                    if ((blk + 1) % gpb == 0) {
                        // end of a group: 256 * P_g exactly; promote with s_g
                        const float sg = s_sm[(kc * KC + blk * 128) / G];
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
            };
            mma_half(0, a0, b0);
            if (un < u1) load_half(un, 0, a0, b0);
            mma_half(1, a1, b1);
            if (un < u1) load_half(un, 1, a1, b1);
            // this unit's sums: rows gq, gq + 8 of the tile; tokens 2 tq, 2 tq + 1 (+ 8)
            float* pc = p.part + (size_t)kc * M * N;
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int row = rt * 16 + gq + (r >= 2 ? 8 : 0);
                const int t0 = 2 * tq + (r & 1);
                if (t0 < M) pc[(size_t)t0 * N + row] = acc0[r];
                if (two && t0 + 8 < M) pc[(size_t)(t0 + 8) * N + row] = acc1[r];
            }
        }
    }
    // every unit's sums are in the workspace
    if (!grid_barrier(p.gbar, p.err, p.limit_ns)) return;

    // ---- phase 4: Y = (sum of the chunk sums, in chunk order) * scale_t * scale_w,
    // one output per thread across the grid, eight chunk loads in flight at a time
    {
        const size_t cs = (size_t)M * N;   // stride between chunks
        for (size_t e = (size_t)blockIdx.x * kThreads + tid; e < cs; e += (size_t)gridDim.x * kThreads) {
            const int t = (int)(e / N);
            const int row = (int)(e % N);
            const float* pp = p.part + e;
            float a = __ldcg(pp);
            int c = 1;
            for (; c + 8 <= p.KCN; c += 8) {
                float w[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) w[q] = __ldcg(pp + (size_t)(c + q) * cs);
#pragma unroll
                for (int q = 0; q < 8; ++q) a = __fadd_rn(a, w[q]);
            }
            for (; c < p.KCN; ++c) a = __fadd_rn(a, __ldcg(pp + (size_t)c * cs));
            const float y = __fmul_rn(__fmul_rn(a, sc_sm[t]), __ldg(p.scale_w + row));
            if (p.ybf16)
                reinterpret_cast<__nv_bfloat16*>(p.Y)[e] = __float2bfloat16_rn(y);
            else
                reinterpret_cast<float*>(p.Y)[e] = y;
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
    if (!(M >= 1 && M <= kMaxTokens && N >= 16 && N % 16 == 0 && K % KC == 0 && K <= kMaxK && G >= 128 &&
          G % 128 == 0 && KC % G == 0 && K / G <= kMaxGroups && n >= 1 && n <= kMaxChunk))
        return false;
    // every CTA's units (chunk-major) span at most kMaxSlots chunks of staged codes
    const int grid = decode_grid();
    if (grid < 1 || K / G > kMaxOwned * grid) return false;
    const long long RT = N / 16, U = RT * (K / KC);
    for (int c = 0; c < grid; ++c) {
        const long long u0 = c * U / grid, u1 = (c + 1) * U / grid;
        if (u1 > u0 && (u1 - 1) / RT - u0 / RT + 1 > kMaxSlots) return false;
    }
    return true;
}

// Where the single launch is the faster form (measured on the 70B decode layers):
// few tokens, or a weight stream large enough to hide the activation phases.
bool decode_preferred(int M, int N, int K) { return M <= 6 || (long long)N * K >= (1LL << 27); }

// Workspace bytes after the 256-byte header: X_rot, the per-item group maxima
// and the per-chunk sums, each 256-byte aligned.
static size_t al256(size_t x) { return (x + 255) & ~size_t(255); }
static size_t gtab_bytes(int M, int K) { return (size_t)M * (K / dec::kMinChunk) * (K / 128) * 4; }
size_t decode_ws_bytes(int M, int N, int K) {
    return al256((size_t)M * K * 4) + al256(gtab_bytes(M, K)) + al256((size_t)(K / dec::KC) * M * N * 4);
}

cudaError_t launch_decode(const DecodeLaunch& dl, cudaStream_t st) {
    using namespace dec;
    static KernelSetup setup[2];
    const bool two = dl.M > 8;
    const auto kern = two ? decode_kernel<true> : decode_kernel<false>;
    int occ = 0;
    cudaError_t e = kernel_setup(reinterpret_cast<const void*>(kern), kThreads, kSmemBytes, setup[two ? 1 : 0], &occ);
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
    a.gtab = reinterpret_cast<float*>(w);
    w += al256(gtab_bytes(dl.M, dl.K));
    a.part = reinterpret_cast<float*>(w);
    a.L = dl.n > kMinChunk ? dl.n : kMinChunk;
    a.RT = dl.N / 16;
    a.KCN = dl.K / KC;
    a.U = a.RT * a.KCN;
    a.gbar = dl.gbar;
    a.err = dl.err;
    a.limit_ns = kWaitLimitNs;
    void* params[] = {&a};
    return cudaLaunchCooperativeKernel(reinterpret_cast<void*>(kern), dim3(grid), dim3(kThreads), params,
                                       kSmemBytes, st);
}

}  // namespace rrs
