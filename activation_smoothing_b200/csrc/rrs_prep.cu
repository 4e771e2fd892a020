// rrs_prep.cu -- online activation path of Rotated Runtime Smooth on sm_100a:
// block-diagonal Hadamard rotation (fp32 FWHT in registers + shared memory),
// reorder gather, group-wise runtime max, per-token INT4 quantise and pack.
//
// One kernel body serves four modes:
//   kQuant        pass B: X -> qX (packed INT4), scale_t   (needs s)
//   kGroupMax     pass A: X -> s[g] = max over tokens and group channels |X'|
//   kChannelMax   calibration: X -> cmax[k] = max over tokens |X_rot[:, k]|
//   (weights use kQuant with unit scales: qW, scale_w)
//
// Work split: a "team" of T = K/E threads owns one row at a time, each thread
// E elements (E = 64 for K >= 2048).  A row is staged as fp16 in shared memory
// by cp.async (two stages, prefetching the team's next row), rotated in
// rounds of up to log2(E) butterfly stages held in registers, exchanged
// through a swizzled fp32 row buffer between rounds, then gathered through
// perm for the quantiser.  R teams share a CTA.
//
// Arithmetic follows the library's contract exactly (see include/rrs.h): the
// butterfly stages run in the order h = 1, 2, 4, ... with (a + b, a - b) on
// pairs (j, j + h); every operation is an explicit round-to-nearest
// intrinsic, so no contraction or reassociation can change a bit.
#include <cuda_runtime.h>

#include <cstdint>

#include "rrs_device.cuh"
#include "rrs_internal.h"

namespace rrs {

enum PrepMode : int { kQuant = 0, kGroupMax = 1, kChannelMax = 2 };

// Swizzled word address of element `idx` in the fp32 row buffer: the 16-byte
// chunk index (bits 2..4) is XORed with bits e..e+2 (e = log2 E >= 5), which makes both the
// first-round vector stores (each thread a contiguous run of E elements) and the
// later strided scalar accesses bank-conflict free.
template <int LOGE>
__device__ __forceinline__ int swz(int idx) {
    // The XOR source bits must lie above the target bits 2..4 to keep this a
    // bijection; for E < 32 (LOGE < 5) they are taken from bits 5..7.
    constexpr int SRC = LOGE < 5 ? 5 : LOGE;
    return idx ^ (((idx >> SRC) & 7) << 2);
}

// Returns x through an opaque move, so address arithmetic derived from it is
// recomputed where it is used instead of being hoisted out of the row loop
// (hoisting every round's addresses would exhaust the registers).
__device__ __forceinline__ int opaque(int x) {
    int y;
    asm volatile("mov.b32 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

// Butterfly stages k in [0, a) over the thread's E registers (stage k pairs
// local index l with l + 2^k), in increasing k.
template <int E, int LOGE>
__device__ __forceinline__ void fwht_stages(float (&v)[E], int a) {
#pragma unroll
    for (int k = 0; k < LOGE; ++k) {
        if (k < a) {
#pragma unroll
            for (int l = 0; l < E; ++l) {
                if (!(l & (1 << k))) {
                    const float x = v[l];
                    const float y = v[l | (1 << k)];
                    v[l] = __fadd_rn(x, y);
                    v[l | (1 << k)] = __fsub_rn(x, y);
                }
            }
        }
    }
}

// Element index held in register l by team thread t in a round whose active
// bits are [b0, b0 + a) (rounds after the first).
__device__ __forceinline__ int round_index(int t, int l, int T, int b0, int a) {
    const int j = l >> a;
    const int mid = l & ((1 << a) - 1);
    const int q = t + j * T;
    const int hi = q >> b0;
    const int lo = q & ((1 << b0) - 1);
    return (hi << (b0 + a)) | (mid << b0) | lo;
}

// Shared-memory word address of register l in a round whose first active bit
// is B0 and which has A active bits (both compile-time): thread t holds groups
// j = l >> A (q = t + j*T) and within each group the 2^A elements
// base_j + mid * 2^B0.  For E >= 32 the swizzle term of base_j is computed
// once per group and the per-register part is an immediate.
template <int LOGE, int B0, int A>
__device__ __forceinline__ int raddr(int t, int T, int l) {
    const int j = l >> A;
    const int mid = l & ((1 << A) - 1);
    const int q = t + j * T;
    const int base = ((q >> B0) << (B0 + A)) | (q & ((1 << B0) - 1));
    if constexpr (LOGE >= 5) {
        const int sb = swz<LOGE>(base);
        if constexpr (B0 == LOGE) return (sb ^ ((mid & 7) << 2)) + (mid << B0);
        else return sb + (mid << B0);
    } else {
        return swz<LOGE>(base | (mid << B0));
    }
}

template <int E, int LOGE, int B0, int A>
__device__ __forceinline__ void rload(float (&v)[E], const float* buf, int t, int T) {
#pragma unroll
    for (int l = 0; l < E; ++l) v[l] = buf[raddr<LOGE, B0, A>(t, T, l)];
}

template <int E, int LOGE, int B0, int A>
__device__ __forceinline__ void rstore(const float (&v)[E], float* buf, int t, int T, float mul) {
#pragma unroll
    for (int l = 0; l < E; ++l) buf[raddr<LOGE, B0, A>(t, T, l)] = __fmul_rn(v[l], mul);
}

template <int LOGE, int B0, int A>
__device__ __forceinline__ int rindex(int t, int T, int l) {
    const int j = l >> A;
    const int mid = l & ((1 << A) - 1);
    const int q = t + j * T;
    return (((q >> B0) << (B0 + A)) | (q & ((1 << B0) - 1))) | (mid << B0);
}

// Dispatch a runtime active-bit count a in [1, LOGE] to the templates.
#define RRS_A_SWITCH(a, CALL)                       \
    switch (a) {                                    \
        case 1: { constexpr int AA = 1; CALL; } break;                         \
        case 2: if constexpr (LOGE >= 2) { constexpr int AA = 2; CALL; } break; \
        case 3: if constexpr (LOGE >= 3) { constexpr int AA = 3; CALL; } break; \
        case 4: if constexpr (LOGE >= 4) { constexpr int AA = 4; CALL; } break; \
        case 5: if constexpr (LOGE >= 5) { constexpr int AA = 5; CALL; } break; \
        default: if constexpr (LOGE >= 6) { constexpr int AA = LOGE; CALL; } break; \
    }

template <int E, int LOGE, int B0>
__device__ __forceinline__ void round_load(float (&v)[E], const float* buf, int t, int T, int a) {
    RRS_A_SWITCH(a, (rload<E, LOGE, B0, AA>(v, buf, t, T)))
}

template <int E, int LOGE, int B0>
__device__ __forceinline__ void round_store(const float (&v)[E], float* buf, int t, int T, int a, float mul) {
    RRS_A_SWITCH(a, (rstore<E, LOGE, B0, AA>(v, buf, t, T, mul)))
}

template <int E, int LOGE>
__device__ __forceinline__ void contig_store(const float (&v)[E], float* buf, int t, float mul) {
#pragma unroll
    for (int l = 0; l < E; l += 4) {
        *reinterpret_cast<float4*>(buf + swz<LOGE>(t * E + l)) =
            make_float4(__fmul_rn(v[l], mul), __fmul_rn(v[l + 1], mul), __fmul_rn(v[l + 2], mul),
                        __fmul_rn(v[l + 3], mul));
    }
}

// Element index of register l in the final layout of a transform with
// `nrounds` rounds, the last one having `al` active bits.
template <int E, int LOGE>
__device__ __forceinline__ int final_index(int t, int l, int T, int nrounds, int al) {
    if (nrounds == 1) return t * E + l;
    return round_index(t, l, T, (nrounds - 1) * LOGE, al);
}

// Stores the final registers (times `mul`) in the final layout.
template <int E, int LOGE>
__device__ __forceinline__ void final_store(const float (&v)[E], float* buf, int t, int T, int nrounds,
                                            int al, float mul) {
    if (nrounds == 1) contig_store<E, LOGE>(v, buf, t, mul);
    else if (nrounds == 2) round_store<E, LOGE, LOGE>(v, buf, t, T, al, mul);
    else if (nrounds == 3) round_store<E, LOGE, 2 * LOGE>(v, buf, t, T, al, mul);
    else round_store<E, LOGE, 3 * LOGE>(v, buf, t, T, al, mul);
}

struct PrepArgs {
    const __half* X;        // [rows, K] fp16
    int rows, K, L;         // L = log2(n)
    float c_n;              // fl32(1/sqrt(n)), from the host
    const int32_t* perm;    // [K]
    int G;
    int mode;
    int unit_scales;
    int stages;             // fp16 staging buffers per team (1 or 2)
    const float* s_in;      // [K/G] (kQuant without unit scales)
    uint8_t* q_out;         // [rows, K/2] (kQuant)
    float* scale_out;       // [rows] (kQuant)
    float* s_unit_out;      // [K/G] written as 1 (kQuant with unit scales), may be null
    uint32_t* max_out;      // [K/G] (kGroupMax) or [K] (kChannelMax): fp32 bits, zeroed by the host
};

template <int E, int LOGE, int MODE, int MAXT>
__global__ void __launch_bounds__(MAXT) prep_kernel(PrepArgs p) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int K = p.K;
    const int T = K / E;                       // team threads
    const int R = blockDim.x / T;              // teams per CTA
    const int team = threadIdx.x / T;
    const int t = threadIdx.x % T;
    float* rowbuf = reinterpret_cast<float*>(smem_raw) + (size_t)team * K;
    __half* stage0 = reinterpret_cast<__half*>(reinterpret_cast<float*>(smem_raw) + (size_t)R * K) +
                     (size_t)team * p.stages * K;
    __shared__ float red[16][16];              // [team][warp in team] per-row amax

    const int L = p.L;
    const int nrounds = (L <= LOGE) ? 1 : (L + LOGE - 1) / LOGE;
    const int a1 = L < LOGE ? L : LOGE;
    // Active bits of the last round (the layout of the final registers).
    const int al = L - (nrounds - 1) * LOGE < LOGE ? L - (nrounds - 1) * LOGE : LOGE;

    // Per-thread gather addresses for the outputs j in [t*E, t*E + E) (kQuant).
    constexpr int CH = E >= 8 ? E / 8 : 1;     // 16-byte fp16 chunks per thread in the first round
    constexpr int EG = (MODE == kQuant) ? E / 2 : 1;
    uint32_t gaddr[EG];
    float d = 1.0f;
    if constexpr (MODE == kQuant) {
#pragma unroll
        for (int l = 0; l < E; l += 2) {
            const int j = t * E + l;
            // a null index means no reorder (the KV-cache path)
            const uint32_t lo16 = (uint32_t)swz<LOGE>(p.perm ? p.perm[j] : j);
            const uint32_t hi16 = (uint32_t)swz<LOGE>(p.perm ? p.perm[j + 1] : j + 1);
            gaddr[l / 2] = lo16 | (hi16 << 16);
        }
        if (!p.unit_scales) {
            const float sg = p.s_in[(t * E) / p.G];
            d = (sg == 0.0f) ? 1.0f : sg;
        }
        if (p.unit_scales && p.s_unit_out && blockIdx.x == 0) {
            for (int g = threadIdx.x; g < K / p.G; g += blockDim.x) p.s_unit_out[g] = 1.0f;
        }
    }

    constexpr int EM = (MODE == kQuant) ? 1 : E;   // running channel maxima (max modes)
    float vmax[EM];
#pragma unroll
    for (int l = 0; l < EM; ++l) vmax[l] = 0.0f;

    const int team_global = blockIdx.x * R + team;
    const int team_stride = gridDim.x * R;
    const int bar_id = 1 + team;

    // Issue the cp.async copies of row `r` into staging buffer `sb`.
    auto issue_row = [&](int r, int sb) {
        const __half* src = p.X + (size_t)r * K;
        __half* dst = stage0 + (size_t)sb * K;
        const int nchunks = K / 8;
        for (int u = t; u < nchunks; u += T) {
            int pos = u;
            if constexpr (E >= 8) {
                const int owner = u / CH;
                const int c = u % CH;
                pos = owner * CH + (c ^ (owner & (CH - 1)));
            }
            cp_async16(dst + (size_t)pos * 8, src + (size_t)u * 8);
        }
    };

    int r = team_global;
    int it = 0;
    if (r < p.rows) issue_row(r, 0);
    cp_async_commit();
    for (; r < p.rows; r += team_stride, ++it) {
        const int sb = (p.stages == 2) ? (it & 1) : 0;
        const int rn = r + team_stride;
        if (p.stages == 2) {
            if (rn < p.rows) issue_row(rn, sb ^ 1);
            cp_async_commit();
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        named_bar(bar_id, T);
        const int tl = opaque(t);

        // ---- first round: E contiguous elements from the staging buffer.
        float v[E];
        {
            const __half* st = stage0 + (size_t)sb * K;
            if constexpr (E >= 8) {
#pragma unroll
                for (int c = 0; c < CH; ++c) {
                    const int pos = t * CH + (c ^ (t & (CH - 1)));
                    const uint4 raw = *reinterpret_cast<const uint4*>(st + (size_t)pos * 8);
                    const __half2* h2 = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float2 f = __half22float2(h2[q]);
                        v[c * 8 + 2 * q] = f.x;
                        v[c * 8 + 2 * q + 1] = f.y;
                    }
                }
            } else {
                const uint2 raw = *reinterpret_cast<const uint2*>(st + (size_t)t * 4);
                const __half2* h2 = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const float2 f = __half22float2(h2[q]);
                    v[2 * q] = f.x;
                    v[2 * q + 1] = f.y;
                }
            }
        }
        if (p.stages == 1) {
            named_bar(bar_id, T);                       // staging buffer free
            if (rn < p.rows) issue_row(rn, 0);
            cp_async_commit();
        }
        fwht_stages<E, LOGE>(v, a1);

        // ---- further rounds through the fp32 row buffer (at most 4 rounds in
        // total; each thread re-reads exactly the elements it will rewrite, so
        // only the store -> load transition needs a barrier).
        if (nrounds >= 2) {
            contig_store<E, LOGE>(v, rowbuf, tl, 1.0f);
            named_bar(bar_id, T);
            const int a = (L - LOGE) < LOGE ? (L - LOGE) : LOGE;
            round_load<E, LOGE, LOGE>(v, rowbuf, tl, T, a);
            fwht_stages<E, LOGE>(v, a);
        }
        if (nrounds >= 3) {
            round_store<E, LOGE, LOGE>(v, rowbuf, tl, T, LOGE, 1.0f);
            named_bar(bar_id, T);
            const int a = (L - 2 * LOGE) < LOGE ? (L - 2 * LOGE) : LOGE;
            round_load<E, LOGE, 2 * LOGE>(v, rowbuf, tl, T, a);
            fwht_stages<E, LOGE>(v, a);
        }
        if (nrounds >= 4) {
            round_store<E, LOGE, 2 * LOGE>(v, rowbuf, tl, T, LOGE, 1.0f);
            named_bar(bar_id, T);
            const int a = (L - 3 * LOGE) < LOGE ? (L - 3 * LOGE) : LOGE;
            round_load<E, LOGE, 3 * LOGE>(v, rowbuf, tl, T, a);
            fwht_stages<E, LOGE>(v, a);
        }

        if constexpr (MODE != kQuant) {
#pragma unroll
            for (int l = 0; l < EM; ++l) vmax[l] = fmaxf(vmax[l], fabsf(v[l]));
            // The row buffer and staging buffer are reused by the next row.
            named_bar(bar_id, T);
            continue;
        }

        if constexpr (MODE == kQuant) {
        // ---- normalise and write X_rot for the gather.
        final_store<E, LOGE>(v, rowbuf, tl, T, nrounds, al, p.c_n);
        named_bar(bar_id, T);

        // ---- gather through perm, smooth, per-token amax.
        float amax = 0.0f;
#pragma unroll
        for (int l = 0; l < E; l += 2) {
            const uint32_t ga = gaddr[l / 2];
            float x0 = rowbuf[ga & 0xFFFFu];
            float x1 = rowbuf[ga >> 16];
            if (!p.unit_scales) {
                x0 = __fdiv_rn(x0, d);
                x1 = __fdiv_rn(x1, d);
            }
            v[l] = x0;
            v[l + 1] = x1;
            amax = fmaxf(amax, fmaxf(fabsf(x0), fabsf(x1)));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const int nw = (T + 31) / 32;
        if (T >= 32) {
            if ((t & 31) == 0) red[team][t >> 5] = amax;
            named_bar(bar_id, T);
            amax = red[team][0];
            for (int w = 1; w < nw; ++w) amax = fmaxf(amax, red[team][w]);
        }
        const float scale = __fdiv_rn(amax, 7.0f);

        // ---- quantise (round half to even), clamp, pack two codes per byte.
        uint32_t packed[E / 8 > 0 ? E / 8 : 1];
#pragma unroll
        for (int w = 0; w < (E / 8 > 0 ? E / 8 : 1); ++w) packed[w] = 0u;
#pragma unroll
        for (int l = 0; l < E; ++l) {
            int q = 0;
            if (scale != 0.0f) {
                q = __float2int_rn(__fdiv_rn(v[l], scale));
                q = q > 7 ? 7 : (q < -8 ? -8 : q);
            }
            packed[l / 8] |= ((uint32_t)q & 0xFu) << (4 * (l % 8));
        }
        uint8_t* dst = p.q_out + (size_t)r * (K / 2) + (size_t)t * (E / 2);
        if constexpr (E == 64) {
            reinterpret_cast<uint4*>(dst)[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
            reinterpret_cast<uint4*>(dst)[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
        } else if constexpr (E == 32) {
            reinterpret_cast<uint4*>(dst)[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        } else if constexpr (E == 16) {
            reinterpret_cast<uint2*>(dst)[0] = make_uint2(packed[0], packed[1]);
        } else if constexpr (E == 8) {
            reinterpret_cast<uint32_t*>(dst)[0] = packed[0];
        } else {
            reinterpret_cast<uint16_t*>(dst)[0] = (uint16_t)packed[0];
        }
        if (t == 0) p.scale_out[r] = scale;
        named_bar(bar_id, T);   // row buffer and red[] free for the next row
        }  // kQuant
    }
    cp_async_wait<0>();

    if constexpr (MODE != kQuant) {
    // ---- combine the per-thread channel maxima of all teams of this CTA.
    __syncthreads();
    uint32_t* cm = reinterpret_cast<uint32_t*>(smem_raw);   // K words (team 0's row buffer)
    for (int i = threadIdx.x; i < K; i += blockDim.x) cm[i] = 0u;
    __syncthreads();
#pragma unroll
    for (int l = 0; l < EM; ++l) {
        const int idx = final_index<E, LOGE>(t, l, T, nrounds, al);
        if (vmax[l] > 0.0f) atomicMax(&cm[idx], __float_as_uint(vmax[l]));
    }
    __syncthreads();
    if constexpr (MODE == kChannelMax) {
        for (int i = threadIdx.x; i < K; i += blockDim.x) {
            const float m = __uint_as_float(cm[i]);
            if (m > 0.0f) atomicMax(&p.max_out[i], __float_as_uint(__fmul_rn(m, p.c_n)));
        }
    } else {
    // kGroupMax: s[g] = c_n * max over the group's channels (RN is monotone, so
    // scaling the max equals the max of the scaled values).
    for (int j0 = 0; j0 < K; j0 += blockDim.x) {
        const int j = j0 + threadIdx.x;
        float m = (j < K) ? __uint_as_float(cm[p.perm ? p.perm[j] : j]) : 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if ((threadIdx.x & 31) == 0 && j < K && m > 0.0f)
            atomicMax(&p.max_out[j / p.G], __float_as_uint(__fmul_rn(m, p.c_n)));
    }
    }
    }  // max modes
}

// ------------------------------------------------------------------ launch ---

static int pick_E(int K) {
    for (int E = 64; E >= 4; E >>= 1)
        if (K % (32 * E) == 0) return E;
    return 0;
}

template <int E, int LOGE, int MODE, int MAXT>
static cudaError_t launch_one(const PrepArgs& a, int threads, size_t smem, int nsm, int teams_needed,
                              cudaStream_t stream) {
    if (threads > MAXT) return cudaErrorInvalidValue;
    auto kern = prep_kernel<E, LOGE, MODE, MAXT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int occ = 1;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, threads, smem);
    if (occ < 1) occ = 1;
    int grid = nsm * occ;
    if (grid > teams_needed) grid = teams_needed;
    if (grid < 1) grid = 1;
    kern<<<grid, threads, smem, stream>>>(a);
    return cudaGetLastError();
}

template <int E, int LOGE, int MAXT>
static cudaError_t launch_mode(const PrepArgs& a, int mode, int threads, size_t smem, int nsm,
                               int teams_needed, cudaStream_t stream) {
    if (mode == kQuant) return launch_one<E, LOGE, kQuant, MAXT>(a, threads, smem, nsm, teams_needed, stream);
    if (mode == kGroupMax)
        return launch_one<E, LOGE, kGroupMax, MAXT>(a, threads, smem, nsm, teams_needed, stream);
    return launch_one<E, LOGE, kChannelMax, MAXT>(a, threads, smem, nsm, teams_needed, stream);
}

size_t prep_smem_bytes(int K, int R, int stages) {
    return (size_t)R * K * 4 + (size_t)R * stages * K * 2;
}

cudaError_t launch_prep(const PrepLaunch& pl, cudaStream_t stream) {
    const int K = pl.K;
    const int E = pick_E(K);
    if (E == 0) return cudaErrorInvalidValue;
    const int T = K / E;
    int R = 1;
    if (T < 256 && 256 % T == 0) R = 256 / T;
    if (R > 8) R = 8;
    int stages = 2;
    size_t smem = prep_smem_bytes(K, R, stages);
    const size_t kMaxSmem = 227 * 1024 - 2048;
    while (smem > kMaxSmem && R > 1) {
        R >>= 1;
        smem = prep_smem_bytes(K, R, stages);
    }
    if (smem > kMaxSmem) {
        stages = 1;
        smem = prep_smem_bytes(K, R, stages);
    }
    if (smem > kMaxSmem || T * R > 512) return cudaErrorInvalidValue;

    PrepArgs a;
    a.X = reinterpret_cast<const __half*>(pl.X);
    a.rows = pl.rows;
    a.K = K;
    int L = 0;
    while ((1 << L) < pl.n) ++L;
    a.L = L;
    a.c_n = pl.c_n;
    a.perm = pl.perm;
    a.G = pl.G;
    a.mode = pl.mode;
    a.unit_scales = pl.unit_scales;
    a.stages = stages;
    a.s_in = pl.s_in;
    a.q_out = pl.q_out;
    a.scale_out = pl.scale_out;
    a.s_unit_out = pl.s_unit_out;
    a.max_out = pl.max_out;

    int dev = 0;
    cudaGetDevice(&dev);
    int nsm = 148;
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    const int threads = T * R;
    const int teams_needed = (pl.rows + R - 1) / R;
    int nrounds = (L <= 0) ? 1 : 0;
    {
        int logE = 0;
        while ((1 << logE) < E) ++logE;
        if (nrounds == 0) nrounds = (L + logE - 1) / logE;
        if (nrounds < 1) nrounds = 1;
    }
    if (nrounds > 4) return cudaErrorInvalidValue;

    switch (E) {
        case 64:
            return threads <= 256 ? launch_mode<64, 6, 256>(a, pl.mode, threads, smem, nsm, teams_needed, stream)
                                  : launch_mode<64, 6, 512>(a, pl.mode, threads, smem, nsm, teams_needed, stream);
        case 32: return launch_mode<32, 5, 256>(a, pl.mode, threads, smem, nsm, teams_needed, stream);
        case 16: return launch_mode<16, 4, 256>(a, pl.mode, threads, smem, nsm, teams_needed, stream);
        case 8: return launch_mode<8, 3, 256>(a, pl.mode, threads, smem, nsm, teams_needed, stream);
        case 4: return launch_mode<4, 2, 512>(a, pl.mode, threads, smem, nsm, teams_needed, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace rrs
