// rrs_prep_fast.cu -- online activation path for K a multiple of 2048 (every
// LLaMA projection shape): one cooperative persistent kernel in two phases
// (the kernel itself is in rrs_act.cuh, instantiated in rrs_act_*.cu).
//
//   phase A   X (fp16) -> Hadamard rotation of every row this CTA owns; each
//             thread keeps, per register, the largest |v| of its channel over
//             its rows, and at the end the CTA's per-channel maxima are gathered
//             by the reorder into its row of a group-maxima table in the
//             workspace (fl(c_n |v|) is monotone in |v|, so c_n is applied once)
//   barrier   a grid-wide barrier (bounded wait); every CTA then reduces the
//             table: s[g] = max over all tokens and group channels of |X'|
//   phase B   X again (an L2 hit) -> the same rotation bit for bit, reorder
//             gather, division by s_g, per-token INT4 quantisation; writes qX
//             (packed), scale_t and the GEMM operand (e4m3 or int8).  When every
//             team owns at most one row (decode token counts), phase A keeps the
//             rotated row in shared memory and phase B does not recompute it.
//
// Nothing of size M x K passes between the phases: the rotation is recomputed
// (or kept on chip) instead of stored.  The host picks one of eight kernel forms
// (up to 320 or 512 threads, rows kept or not, e4m3 or int8 operand), each a smaller
// kernel: in a layer sequence the kernel follows a GEMM and its code is fetched
// cold, so code size is time.
//
// Work split: a team of T = K/64 threads (a multiple of 32) owns one row at a
// time; each thread holds 64 elements.  Rotation rounds: up to 6 butterfly
// stages on the 64 registers (f32x2 packed add/sub for every stage but the
// first of a round), an exchange through a swizzled fp32 row buffer, the next 6
// stages (and a third round for n = 8192).
//
// Arithmetic is bit-identical to the library contract: stage order h = 1, 2, 4,
// ... with (a + b, a - b); one multiply by c_n; IEEE division (computed with
// Markstein's correction from a correctly rounded reciprocal, see
// div_markstein); round half to even; clamp to [-8, 7].
#include <cuda_runtime.h>

#include <cstdint>

#include "rrs_act.cuh"
#include "rrs_device.cuh"
#include "rrs_internal.h"

namespace rrs {
namespace fast {

// instantiated in rrs_act_*.cu (several files, compiled in parallel)
extern template cudaError_t launch_act<0>(const ActArgs&, bool, int, size_t, int, cudaStream_t);
extern template cudaError_t launch_act<1>(const ActArgs&, bool, int, size_t, int, cudaStream_t);
extern template cudaError_t launch_act<2>(const ActArgs&, bool, int, size_t, int, cudaStream_t);
extern template cudaError_t launch_act<3>(const ActArgs&, bool, int, size_t, int, cudaStream_t);
extern template cudaError_t launch_act<4>(const ActArgs&, bool, int, size_t, int, cudaStream_t);
extern template cudaError_t launch_act<5>(const ActArgs&, bool, int, size_t, int, cudaStream_t);
extern template cudaError_t launch_act<6>(const ActArgs&, bool, int, size_t, int, cudaStream_t);
extern template cudaError_t launch_act<7>(const ActArgs&, bool, int, size_t, int, cudaStream_t);
extern template cudaError_t launch_act<8>(const ActArgs&, bool, int, size_t, int, cudaStream_t);
extern template cudaError_t launch_act<9>(const ActArgs&, bool, int, size_t, int, cudaStream_t);
extern template cudaError_t launch_act<10>(const ActArgs&, bool, int, size_t, int, cudaStream_t);
extern template cudaError_t launch_act<11>(const ActArgs&, bool, int, size_t, int, cudaStream_t);
extern template cudaError_t launch_act<12>(const ActArgs&, bool, int, size_t, int, cudaStream_t);
extern template cudaError_t launch_act<13>(const ActArgs&, bool, int, size_t, int, cudaStream_t);

// Packed INT4 rows -> int8 GEMM operand rows (the k order of the activation
// kernel's int8 operand: 0, 2, 4, 6, 1, 3, 5, 7 within each 8 channels).
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

// Packed INT4 rows -> e4m3 codes in natural k order (byte 2i from the low
// nibble of packed byte i, byte 2i + 1 from its high nibble).  A nibble n is
// the two's-complement code q = n - 16 * (n >> 3); its e4m3 byte comes from a
// 16-entry table held in two pairs of registers and read with byte permutes.
__device__ __forceinline__ uint32_t e4m3_of_nibbles(uint32_t nib4) {
    // nib4: four nibbles, one per byte (values 0..15).  Codes 0..7 (n < 8) and
    // -8..-1 (n >= 8) read separate 8-entry tables, selected per byte.
    const uint32_t idx = nib4 & 0x07070707u;
    const uint32_t sel = __byte_perm(idx | (idx >> 4), 0u, 0x0020) & 0x7777u;
    // e4m3 of 0..7 and of -8..-1
    const uint32_t pos = __byte_perm(0x44403800u, 0x4E4C4A48u, sel);
    const uint32_t neg = __byte_perm(0xCACCCED0u, 0xB8C0C4C8u, sel);
    const uint32_t negmask = ((nib4 >> 3) & 0x01010101u) * 0xFFu;
    return (pos & ~negmask) | (neg & negmask);
}

__global__ void expand_e4m3_kernel(const uint8_t* q, uint8_t* out, size_t nwords) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < nwords; i += (size_t)gridDim.x * blockDim.x) {
        const uint32_t w = reinterpret_cast<const uint32_t*>(q)[i];
        // bytes b0..b3 hold codes (2i, 2i+1): output order lo0 hi0 lo1 hi1 ...
        const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
        const uint32_t elo = e4m3_of_nibbles(lo), ehi = e4m3_of_nibbles(hi);
        reinterpret_cast<uint2*>(out)[i] = make_uint2(__byte_perm(elo, ehi, 0x5140), __byte_perm(elo, ehi, 0x7362));
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



}  // namespace fast

bool prep_fast_supported(int K, int n) {
    // whole warps per row team, at most 512 threads, and the row buffers of a CTA in shared memory
    return K % 2048 == 0 && K / 64 <= 512 && n >= 1 && n <= 8192 && fast::act_smem_bytes(K, 2) <= fast::kActSmemLimit;
}

int prep_fast_rows_per_cta(int K) { return fast::act_rows_per_cta(K); }

cudaError_t launch_prep_fast(const PrepFastLaunch& pl, cudaStream_t st) {
    using namespace fast;
    const int K = pl.K;
    const int T = K / E;
    const int R = act_rows_per_cta(K);
    const int threads = T * R;
    const int nst = act_stages(K);
    const size_t smem = act_smem_bytes(K, nst);
    int L = 0;
    while ((1 << L) < pl.n) ++L;
    ActArgs a;
    a.X = reinterpret_cast<const __half*>(pl.X);
    a.rows = pl.rows;
    a.K = K;
    a.G = pl.G;
    a.NG = K / pl.G;
    a.c_n = pl.c_n;
    a.perm = pl.perm;
    a.phase = pl.unit_scales ? 2 : pl.phase;
    a.unit_scales = pl.unit_scales;
    a.s = pl.s;
    a.qX = pl.qX;
    a.a8 = reinterpret_cast<uint8_t*>(pl.qX8);
    if (pl.qX8 == nullptr) return cudaErrorInvalidValue;   // the GEMM operand is always written
    a.scale_t = pl.scale_t;
    a.partial = pl.partial;
    a.gbar = pl.gbar;
    a.err = pl.err;
    a.limit_ns = kWaitLimitNs;
    a.nst = nst;
    cudaError_t e;
    switch (L) {
#define RRS_ACT_CASE(LL) \
    case LL: e = launch_act<LL>(a, pl.a_e4m3, threads, smem, pl.partial_rows, st); break;
        RRS_ACT_CASE(0) RRS_ACT_CASE(1) RRS_ACT_CASE(2) RRS_ACT_CASE(3) RRS_ACT_CASE(4)
        RRS_ACT_CASE(5) RRS_ACT_CASE(6) RRS_ACT_CASE(7) RRS_ACT_CASE(8) RRS_ACT_CASE(9)
        RRS_ACT_CASE(10) RRS_ACT_CASE(11) RRS_ACT_CASE(12) RRS_ACT_CASE(13)
#undef RRS_ACT_CASE
        default: return cudaErrorInvalidValue;
    }
    return e;
}

namespace fast {
__global__ void fill_kernel(float* p, int n, float v) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) p[i] = v;
}
}  // namespace fast

cudaError_t launch_fill(float* p, int n, float v, cudaStream_t st) {
    int blocks = (n + 255) / 256;
    if (blocks > 1024) blocks = 1024;
    fast::fill_kernel<<<blocks, 256, 0, st>>>(p, n, v);
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
    const int nsm = device_sm_count();
    size_t blocks = (nwords + 255) / 256;
    if (blocks > (size_t)nsm * 8) blocks = (size_t)nsm * 8;
    fast::expand_kernel<<<(unsigned)blocks, 256, 0, st>>>(qX, qX8, nwords);
    return cudaGetLastError();
}

cudaError_t launch_expand_e4m3(const uint8_t* q, uint8_t* out, int rows, int K, cudaStream_t st) {
    const size_t nwords = (size_t)rows * K / 8;
    const int nsm = device_sm_count();
    size_t blocks = (nwords + 255) / 256;
    if (blocks > (size_t)nsm * 8) blocks = (size_t)nsm * 8;
    fast::expand_e4m3_kernel<<<(unsigned)blocks, 256, 0, st>>>(q, out, nwords);
    return cudaGetLastError();
}


}  // namespace rrs
