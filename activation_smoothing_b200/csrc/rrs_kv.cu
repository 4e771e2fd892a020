// rrs_kv.cu -- the KV cache of the 4-4-4 setting (Rotated Runtime Smooth
// summary page, "Key results": weights, activations and KV cache in 4 bits).
//
// Quantisation reuses the activation path's general kernel (rrs_prep.cu):
// every head vector of length D is one row, rotated by the normalised Hadamard
// transform of size D and quantised per row to symmetric INT4, with no reorder
// and no runtime smoothing.  This file holds the way back: the cached codes
// times their scale, in the rotated space (a query rotated by the same
// transform gives the same attention scores, since the transform is
// orthogonal).
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "rrs_device.cuh"
#include "rrs_internal.h"

namespace rrs {
namespace kv {

// out[r][j] = fp16(code_j * scale[r]), code_j the signed nibble j of row r
// (low nibble = even j).  Eight outputs per thread: one 4-byte load, one
// 16-byte store.
__global__ void dequant_kernel(const uint8_t* q, const float* scale, size_t rows, int D, __half* out) {
    const int W = D / 8;                          // 8-output words per row
    const size_t total = rows * (size_t)W;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
        const size_t r = i / W;
        const uint32_t w = reinterpret_cast<const uint32_t*>(q)[i];
        const float sc = scale[r];
        uint32_t o[4];
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int byte = (int)((w >> (8 * b)) & 0xFFu);
            const int lo = (byte & 0x0F) - ((byte & 0x08) << 1);
            const int hi = ((byte >> 4) & 0x0F) - ((byte & 0x80) >> 3);
            const __half2 h = __floats2half2_rn(__fmul_rn((float)lo, sc), __fmul_rn((float)hi, sc));
            o[b] = *reinterpret_cast<const uint32_t*>(&h);
        }
        reinterpret_cast<uint4*>(out)[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// Two codes (one byte: low nibble the even channel) times the vector's scale, as
// a half2.
__device__ __forceinline__ uint32_t half2_codes(uint32_t byte, float sc) {
    const int lo = (int)(byte & 0x0Fu) - (int)((byte & 0x08u) << 1);
    const int hi = (int)((byte >> 4) & 0x0Fu) - (int)((byte & 0x80u) >> 3);
    const __half2 h = __floats2half2_rn(__fmul_rn((float)lo, sc), __fmul_rn((float)hi, sc));
    return *reinterpret_cast<const uint32_t*>(&h);
}

// The same for D a power of two >= 32, by 4-byte code words (8 outputs, one
// 16-byte store): consecutive threads take consecutive words, so a warp reads 128
// contiguous bytes of codes and writes 512 contiguous bytes of fp16 per
// instruction (whole sectors); four words per thread and pass are in flight.
__global__ void dequant_words_kernel(const uint32_t* q, const float* scale, size_t words, int lg_wpr, uint4* out) {
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (size_t w0 = blockIdx.x * (size_t)blockDim.x + threadIdx.x; w0 < words; w0 += 4 * stride) {
        uint32_t c[4];
        float sc[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const size_t w = w0 + j * stride;
            c[j] = w < words ? q[w] : 0u;
            sc[j] = w < words ? scale[w >> lg_wpr] : 0.0f;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const size_t w = w0 + j * stride;
            if (w < words)
                out[w] = make_uint4(half2_codes(c[j] & 0xFFu, sc[j]), half2_codes((c[j] >> 8) & 0xFFu, sc[j]),
                                    half2_codes((c[j] >> 16) & 0xFFu, sc[j]), half2_codes(c[j] >> 24, sc[j]));
        }
    }
}

// Quantisation of head vectors of D channels by LPV = D / 32 lanes each (32
// channels per lane, in registers; a warp takes 32 / LPV vectors at a time).  The
// normalised Hadamard transform runs in the library's stage order (h = 1, 2, 4,
// ...; pair (a + b, a - b), a the lower index): the stages h < 32 inside a lane,
// the stages h = 32, 64, ... across the vector's lanes by shuffles (the lane with
// the clear bit holds the lower index).  Then x = fl(c_n v), amax = max |x| over
// the vector, scale = amax / 7, q = clamp(rint(x / scale), -8, 7), the division
// correctly rounded by Markstein's correction as in the activation kernels (a
// zero scale gives zero codes).
template <int LPV>
__global__ void __launch_bounds__(256) quant_kernel(const __half* kv, size_t rows, float c_n, uint8_t* q,
                                                    float* scale) {
    constexpr int E = 32;                         // channels per lane, held as 16 float2
    constexpr int D = LPV * E;
    constexpr int VPW = 32 / LPV;                 // vectors per warp per pass
    constexpr float kMagic = 12582912.0f;         // 1.5 * 2^23: adding it rounds to an integer, half to even
    const int lane = threadIdx.x & 31;
    const int sub = lane % LPV;                   // this lane's part of its vector
    const size_t warp0 = (blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5;
    const size_t nwarps = (gridDim.x * (size_t)blockDim.x) >> 5;
    const float2 neg1 = make_float2(-1.0f, -1.0f);
    for (size_t rb = warp0 * VPW; rb < rows; rb += nwarps * VPW) {
        const size_t r = rb + lane / LPV;
        const bool live = r < rows;
        float2 v[E / 2];
        const __half* src = kv + (live ? r : 0) * D + (size_t)sub * E;
#pragma unroll
        for (int c = 0; c < E; c += 8) {
            const uint4 w = *reinterpret_cast<const uint4*>(src + c);
            const __half2* h = reinterpret_cast<const __half2*>(&w);
#pragma unroll
            for (int k = 0; k < 4; ++k) v[c / 2 + k] = __half22float2(h[k]);
        }
        // stage h = 1: the two channels of one float2
#pragma unroll
        for (int i = 0; i < E / 2; ++i) {
            const float a = v[i].x, b = v[i].y;
            v[i] = make_float2(__fadd_rn(a, b), __fsub_rn(a, b));
        }
        // stages h = 2 .. 16: pairs of float2, lane by lane with packed add / sub
        // (a - b as fma(b, -1, a), which is exactly RN(a - b))
#pragma unroll
        for (int hh = 1; hh < E / 2; hh <<= 1) {
#pragma unroll
            for (int i = 0; i < E / 2; ++i) {
                if (!(i & hh)) {
                    const float2 a = v[i], b = v[i + hh];
                    v[i] = __fadd2_rn(a, b);
                    v[i + hh] = __ffma2_rn(b, neg1, a);
                }
            }
        }
        // stages h = 32, 64, ...: the partner lane's value p; the lower lane keeps
        // RN(v + p), the upper RN(p - v): both are fma(v, +-1, p)
#pragma unroll
        for (int m = 1; m < LPV; m <<= 1) {
            const float sg = (lane & m) ? -1.0f : 1.0f;
            const float2 sg2 = make_float2(sg, sg);
#pragma unroll
            for (int i = 0; i < E / 2; ++i) {
                const float2 pv = make_float2(__shfl_xor_sync(0xFFFFFFFFu, v[i].x, m),
                                              __shfl_xor_sync(0xFFFFFFFFu, v[i].y, m));
                v[i] = __ffma2_rn(v[i], sg2, pv);
            }
        }
        const float2 c2 = make_float2(c_n, c_n);
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < E / 2; ++i) {
            v[i] = __fmul2_rn(v[i], c2);
            amax = fmaxf(amax, fmaxf(fabsf(v[i].x), fabsf(v[i].y)));
        }
#pragma unroll
        for (int m = 1; m < LPV; m <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, m));
        const float sc = __fdiv_rn(amax, 7.0f);
        uint32_t packed[4] = {0u, 0u, 0u, 0u};
        if (sc != 0.0f) {
            // |x| / scale <= 7 (to within an ulp: scale = RN(amax / 7)), so rint needs no clamp
            const float ys = __frcp_rn(sc);
            const float2 ns2 = make_float2(-sc, -sc), ys2 = make_float2(ys, ys);
            const float2 magic2 = make_float2(kMagic, kMagic);
#pragma unroll
            for (int w = 0; w < 4; ++w) {   // 8 channels (4 float2) per packed word
                uint32_t ev[4], od[4];
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const float2 z = __fadd2_rn(div_markstein(v[4 * w + h], ns2, ys2), magic2);   // low byte: the code
                    ev[h] = __float_as_uint(z.x);
                    od[h] = __float_as_uint(z.y);
                }
                // byte h of lo / hi: the code of channel 2h / 2h + 1 of the word
                const uint32_t lo = __byte_perm(__byte_perm(ev[0], ev[1], 0x0040), __byte_perm(ev[2], ev[3], 0x0040), 0x5410);
                const uint32_t hi = __byte_perm(__byte_perm(od[0], od[1], 0x0040), __byte_perm(od[2], od[3], 0x0040), 0x5410);
                packed[w] = (lo & 0x0F0F0F0Fu) | ((hi << 4) & 0xF0F0F0F0u);
            }
        }
        if (live) {
            *reinterpret_cast<uint4*>(q + r * (D / 2) + (size_t)sub * (E / 2)) =
                make_uint4(packed[0], packed[1], packed[2], packed[3]);
            if (sub == 0) scale[r] = sc;
        }
    }
}

}  // namespace kv

bool kv_quant_warp_supported(int D) { return D == 128 || D == 256 || D == 512; }

cudaError_t launch_kv_quant_warp(const void* kv, size_t rows, int D, float c_n, uint8_t* q, float* scale,
                                 cudaStream_t st) {
    const int LPV = D / 32;
    const size_t per_block = 8 * (size_t)(32 / LPV);        // vectors per block per pass
    size_t blocks = (rows + per_block - 1) / per_block;
    const size_t cap = (size_t)device_sm_count() * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    const __half* x = reinterpret_cast<const __half*>(kv);
    if (LPV == 4) kv::quant_kernel<4><<<(unsigned)blocks, 256, 0, st>>>(x, rows, c_n, q, scale);
    else if (LPV == 8) kv::quant_kernel<8><<<(unsigned)blocks, 256, 0, st>>>(x, rows, c_n, q, scale);
    else if (LPV == 16) kv::quant_kernel<16><<<(unsigned)blocks, 256, 0, st>>>(x, rows, c_n, q, scale);
    else return cudaErrorInvalidValue;
    return cudaGetLastError();
}

cudaError_t launch_kv_dequant(const uint8_t* q, const float* scale, size_t rows, int D, void* out,
                              cudaStream_t st) {
    const size_t cap = (size_t)device_sm_count() * 16;
    if (D >= 32 && (D & (D - 1)) == 0) {
        int lg = 0;                       // log2 of the code words per row (D / 8)
        while ((8 << lg) < D) ++lg;
        const size_t words = rows << lg;
        size_t blocks = (words + 1023) / 1024;
        if (blocks > cap) blocks = cap;
        if (blocks < 1) blocks = 1;
        kv::dequant_words_kernel<<<(unsigned)blocks, 256, 0, st>>>(reinterpret_cast<const uint32_t*>(q), scale, words,
                                                                    lg, reinterpret_cast<uint4*>(out));
        return cudaGetLastError();
    }
    const size_t total = rows * (size_t)(D / 8);
    size_t blocks = (total + 255) / 256;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    kv::dequant_kernel<<<(unsigned)blocks, 256, 0, st>>>(q, scale, rows, D, reinterpret_cast<__half*>(out));
    return cudaGetLastError();
}

}  // namespace rrs
