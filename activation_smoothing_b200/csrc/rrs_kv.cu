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

}  // namespace kv

cudaError_t launch_kv_dequant(const uint8_t* q, const float* scale, size_t rows, int D, void* out,
                              cudaStream_t st) {
    const size_t total = rows * (size_t)(D / 8);
    size_t blocks = (total + 255) / 256;
    const size_t cap = (size_t)device_sm_count() * 16;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    kv::dequant_kernel<<<(unsigned)blocks, 256, 0, st>>>(q, scale, rows, D, reinterpret_cast<__half*>(out));
    return cudaGetLastError();
}

}  // namespace rrs
