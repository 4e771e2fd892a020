// rrs_mlp.cu -- the step between the two RRS linears of a gated MLP block:
// H = silu(gate) * up, from the fused gate/up projection's fp32 output, as the
// fp16 activations of the down projection.
//
// GU is [M, 2F] row-major with the gate columns first (the weight rows of the
// fused projection are [W_gate; W_up]).  silu(g) = g / (1 + exp(-g)) in fp32;
// the product is rounded to fp16 and saturated to +-65504, the range the down
// projection's activation path accepts.  Element-wise and HBM-bound: 8 bytes
// read and 2 bytes written per output.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "rrs_device.cuh"
#include "rrs_internal.h"

namespace rrs {
namespace mlp {


// Four outputs per thread when F % 4 == 0 (16-byte loads, 8-byte stores).
__global__ void silu_mul_vec4_kernel(const float* GU, int M, int F, __half* H) {
    const int F4 = F / 4;
    const size_t total = (size_t)M * F4;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
        const size_t m = i / F4;
        const int c = (int)(i % F4);
        const float4 g = reinterpret_cast<const float4*>(GU + m * 2 * F)[c];
        const float4 u = reinterpret_cast<const float4*>(GU + m * 2 * F + F)[c];
        const __half2 a = __floats2half2_rn(silu_mul(g.x, u.x), silu_mul(g.y, u.y));
        const __half2 b = __floats2half2_rn(silu_mul(g.z, u.z), silu_mul(g.w, u.w));
        uint2 o;
        o.x = *reinterpret_cast<const uint32_t*>(&a);
        o.y = *reinterpret_cast<const uint32_t*>(&b);
        reinterpret_cast<uint2*>(H + m * F)[c] = o;
    }
}

__global__ void silu_mul_kernel(const float* GU, int M, int F, __half* H) {
    const size_t total = (size_t)M * F;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
        const size_t m = i / F;
        const int c = (int)(i % F);
        H[i] = __float2half_rn(silu_mul(GU[m * 2 * F + c], GU[m * 2 * F + F + c]));
    }
}

}  // namespace mlp

cudaError_t launch_silu_mul(const float* GU, int M, int F, void* H, cudaStream_t st) {
    const int nsm = device_sm_count();
    __half* h = reinterpret_cast<__half*>(H);
    const bool vec = F % 4 == 0;
    const size_t items = (size_t)M * (vec ? F / 4 : F);
    size_t blocks = (items + 255) / 256;
    if (blocks > (size_t)nsm * 16) blocks = (size_t)nsm * 16;
    if (vec) mlp::silu_mul_vec4_kernel<<<(unsigned)blocks, 256, 0, st>>>(GU, M, F, h);
    else mlp::silu_mul_kernel<<<(unsigned)blocks, 256, 0, st>>>(GU, M, F, h);
    return cudaGetLastError();
}

}  // namespace rrs
