// rrs_internal.h -- host-side launch interfaces between the C-ABI layer
// (rrs_api.cu) and the kernel files.  Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace rrs {

struct PrepLaunch {
    const void* X;          // fp16 [rows, K]
    int rows, K, n, G;
    float c_n;
    const int32_t* perm;
    int mode;               // 0 quantise, 1 group max, 2 channel max
    int unit_scales;
    const float* s_in;
    uint8_t* q_out;
    float* scale_out;
    float* s_unit_out;
    uint32_t* max_out;
};

cudaError_t launch_prep(const PrepLaunch& pl, cudaStream_t stream);

struct GemmLaunch {
    const uint8_t* qX;      // [M, K/2]
    const uint8_t* qW;      // [N, K/2]
    const float* s;         // [K/G] (null = all ones)
    const float* scale_t;   // [M]
    const float* scale_w;   // [N]
    int M, N, K, G;
    float* Y;               // [M, N] (null in debug mode)
    int32_t* P;             // [K/G, M, N] debug partials (null in normal mode)
    uint32_t* err;          // workspace error word
};

cudaError_t launch_gemm(const GemmLaunch& gl, cudaStream_t stream);

cudaError_t launch_wait_probe(uint64_t limit_ns, uint32_t* err, cudaStream_t stream);

}  // namespace rrs
