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
    const int8_t* qX8;      // [M, K] int8 activation codes (k order of the fast prep / expand kernels)
    const uint8_t* qW;      // [N, K/2] packed INT4 weights, or [N, K] int8 16 q when w_expanded
    const float* s;         // [K/G]
    const float* scale_t;   // [M]
    const float* scale_w;   // [N]
    int M, N, K, G;
    float* Y;               // [M, N] (null in debug mode)
    int32_t* P;             // [K/G, M, N] debug partials (null in normal mode)
    uint32_t* err;          // workspace error word
    bool w_expanded;        // qW holds the expanded operand written by launch_expand_weights
    float* part;            // workspace room for split-k partial sums (may be null)
    size_t part_bytes;
    bool y_bf16;            // Y is bf16 [M, N] instead of fp32
};

// Token counts up to this may split k across CTAs; the workspace then holds
// up to kSplitRoom * M * N fp32 partial sums after the int8 operand.
constexpr int kSplitRoomMaxM = 16;
constexpr int kSplitRoom = 16;

// Fast activation path (K % 2048 == 0): rotation + reorder + group max into an
// fp32 scratch, then smoothing + quantisation.
struct PrepFastLaunch {
    const void* X;          // fp16 [rows, K]
    int rows, K, n, G;
    float c_n;
    const int32_t* perm;
    int unit_scales;
    float* s;               // [K/G] output (max of |X'| per group, or 1)
    uint8_t* qX;            // [rows, K/2]
    int8_t* qX8;            // [rows, K]
    float* scale_t;         // [rows]
    float* scratch;         // [rows, K] fp32
};

bool prep_fast_supported(int K, int n);
size_t prep_fast_scratch_bytes(int M, int K);
cudaError_t launch_prep_fast(const PrepFastLaunch& pl, cudaStream_t stream);
// Packed INT4 rows -> int8 rows in the GEMM's k order.
cudaError_t launch_expand(const uint8_t* qX, int8_t* qX8, int M, int K, cudaStream_t stream);
// Packed INT4 weight rows -> int8 rows holding 16 q, in the same k order.
cudaError_t launch_expand_weights(const uint8_t* qW, int8_t* qW8, int N, int K, cudaStream_t stream);

cudaError_t launch_gemm(const GemmLaunch& gl, cudaStream_t stream);
// H fp16 [M, F] = silu(GU[:, :F]) * GU[:, F:], GU fp32 [M, 2F].
cudaError_t launch_silu_mul(const float* GU, int M, int F, void* H, cudaStream_t stream);
cudaError_t launch_divide_check(const float* a, const float* b, int n, float* q_fast, float* q_ieee,
                                cudaStream_t stream);

cudaError_t launch_wait_probe(uint64_t limit_ns, uint32_t* err, cudaStream_t stream);

}  // namespace rrs
