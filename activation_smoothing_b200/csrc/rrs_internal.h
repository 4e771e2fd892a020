// rrs_internal.h -- host-side launch interfaces between the C-ABI layer
// (rrs_api.cu) and the kernel files.  Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace rrs {

// Per-device launch facts, looked up once per device and kept: the number of
// SMs, and for a kernel the dynamic shared memory attribute already set and
// its occupancy.  Launch paths call these instead of querying the runtime on
// every call (the queries cost more host time than a small kernel runs).
int device_sm_count();
// Raises the kernel's dynamic shared-memory limit to `smem` when needed (it only
// ever grows, per device) and returns blocks per SM for (threads, smem); `cache`
// is the kernel's own slot and remembers the last (threads, smem) per device.
struct KernelSetup {
    size_t attr[16] = {0};
    int threads[16] = {0};
    size_t smem[16] = {0};
    int occ[16] = {0};
};
cudaError_t kernel_setup(const void* kern, int threads, size_t smem, KernelSetup& cache, int* occ_out);

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
    const uint8_t* qW;      // [N, K/2] packed INT4 weights
    const float* s;         // [K/G]
    const float* scale_t;   // [M]
    const float* scale_w;   // [N]
    int M, N, K, G;
    float* Y;               // [M, N] (null in debug mode)
    int32_t* P;             // [K/G, M, N] debug partials (null in normal mode)
    uint32_t* err;          // workspace error word
    float* part;            // workspace room for split-k partial sums (may be null)
    size_t part_bytes;
    bool y_bf16;            // Y is bf16 [M, N] instead of fp32
};

// Token counts up to this may split k across CTAs; the workspace then holds
// up to kSplitRoom * M * N fp32 partial sums after the int8 operand.
constexpr int kSplitRoomMaxM = 16;
constexpr int kSplitRoom = 16;

// Fast activation path (K % 2048 == 0): one cooperative kernel, phase A (group
// maxima -> s) and phase B (quantise with s), no M x K intermediate.
struct PrepFastLaunch {
    const void* X;          // fp16 [rows, K]
    int rows, K, n, G;
    float c_n;
    const int32_t* perm;
    int unit_scales;
    int phase;              // 3: both phases; 1: phase A only (writes s); 2: phase B only (reads s)
    float* s;               // [K/G]
    uint8_t* qX;            // [rows, K/2]
    int8_t* qX8;            // [rows, K] GEMM operand or null: int8 codes (GEMM k order), or e4m3 (natural) if a_e4m3
    float* scale_t;         // [rows]
    bool a_e4m3;            // write the fp8 GEMM operand instead of the int8 one
    float* partial;         // per-CTA group maxima: partial_rows x K/G floats (workspace)
    int partial_rows;       // capacity of that table in CTAs (caps the grid)
    uint32_t* gbar;         // grid barrier words (workspace header, zero-filled)
    uint32_t* err;          // workspace error word
};

bool prep_fast_supported(int K, int n);
int prep_fast_rows_per_cta(int K);
cudaError_t launch_prep_fast(const PrepFastLaunch& pl, cudaStream_t stream);
// KV cache: out fp16 [rows, D] = code * scale[row] from packed INT4 q [rows, D/2].
// KV-cache quantisation for head sizes 128, 256, 512: 32 channels per lane.
bool kv_quant_warp_supported(int D);
cudaError_t launch_kv_quant_warp(const void* kv, size_t rows, int D, float c_n, uint8_t* q, float* scale,
                                 cudaStream_t stream);
cudaError_t launch_kv_dequant(const uint8_t* q, const float* scale, size_t rows, int D, void* out,
                              cudaStream_t stream);
// p[0..n) = v.
cudaError_t launch_fill(float* p, int n, float v, cudaStream_t stream);
// The whole linear layer for M <= 16 tokens in one cooperative launch
// (rrs_decode.cu).  `body` is the workspace past its 256-byte header, at least
// decode_ws_bytes(M, N, K) bytes; gbar and err are the header's words.
struct DecodeLaunch {
    const void* X;             // fp16 [M, K]
    const int32_t* perm;
    const uint8_t* qW;         // packed [N, K/2]
    const float* scale_w;
    int M, N, K, G, n;
    float c_n;
    int unit_scales;
    uint8_t* qX;
    float* s;
    float* scale_t;
    void* Y;                   // fp32 or bf16 [M, N]
    int ybf16;
    void* body;
    uint32_t* gbar;
    uint32_t* err;
};
bool decode_supported(int M, int N, int K, int G, int n);
bool decode_preferred(int M, int N, int K);
size_t decode_ws_bytes(int M, int N, int K);
cudaError_t launch_decode(const DecodeLaunch& dl, cudaStream_t stream);

// Reorder-index check (rrs_check.cu): scratch of perm_check_bytes(K) bytes;
// words 0 and 1 of it receive the first out-of-range position and the smallest
// missing value (K when there is none).
size_t perm_check_bytes(int K);
cudaError_t launch_perm_check(const int32_t* perm, int K, void* scratch, cudaStream_t stream);
// Packed INT4 rows -> int8 rows in the GEMM's k order.
cudaError_t launch_expand(const uint8_t* qX, int8_t* qX8, int M, int K, cudaStream_t stream);

cudaError_t launch_gemm(const GemmLaunch& gl, cudaStream_t stream);

// Prefill GEMM on fp8 (e4m3) operands: both INT4 code sets stored one code per
// byte as e4m3 numbers in natural k order (exact; see rrs_gemm_f8.cu).
struct GemmF8Launch {
    const void* A;          // e4m3 [M, K] activation codes
    const void* B;          // e4m3 [N, K] weight codes
    const float* s;         // [K/G]
    const float* scale_t;   // [M]
    const float* scale_w;   // [N]
    int M, N, K, G, PB;     // PB: promotion block (a multiple of 128 dividing G, <= 4096)
    void* Y;                // fp32 or bf16 [M, N] (null in debug mode)
    int32_t* P;             // [K/G, M, N] debug partials (null in normal mode)
    uint32_t* err;          // workspace error word
    int ymode;              // 0 fp32 Y, 1 bf16 Y, 2 H = fp16(silu(y[2f]) * y[2f+1]) [M, N/2]
    int bn;                 // tile width 128 or 256; 0 = chosen from the shape
    cudaStream_t stream;
};
cudaError_t launch_gemm_f8(const GemmF8Launch& gl);
// Tile choice of the fp8 GEMM: 128 or 256 (one CTA, 128 rows x that many
// columns), or a CTA pair of 256 rows x 256 / 128 columns.
constexpr int kPickPair256 = 512;
constexpr int kPickPair128 = 640;
int gemm_f8_pick_bn(int M, int N, int nsm);
// Packed INT4 rows [rows, K/2] -> e4m3 codes [rows, K], natural k order.
cudaError_t launch_expand_e4m3(const uint8_t* q, uint8_t* out, int rows, int K, cudaStream_t stream);
// Longest block of k, a multiple of 128 and at most 4096, that divides G: the
// unit in which both GEMMs promote exact partial sums.
int promotion_block(int G);
// H fp16 [M, F] = silu(GU[:, :F]) * GU[:, F:], GU fp32 [M, 2F].
cudaError_t launch_silu_mul(const float* GU, int M, int F, void* H, cudaStream_t stream);
cudaError_t launch_divide_check(const float* a, const float* b, int n, float* q_fast, float* q_ieee,
                                cudaStream_t stream);

cudaError_t launch_wait_probe(uint64_t limit_ns, uint32_t* err, cudaStream_t stream);

}  // namespace rrs
