// rrs_api.cu -- the extern "C" entry points declared in include/rrs.h:
// argument validation on the host, then stream-ordered kernel launches.
// No entry point allocates memory; only rrs_check_workspace, rrs_check_perm
// and rrs_linear_from_host synchronise the host.
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <numeric>
#include <vector>

#include "rrs.h"
#include "rrs_device.cuh"
#include "rrs_internal.h"

namespace {

thread_local char g_last_error[512] = "no error";

rrs_status fail(rrs_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return st;
}

rrs_status cuda_fail(cudaError_t e, const char* what) {
    return fail(RRS_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

// One NVTX range per entry point, named after it, for timeline tools; without
// a tool attached the push and pop return at once.
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
};
#define RRS_TRACE() NvtxRange rrs_trace_range_(__func__)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int kMaxK = 32768;
constexpr int kMaxHadamard = 8192;
constexpr size_t kHeaderBytes = 256;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace layout: [header 256 B: error word at 0, grid-barrier words at 64]
// [activation operand for the GEMM, M*K bytes] [per-CTA group maxima of the
// activation kernel: one row of K/128 floats per CTA, fast path only].  For
// M <= 16 the space after the operand also takes the GEMM's split-k partial
// sums (the activation kernel's table is dead by then).
constexpr size_t kBarrierOffset = 64;
constexpr int kMaxPartialRows = 1024;
size_t ws_a8_offset() { return kHeaderBytes; }
size_t ws_bytes_gemm(int M, int K) { return kHeaderBytes + align256((size_t)M * K); }
int ws_partial_rows(int M, int K) {
    const int R = rrs::prep_fast_rows_per_cta(K);
    const int rows = (M + R - 1) / R;
    return rows < kMaxPartialRows ? rows : kMaxPartialRows;
}
size_t ws_bytes_full(int M, int K, int n) {
    size_t b = ws_bytes_gemm(M, K);
    if (rrs::prep_fast_supported(K, n)) b += align256((size_t)ws_partial_rows(M, K) * (K / 128) * 4);
    return b;
}

#define RRS_REQUIRE_PTR(p)                                                          \
    do {                                                                            \
        if ((p) == nullptr) return fail(RRS_ERR_INVALID_ARG, "%s is null", #p);     \
        if (!aligned16(p))                                                          \
            return fail(RRS_ERR_INVALID_ARG, "%s is not 16-byte aligned", #p);      \
    } while (0)

rrs_status check_K(int K) {
    if (K < 128 || K % 128 != 0)
        return fail(K > 0 && K % 2 == 0 ? RRS_ERR_UNSUPPORTED : RRS_ERR_INVALID_ARG,
                    "K = %d: the CUDA path needs K a positive multiple of 128", K);
    if (K > kMaxK) return fail(RRS_ERR_UNSUPPORTED, "K = %d exceeds the limit %d", K, kMaxK);
    return RRS_OK;
}

// Resolves the Hadamard block size (1 under RRS_NO_ROTATE) and its scale.
rrs_status check_hadamard(int K, int had_block, unsigned flags, int* n, float* c_n) {
    int nn = (flags & RRS_NO_ROTATE) ? 1 : had_block;
    if (nn < 1 || (nn & (nn - 1)) != 0)
        return fail(RRS_ERR_INVALID_ARG, "had_block = %d is not a power of two", had_block);
    if (nn > kMaxHadamard)
        return fail(RRS_ERR_UNSUPPORTED, "had_block = %d exceeds %d", nn, kMaxHadamard);
    if (K % nn != 0) return fail(RRS_ERR_INVALID_ARG, "K = %d is not a multiple of had_block = %d", K, nn);
    *n = nn;
    *c_n = (float)(1.0 / std::sqrt((double)nn));
    return RRS_OK;
}

rrs_status check_G(int K, int G) {
    if (G < 1 || K % G != 0) return fail(RRS_ERR_INVALID_ARG, "G = %d does not divide K = %d", G, K);
    if (G % 128 != 0) return fail(RRS_ERR_UNSUPPORTED, "G = %d: the CUDA path needs G %% 128 == 0", G);
    return RRS_OK;
}

rrs_status check_ws(void* ws, size_t ws_bytes, size_t need) {
    if (ws == nullptr || ws_bytes < need)
        return fail(RRS_ERR_WORKSPACE, "workspace %p of %zu bytes, need %zu (rrs_workspace_size)", ws, ws_bytes, need);
    if (!aligned16(ws)) return fail(RRS_ERR_INVALID_ARG, "workspace is not 16-byte aligned");
    return RRS_OK;
}

// phase 3: group maxima then quantisation (rrs_smooth_quant); 1: group maxima
// only (pass A, writes s); 2: quantisation with the caller's s (pass B).
rrs_status launch_smooth_quant(const void* X, int M, int K, int G, int n, float c_n, const int32_t* perm,
                               uint8_t* qX, float* s, float* scale_t, void* ws, unsigned flags, cudaStream_t st,
                               int phase = 3) {
    const int unit = (flags & RRS_FORCE_UNIT_SCALES) ? 1 : 0;
    int8_t* qX8 = reinterpret_cast<int8_t*>(static_cast<unsigned char*>(ws) + ws_a8_offset());
    if (rrs::prep_fast_supported(K, n)) {
        rrs::PrepFastLaunch pf{};
        pf.X = X;
        pf.rows = M;
        pf.K = K;
        pf.n = n;
        pf.G = G;
        pf.c_n = c_n;
        pf.perm = perm;
        pf.unit_scales = unit;
        pf.s = s;
        pf.qX = qX;
        pf.qX8 = qX8;
        pf.scale_t = scale_t;
        pf.phase = phase;
        pf.a_e4m3 = (flags & RRS_W_EXPANDED) != 0;
        pf.partial = reinterpret_cast<float*>(static_cast<unsigned char*>(ws) + ws_bytes_gemm(M, K));
        pf.partial_rows = ws_partial_rows(M, K);
        pf.gbar = reinterpret_cast<uint32_t*>(static_cast<unsigned char*>(ws) + kBarrierOffset);
        pf.err = reinterpret_cast<uint32_t*>(ws);
        cudaError_t e = rrs::launch_prep_fast(pf, st);
        if (e != cudaSuccess) return cuda_fail(e, "rotation/quantise kernels");
        return RRS_OK;
    }
    // General shapes: two passes that each rotate, then the int8 operand.
    rrs::PrepLaunch pl{};
    pl.X = X;
    pl.rows = M;
    pl.K = K;
    pl.n = n;
    pl.G = G;
    pl.c_n = c_n;
    pl.perm = perm;
    if (!unit && (phase & 1)) {
        cudaError_t e = cudaMemsetAsync(s, 0, sizeof(float) * (size_t)(K / G), st);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(s)");
        pl.mode = 1;
        pl.max_out = reinterpret_cast<uint32_t*>(s);
        e = rrs::launch_prep(pl, st);
        if (e != cudaSuccess) return cuda_fail(e, "group-max kernel");
    }
    if (!(phase & 2)) return RRS_OK;
    pl.mode = 0;
    pl.max_out = nullptr;
    pl.unit_scales = unit;
    pl.s_in = s;
    pl.q_out = qX;
    pl.scale_out = scale_t;
    pl.s_unit_out = unit ? s : nullptr;
    cudaError_t e = rrs::launch_prep(pl, st);
    if (e != cudaSuccess) return cuda_fail(e, "quantise kernel");
    e = (flags & RRS_W_EXPANDED) ? rrs::launch_expand_e4m3(qX, reinterpret_cast<uint8_t*>(qX8), M, K, st)
                                 : rrs::launch_expand(qX, qX8, M, K, st);
    if (e != cudaSuccess) return cuda_fail(e, "expand kernel");
    return RRS_OK;
}

rrs_status launch_gemm_checked(const uint8_t* qX, const float* s, const float* scale_t, const uint8_t* qW,
                               const float* scale_w, int M, int N, int K, int G, float* Y, int32_t* P,
                               void* ws, size_t ws_bytes, unsigned flags, cudaStream_t st) {
    int8_t* qX8 = reinterpret_cast<int8_t*>(static_cast<unsigned char*>(ws) + ws_a8_offset());
    if (flags & RRS_W_EXPANDED) {
        // fp8 operands: e4m3 activation codes in the workspace, e4m3 weight codes
        if (!(flags & RRS_WS_HOLDS_A8)) {
            cudaError_t e = rrs::launch_expand_e4m3(qX, reinterpret_cast<uint8_t*>(qX8), M, K, st);
            if (e != cudaSuccess) return cuda_fail(e, "expand kernel");
        }
        rrs::GemmF8Launch gf{};
        gf.A = qX8;
        gf.B = qW;
        gf.s = s;
        gf.scale_t = scale_t;
        gf.scale_w = scale_w;
        gf.M = M;
        gf.N = N;
        gf.K = K;
        gf.G = G;
        gf.PB = rrs::promotion_block(G);
        gf.Y = Y;
        gf.P = P;
        gf.err = reinterpret_cast<uint32_t*>(ws);
        gf.ymode = P != nullptr ? 0 : (flags & RRS_Y_SILU_MUL) ? 2 : (flags & RRS_Y_BF16) ? 1 : 0;
        gf.bn = 0;
        gf.stream = st;
        cudaError_t e = rrs::launch_gemm_f8(gf);
        if (e != cudaSuccess) return cuda_fail(e, "GEMM kernel");
        return RRS_OK;
    }
    if (!(flags & RRS_WS_HOLDS_A8)) {
        cudaError_t e = rrs::launch_expand(qX, qX8, M, K, st);
        if (e != cudaSuccess) return cuda_fail(e, "expand kernel");
    }
    rrs::GemmLaunch gl{};
    gl.qX8 = qX8;
    gl.qW = qW;
    gl.s = s;
    gl.scale_t = scale_t;
    gl.scale_w = scale_w;
    gl.M = M;
    gl.N = N;
    gl.K = K;
    gl.G = G;
    gl.Y = Y;
    gl.P = P;
    gl.err = reinterpret_cast<uint32_t*>(ws);
    gl.y_bf16 = P == nullptr && (flags & RRS_Y_BF16) != 0;
    // Room after the int8 operand (the activation scratch, dead once the
    // activation kernels have run) takes split-k partial sums for small M.
    const size_t used = ws_bytes_gemm(M, K);
    gl.part = ws_bytes > used ? reinterpret_cast<float*>(static_cast<unsigned char*>(ws) + used) : nullptr;
    gl.part_bytes = ws_bytes > used ? ws_bytes - used : 0;
    cudaError_t e = rrs::launch_gemm(gl, st);
    if (e != cudaSuccess) return cuda_fail(e, "GEMM kernel");
    return RRS_OK;
}

}  // namespace

// ---------------------------------------------------------------------------
// Scratch for rrs_smooth_quant_noalloc: a fixed device array, so that the call
// needs no workspace from the caller.  Every device that loads this library
// holds it (about 5 MiB) until the process exits.  In host code the name
// g_noalloc_ws is only a host-side stand-in; the device address comes from
// cudaGetSymbolAddress, once per device.
namespace {
constexpr size_t kNoAllocMaxElems = (size_t)1 << 20;   // M * K limit
constexpr size_t kNoAllocBytes = kHeaderBytes + kNoAllocMaxElems + kNoAllocMaxElems * 4;
}  // namespace

static __device__ __align__(256) unsigned char g_noalloc_ws[kNoAllocBytes];

namespace {
// Device address of g_noalloc_ws on the current device.  Looked up on every
// call (cheap once the module is loaded), so that it stays right after the
// device's context is reset and the module reloaded.
rrs_status noalloc_scratch(void** out) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_ws);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-allocation scratch)");
    *out = p;
    return RRS_OK;
}
}  // namespace

namespace rrs {

int device_sm_count() {
    static int cached[16] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev < 0 || dev >= 16) {
        int n = 148;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        return n;
    }
    if (cached[dev] == 0) {
        int n = 148;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        cached[dev] = n;
    }
    return cached[dev];
}

cudaError_t kernel_setup(const void* kern, int threads, size_t smem, KernelSetup& cache, int* occ_out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const bool cacheable = dev >= 0 && dev < 16;
    if (cacheable && cache.occ[dev] > 0 && cache.threads[dev] == threads && cache.smem[dev] == smem) {
        *occ_out = cache.occ[dev];
        return cudaSuccess;
    }
    if (!cacheable || smem > cache.attr[dev]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        if (cacheable) cache.attr[dev] = smem;
    }
    int occ = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, threads, smem);
    if (e != cudaSuccess) return e;
    if (cacheable) {
        cache.threads[dev] = threads;
        cache.smem[dev] = smem;
        cache.occ[dev] = occ;
    }
    *occ_out = occ;
    return cudaSuccess;
}

}  // namespace rrs

extern "C" {

size_t rrs_workspace_size(int M, int N, int K, int G, int had_block, unsigned flags) {
    (void)G;
    if (M < 1 || K < 1) return kHeaderBytes;
    const int n = (flags & RRS_NO_ROTATE) ? 1 : had_block;
    size_t b = ws_bytes_full(M, K, n);
    if (M <= 16 && N > 0) b = std::max(b, kHeaderBytes + rrs::decode_ws_bytes(M, N, K));
    if (M <= rrs::kSplitRoomMaxM && N > 0) {
        // split-k partial sums share the space after the int8 operand with the scratch
        const size_t room = align256((size_t)rrs::kSplitRoom * M * N * 4);
        const size_t after = b - ws_bytes_gemm(M, K);
        if (room > after) b += room - after;
    }
    return b;
}

rrs_status rrs_prepare_weights(const void* W, int N, int K, int had_block, const int32_t* perm, uint8_t* qW,
                               float* scale_w, unsigned flags, rrs_stream_t stream) {
    RRS_TRACE();
    RRS_REQUIRE_PTR(W);
    RRS_REQUIRE_PTR(perm);
    RRS_REQUIRE_PTR(qW);
    RRS_REQUIRE_PTR(scale_w);
    if (N < 1) return fail(RRS_ERR_INVALID_ARG, "N = %d", N);
    rrs_status r = check_K(K);
    if (r != RRS_OK) return r;
    int n;
    float c_n;
    r = check_hadamard(K, had_block, flags, &n, &c_n);
    if (r != RRS_OK) return r;
    rrs::PrepLaunch pl{};
    pl.X = W;
    pl.rows = N;
    pl.K = K;
    pl.n = n;
    pl.G = K;
    pl.c_n = c_n;
    pl.perm = perm;
    pl.mode = 0;
    pl.unit_scales = 1;
    pl.q_out = qW;
    pl.scale_out = scale_w;
    cudaError_t e = rrs::launch_prep(pl, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "weight prep kernel");
    return RRS_OK;
}

rrs_status rrs_smooth_quant(const void* X, int M, int K, int G, int had_block, const int32_t* perm, uint8_t* qX,
                            float* s, float* scale_t, void* ws, size_t ws_bytes, unsigned flags,
                            rrs_stream_t stream) {
    RRS_TRACE();
    RRS_REQUIRE_PTR(X);
    RRS_REQUIRE_PTR(perm);
    RRS_REQUIRE_PTR(qX);
    RRS_REQUIRE_PTR(s);
    RRS_REQUIRE_PTR(scale_t);
    if (M < 1) return fail(RRS_ERR_INVALID_ARG, "M = %d", M);
    rrs_status r = check_K(K);
    if (r != RRS_OK) return r;
    r = check_G(K, G);
    if (r != RRS_OK) return r;
    int n;
    float c_n;
    r = check_hadamard(K, had_block, flags, &n, &c_n);
    if (r != RRS_OK) return r;
    r = check_ws(ws, ws_bytes, ws_bytes_full(M, K, n));
    if (r != RRS_OK) return r;
    return launch_smooth_quant(X, M, K, G, n, c_n, perm, qX, s, scale_t, ws, flags,
                               reinterpret_cast<cudaStream_t>(stream));
}

rrs_status rrs_group_max(const void* X, int M, int K, int G, int had_block, const int32_t* perm, float* s,
                         void* ws, size_t ws_bytes, unsigned flags, rrs_stream_t stream) {
    RRS_TRACE();
    RRS_REQUIRE_PTR(X);
    RRS_REQUIRE_PTR(perm);
    RRS_REQUIRE_PTR(s);
    if (M < 1) return fail(RRS_ERR_INVALID_ARG, "M = %d", M);
    rrs_status r = check_K(K);
    if (r != RRS_OK) return r;
    r = check_G(K, G);
    if (r != RRS_OK) return r;
    int n;
    float c_n;
    r = check_hadamard(K, had_block, flags, &n, &c_n);
    if (r != RRS_OK) return r;
    r = check_ws(ws, ws_bytes, ws_bytes_full(M, K, n));
    if (r != RRS_OK) return r;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (flags & RRS_FORCE_UNIT_SCALES) {
        // no smoothing: every scale is 1
        cudaError_t e = rrs::launch_fill(s, K / G, 1.0f, st);
        if (e != cudaSuccess) return cuda_fail(e, "fill kernel");
        return RRS_OK;
    }
    return launch_smooth_quant(X, M, K, G, n, c_n, perm, nullptr, s, nullptr, ws, flags & ~RRS_W_EXPANDED, st, 1);
}

rrs_status rrs_smooth_quant_scaled(const void* X, int M, int K, int G, int had_block, const int32_t* perm,
                                   const float* s, uint8_t* qX, float* scale_t, void* ws, size_t ws_bytes,
                                   unsigned flags, rrs_stream_t stream) {
    RRS_TRACE();
    RRS_REQUIRE_PTR(X);
    RRS_REQUIRE_PTR(perm);
    RRS_REQUIRE_PTR(s);
    RRS_REQUIRE_PTR(qX);
    RRS_REQUIRE_PTR(scale_t);
    if (M < 1) return fail(RRS_ERR_INVALID_ARG, "M = %d", M);
    rrs_status r = check_K(K);
    if (r != RRS_OK) return r;
    r = check_G(K, G);
    if (r != RRS_OK) return r;
    int n;
    float c_n;
    r = check_hadamard(K, had_block, flags, &n, &c_n);
    if (r != RRS_OK) return r;
    r = check_ws(ws, ws_bytes, ws_bytes_full(M, K, n));
    if (r != RRS_OK) return r;
    if (flags & RRS_FORCE_UNIT_SCALES)
        return fail(RRS_ERR_INVALID_ARG, "rrs_smooth_quant_scaled takes its scales from s; RRS_FORCE_UNIT_SCALES "
                                         "does not apply (pass s filled with 1 instead)");
    return launch_smooth_quant(X, M, K, G, n, c_n, perm, qX, const_cast<float*>(s), scale_t, ws, flags,
                               reinterpret_cast<cudaStream_t>(stream), 2);
}

rrs_status rrs_w4a4_gemm(const uint8_t* qX, const float* s, const float* scale_t, const uint8_t* qW,
                         const float* scale_w, int M, int N, int K, int G, float* Y, void* ws, size_t ws_bytes,
                         unsigned flags, rrs_stream_t stream) {
    RRS_TRACE();
    RRS_REQUIRE_PTR(qX);
    RRS_REQUIRE_PTR(s);
    RRS_REQUIRE_PTR(scale_t);
    RRS_REQUIRE_PTR(qW);
    RRS_REQUIRE_PTR(scale_w);
    RRS_REQUIRE_PTR(Y);
    if (M < 1 || N < 1) return fail(RRS_ERR_INVALID_ARG, "M = %d, N = %d", M, N);
    rrs_status r = check_K(K);
    if (r != RRS_OK) return r;
    r = check_G(K, G);
    if (r != RRS_OK) return r;
    r = check_ws(ws, ws_bytes, ws_bytes_gemm(M, K));
    if (r != RRS_OK) return r;
    if (flags & RRS_Y_SILU_MUL) {
        if (!(flags & RRS_W_EXPANDED))
            return fail(RRS_ERR_UNSUPPORTED, "RRS_Y_SILU_MUL needs the fp8 path (RRS_W_EXPANDED)");
        if (N % 2 != 0) return fail(RRS_ERR_INVALID_ARG, "RRS_Y_SILU_MUL needs N even (interleaved gate/up rows), N = %d", N);
    }
    return launch_gemm_checked(qX, s, scale_t, qW, scale_w, M, N, K, G, Y, nullptr, ws, ws_bytes, flags,
                               reinterpret_cast<cudaStream_t>(stream));
}

rrs_status rrs_linear(const void* X, const uint8_t* qW, const float* scale_w, const int32_t* perm, int M, int N,
                      int K, int G, int had_block, uint8_t* qX, float* s, float* scale_t, float* Y, void* ws,
                      size_t ws_bytes, unsigned flags, rrs_stream_t stream) {
    RRS_TRACE();
    if (M >= 1 && M <= 16 && !(flags & (RRS_W_EXPANDED | RRS_Y_SILU_MUL))) {
        // few tokens: the whole layer in one launch when the shape and workspace allow
        RRS_REQUIRE_PTR(X);
        RRS_REQUIRE_PTR(perm);
        RRS_REQUIRE_PTR(qX);
        RRS_REQUIRE_PTR(s);
        RRS_REQUIRE_PTR(scale_t);
        RRS_REQUIRE_PTR(qW);
        RRS_REQUIRE_PTR(scale_w);
        RRS_REQUIRE_PTR(Y);
        if (N < 1) return fail(RRS_ERR_INVALID_ARG, "M = %d, N = %d", M, N);
        rrs_status r = check_K(K);
        if (r != RRS_OK) return r;
        r = check_G(K, G);
        if (r != RRS_OK) return r;
        int n;
        float c_n;
        r = check_hadamard(K, had_block, flags, &n, &c_n);
        if (r != RRS_OK) return r;
        r = check_ws(ws, ws_bytes, ws_bytes_full(M, K, n));
        if (r != RRS_OK) return r;
        if (ws_bytes >= kHeaderBytes + rrs::decode_ws_bytes(M, N, K) && rrs::decode_supported(M, N, K, G, n) &&
            ((flags & RRS_ONE_LAUNCH) || rrs::decode_preferred(M, N, K))) {
            rrs::DecodeLaunch dl{};
            dl.X = X;
            dl.perm = perm;
            dl.qW = qW;
            dl.scale_w = scale_w;
            dl.M = M;
            dl.N = N;
            dl.K = K;
            dl.G = G;
            dl.n = n;
            dl.c_n = c_n;
            dl.unit_scales = (flags & RRS_FORCE_UNIT_SCALES) ? 1 : 0;
            dl.qX = qX;
            dl.s = s;
            dl.scale_t = scale_t;
            dl.Y = Y;
            dl.ybf16 = (flags & RRS_Y_BF16) ? 1 : 0;
            dl.body = static_cast<unsigned char*>(ws) + kHeaderBytes;
            dl.gbar = reinterpret_cast<uint32_t*>(static_cast<unsigned char*>(ws) + kBarrierOffset);
            dl.err = reinterpret_cast<uint32_t*>(ws);
            cudaError_t e = rrs::launch_decode(dl, reinterpret_cast<cudaStream_t>(stream));
            if (e != cudaSuccess) return cuda_fail(e, "single-launch linear kernel");
            return RRS_OK;
        }
    }
    rrs_status r = rrs_smooth_quant(X, M, K, G, had_block, perm, qX, s, scale_t, ws, ws_bytes, flags, stream);
    if (r != RRS_OK) return r;
    return rrs_w4a4_gemm(qX, s, scale_t, qW, scale_w, M, N, K, G, Y, ws, ws_bytes,
                         RRS_WS_HOLDS_A8 | (flags & (RRS_W_EXPANDED | RRS_Y_BF16 | RRS_Y_SILU_MUL)), stream);
}

rrs_status rrs_linear_from_host(const void* X_host, void* X_dev, const uint8_t* qW, const float* scale_w,
                                const int32_t* perm, int M, int N, int K, int G, int had_block, uint8_t* qX,
                                float* s, float* scale_t, float* Y_dev, float* Y_host, void* ws,
                                size_t ws_bytes, unsigned flags, rrs_stream_t stream) {
    RRS_TRACE();
    if (X_host == nullptr || Y_host == nullptr) return fail(RRS_ERR_INVALID_ARG, "host buffer is null");
    RRS_REQUIRE_PTR(X_dev);
    RRS_REQUIRE_PTR(Y_dev);
    if (M < 1 || N < 1 || K < 1) return fail(RRS_ERR_INVALID_ARG, "M = %d, N = %d, K = %d", M, N, K);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(X_dev, X_host, (size_t)M * K * 2, cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess) return cuda_fail(e, "host-to-device copy of X");
    rrs_status r = rrs_linear(X_dev, qW, scale_w, perm, M, N, K, G, had_block, qX, s, scale_t, Y_dev, ws,
                              ws_bytes, flags, stream);
    if (r != RRS_OK) return r;
    const size_t ybytes = (flags & RRS_Y_SILU_MUL) ? (size_t)M * (N / 2) * 2 : (size_t)M * N * ((flags & RRS_Y_BF16) ? 2 : 4);
    e = cudaMemcpyAsync(Y_host, Y_dev, ybytes, cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess) return cuda_fail(e, "device-to-host copy of Y");
    e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    return RRS_OK;
}

rrs_status rrs_w4a4_gemm_debug_partials(const uint8_t* qX, const uint8_t* qW, int M, int N, int K, int G,
                                        int32_t* P, void* ws, size_t ws_bytes, unsigned flags,
                                        rrs_stream_t stream) {
    RRS_TRACE();
    RRS_REQUIRE_PTR(qX);
    RRS_REQUIRE_PTR(qW);
    RRS_REQUIRE_PTR(P);
    if (M < 1 || N < 1) return fail(RRS_ERR_INVALID_ARG, "M = %d, N = %d", M, N);
    rrs_status r = check_K(K);
    if (r != RRS_OK) return r;
    r = check_G(K, G);
    if (r != RRS_OK) return r;
    r = check_ws(ws, ws_bytes, ws_bytes_gemm(M, K));
    if (r != RRS_OK) return r;
    return launch_gemm_checked(qX, nullptr, nullptr, qW, nullptr, M, N, K, G, nullptr, P, ws, ws_bytes,
                               flags & RRS_W_EXPANDED, reinterpret_cast<cudaStream_t>(stream));
}

rrs_status rrs_silu_mul(const float* GU, int M, int F, void* H, rrs_stream_t stream) {
    RRS_TRACE();
    RRS_REQUIRE_PTR(GU);
    RRS_REQUIRE_PTR(H);
    if (M < 1 || F < 1) return fail(RRS_ERR_INVALID_ARG, "M = %d, F = %d", M, F);
    cudaError_t e = rrs::launch_silu_mul(GU, M, F, H, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "silu_mul kernel");
    return RRS_OK;
}

rrs_status rrs_expand_weights(const uint8_t* qW, int N, int K, uint8_t* qW8, rrs_stream_t stream) {
    RRS_TRACE();
    RRS_REQUIRE_PTR(qW);
    RRS_REQUIRE_PTR(qW8);
    if (N < 1) return fail(RRS_ERR_INVALID_ARG, "N = %d", N);
    rrs_status r = check_K(K);
    if (r != RRS_OK) return r;
    cudaError_t e = rrs::launch_expand_e4m3(qW, qW8, N, K, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "expand_weights kernel");
    return RRS_OK;
}

rrs_status rrs_kv_quant(const void* KV, int T, int H, int D, uint8_t* q, float* scale, unsigned flags,
                        rrs_stream_t stream) {
    RRS_TRACE();
    RRS_REQUIRE_PTR(KV);
    RRS_REQUIRE_PTR(q);
    RRS_REQUIRE_PTR(scale);
    if (T < 1 || H < 1) return fail(RRS_ERR_INVALID_ARG, "T = %d, H = %d", T, H);
    if (D < 1 || (D & (D - 1)) != 0) return fail(RRS_ERR_INVALID_ARG, "D = %d is not a power of two", D);
    if (D < 128 || D > kMaxHadamard)
        return fail(RRS_ERR_UNSUPPORTED, "D = %d: the CUDA path takes head sizes 128..%d", D, kMaxHadamard);
    if (flags != 0) return fail(RRS_ERR_INVALID_ARG, "rrs_kv_quant takes no flags (got 0x%x)", flags);
    if (rrs::kv_quant_warp_supported(D)) {
        cudaError_t e = rrs::launch_kv_quant_warp(KV, (size_t)T * H, D, (float)(1.0 / std::sqrt((double)D)), q, scale,
                                                  reinterpret_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return cuda_fail(e, "KV quantise kernel");
        return RRS_OK;
    }
    rrs::PrepLaunch pl{};
    pl.X = KV;
    pl.rows = T * H;
    pl.K = D;
    pl.n = D;
    pl.G = D;
    pl.c_n = (float)(1.0 / std::sqrt((double)D));
    pl.perm = nullptr;           // no reorder
    pl.mode = 0;
    pl.unit_scales = 1;          // no runtime smoothing
    pl.q_out = q;
    pl.scale_out = scale;
    cudaError_t e = rrs::launch_prep(pl, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "KV quantise kernel");
    return RRS_OK;
}

rrs_status rrs_kv_dequant(const uint8_t* q, const float* scale, int T, int H, int D, void* out,
                          rrs_stream_t stream) {
    RRS_TRACE();
    RRS_REQUIRE_PTR(q);
    RRS_REQUIRE_PTR(scale);
    RRS_REQUIRE_PTR(out);
    if (T < 1 || H < 1) return fail(RRS_ERR_INVALID_ARG, "T = %d, H = %d", T, H);
    if (D < 8 || D % 8 != 0) return fail(RRS_ERR_INVALID_ARG, "D = %d is not a positive multiple of 8", D);
    cudaError_t e = rrs::launch_kv_dequant(q, scale, (size_t)T * H, D, out, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "KV dequantise kernel");
    return RRS_OK;
}

rrs_status rrs_check_perm(const int32_t* perm, int K, void* ws, size_t ws_bytes, rrs_stream_t stream) {
    RRS_TRACE();
    RRS_REQUIRE_PTR(perm);
    if (K < 1) return fail(RRS_ERR_INVALID_ARG, "K = %d", K);
    const size_t need = kHeaderBytes + rrs::perm_check_bytes(K);
    rrs_status r = check_ws(ws, ws_bytes, need);
    if (r != RRS_OK) return r;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    unsigned char* scratch = static_cast<unsigned char*>(ws) + kHeaderBytes;
    cudaError_t e = rrs::launch_perm_check(perm, K, scratch, st);
    if (e != cudaSuccess) return cuda_fail(e, "reorder-index check kernels");
    e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    uint32_t words[2] = {0, 0};
    e = cudaMemcpy(words, scratch, sizeof(words), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "reading the check result");
    if (words[0] < (uint32_t)K)
        return fail(RRS_ERR_INVALID_ARG, "perm[%u] is outside [0, %d)", words[0], K);
    if (words[1] < (uint32_t)K)
        return fail(RRS_ERR_INVALID_ARG, "perm is not a permutation: no position holds %u", words[1]);
    return RRS_OK;
}

rrs_status rrs_channel_absmax(const void* X, int M, int K, int had_block, float* cmax, unsigned flags,
                              rrs_stream_t stream) {
    RRS_TRACE();
    RRS_REQUIRE_PTR(X);
    RRS_REQUIRE_PTR(cmax);
    if (M < 1) return fail(RRS_ERR_INVALID_ARG, "M = %d", M);
    rrs_status r = check_K(K);
    if (r != RRS_OK) return r;
    int n;
    float c_n;
    r = check_hadamard(K, had_block, flags, &n, &c_n);
    if (r != RRS_OK) return r;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(cmax, 0, sizeof(float) * (size_t)K, st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(cmax)");
    rrs::PrepLaunch pl{};
    pl.X = X;
    pl.rows = M;
    pl.K = K;
    pl.n = n;
    pl.G = K;
    pl.c_n = c_n;
    pl.mode = 2;
    pl.max_out = reinterpret_cast<uint32_t*>(cmax);
    e = rrs::launch_prep(pl, st);
    if (e != cudaSuccess) return cuda_fail(e, "channel-max kernel");
    return RRS_OK;
}

rrs_status rrs_perm_from_channel_max(const float* cmax_host, int K, int32_t* perm_host) {
    RRS_TRACE();
    if (cmax_host == nullptr || perm_host == nullptr) return fail(RRS_ERR_INVALID_ARG, "null host buffer");
    if (K < 1) return fail(RRS_ERR_INVALID_ARG, "K = %d", K);
    std::vector<int32_t> idx((size_t)K);
    std::iota(idx.begin(), idx.end(), 0);
    std::stable_sort(idx.begin(), idx.end(),
                     [&](int32_t a, int32_t b) { return cmax_host[a] > cmax_host[b]; });
    std::memcpy(perm_host, idx.data(), sizeof(int32_t) * (size_t)K);
    return RRS_OK;
}

rrs_status rrs_check_workspace(void* ws, rrs_stream_t stream) {
    RRS_TRACE();
    if (ws == nullptr) return fail(RRS_ERR_WORKSPACE, "workspace is null");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    uint32_t word = 0;
    e = cudaMemcpy(&word, ws, sizeof(word), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "reading the workspace error word");
    if (word != 0) {
        const uint32_t zero = 0;
        e = cudaMemcpy(ws, &zero, sizeof(zero), cudaMemcpyHostToDevice);
        if (e != cudaSuccess) return cuda_fail(e, "clearing the workspace error word");
        return fail(RRS_ERR_TIMEOUT, "a kernel gave up on a bounded wait (error word 0x%x)", word);
    }
    return RRS_OK;
}

rrs_status rrs_debug_wait_timeout(int limit_us, void* ws, size_t ws_bytes, rrs_stream_t stream) {
    RRS_TRACE();
    rrs_status r = check_ws(ws, ws_bytes, kHeaderBytes);
    if (r != RRS_OK) return r;
    if (limit_us < 1 || limit_us > 1000000) return fail(RRS_ERR_INVALID_ARG, "limit_us = %d", limit_us);
    cudaError_t e = rrs::launch_wait_probe((uint64_t)limit_us * 1000ull, reinterpret_cast<uint32_t*>(ws),
                                           reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "wait probe kernel");
    return RRS_OK;
}

rrs_status rrs_debug_divide(const float* a, const float* b, int n, float* q_fast, float* q_ieee,
                            rrs_stream_t stream) {
    RRS_TRACE();
    if (!a || !b || !q_fast || !q_ieee || n < 1) return fail(RRS_ERR_INVALID_ARG, "rrs_debug_divide arguments");
    cudaError_t e = rrs::launch_divide_check(a, b, n, q_fast, q_ieee, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "divide check kernel");
    return RRS_OK;
}

rrs_status rrs_smooth_quant_noalloc(const void* X, int M, int K, int G, int had_block, const int32_t* perm,
                                    uint8_t* qX, float* s, float* scale_t, unsigned flags, rrs_stream_t stream) {
    RRS_TRACE();
    RRS_REQUIRE_PTR(X);
    RRS_REQUIRE_PTR(perm);
    RRS_REQUIRE_PTR(qX);
    RRS_REQUIRE_PTR(s);
    RRS_REQUIRE_PTR(scale_t);
    if (M < 1) return fail(RRS_ERR_INVALID_ARG, "M = %d", M);
    rrs_status r = check_K(K);
    if (r != RRS_OK) return r;
    r = check_G(K, G);
    if (r != RRS_OK) return r;
    int n;
    float c_n;
    r = check_hadamard(K, had_block, flags, &n, &c_n);
    if (r != RRS_OK) return r;
    const size_t need = ws_bytes_full(M, K, n);
    if ((size_t)M * (size_t)K > kNoAllocMaxElems || need > kNoAllocBytes)
        return fail(RRS_ERR_UNSUPPORTED,
                    "rrs_smooth_quant_noalloc: M*K = %zu exceeds its fixed scratch limit of %zu elements; "
                    "use rrs_smooth_quant with a workspace",
                    (size_t)M * (size_t)K, kNoAllocMaxElems);
    void* ws = nullptr;
    r = noalloc_scratch(&ws);
    if (r != RRS_OK) return r;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // The array keeps the previous call's contents: clear the error word.
    cudaError_t e = cudaMemsetAsync(ws, 0, kHeaderBytes, st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(no-allocation scratch header)");
    return launch_smooth_quant(X, M, K, G, n, c_n, perm, qX, s, scale_t, ws, flags, st);
}

const char* rrs_last_error_string(void) { return g_last_error; }

}  // extern "C"
