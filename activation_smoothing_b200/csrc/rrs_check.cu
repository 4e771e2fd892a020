// rrs_check.cu -- validity check of the reorder index (debug entry).
//
// The reorder of the rebuttal page ("Description of the reorder process")
// permutes channels, and the hot path trusts the index it is given: a value out
// of range would read outside a row.  This check marks every value in a bitmap
// and reports the first position holding an out-of-range value, then the
// smallest value that no position holds (with K in-range entries, a missing
// value is the same thing as a repeated one).
#include <cuda_runtime.h>

#include <cstdint>

#include "rrs_internal.h"

namespace rrs {
namespace check {

// words[0] = smallest position j with perm[j] outside [0, K) (K if none),
// words[1] = smallest value in [0, K) that no position holds (K if none).
__global__ void mark_kernel(const int32_t* perm, int K, uint32_t* bitmap, uint32_t* words) {
    for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < K; j += gridDim.x * blockDim.x) {
        const int32_t v = perm[j];
        if (v < 0 || v >= K)
            atomicMin(&words[0], (uint32_t)j);
        else
            atomicOr(&bitmap[v >> 5], 1u << (v & 31));
    }
}

__global__ void missing_kernel(int K, const uint32_t* bitmap, uint32_t* words) {
    const int nwords = (K + 31) / 32;
    for (int w = blockIdx.x * blockDim.x + threadIdx.x; w < nwords; w += gridDim.x * blockDim.x) {
        const int bits = (K - 32 * w) < 32 ? (K - 32 * w) : 32;
        const uint32_t want = bits == 32 ? 0xFFFFFFFFu : ((1u << bits) - 1u);
        const uint32_t gap = ~bitmap[w] & want;
        if (gap) atomicMin(&words[1], (uint32_t)(32 * w + __ffs(gap) - 1));
    }
}

__global__ void init_kernel(int K, uint32_t* bitmap, uint32_t* words) {
    const int nwords = (K + 31) / 32;
    for (int w = blockIdx.x * blockDim.x + threadIdx.x; w < nwords; w += gridDim.x * blockDim.x) bitmap[w] = 0;
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        words[0] = (uint32_t)K;
        words[1] = (uint32_t)K;
    }
}

}  // namespace check

size_t perm_check_bytes(int K) { return 16 + 4 * (size_t)((K + 31) / 32); }

cudaError_t launch_perm_check(const int32_t* perm, int K, void* scratch, cudaStream_t st) {
    uint32_t* words = reinterpret_cast<uint32_t*>(scratch);
    uint32_t* bitmap = words + 4;
    const int nwords = (K + 31) / 32;
    const int b_words = (nwords + 255) / 256;
    const int b_perm = (K + 255) / 256;
    check::init_kernel<<<b_words, 256, 0, st>>>(K, bitmap, words);
    check::mark_kernel<<<b_perm, 256, 0, st>>>(perm, K, bitmap, words);
    check::missing_kernel<<<b_words, 256, 0, st>>>(K, bitmap, words);
    return cudaGetLastError();
}

}  // namespace rrs
