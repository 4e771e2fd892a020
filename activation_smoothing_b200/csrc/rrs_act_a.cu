// rrs_act_a.cu -- instantiations of the activation kernel (rrs_act.cuh) for
// Hadamard sizes 2^L, L in {0, 1, 2, 3, 4, 5, 6, 7, 8}; split from the other sizes so that they compile
// in parallel.
#include "rrs_act.cuh"

namespace rrs {
namespace fast {
template cudaError_t launch_act<0>(const ActArgs&, bool, int, size_t, int, cudaStream_t);
template cudaError_t launch_act<1>(const ActArgs&, bool, int, size_t, int, cudaStream_t);
template cudaError_t launch_act<2>(const ActArgs&, bool, int, size_t, int, cudaStream_t);
template cudaError_t launch_act<3>(const ActArgs&, bool, int, size_t, int, cudaStream_t);
template cudaError_t launch_act<4>(const ActArgs&, bool, int, size_t, int, cudaStream_t);
template cudaError_t launch_act<5>(const ActArgs&, bool, int, size_t, int, cudaStream_t);
template cudaError_t launch_act<6>(const ActArgs&, bool, int, size_t, int, cudaStream_t);
template cudaError_t launch_act<7>(const ActArgs&, bool, int, size_t, int, cudaStream_t);
template cudaError_t launch_act<8>(const ActArgs&, bool, int, size_t, int, cudaStream_t);
}  // namespace fast
}  // namespace rrs
