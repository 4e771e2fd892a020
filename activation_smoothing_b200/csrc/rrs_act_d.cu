// rrs_act_d.cu -- instantiations of the activation kernel (rrs_act.cuh) for
// Hadamard sizes 2^L, L in {12}; split from the other sizes so that they compile
// in parallel.
#include "rrs_act.cuh"

namespace rrs {
namespace fast {
template cudaError_t launch_act<12>(const ActArgs&, bool, int, size_t, int, cudaStream_t);
}  // namespace fast
}  // namespace rrs
