// Decode-step and dense kernels instantiated for group sizes 5 and 6.
#include "hhr_dense.cuh"

namespace hhr {
HHR_INSTANTIATE_DECODE(5)
HHR_INSTANTIATE_DECODE(6)
}  // namespace hhr
