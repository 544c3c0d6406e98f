// Decode-step and dense kernels instantiated for group sizes 1 and 2.
#include "hhr_dense.cuh"

namespace hhr {
HHR_INSTANTIATE_DECODE(1)
HHR_INSTANTIATE_DECODE(2)
}  // namespace hhr
