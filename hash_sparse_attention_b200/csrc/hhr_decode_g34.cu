// Decode-step and dense kernels instantiated for group sizes 3 and 4.
#include "hhr_dense.cuh"

namespace hhr {
HHR_INSTANTIATE_DECODE(3)
HHR_INSTANTIATE_DECODE(4)
}  // namespace hhr
