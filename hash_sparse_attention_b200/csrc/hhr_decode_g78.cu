// Decode-step and dense kernels instantiated for group sizes 7 and 8.
#include "hhr_dense.cuh"

namespace hhr {
HHR_INSTANTIATE_DECODE(7)
HHR_INSTANTIATE_DECODE(8)
}  // namespace hhr
