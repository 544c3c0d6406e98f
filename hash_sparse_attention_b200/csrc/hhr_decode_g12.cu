// Decode kernels instantiated for group sizes 1 and 2.
#include "hhr_group.cuh"

namespace hhr {
HHR_INSTANTIATE_DECODE(1)
HHR_INSTANTIATE_DECODE(2)
}  // namespace hhr
