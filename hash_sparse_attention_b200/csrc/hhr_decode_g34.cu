// Decode kernels instantiated for group sizes 3 and 4.
#include "hhr_group.cuh"

namespace hhr {
HHR_INSTANTIATE_DECODE(3)
HHR_INSTANTIATE_DECODE(4)
}  // namespace hhr
