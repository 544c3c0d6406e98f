// Decode kernels instantiated for group sizes 7 and 8.
#include "hhr_group.cuh"

namespace hhr {
HHR_INSTANTIATE_DECODE(7)
HHR_INSTANTIATE_DECODE(8)
}  // namespace hhr
