// Cache-build kernel instantiations and launcher.
#include "hhr_build.cuh"

namespace hhr {

template <int NB>
static cudaError_t launch_build_nb(const Dims& dm, const __nv_bfloat16* K, const float* R, const __nv_bfloat16* W,
                                   const int* seq_lens, const int* table, __nv_bfloat16* Krot, __nv_bfloat16* pmin,
                                   __nv_bfloat16* pmax, uint64_t* codes, int* status, cudaStream_t st) {
  const size_t smem = BuildSmem::bytes(NB);
  // the attribute belongs to the function; setting it again is harmless
  cudaError_t e = cudaFuncSetAttribute(build_cache_kernel<NB>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 grid((dm.T + BUILD_ROWS * BUILD_TILES - 1) / (BUILD_ROWS * BUILD_TILES), dm.Hkv, dm.B);
  build_cache_kernel<NB><<<grid, BUILD_THREADS, smem, st>>>(dm, K, R, W, seq_lens, table, Krot, pmin, pmax, codes,
                                                             status);
  return cudaGetLastError();
}

cudaError_t launch_build(const Dims& dm, const __nv_bfloat16* K, const float* R, const __nv_bfloat16* W,
                         const int* seq_lens, const int* table, __nv_bfloat16* Krot, __nv_bfloat16* pmin,
                         __nv_bfloat16* pmax, uint64_t* codes, int* status, cudaStream_t st) {
  switch (dm.nb) {
    case 64: return launch_build_nb<64>(dm, K, R, W, seq_lens, table, Krot, pmin, pmax, codes, status, st);
    case 128: return launch_build_nb<128>(dm, K, R, W, seq_lens, table, Krot, pmin, pmax, codes, status, st);
    case 256: return launch_build_nb<256>(dm, K, R, W, seq_lens, table, Krot, pmin, pmax, codes, status, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace hhr
