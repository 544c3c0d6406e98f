// Cache-build kernel instantiations and launcher.
#include "hhr_build.cuh"

namespace hhr {

template <int NB>
static cudaError_t launch_build_nb(const BuildArgs& a) {
  const size_t smem = BuildSmem::bytes(NB);
  // the attribute belongs to the function; setting it again is harmless
  cudaError_t e = cudaFuncSetAttribute(build_cache_kernel<NB>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // rows per sequence the launch must cover: all of them, or the appended ones
  // (they start inside a 128-row tile, hence one tile more)
  const int span = a.max_rows + (a.starts ? BT_ROWS : 0);
  const dim3 grid((span + BT_ROWS * BT_TILES - 1) / (BT_ROWS * BT_TILES), a.dm.Hkv, a.dm.B);
  build_cache_kernel<NB><<<grid, BT_THREADS, smem, a.stream>>>(a.dm, a.K, a.V, a.R, a.W, a.starts, a.seq_lens, a.table,
                                                               a.Krot, a.Vcache, a.pmin, a.pmax, a.codes, a.status,
                                                               a.wait_limit);
  return cudaGetLastError();
}

cudaError_t launch_build(const BuildArgs& a) {
  switch (a.dm.nb) {
    case 64: return launch_build_nb<64>(a);
    case 128: return launch_build_nb<128>(a);
    case 256: return launch_build_nb<256>(a);
  }
  return cudaErrorInvalidValue;
}

}  // namespace hhr
