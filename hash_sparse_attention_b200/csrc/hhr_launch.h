// Host-side launch interface between the C ABI (hhr_api.cu) and the kernel
// translation units.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "hhr.h"
#include "hhr_common.cuh"

namespace hhr {

constexpr int PREP_THREADS = 256;
constexpr int SCAN_THREADS = 512;
constexpr int SCAN_PAGES = 128;          // pages per scan CTA: 4 per half-warp
constexpr int SEL_KPT = 32;              // keys per thread in the page select
constexpr int MAX_SELECT_PAGES = SCAN_THREADS * SEL_KPT;  // 16384 pages
constexpr int LHP_THREADS = 256;         // one candidate row per thread
constexpr int LHP_KPT = 16;              // candidates per thread per compaction tile
constexpr int ATT_THREADS = 128;         // 8 half-warps
constexpr int ATT_SPLIT = 128;           // kept rows per attention CTA
constexpr int DENSE_SPLIT = 1024;        // rows per dense-attention CTA

struct DecodeArgs {
  Dims dm;
  Work wk;
  const __nv_bfloat16* q;
  const float* R;
  const __nv_bfloat16* W;
  const __nv_bfloat16* Kr;
  const __nv_bfloat16* Vc;
  const __nv_bfloat16* pmin;
  const __nv_bfloat16* pmax;
  const uint64_t* codes;
  const int* seq_lens;
  const int* table;
  const int* n_keep;
  const int* top_k;
  float sm_scale;
  float* out;
  hhr_debug dbg;
  int* status;
  cudaStream_t stream;
};

hhr_status record_error(hhr_status s, const char* msg);

template <int G> cudaError_t launch_decode(const DecodeArgs& a);
template <int G> cudaError_t launch_dense(const DecodeArgs& a);

cudaError_t launch_build(const Dims& dm, const __nv_bfloat16* K, const float* R, const __nv_bfloat16* W,
                         const int* seq_lens, const int* table, __nv_bfloat16* Krot, __nv_bfloat16* pmin,
                         __nv_bfloat16* pmax, uint64_t* codes, int* status, cudaStream_t st);

}  // namespace hhr
