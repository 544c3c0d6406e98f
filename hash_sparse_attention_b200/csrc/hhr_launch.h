// Host-side launch interface between the C ABI (hhr_api.cu) and the kernel
// translation units.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "hhr.h"
#include "hhr_common.cuh"

namespace hhr {

constexpr int MAX_SELECT_PAGES = 8192;   // pages of one sequence in the page select (shared memory)
constexpr int MAX_DENSE_PAGES = 16384;   // pages of one sequence elsewhere
constexpr int MAX_KEEP_PAGES = 2048;     // kept pages per sequence
constexpr int MAX_CANDIDATES = 16384;    // kept pages x page size (scores in shared memory)
constexpr int FUSED_ROWS = 128;          // pages per scan item, rows per gather item
constexpr int MAX_GRID = 160;            // CTAs of the fused kernel (one per SM)
constexpr int FUSED_GROUP = 16;          // gather chunks merged together first
constexpr int FUSED_SCORE = 1024;        // candidate rows per score item
constexpr int MAX_GATHER_GROUPS = 256;   // groups per unit (final merge width)
constexpr int GROUP_GX_WORDS = 4;       // per-unit counters of the group kernel

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
  int num_sms;
};

hhr_status record_error(hhr_status s, const char* msg);

template <int G> cudaError_t launch_decode(const DecodeArgs& a);
template <int G> cudaError_t launch_dense(const DecodeArgs& a);

cudaError_t launch_build(const Dims& dm, const __nv_bfloat16* K, const float* R, const __nv_bfloat16* W,
                         const int* seq_lens, const int* table, __nv_bfloat16* Krot, __nv_bfloat16* pmin,
                         __nv_bfloat16* pmax, uint64_t* codes, int* status, cudaStream_t st);

}  // namespace hhr
