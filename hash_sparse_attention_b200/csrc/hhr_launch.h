// Host-side launch interface between the C ABI (hhr_api.cu) and the kernel
// translation units.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "hhr.h"
#include "hhr_common.cuh"

namespace hhr {

constexpr int MAX_SELECT_PAGES = 8192;   // pages of one sequence in the page select (16 per thread)
constexpr int MAX_DENSE_PAGES = 16384;   // pages of one sequence elsewhere
constexpr int MAX_KEEP_PAGES = 2048;     // kept pages per sequence (shared memory list)
constexpr int MAX_CANDIDATES = 16384;    // kept pages x page size
constexpr int MAX_GRID = 160;            // CTAs of a launch (one per SM)
constexpr int MAX_KEPT_PER_CTA = 10944;  // kept rows one CTA of a decode group gathers (shared memory list)
constexpr int GATHER_ROWS = 128;         // rows per dense split granule
constexpr int GX_STRIDE = 4;             // per-unit counter words
constexpr long long DEFAULT_WAIT_CYCLES = 4000000000ll;  // ~2 s at 1.9 GHz

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
  long long wait_limit;
  int dense_nsplit, dense_rows;
};

hhr_status record_error(hhr_status s, const char* msg);
long long wait_limit_cycles();

// splits per unit and rows per split of the dense kernel
void dense_split(const Dims& dm, int sms, int* nsplit, int* rows);

template <int G> cudaError_t launch_decode(const DecodeArgs& a);
template <int G> cudaError_t launch_dense(const DecodeArgs& a);

// Cache build over rows [starts[b], seq_lens[b]) of every sequence (starts
// NULL: from row 0); max_rows bounds seq_lens[b] - starts[b].
struct BuildArgs {
  Dims dm;
  const __nv_bfloat16* K;
  const __nv_bfloat16* V;
  const float* R;
  const __nv_bfloat16* W;
  const int* starts;
  const int* seq_lens;
  const int* table;
  __nv_bfloat16* Krot;
  __nv_bfloat16* Vcache;
  __nv_bfloat16* pmin;
  __nv_bfloat16* pmax;
  uint64_t* codes;
  int* status;
  int max_rows;
  long long wait_limit;  // SM clock cycles of the bounded wait for the tensor cores
  cudaStream_t stream;
};
cudaError_t launch_build(const BuildArgs& a);

}  // namespace hhr
