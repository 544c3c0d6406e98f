// Host-side helpers shared by the C ABI translation units (not exported).
#pragma once

#include "hhr_launch.h"

namespace hhr {

hhr_status make_dims(const hhr_config* cfg, Dims* dm);
size_t carve(const Dims& dm, int Nmax, int Kmax, bool dense, char* base, Work* wk);

// Every host-side check of hhr_decode_step's arguments except the workspace;
// fills the dimensions, the kept-page capacity and the workspace size.  No
// CUDA call is made.
hhr_status decode_check(const hhr_config* cfg, const void* q, const float* R, const void* W, const void* Krot,
                        const void* Vcache, const void* page_min, const void* page_max, const uint64_t* codes,
                        const int32_t* seq_lens, const int32_t* block_table, const int32_t* n_keep_pages,
                        const int32_t* top_k, int32_t max_keep_pages, int32_t max_top_k, float sm_scale,
                        const float* out, const char* who, Dims* dm, int* Nmax, size_t* need);

// Launches the decode step on a checked, zero-initialised workspace.
hhr_status decode_launch(const Dims& dm, int Nmax, int32_t max_top_k, const void* q, const float* R, const void* W,
                         const void* Krot, const void* Vcache, const void* page_min, const void* page_max,
                         const uint64_t* codes, const int32_t* seq_lens, const int32_t* block_table,
                         const int32_t* n_keep_pages, const int32_t* top_k, float sm_scale, float* out,
                         const hhr_debug* dbg, void* workspace, int32_t* device_status, hhr_stream_t stream,
                         const char* who);

}  // namespace hhr
