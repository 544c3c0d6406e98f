// hhr_decode_step_noalloc: the decode step for callers that cannot allocate
// device memory.  Its workspace is a fixed array in the library's own device
// memory (every GPU that loads the library holds it until the process exits).
#include <cstdio>
#include <mutex>

#include "hhr_api_internal.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[HHR_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device.  The symbol's
// host-side name is only a stand-in, so the address is looked up once per
// device, with that device current, and cached.
hhr_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return hhr::record_error(HHR_ERR_CUDA, "hhr_decode_step_noalloc: no current CUDA device");
  }
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      char msg[256];
      snprintf(msg, sizeof(msg), "hhr_decode_step_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
      cudaGetLastError();
      return hhr::record_error(HHR_ERR_CUDA, msg);
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return HHR_OK;
}

}  // namespace

extern "C" hhr_status hhr_decode_step_noalloc(
    const hhr_config* cfg, const void* q, const float* R, const void* W, const void* Krot, const void* Vcache,
    const void* page_min, const void* page_max, const uint64_t* codes, const int32_t* seq_lens,
    const int32_t* block_table, const int32_t* n_keep_pages, const int32_t* top_k, int32_t max_keep_pages,
    int32_t max_top_k, float sm_scale, float* out, const hhr_debug* dbg, int32_t* device_status,
    hhr_stream_t stream) {
  static const char* who = "hhr_decode_step_noalloc";
  // the same checks, status codes and messages as hhr_decode_step, before any stream work
  hhr::Dims dm;
  int Nmax = 0;
  size_t need = 0;
  hhr_status s = hhr::decode_check(cfg, q, R, W, Krot, Vcache, page_min, page_max, codes, seq_lens, block_table,
                                   n_keep_pages, top_k, max_keep_pages, max_top_k, sm_scale, out, who, &dm, &Nmax,
                                   &need);
  if (s != HHR_OK) return s;
  if (need > (size_t)HHR_NOALLOC_SCRATCH_BYTES) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "%s: these sizes need %zu bytes of scratch; the built-in scratch holds %zu "
             "(use hhr_decode_step with a caller-provided workspace)",
             who, need, (size_t)HHR_NOALLOC_SCRATCH_BYTES);
    return hhr::record_error(HHR_ERR_WORKSPACE, msg);
  }
  void* scratch = nullptr;
  s = scratch_address(&scratch);
  if (s != HHR_OK) return s;
  // the scratch keeps the previous call's contents: clear the part this call uses
  s = hhr_workspace_init(scratch, need, stream);
  if (s != HHR_OK) return s;
  return hhr::decode_launch(dm, Nmax, max_top_k, q, R, W, Krot, Vcache, page_min, page_max, codes, seq_lens,
                            block_table, n_keep_pages, top_k, sm_scale, out, dbg, scratch, device_status, stream,
                            who);
}
