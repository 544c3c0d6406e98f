// C ABI of libhhr.so: argument validation, workspace carve-out and launches.
// The kernels live in hhr_build.cuh (cache build), hhr_decode.cuh (decode
// step) and hhr_dense.cuh (dense comparison).
#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "hhr_api_internal.h"

using namespace hhr;

namespace {

thread_local char g_err[512] = {0};
std::atomic<long long> g_wait_cycles{DEFAULT_WAIT_CYCLES};

hhr_status fail(hhr_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return s;
}

hhr_status ok() {
  g_err[0] = 0;
  return HHR_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

hhr_status check_cuda(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(HHR_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return HHR_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int ceil_div(long long a, long long b) { return (int)((a + b - 1) / b); }

// SMs of the current device (cached per device), at most MAX_GRID.
int device_sms() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 0;
    cache[dev] = std::min(n, MAX_GRID);
  }
  return cache[dev];
}

// ---- group-size dispatch -------------------------------------------------
#define HHR_DISPATCH_G(G_, ...)                          \
  switch (G_) {                                          \
    case 1: { constexpr int GG = 1; __VA_ARGS__; } break; \
    case 2: { constexpr int GG = 2; __VA_ARGS__; } break; \
    case 3: { constexpr int GG = 3; __VA_ARGS__; } break; \
    case 4: { constexpr int GG = 4; __VA_ARGS__; } break; \
    case 5: { constexpr int GG = 5; __VA_ARGS__; } break; \
    case 6: { constexpr int GG = 6; __VA_ARGS__; } break; \
    case 7: { constexpr int GG = 7; __VA_ARGS__; } break; \
    case 8: { constexpr int GG = 8; __VA_ARGS__; } break; \
    default: break;                                      \
  }

}  // namespace

namespace hhr {

// Records a host-side error message for hhr_last_error() (used by entry
// points defined in other translation units).
hhr_status record_error(hhr_status s, const char* msg) { return fail(s, "%s", msg); }

long long wait_limit_cycles() { return g_wait_cycles.load(std::memory_order_relaxed); }

void dense_split(const Dims& dm, int sms, int* nsplit, int* rows) {
  const int U = dm.B * dm.Hkv;
  int ns = std::max(1, std::min(MAX_GRID, sms / U));
  ns = std::min(ns, ceil_div(dm.T, GATHER_ROWS));
  const int r = ceil_div(ceil_div(dm.T, ns), GATHER_ROWS) * GATHER_ROWS;
  *rows = r;
  *nsplit = ceil_div(dm.T, r);
}

// Validates the configuration and fills the kernel-side dimensions.
hhr_status make_dims(const hhr_config* cfg, Dims* dm) {
  if (!cfg) return fail(HHR_ERR_INVALID_ARG, "cfg is NULL");
  if (cfg->head_dim != D) return fail(HHR_ERR_UNSUPPORTED, "head_dim %d (only 128)", cfg->head_dim);
  if (cfg->batch < 1 || cfg->num_kv_heads < 1 || cfg->num_q_heads < 1 || cfg->max_seq_len < 1)
    return fail(HHR_ERR_INVALID_ARG, "batch, heads and max_seq_len must be >= 1");
  if (cfg->num_q_heads % cfg->num_kv_heads != 0)
    return fail(HHR_ERR_INVALID_ARG, "num_q_heads %d not a multiple of num_kv_heads %d", cfg->num_q_heads,
                cfg->num_kv_heads);
  const int G = cfg->num_q_heads / cfg->num_kv_heads;
  if (G > 8) return fail(HHR_ERR_UNSUPPORTED, "group size %d (1..8)", G);
  if (cfg->page_size != 16 && cfg->page_size != 32)
    return fail(HHR_ERR_UNSUPPORTED, "page_size %d (16 or 32)", cfg->page_size);
  if (cfg->hash_bits != 64 && cfg->hash_bits != 128 && cfg->hash_bits != 256)
    return fail(HHR_ERR_UNSUPPORTED, "hash_bits %d (64, 128 or 256)", cfg->hash_bits);
  const long long np_max = ((long long)cfg->max_seq_len + cfg->page_size - 1) / cfg->page_size;
  if (np_max > MAX_DENSE_PAGES)
    return fail(HHR_ERR_UNSUPPORTED, "%lld pages per sequence (at most %d)", np_max, MAX_DENSE_PAGES);
  if ((long long)cfg->batch * cfg->num_kv_heads * cfg->max_seq_len * D >= (1ll << 31) * D)
    return fail(HHR_ERR_UNSUPPORTED, "cache of %lld rows (at most 2^31)",
                (long long)cfg->batch * cfg->num_kv_heads * cfg->max_seq_len);
  if (cfg->paged) {
    if (cfg->num_blocks < 1) return fail(HHR_ERR_INVALID_ARG, "paged: num_blocks must be >= 1");
    if (cfg->max_blocks_per_seq < np_max)
      return fail(HHR_ERR_INVALID_ARG, "paged: max_blocks_per_seq %d < ceil(max_seq_len / page_size) %lld",
                  cfg->max_blocks_per_seq, np_max);
    if ((long long)cfg->num_blocks * cfg->num_kv_heads * cfg->page_size >= (1ll << 31))
      return fail(HHR_ERR_UNSUPPORTED, "block pool of %lld rows (at most 2^31)",
                  (long long)cfg->num_blocks * cfg->num_kv_heads * cfg->page_size);
  }
  dm->B = cfg->batch;
  dm->Hq = cfg->num_q_heads;
  dm->Hkv = cfg->num_kv_heads;
  dm->G = G;
  dm->P = cfg->page_size;
  dm->lgP = cfg->page_size == 16 ? 4 : 5;
  dm->nb = cfg->hash_bits;
  dm->words = cfg->hash_bits / 64;
  dm->T = cfg->max_seq_len;
  dm->np_max = (int)np_max;
  dm->paged = cfg->paged ? 1 : 0;
  dm->num_blocks = cfg->paged ? cfg->num_blocks : 0;
  dm->max_blocks = cfg->paged ? cfg->max_blocks_per_seq : 0;
  if (cfg->page_group_agg != 0 && cfg->page_group_agg != 1)
    return fail(HHR_ERR_INVALID_ARG, "page_group_agg %d (0 max, 1 sum)", cfg->page_group_agg);
  if (cfg->key_group_agg != 0 && cfg->key_group_agg != 1)
    return fail(HHR_ERR_INVALID_ARG, "key_group_agg %d (0 sum, 1 min)", cfg->key_group_agg);
  dm->page_sum = cfg->page_group_agg;
  dm->key_min = cfg->key_group_agg;
  return HHR_OK;
}

// Carves the workspace; with base == nullptr only the size is computed.
// Sparse: per-unit counters, page bounds, one attention partial per CTA of
// the unit's group, one cumulative score histogram per CTA and one score
// histogram per unit.  Dense: counters and one partial per split.
size_t carve(const Dims& dm, int Nmax, int Kmax, bool dense, char* base, Work* wk) {
  const size_t BH = (size_t)dm.B * dm.Hkv;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* p = base ? base + off : nullptr;
    off += align256(bytes);
    return p;
  };
  Work w{};
  w.gx_stride = GX_STRIDE;
  w.gx = reinterpret_cast<unsigned*>(take(sizeof(unsigned) * BH * GX_STRIDE));
  const size_t PS = (size_t)dm.G * D + 16;
  if (dense) {
    w.C3 = std::min(MAX_GRID, ceil_div(dm.T, GATHER_ROWS));
    w.part = reinterpret_cast<float*>(take(sizeof(float) * BH * w.C3 * PS));
  } else {
    // one partial per CTA of a unit's group: at most max(1, 160 / units) CTAs,
    // or as many as the kept rows need (sparse_group_shape)
    const long long kcap = std::min<long long>(Kmax, (long long)Nmax * dm.P);
    w.C3 = std::max({1, MAX_GRID / (int)BH, ceil_div(kcap, MAX_KEPT_PER_CTA)});
    w.Ustride = (dm.np_max + 31) / 32 * 32;
    w.HB = (dm.G * dm.nb + 1 + 7) / 8 * 8;
    w.U = reinterpret_cast<float*>(take(sizeof(float) * BH * w.Ustride));
    w.part = reinterpret_cast<float*>(take(sizeof(float) * BH * w.C3 * PS));
    w.khist = reinterpret_cast<int*>(take(sizeof(int) * (size_t)MAX_GRID * w.HB));
    w.ktot = reinterpret_cast<int*>(take(sizeof(int) * BH * w.HB));
  }
  w.Nmax = Nmax;
  w.Kmax = Kmax;
  if (wk) *wk = w;
  return off;
}

hhr_status decode_check(const hhr_config* cfg, const void* q, const float* R, const void* W, const void* Krot,
                        const void* Vcache, const void* page_min, const void* page_max, const uint64_t* codes,
                        const int32_t* seq_lens, const int32_t* block_table, const int32_t* n_keep_pages,
                        const int32_t* top_k, int32_t max_keep_pages, int32_t max_top_k, float sm_scale,
                        const float* out, const char* who, Dims* dm, int* Nmax, size_t* need) {
  hhr_status s = make_dims(cfg, dm);
  if (s != HHR_OK) return s;
  if (dm->np_max > MAX_SELECT_PAGES)
    return fail(HHR_ERR_UNSUPPORTED, "%s: %d pages per sequence (at most %d)", who, dm->np_max, MAX_SELECT_PAGES);
  if (!q || !R || !W || !Krot || !Vcache || !page_min || !page_max || !codes || !seq_lens || !n_keep_pages ||
      !top_k || !out)
    return fail(HHR_ERR_INVALID_ARG, "%s: NULL pointer", who);
  if (dm->paged && !block_table) return fail(HHR_ERR_INVALID_ARG, "%s: paged needs block_table", who);
  const void* al[] = {q, R, W, Krot, Vcache, page_min, page_max, codes};
  for (const void* p : al)
    if (!aligned16(p)) return fail(HHR_ERR_INVALID_ARG, "%s: tensor not 16-byte aligned", who);
  if (max_keep_pages < 1 || max_top_k < 1)
    return fail(HHR_ERR_INVALID_ARG, "%s: max_keep_pages and max_top_k must be >= 1", who);
  if (!(sm_scale > 0.f)) return fail(HHR_ERR_INVALID_ARG, "%s: sm_scale must be > 0", who);
  const int nm = std::min(max_keep_pages, dm->np_max);
  if (nm > MAX_KEEP_PAGES)
    return fail(HHR_ERR_UNSUPPORTED, "%s: max_keep_pages %d (at most %d)", who, nm, MAX_KEEP_PAGES);
  if ((long long)nm * dm->P > MAX_CANDIDATES)
    return fail(HHR_ERR_UNSUPPORTED, "%s: max_keep_pages x page_size = %lld candidates (at most %d)", who,
                (long long)nm * dm->P, MAX_CANDIDATES);
  *Nmax = nm;
  *need = carve(*dm, nm, max_top_k, false, nullptr, nullptr);
  return HHR_OK;
}

hhr_status decode_launch(const Dims& dm, int Nmax, int32_t max_top_k, const void* q, const float* R, const void* W,
                         const void* Krot, const void* Vcache, const void* page_min, const void* page_max,
                         const uint64_t* codes, const int32_t* seq_lens, const int32_t* block_table,
                         const int32_t* n_keep_pages, const int32_t* top_k, float sm_scale, float* out,
                         const hhr_debug* dbg, void* workspace, int32_t* device_status, hhr_stream_t stream,
                         const char* who) {
  Work wk;
  carve(dm, Nmax, max_top_k, false, static_cast<char*>(workspace), &wk);
  const int sms = device_sms();
  if (sms <= 0) return fail(HHR_ERR_CUDA, "%s: cannot query the device", who);
  DecodeArgs a = {};
  a.dm = dm;
  a.wk = wk;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.R = R;
  a.W = static_cast<const __nv_bfloat16*>(W);
  a.Kr = static_cast<const __nv_bfloat16*>(Krot);
  a.Vc = static_cast<const __nv_bfloat16*>(Vcache);
  a.pmin = static_cast<const __nv_bfloat16*>(page_min);
  a.pmax = static_cast<const __nv_bfloat16*>(page_max);
  a.codes = codes;
  a.seq_lens = seq_lens;
  a.table = block_table;
  a.n_keep = n_keep_pages;
  a.top_k = top_k;
  a.sm_scale = sm_scale;
  a.out = out;
  if (dbg) a.dbg = *dbg;
  a.status = device_status;
  a.stream = reinterpret_cast<cudaStream_t>(stream);
  a.num_sms = sms;
  a.wait_limit = wait_limit_cycles();
  cudaError_t e = cudaErrorInvalidValue;
  HHR_DISPATCH_G(dm.G, e = launch_decode<GG>(a));
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(HHR_ERR_CUDA, "%s: launch failed: %s", who, cudaGetErrorString(e));
  }
  return ok();
}

}  // namespace hhr

extern "C" {

const char* hhr_status_string(hhr_status s) {
  switch (s) {
    case HHR_OK: return "HHR_OK";
    case HHR_ERR_INVALID_ARG: return "HHR_ERR_INVALID_ARG";
    case HHR_ERR_UNSUPPORTED: return "HHR_ERR_UNSUPPORTED";
    case HHR_ERR_WORKSPACE: return "HHR_ERR_WORKSPACE";
    case HHR_ERR_CUDA: return "HHR_ERR_CUDA";
    case HHR_ERR_TIMEOUT: return "HHR_ERR_TIMEOUT";
    case HHR_ERR_BAD_BLOCK: return "HHR_ERR_BAD_BLOCK";
  }
  return "HHR_ERR_UNKNOWN";
}

const char* hhr_last_error(void) { return g_err; }

void hhr_set_wait_limit(int64_t cycles) {
  g_wait_cycles.store(cycles > 0 ? (long long)cycles : DEFAULT_WAIT_CYCLES, std::memory_order_relaxed);
}

static hhr_status build_rows(const char* who, const hhr_config* cfg, const void* K, const void* V, const float* R,
                             const void* W, const int32_t* starts, const int32_t* seq_lens, int32_t max_rows,
                             const int32_t* block_table, void* Krot, void* Vcache, void* page_min, void* page_max,
                             uint64_t* codes, hhr_stream_t stream) {
  Dims dm;
  hhr_status s = make_dims(cfg, &dm);
  if (s != HHR_OK) return s;
  if (!K || !V || !R || !W || !seq_lens || !Krot || !Vcache || !page_min || !page_max || !codes)
    return fail(HHR_ERR_INVALID_ARG, "%s: NULL tensor pointer", who);
  if (dm.paged && !block_table) return fail(HHR_ERR_INVALID_ARG, "%s: paged needs block_table", who);
  const void* al[] = {K, V, R, W, Krot, Vcache, page_min, page_max, codes};
  for (const void* p : al)
    if (!aligned16(p)) return fail(HHR_ERR_INVALID_ARG, "%s: tensor not 16-byte aligned", who);
  if (max_rows < 1) return ok();  // nothing to build
  BuildArgs a = {};
  a.dm = dm;
  a.K = static_cast<const __nv_bfloat16*>(K);
  a.V = static_cast<const __nv_bfloat16*>(V);
  a.R = R;
  a.W = static_cast<const __nv_bfloat16*>(W);
  a.starts = starts;
  a.seq_lens = seq_lens;
  a.table = block_table;
  a.Krot = static_cast<__nv_bfloat16*>(Krot);
  a.Vcache = static_cast<__nv_bfloat16*>(Vcache);
  a.pmin = static_cast<__nv_bfloat16*>(page_min);
  a.pmax = static_cast<__nv_bfloat16*>(page_max);
  a.codes = codes;
  a.status = nullptr;
  a.max_rows = std::min(max_rows, dm.T);
  a.wait_limit = wait_limit_cycles();
  a.stream = reinterpret_cast<cudaStream_t>(stream);
  const cudaError_t e = launch_build(a);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(HHR_ERR_CUDA, "%s: %s", who, cudaGetErrorString(e));
  }
  return ok();
}

hhr_status hhr_build_cache(const hhr_config* cfg, const void* K, const void* V, const float* R, const void* W,
                           const int32_t* seq_lens, const int32_t* block_table, void* Krot, void* Vcache,
                           void* page_min, void* page_max, uint64_t* codes, hhr_stream_t stream) {
  return build_rows("hhr_build_cache", cfg, K, V, R, W, nullptr, seq_lens, cfg ? cfg->max_seq_len : 0, block_table,
                    Krot, Vcache, page_min, page_max, codes, stream);
}

hhr_status hhr_append_cache(const hhr_config* cfg, const void* K, const void* V, const float* R, const void* W,
                            const int32_t* old_lens, const int32_t* new_lens, int32_t max_new,
                            const int32_t* block_table, void* Krot, void* Vcache, void* page_min, void* page_max,
                            uint64_t* codes, hhr_stream_t stream) {
  if (!old_lens) return fail(HHR_ERR_INVALID_ARG, "hhr_append_cache: NULL old_lens");
  if (max_new < 0) return fail(HHR_ERR_INVALID_ARG, "hhr_append_cache: max_new must be >= 0");
  return build_rows("hhr_append_cache", cfg, K, V, R, W, old_lens, new_lens, max_new, block_table, Krot, Vcache,
                    page_min, page_max, codes, stream);
}

size_t hhr_decode_workspace_size(const hhr_config* cfg, int32_t max_keep_pages, int32_t max_top_k) {
  Dims dm;
  if (make_dims(cfg, &dm) != HHR_OK || max_keep_pages < 1 || max_top_k < 1) return 0;
  const int Nmax = std::min(max_keep_pages, dm.np_max);
  if (dm.np_max > MAX_SELECT_PAGES || Nmax > MAX_KEEP_PAGES || (long long)Nmax * dm.P > MAX_CANDIDATES) return 0;
  return carve(dm, Nmax, max_top_k, false, nullptr, nullptr);
}

hhr_status hhr_workspace_init(void* workspace, size_t workspace_bytes, hhr_stream_t stream) {
  if (!workspace) return fail(HHR_ERR_INVALID_ARG, "hhr_workspace_init: NULL workspace");
  if (cudaMemsetAsync(workspace, 0, workspace_bytes, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return check_cuda("hhr_workspace_init");
  return ok();
}

hhr_status hhr_decode_step(const hhr_config* cfg, const void* q, const float* R, const void* W, const void* Krot,
                           const void* Vcache, const void* page_min, const void* page_max, const uint64_t* codes,
                           const int32_t* seq_lens, const int32_t* block_table, const int32_t* n_keep_pages,
                           const int32_t* top_k, int32_t max_keep_pages, int32_t max_top_k, float sm_scale,
                           float* out, const hhr_debug* dbg, void* workspace, size_t workspace_bytes,
                           int32_t* device_status, hhr_stream_t stream) {
  static const char* who = "hhr_decode_step";
  Dims dm;
  int Nmax = 0;
  size_t need = 0;
  hhr_status s = decode_check(cfg, q, R, W, Krot, Vcache, page_min, page_max, codes, seq_lens, block_table,
                              n_keep_pages, top_k, max_keep_pages, max_top_k, sm_scale, out, who, &dm, &Nmax, &need);
  if (s != HHR_OK) return s;
  if (!workspace) return fail(HHR_ERR_INVALID_ARG, "%s: NULL workspace", who);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(HHR_ERR_INVALID_ARG, "%s: workspace not 256-byte aligned", who);
  if (workspace_bytes < need) return fail(HHR_ERR_WORKSPACE, "%s: workspace %zu bytes < %zu", who, workspace_bytes, need);
  return decode_launch(dm, Nmax, max_top_k, q, R, W, Krot, Vcache, page_min, page_max, codes, seq_lens, block_table,
                       n_keep_pages, top_k, sm_scale, out, dbg, workspace, device_status, stream, who);
}

size_t hhr_dense_workspace_size(const hhr_config* cfg) {
  Dims dm;
  if (make_dims(cfg, &dm) != HHR_OK) return 0;
  return carve(dm, 1, 1, true, nullptr, nullptr);
}

hhr_status hhr_dense_decode(const hhr_config* cfg, const void* q, const float* R, const void* Krot,
                            const void* Vcache, const int32_t* seq_lens, const int32_t* block_table, float sm_scale,
                            float* out, void* workspace, size_t workspace_bytes, int32_t* device_status,
                            hhr_stream_t stream) {
  Dims dm;
  hhr_status s = make_dims(cfg, &dm);
  if (s != HHR_OK) return s;
  if (!q || !R || !Krot || !Vcache || !seq_lens || !out || !workspace)
    return fail(HHR_ERR_INVALID_ARG, "hhr_dense_decode: NULL pointer");
  if (dm.paged && !block_table) return fail(HHR_ERR_INVALID_ARG, "hhr_dense_decode: paged needs block_table");
  const void* al[] = {q, R, Krot, Vcache};
  for (const void* p : al)
    if (!aligned16(p)) return fail(HHR_ERR_INVALID_ARG, "hhr_dense_decode: tensor not 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(HHR_ERR_INVALID_ARG, "hhr_dense_decode: workspace not 256-byte aligned");
  if (!(sm_scale > 0.f)) return fail(HHR_ERR_INVALID_ARG, "hhr_dense_decode: sm_scale must be > 0");
  const size_t need = carve(dm, 1, 1, true, nullptr, nullptr);
  if (workspace_bytes < need)
    return fail(HHR_ERR_WORKSPACE, "hhr_dense_decode: workspace %zu bytes < %zu", workspace_bytes, need);
  Work wk;
  carve(dm, 1, 1, true, static_cast<char*>(workspace), &wk);
  const int sms = device_sms();
  if (sms <= 0) return fail(HHR_ERR_CUDA, "hhr_dense_decode: cannot query the device");
  DecodeArgs a = {};
  a.dm = dm;
  a.wk = wk;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.R = R;
  a.Kr = static_cast<const __nv_bfloat16*>(Krot);
  a.Vc = static_cast<const __nv_bfloat16*>(Vcache);
  a.seq_lens = seq_lens;
  a.table = block_table;
  a.sm_scale = sm_scale;
  a.out = out;
  a.status = device_status;
  a.stream = reinterpret_cast<cudaStream_t>(stream);
  a.num_sms = sms;
  a.wait_limit = wait_limit_cycles();
  dense_split(dm, sms, &a.dense_nsplit, &a.dense_rows);
  if (a.dense_nsplit > wk.C3) return fail(HHR_ERR_UNSUPPORTED, "hhr_dense_decode: %d splits", a.dense_nsplit);
  cudaError_t e = cudaErrorInvalidValue;
  HHR_DISPATCH_G(dm.G, e = launch_dense<GG>(a));
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(HHR_ERR_CUDA, "hhr_dense_decode: launch failed: %s", cudaGetErrorString(e));
  }
  return ok();
}

}  // extern "C"
