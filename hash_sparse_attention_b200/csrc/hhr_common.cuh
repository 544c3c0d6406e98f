// Device helpers shared by the HHR kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "hhr.h"

namespace hhr {

constexpr int D = 128;  // head_dim: the only supported value

// Problem dimensions passed by value to every kernel.
struct Dims {
  int B, Hq, Hkv, G, P, nb, words, T, np_max, paged, num_blocks, max_blocks;
  int lgP;  // log2 of the page size (a power of two)
  int page_sum;  // U_p: 0 max over the group's heads, 1 sum
  int key_min;   // S_j: 0 sum over the group's heads, 1 min
};

// Workspace carve-out of one decode step (device pointers).  The per-unit
// counters `gx` and histograms `ktot` are zero between calls (the kernels
// reset what they use); everything else is overwritten by every call.
struct Work {
  float* U;            // [B Hkv, Ustride] page bounds (aggregated over the group's query heads)
  float* part;         // [B Hkv, C3, G D + 16] softmax partials (CTAs of a unit's group, or dense splits)
  int* khist;          // [grid, HB] cumulative score histogram of every CTA
  int* ktot;           // [B Hkv, HB] score histogram of every unit (zero between calls)
  unsigned* gx;        // [B Hkv, gx_stride] per-unit barrier and arrival counters
  int Nmax, Kmax;      // budgets the workspace was sized for
  int HB;              // histogram stride (>= G nb + 1, a multiple of 8)
  int Ustride;         // row stride of U (np_max rounded up to 32)
  int C3;              // partials per unit
  int gx_stride;       // 32-bit words per unit exchange area
};

// --- bf16 ---------------------------------------------------------------
__device__ __forceinline__ float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// 8 bf16 (one 16-byte vector) to fp32
__device__ __forceinline__ void unpack8(const uint4& v, float* f) {
  f[0] = bf_lo(v.x); f[1] = bf_hi(v.x);
  f[2] = bf_lo(v.y); f[3] = bf_hi(v.y);
  f[4] = bf_lo(v.z); f[5] = bf_hi(v.z);
  f[6] = bf_lo(v.w); f[7] = bf_hi(v.w);
}

__device__ __forceinline__ uint4 ldg16(const void* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}

// streaming 16-byte load (read once: do not keep in L1)
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

// --- ordering ---------------------------------------------------------------
// Order-preserving map fp32 -> uint32 (a larger float gives a larger key).
// -0 is mapped like +0 so that equal values tie and go to the lower index.
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u << 1) == 0u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// --- status ------------------------------------------------------------------
__device__ __forceinline__ void set_status(int* st, int code) {
  if (st) atomicCAS(st, 0, code);
}

// Sequence length clamped to [0, T] (a longer value would address past the cache).
__device__ __forceinline__ int seq_len_of(const Dims& dm, const int* __restrict__ seq_lens, int b) {
  return min(max(__ldg(seq_lens + b), 0), dm.T);
}

// --- cache addressing -------------------------------------------------------
// Element offset of row t of (sequence b, KV head h) in a [.., D]-row tensor
// (K', V).  Returns -1 (and records HHR_ERR_BAD_BLOCK) for a bad block id.
__device__ __forceinline__ long long kv_row(const Dims& dm, const int* __restrict__ table,
                                            int b, int h, int t, int* status) {
  if (!dm.paged) return ((long long)(b * dm.Hkv + h) * dm.T + t) * D;
  const int blk = __ldg(table + (long long)b * dm.max_blocks + (t >> dm.lgP));
  if ((unsigned)blk >= (unsigned)dm.num_blocks) { set_status(status, HHR_ERR_BAD_BLOCK); return -1; }
  return (((long long)blk * dm.Hkv + h) * dm.P + (t & (dm.P - 1))) * D;
}

// Element offset of page p's metadata row (page_min / page_max).
__device__ __forceinline__ long long meta_row(const Dims& dm, const int* __restrict__ table,
                                              int b, int h, int p, int* status) {
  if (!dm.paged) return ((long long)(b * dm.Hkv + h) * dm.np_max + p) * D;
  const int blk = __ldg(table + (long long)b * dm.max_blocks + p);
  if ((unsigned)blk >= (unsigned)dm.num_blocks) { set_status(status, HHR_ERR_BAD_BLOCK); return -1; }
  return ((long long)blk * dm.Hkv + h) * D;
}

// Word offset of row t's code (uint64 units).
__device__ __forceinline__ long long code_row(const Dims& dm, const int* __restrict__ table,
                                              int b, int h, int t, int* status) {
  if (!dm.paged) return ((long long)(b * dm.Hkv + h) * dm.T + t) * dm.words;
  const int blk = __ldg(table + (long long)b * dm.max_blocks + (t >> dm.lgP));
  if ((unsigned)blk >= (unsigned)dm.num_blocks) { set_status(status, HHR_ERR_BAD_BLOCK); return -1; }
  return (((long long)blk * dm.Hkv + h) * dm.P + (t & (dm.P - 1))) * dm.words;
}

}  // namespace hhr
