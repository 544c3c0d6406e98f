// Device primitives shared by the HHR kernels (sm_100a): asynchronous copies,
// acquire/release words, tensor-core fragments, block scans and the bounded
// wait used by every spin in the library.
#pragma once

#include <climits>

#include "hhr_common.cuh"

namespace hhr {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// --- cp.async (16 bytes, through L2 only) --------------------------------------
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// --- TMA bulk copies (global -> shared, no tensor map) and mbarriers --------
// A phase of a barrier initialised with count 1 completes when its one arrival
// (mbar_arrive_expect_tx, which also adds the phase's byte count) has happened
// and the bulk copies have delivered those bytes.  Addresses and sizes of a
// bulk copy are multiples of 16 bytes.
__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
// makes barrier initialisation visible to the asynchronous (TMA) proxy
__device__ __forceinline__ void mbar_fence_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
// orders this thread's earlier shared-memory accesses before later TMA writes
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ bool mbar_test(uint64_t* bar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// --- global words with gpu-scope ordering --------------------------------------
__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ int ld_relaxed_s32(const int* p) {
  int v;
  asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_add(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned atom_add_acq_rel(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// --- programmatic dependent launch ------------------------------------------
// wait: every prior grid of the stream has completed and its writes are
// visible; launch_dependents: the next grid of the stream may be scheduled.
// Both are no-ops for a launch without the programmatic attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// --- bounded waits -------------------------------------------------------------
// Every spin in the library gives up after `limit` SM clock cycles (a kernel
// parameter; about two seconds by default).  On expiry the caller records
// HHR_ERR_TIMEOUT and raises the CTA's abort flag.
struct Spin {
  long long t0, limit;
  __device__ __forceinline__ explicit Spin(long long lim) {
    t0 = clock64();
    limit = lim;
  }
  __device__ __forceinline__ bool expired() const { return clock64() - t0 > limit; }
};

// Bounded wait for the phase of `bar` with the given parity; false on timeout.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, unsigned parity, long long limit) {
  if (mbar_test(bar, parity)) return true;
  Spin sp(limit);
  while (!mbar_test(bar, parity))
    if (sp.expired()) return false;
  return true;
}

// --- tensor-core fragments (mma.sync m16n8k16, bf16 in, fp32 accumulate) -------
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x2(uint32_t (&r)[2], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r[0]), "=r"(r[1]) : "r"(smem_u32(p)));
}
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// x as bf16 hi + lo (hi = RNE(x), lo = RNE(x - hi)): |x - hi - lo| <= 2^-17 |x|
__device__ __forceinline__ void split_bf16(float x, __nv_bfloat16& hi, __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(x);
  lo = __float2bfloat16_rn(x - __bfloat162float(hi));
}

// --- block scan ----------------------------------------------------------------
// Named barrier `id` over the first `n` threads that reach it (id 0 with the
// whole block is __syncthreads).
__device__ __forceinline__ void bar_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }
// arrive at named barrier id without waiting (the other n - 32 k threads wait in bar_sync)
__device__ __forceinline__ void bar_arrive(int id, int n) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void prefetch_l2(const void* p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }

// Exclusive prefix of v over the threads of a group of nw consecutive warps
// (warps wbase .. wbase + nw - 1, nw <= 16, synchronised by named barrier
// `bar`) in thread order, and the group total.  `red` holds 2 x 32 ints;
// `parity` alternates between calls so that one barrier per call suffices.
// Every thread of the group must call it.  Out of line: one copy serves every
// call site.
static __device__ __noinline__ int block_scan_excl(int v, int* red, int parity, int* total, int wbase = 0,
                                                   int nw = 16, int bar = 0) {
  const int lane = threadIdx.x & 31, warp = (threadIdx.x >> 5) - wbase;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  int* r = red + 32 * (parity & 1);
  if (lane == 31) r[warp] = x;
  bar_sync(bar, nw * 32);
  // lane l < nw holds warp l's total; a scan of the totals in every warp
  int t = lane < nw ? r[lane] : 0;
#pragma unroll
  for (int o = 1; o < 16; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, t, o);
    if (lane >= o) t += y;
  }
  *total = __shfl_sync(0xffffffffu, t, nw - 1);
  const int before = warp > 0 ? __shfl_sync(0xffffffffu, t, (warp - 1) & 31) : 0;
  return before + x - v;
}

// Block-wide minimum and maximum of unsigned values over a 512-thread block
// (one barrier; `red` 2 x 32).
static __device__ __noinline__ void block_minmax_u32(unsigned& lo, unsigned& hi, unsigned* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if (lane == 0) {
    red[warp] = lo;
    red[32 + warp] = hi;
  }
  __syncthreads();
  // lanes 16-31 hold the identities, so the butterfly over all 32 lanes
  // leaves the block's result in every lane
  lo = lane < 16 ? red[lane] : 0xffffffffu;
  hi = lane < 16 ? red[32 + lane] : 0u;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
}

__host__ __device__ constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x >> 1); }

// Transposed butterfly over the NL lanes of an aligned lane group (NV, NL
// powers of two): v[0..NV) are per-lane partial sums of NV quantities.
// Afterwards, with NV >= NL, lane l of the group holds the group totals of
// quantities l*(NV/NL) + e in v[e], e < NV/NL; with NV < NL it holds the total
// of quantity l*NV/NL in v[0].  Each round halves the values a lane keeps.
template <int NV, int NL>
__device__ __forceinline__ void group_reduce_scatter(float (&v)[NV], int lane) {
  static_assert((NV & (NV - 1)) == 0 && (NL & (NL - 1)) == 0 && NL <= 32, "powers of two");
  constexpr int ROUNDS = ilog2(NV < NL ? NV : NL);
#pragma unroll
  for (int k = 0; k < ROUNDS; ++k) {
    const int half = NV >> (k + 1), o = NL >> (k + 1);
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = upper ? v[i] : v[i + half];
      const float keep = upper ? v[i + half] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  // NV < NL: the remaining lane levels add up copies of the same quantity
#pragma unroll
  for (int o = (NV < NL ? NL / (2 * NV) : 0); o >= 1; o >>= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
}

}  // namespace hhr
