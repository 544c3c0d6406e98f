// HHR cache build and append (sm_100a) on the 5th-generation tensor cores.
//
// For each sequence b the kernel (re)builds rows t in [S_b, L_b): S_b = 0 for
// a full build, the old length for an append of new tokens.  Per 128-row tile
// of one (sequence, KV head), one tcgen05.mma chain per product, operands in
// shared memory (no-swizzle K-major core-matrix layout), accumulators in TMEM:
//   K'  = bf16_rne(K R_h^T)          R_h (fp32) as bf16 hi + mid + lo, the
//                                      three products into one fp32
//                                      accumulator (|R - hi - mid - lo| <=
//                                      2^-26 |R|); an element whose
//                                      accumulator lies within 2^-20 |k| of
//                                      a bf16 rounding midpoint is recomputed
//                                      in fp64 and rounded once, so K' is the
//                                      correctly rounded product; every
//                                      row gets the same arithmetic whatever
//                                      its tile, so an append gives
//                                      bit-identical rows
//   code bit j = [ (K W_h^T)_j > 0 ]  unrotated K; the products are exact
//                                      bf16 x bf16 and the fp32 sum is trusted
//                                      only when |sum| > 2^-14 |w_j| |k|,
//                                      otherwise the sign comes from fp64
//   page min / max over the valid stored K' rows of each page; a page that
//   began before S_b merges its stored min / max with the new rows (min and
//   max are exact, so the result equals a build over the whole page)
//   V rows copied to the cache unless it aliases V.
// "HHR" paper card, Abstract (head-wise orthogonal transformation and
// head-wise hash projection of the keys); rit.work explainer, section "Два
// уровня маршрутизации решают разные ошибки" (pages of neighbouring keys with
// stored per-channel bounds).
//
// A CTA (16 warps) walks BT_TILES consecutive tiles, so that R_h and W_h are
// staged once.  Thread 0 issues the MMAs; in the epilogue warp w reads TMEM
// lanes (rows) 32 (w mod 4) .. +31, columns of group w / 4 (a quarter of K'
// and a quarter of the code bits).
#pragma once

#include "hhr_dev.cuh"
#include "hhr_launch.h"

namespace hhr {

constexpr int BT_THREADS = 512;  // 16 warps: warp w reads TMEM lanes 32 (w mod 4) .. +31, column group w / 4
constexpr int BT_ROWS = 128;   // rows per tile: the M of the MMA
constexpr int BT_TILES = 16;   // tiles per CTA
constexpr int BT_FIXCAP = 512; // K' elements per tile queued for the exact recompute

// Byte offset of element (m, k) of a [rows][128] bf16 operand in the
// no-swizzle K-major canonical layout: 8 x 8 core matrices of 128 bytes, the
// 16 along K contiguous (leading byte offset 128), 8-row groups 2048 bytes
// apart (stride byte offset).
__host__ __device__ constexpr int bt_off(int m, int k) {
  return (m >> 3) * 2048 + (k >> 3) * 128 + (m & 7) * 16 + (k & 7) * 2;
}

// Byte offset of element c of row r of the K' tile: 256-byte rows, their
// 16-byte pieces XOR-swizzled by row (a warp's rows spread over the banks).
__host__ __device__ constexpr int bt_koff(int r, int c) { return r * 256 + (((c >> 3) ^ (r & 15)) << 4) + (c & 7) * 2; }

// dynamic shared memory layout of the build kernel
struct BuildSmem {
  static constexpr size_t rhi = 0;                        // R_h hi [128][128] bf16, canonical
  static constexpr size_t rmid = rhi + 32768;             // R_h mid
  static constexpr size_t rlo = rmid + 32768;             // R_h lo
  static constexpr size_t a = rlo + 32768;                // K tile [128][128] bf16, canonical
  static constexpr size_t ko = a + 32768;                 // K' tile [128][128] bf16, swizzled rows
  static constexpr size_t wn = ko + 32768;                // float [256] |w_j|
  static constexpr size_t bar = wn + 1024;                // u64 MMA-done barrier, u32 TMEM address, u32 count
  static constexpr size_t fix = bar + 64;                 // u16 [BT_FIXCAP] K' elements (row << 7 | column)
  static constexpr size_t kn = fix + 2 * BT_FIXCAP;       // float [128] |k| of the tile's rows
  static constexpr size_t w = kn + 512;                   // W_h [nb][128] bf16, canonical
  static size_t bytes(int nb) { return w + 256 * (size_t)nb; }
};

// --- tcgen05 (5th-generation tensor cores, accumulators in TMEM) -------------
// Shared-memory matrix descriptor: start address, leading / stride byte
// offsets (>> 4), descriptor version 1, no swizzle.
__device__ __forceinline__ uint64_t bt_desc(const void* p) {
  const uint32_t addr = smem_u32(p);
  return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)(128 >> 4) << 16) | ((uint64_t)(2048 >> 4) << 32) |
         ((uint64_t)1 << 46);
}
// Instruction descriptor of kind::f16: bf16 A and B (K-major), fp32 D, M = 128.
__host__ __device__ constexpr uint32_t bt_idesc(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}
__device__ __forceinline__ void bt_mma(uint32_t tmem, uint64_t da, uint64_t db, uint32_t idesc, bool acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(
          tmem),
      "l"(da), "l"(db), "r"(idesc), "r"(acc ? 1u : 0u)
      : "memory");
}
__device__ __forceinline__ void bt_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// 16 consecutive fp32 columns of the warp's 32 TMEM lanes (one lane per thread)
__device__ __forceinline__ void tc_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// fp64 partial dot product of K-tile row r and W_h row j (both bf16 in the
// canonical layout) over k = 4 lane .. 4 lane + 3; the products are exact.
__device__ __forceinline__ double bt_dot4(const unsigned char* A, const unsigned char* Bw, int r, int j, int lane) {
  const uint2 a = *reinterpret_cast<const uint2*>(A + bt_off(r, 4 * lane));
  const uint2 w = *reinterpret_cast<const uint2*>(Bw + bt_off(j, 4 * lane));
  return (double)bf_lo(a.x) * bf_lo(w.x) + (double)bf_hi(a.x) * bf_hi(w.x) + (double)bf_lo(a.y) * bf_lo(w.y) +
         (double)bf_hi(a.y) * bf_hi(w.y);
}

// The bf16 value nearest to s (ties to even), from the two bf16 values around
// s: its truncation toward zero and the next one away from zero.
__device__ __forceinline__ uint16_t bt_round_bf16(double s) {
  const float f = (float)s;
  uint32_t c0 = __float_as_uint(f) >> 16;
  // ((float)s may have rounded away from zero past a bf16 value: step back)
  if (fabs((double)__uint_as_float(c0 << 16)) > fabs(s)) c0 -= 1u;
  const uint32_t c1 = c0 + 1u;
  const double d0 = fabs(s - (double)__uint_as_float(c0 << 16)), d1 = fabs(s - (double)__uint_as_float(c1 << 16));
  return (uint16_t)(d0 < d1 ? c0 : d1 < d0 ? c1 : ((c0 & 1u) ? c1 : c0));
}

// K'[r][i] exactly: the fp64 dot product of K-tile row r (bf16) with R_h row i
// (fp32; every product is exact in fp64), rounded once to bf16 (nearest, ties
// to even).  For the rare elements whose fp32 accumulator lies too close to a
// bf16 rounding midpoint to be sure of the rounding.
static __device__ __noinline__ uint16_t bt_kexact(const unsigned char* A, const float* Ri, int r) {
  double s = 0.0;
  #pragma unroll 1
  for (int k0 = 0; k0 < D; k0 += 32) {  // eight 16-byte loads of R in flight at a time
    float4 rv[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) rv[q] = __ldg(reinterpret_cast<const float4*>(Ri + k0) + q);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float rr[4] = {rv[q].x, rv[q].y, rv[q].z, rv[q].w};
#pragma unroll
      for (int u = 0; u < 4; ++u)
        s += (double)__bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(A + bt_off(r, k0 + 4 * q + u))) *
             (double)rr[u];
    }
  }
  return bt_round_bf16(s);
}

// The queued K' elements (row << 7 | column), four lanes per element: lane g
// of a group sums k in [32 g, 32 g + 32) in fp64, the group adds its partial
// sums by shuffles and the result is rounded once.  A lane takes two elements
// per pass, their R loads in flight together.
static __device__ __noinline__ void bt_fixups(const unsigned char* A, const float* __restrict__ Rh,
                                              const uint16_t* fixq, int n, unsigned char* Ko, int warp, int lane) {
  constexpr int PER = BT_THREADS / 4;  // elements per half pass
  const int g = lane & 3;
  #pragma unroll 1
  for (int base = 8 * warp; base < n; base += 2 * PER) {  // (warp-uniform trip count)
    int ent[2];
    float4 x[2][8];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int e = base + u * PER + (lane >> 2);
      ent[u] = e < n ? (int)fixq[e] : -1;
      const float4* Rp = reinterpret_cast<const float4*>(Rh + (ent[u] < 0 ? 0 : ent[u] & 127) * D + 32 * g);
#pragma unroll
      for (int v = 0; v < 8; ++v) x[u][v] = __ldg(Rp + v);
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int r = ent[u] < 0 ? 0 : ent[u] >> 7;
      double s = 0.0;
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        float a[8];
        unpack8(*reinterpret_cast<const uint4*>(A + bt_off(r, 32 * g + 8 * v)), a);
        s += (double)a[0] * x[u][2 * v].x + (double)a[1] * x[u][2 * v].y + (double)a[2] * x[u][2 * v].z +
             (double)a[3] * x[u][2 * v].w + (double)a[4] * x[u][2 * v + 1].x + (double)a[5] * x[u][2 * v + 1].y +
             (double)a[6] * x[u][2 * v + 1].z + (double)a[7] * x[u][2 * v + 1].w;
      }
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      s += __shfl_xor_sync(0xffffffffu, s, 2);
      if (ent[u] >= 0 && g == 0) *reinterpret_cast<uint16_t*>(Ko + bt_koff(r, ent[u] & 127)) = bt_round_bf16(s);
    }
  }
}

// The same recompute with R_h row c read back from its three staged bf16
// terms (their fp32 sum is R_h's element exactly whenever the staging found
// every split exact, which it checks), so that no global load is needed.
static __device__ __noinline__ void bt_fixups_smem(const unsigned char* A, const unsigned char* Bh,
                                                   const unsigned char* Bm, const unsigned char* Bl,
                                                   const uint16_t* fixq, int n, unsigned char* Ko, int warp,
                                                   int lane) {
  constexpr int PER = BT_THREADS / 4;
  const int g = lane & 3;
  #pragma unroll 1
  for (int base = 8 * warp; base < n; base += PER) {  // (warp-uniform trip count)
    const int e = base + (lane >> 2);
    const int ent = e < n ? (int)fixq[e] : 0;
    const int r = ent >> 7, c = ent & 127;
    double s = 0.0;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int k = 32 * g + 8 * v;
      float a[8], h[8], m[8], l[8];
      unpack8(*reinterpret_cast<const uint4*>(A + bt_off(r, k)), a);
      unpack8(*reinterpret_cast<const uint4*>(Bh + bt_off(c, k)), h);
      unpack8(*reinterpret_cast<const uint4*>(Bm + bt_off(c, k)), m);
      unpack8(*reinterpret_cast<const uint4*>(Bl + bt_off(c, k)), l);
#pragma unroll
      for (int u = 0; u < 8; ++u) s += (double)a[u] * (double)((h[u] + m[u]) + l[u]);
    }
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    if (e < n && g == 0) *reinterpret_cast<uint16_t*>(Ko + bt_koff(r, c)) = bt_round_bf16(s);
  }
}

// Issue the copies of K tile rows t0 .. t0 + 127 into the canonical layout
// (cp.async, one commit group); rows outside [S0, L) are zeros.
__device__ __forceinline__ void bt_issue_k(const Dims& dm, const int* __restrict__ table, int b, int h, int t0,
                                           int S0, int L, const __nv_bfloat16* K, unsigned char* A, int tid,
                                           int* status) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = tid + BT_THREADS * i, rr = e >> 4, c = e & 15, t = t0 + rr;
    unsigned char* dst = A + bt_off(rr, c * 8);
    const long long off = (t >= S0 && t < L) ? kv_row(dm, table, b, h, t, status) : -1;
    if (off >= 0) cp_async16(dst, K + off + c * 8);
    else *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
  }
  cp_async_commit();
}

template <int NB>
__global__ void __launch_bounds__(BT_THREADS, 1)
build_cache_kernel(Dims dm, const __nv_bfloat16* K, const __nv_bfloat16* V, const float* __restrict__ R,
                   const __nv_bfloat16* __restrict__ W, const int* __restrict__ starts,
                   const int* __restrict__ seq_lens, const int* __restrict__ table, __nv_bfloat16* Krot,
                   __nv_bfloat16* Vcache, __nv_bfloat16* __restrict__ pmin, __nv_bfloat16* __restrict__ pmax,
                   uint64_t* __restrict__ codes, int* status, long long wait_limit) {
  constexpr int TCOLS = NB <= 128 ? 256 : 512;  // TMEM columns: K' [0, 128), codes [128, 128 + NB)
  extern __shared__ __align__(1024) unsigned char smem[];
  unsigned char* Bh = smem + BuildSmem::rhi;
  unsigned char* Bm = smem + BuildSmem::rmid;
  unsigned char* Bl = smem + BuildSmem::rlo;
  unsigned char* A = smem + BuildSmem::a;
  unsigned char* Ko = smem + BuildSmem::ko;
  float* wn = reinterpret_cast<float*>(smem + BuildSmem::wn);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + BuildSmem::bar);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + BuildSmem::bar + 8);
  int* nfix = reinterpret_cast<int*>(smem + BuildSmem::bar + 16);
  uint16_t* fixq = reinterpret_cast<uint16_t*>(smem + BuildSmem::fix);
  unsigned char* Bw = smem + BuildSmem::w;

  const int h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int L = seq_len_of(dm, seq_lens, b);
  const int S0 = starts ? min(max(__ldg(starts + b), 0), L) : 0;  // first row (re)built
  const int row0 = (S0 & ~(BT_ROWS - 1)) + blockIdx.x * BT_TILES * BT_ROWS;
  if (row0 >= L || S0 >= L) return;

  // ---- stage R_h as bf16 hi + mid + lo and W_h (canonical layout), the norms |w_j| ----
  const float* Rh = R + (long long)h * D * D;
  int inexact = 0;  // an element whose three terms do not add back to it in fp32
  #pragma unroll 4
  for (int e = tid; e < D * 16; e += BT_THREADS) {
    const int i = e >> 4, c = e & 15;
    const float4 x0 = __ldg(reinterpret_cast<const float4*>(Rh + i * D + c * 8));
    const float4 x1 = __ldg(reinterpret_cast<const float4*>(Rh + i * D + c * 8 + 4));
    const float f[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
    uint32_t hi[4], mi[4], lo[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {  // (each residual is exact in fp32)
      const __nv_bfloat162 h2 = __floats2bfloat162_rn(f[2 * q], f[2 * q + 1]);
      const float2 hf = __bfloat1622float2(h2);
      const float r0 = f[2 * q] - hf.x, r1 = f[2 * q + 1] - hf.y;
      const __nv_bfloat162 m2 = __floats2bfloat162_rn(r0, r1);
      const float2 mf = __bfloat1622float2(m2);
      const __nv_bfloat162 l2 = __floats2bfloat162_rn(r0 - mf.x, r1 - mf.y);
      const float2 lf = __bfloat1622float2(l2);
      if ((hf.x + mf.x) + lf.x != f[2 * q] || (hf.y + mf.y) + lf.y != f[2 * q + 1]) inexact = 1;
      hi[q] = *reinterpret_cast<const uint32_t*>(&h2);
      mi[q] = *reinterpret_cast<const uint32_t*>(&m2);
      lo[q] = *reinterpret_cast<const uint32_t*>(&l2);
    }
    *reinterpret_cast<uint4*>(Bh + bt_off(i, c * 8)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4*>(Bm + bt_off(i, c * 8)) = make_uint4(mi[0], mi[1], mi[2], mi[3]);
    *reinterpret_cast<uint4*>(Bl + bt_off(i, c * 8)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  }
  const __nv_bfloat16* Wh = W + (long long)h * NB * D;
  #pragma unroll 4
  for (int e = tid; e < NB * 16; e += BT_THREADS) {
    const int j = e >> 4, c = e & 15;
    *reinterpret_cast<uint4*>(Bw + bt_off(j, c * 8)) = ldg16(Wh + j * D + c * 8);
  }
  const bool split_exact = !__syncthreads_or(inexact);
  #pragma unroll 1
  for (int j = tid; j < NB; j += BT_THREADS) {
    float sq = 0.f;
    #pragma unroll 4
    for (int c = 0; c < 16; ++c) {
      float f[8];
      unpack8(*reinterpret_cast<const uint4*>(Bw + bt_off(j, c * 8)), f);
#pragma unroll
      for (int q = 0; q < 8; ++q) sq = fmaf(f[q], f[q], sq);
    }
    wn[j] = sqrtf(sq) * 1.0001f;  // a hair above |w_j| so the guard stays conservative
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tslot)),
                 "r"(TCOLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_fence_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  float* knr = reinterpret_cast<float*>(smem + BuildSmem::kn);
  bool timed_out = false;
  unsigned phase = 0u;
  const int q = warp & 3, cg = warp >> 2;       // TMEM lane quarter, column group
  const int r = 32 * q + lane;                  // the thread's row of the tile in the epilogue
  const uint32_t tl = tmem + ((uint32_t)(32 * q) << 16);

  bt_issue_k(dm, table, b, h, row0, S0, L, K, A, tid, status);
  #pragma unroll 1
  for (int tile = 0; tile < BT_TILES; ++tile) {
    const int t0 = row0 + tile * BT_ROWS;
    if (t0 >= L) break;
    cp_async_wait_all();  // this tile's K (issued before the previous tile's copy-out)
    if (tid == 0) *nfix = 0;
    fence_proxy_async();  // (the tensor cores read the tile through the async proxy)
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // ---- K' = K R^T (lo, mid, then hi: the small terms first) and K W^T, one thread issues ----
    if (tid == 0) {
      #pragma unroll 1
      for (int ks = 0; ks < 8; ++ks) bt_mma(tmem, bt_desc(A + ks * 256), bt_desc(Bl + ks * 256), bt_idesc(128), ks > 0);
      #pragma unroll 1
      for (int ks = 0; ks < 8; ++ks) bt_mma(tmem, bt_desc(A + ks * 256), bt_desc(Bm + ks * 256), bt_idesc(128), true);
      #pragma unroll 1
      for (int ks = 0; ks < 8; ++ks) bt_mma(tmem, bt_desc(A + ks * 256), bt_desc(Bh + ks * 256), bt_idesc(128), true);
      #pragma unroll 1
      for (int ks = 0; ks < 8; ++ks)
        bt_mma(tmem + 128, bt_desc(A + ks * 256), bt_desc(Bw + ks * 256), bt_idesc(NB), ks > 0);
      bt_commit(bar);
    } else if (tid >= 32 && tid < 32 + BT_ROWS) {  // meanwhile |k| of every row of the tile
      const int rr = tid - 32;
      float sq = 0.f;
      #pragma unroll 4
      for (int c = 0; c < 16; ++c) {
        float f[8];
        unpack8(*reinterpret_cast<const uint4*>(A + bt_off(rr, c * 8)), f);
#pragma unroll
        for (int u = 0; u < 8; ++u) sq = fmaf(f[u], f[u], sq);
      }
      knr[rr] = sqrtf(sq) * 1.0001f;
    }
    if (!mbar_wait(bar, phase, wait_limit)) timed_out = true;
    phase ^= 1u;
    __syncthreads();  // (|k| of every row)
    tc_fence_after();
    // ---- epilogue: row r, K' columns [32 cg, 32 cg + 32), code bits [cg NB/4, (cg + 1) NB/4) ----
    const float kn = knr[r];
    const int t = t0 + r;
    const bool live = t >= S0 && t < L;
    // K' rounded to bf16.  The fp32 accumulator is within a few 2^-24 |k| of
    // the exact value (|R_i| = 1); an element within 2^-20 |k| of a bf16
    // rounding midpoint is queued for the exact recompute below.
    const float kdelta = kn * 9.5367431640625e-07f;  // 2^-20
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int c0 = 32 * cg + 16 * half;
      float v[16];
      tc_ld16(tl + c0, v);
      uint32_t pk[8];
#pragma unroll
      for (int qq = 0; qq < 8; ++qq) {
        uint32_t e2[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const float x = v[2 * qq + u];
          const float mid = __uint_as_float((__float_as_uint(x) & 0xffff0000u) | 0x8000u);
          const __nv_bfloat16 hb = __float2bfloat16_rn(x);
          e2[u] = *reinterpret_cast<const uint16_t*>(&hb);
          if (fabsf(x - mid) < kdelta) {  // (in line if the queue is full)
            const int c = c0 + 2 * qq + u;
            const int slot = atomicAdd(nfix, 1);
            if (slot < BT_FIXCAP) fixq[slot] = (uint16_t)((r << 7) | c);
            else e2[u] = bt_kexact(A, R + ((long long)h * D + c) * D, r);
          }
        }
        pk[qq] = e2[0] | (e2[1] << 16);
      }
      *reinterpret_cast<uint4*>(Ko + bt_koff(r, c0)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      *reinterpret_cast<uint4*>(Ko + bt_koff(r, c0 + 8)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
    }
    // code bits of the group: trusted when |sum| > 2^-14 |w_j| |k|, else fp64
    {
      constexpr int NBQ = NB / 4;  // bits per column group (16, 32 or 64)
      const float kg = kn * 6.103515625e-05f;  // 2^-14 |k|
      uint64_t bits = 0ull, fb = 0ull;  // fb: bits whose sign fp32 cannot decide
#pragma unroll
      for (int c0 = 0; c0 < NBQ; c0 += 16) {
        float v[16];
        tc_ld16(tl + 128 + cg * NBQ + c0, v);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const bool near0 = fabsf(v[i]) <= wn[cg * NBQ + c0 + i] * kg;
          fb |= (uint64_t)near0 << (c0 + i);
          bits |= (uint64_t)(v[i] > 0.f && !near0) << (c0 + i);
        }
      }
      // those signs from fp64, one bit at a time for the whole warp (each
      // lane sums 4 of the 128 exact products)
      unsigned any = __ballot_sync(0xffffffffu, fb != 0ull);
      #pragma unroll 1
      while (any) {
        const int src = __ffs(any) - 1;
        const int bit = __ffsll((long long)__shfl_sync(0xffffffffu, fb, src)) - 1;
        double sd = bt_dot4(A, Bw, 32 * q + src, cg * NBQ + bit, lane);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) sd += __shfl_xor_sync(0xffffffffu, sd, o);
        if (lane == src) {
          bits |= (uint64_t)(sd > 0.0) << bit;
          fb &= fb - 1ull;
        }
        any = __ballot_sync(0xffffffffu, fb != 0ull);
      }
      if (live) {
        const long long off = code_row(dm, table, b, h, t, status);
        if (off >= 0) {
          unsigned char* dst = reinterpret_cast<unsigned char*>(codes + off) + cg * (NBQ / 8);
          if constexpr (NBQ == 16) *reinterpret_cast<uint16_t*>(dst) = (uint16_t)bits;
          else if constexpr (NBQ == 32) *reinterpret_cast<uint32_t*>(dst) = (uint32_t)bits;
          else *reinterpret_cast<uint64_t*>(dst) = bits;
        }
      }
    }
    tc_fence_before();
    __syncthreads();  // TMEM is free for the next tile; the queue is complete
    if (split_exact) bt_fixups_smem(A, Bh, Bm, Bl, fixq, min(*nfix, BT_FIXCAP), Ko, warp, lane);
    else bt_fixups(A, Rh, fixq, min(*nfix, BT_FIXCAP), Ko, warp, lane);
    __syncthreads();  // the K' tile is complete; nothing reads this K tile any more
    if (tile + 1 < BT_TILES && t0 + BT_ROWS < L) bt_issue_k(dm, table, b, h, t0 + BT_ROWS, S0, L, K, A, tid, status);
    // ---- K' and V rows (coalesced; a thread's 4 V loads in flight), page min / max ----
    {
      long long offs[4];
      uint4 vv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int e = tid + BT_THREADS * i, rr = e >> 4, c = e & 15, tt = t0 + rr;
        offs[i] = (tt >= S0 && tt < L) ? kv_row(dm, table, b, h, tt, status) : -1;
        if (offs[i] >= 0 && Vcache != V) vv[i] = ldg16(V + offs[i] + c * 8);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int e = tid + BT_THREADS * i, rr = e >> 4, c = e & 15;
        if (offs[i] >= 0) {
          *reinterpret_cast<uint4*>(Krot + offs[i] + c * 8) = *reinterpret_cast<const uint4*>(Ko + bt_koff(rr, c * 8));
          if (Vcache != V) *reinterpret_cast<uint4*>(Vcache + offs[i] + c * 8) = vv[i];
        }
      }
    }
    const int pages = BT_ROWS / dm.P;
    #pragma unroll 1
    for (int e = tid; e < pages * D; e += BT_THREADS) {
      const int pp = e / D, c = e % D;
      const int tp = t0 + pp * dm.P;
      const int r0 = max(0, S0 - tp), r1 = min(dm.P, L - tp);  // the page's rows built here
      if (r0 >= r1) continue;
      float lo = INFINITY, hi = -INFINITY;
      #pragma unroll 4
      for (int rr = r0; rr < r1; ++rr) {
        const float x = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(Ko + bt_koff(pp * dm.P + rr, c)));
        lo = fminf(lo, x);
        hi = fmaxf(hi, x);
      }
      const long long off = meta_row(dm, table, b, h, tp / dm.P, status);
      if (off >= 0) {
        if (r0 > 0) {  // the page began before S0: merge with its stored rows
          lo = fminf(lo, __bfloat162float(pmin[off + c]));
          hi = fmaxf(hi, __bfloat162float(pmax[off + c]));
        }
        pmin[off + c] = __float2bfloat16_rn(lo);
        pmax[off + c] = __float2bfloat16_rn(hi);
      }
    }
    // (the next tile's K-tile writes come after this tile's MMAs completed;
    // its barrier orders the K' tile reads above before the next epilogue)
  }
  cp_async_wait_all();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TCOLS) : "memory");
  if (timed_out && tid == 0) set_status(status, HHR_ERR_TIMEOUT);
}

}  // namespace hhr
