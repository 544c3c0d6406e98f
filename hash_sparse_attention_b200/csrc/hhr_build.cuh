// HHR cache build and append (sm_100a), CUDA-core version.
//
// For each sequence b the kernel (re)builds rows t in [S_b, L_b): S_b = 0 for
// a full build, the old length for an append of new tokens.  Per 64-row tile
// of one (sequence, KV head):
//   K'  = bf16_rne(K R_h^T)          fp32 accumulation, in channel order j =
//                                      0..127 for every row (the same
//                                      arithmetic whatever the tile, so an
//                                      append gives bit-identical rows)
//   code bit j = [ (K W_h^T)_j > 0 ]  unrotated K; the fp32 sum of exact
//                                      bf16 x bf16 products is trusted only
//                                      when |sum| > 2^-14 |w_j| |k| (the fp32
//                                      error is below 128 * 2^-24 sum|w k|),
//                                      otherwise the sign comes from fp64
//   page min / max over the valid stored K' rows of each page; a page that
//   began before S_b merges its stored min / max with the new rows (min and
//   max are exact, so the result equals a build over the whole page)
//   V rows copied to the cache unless it aliases V.
// A CTA walks BUILD_TILES consecutive tiles so that R_h and W_h are staged
// in shared memory once per CTA.
#pragma once

#include "hhr_common.cuh"
#include "hhr_launch.h"

namespace hhr {

constexpr int BUILD_THREADS = 256;
constexpr int BUILD_ROWS = 64;
constexpr int BUILD_TILES = 8;

// dynamic shared memory layout of the build kernel
struct BuildSmem {
  static constexpr size_t kt = 0;                                    // float [D][64]
  static constexpr size_t rt = kt + sizeof(float) * D * BUILD_ROWS;   // float [D][D]
  static constexpr size_t ko = rt + sizeof(float) * D * D;            // bf16 [64][D]
  static constexpr size_t wn = ko + 2 * BUILD_ROWS * D;               // float [256] |w_j|
  static constexpr size_t kn = wn + sizeof(float) * 256;              // float [64]  |k|
  static constexpr size_t cd = kn + sizeof(float) * BUILD_ROWS;       // u64 [64][4]
  static constexpr size_t wt = cd + sizeof(uint64_t) * BUILD_ROWS * 4;  // bf16 [D][nb]
  static size_t bytes(int nb) { return wt + 2 * (size_t)D * nb; }
};

template <int NB>
__global__ void __launch_bounds__(BUILD_THREADS)
build_cache_kernel(Dims dm, const __nv_bfloat16* K, const __nv_bfloat16* V, const float* __restrict__ R,
                   const __nv_bfloat16* __restrict__ W, const int* __restrict__ starts,
                   const int* __restrict__ seq_lens, const int* __restrict__ table, __nv_bfloat16* Krot,
                   __nv_bfloat16* Vcache, __nv_bfloat16* __restrict__ pmin, __nv_bfloat16* __restrict__ pmax,
                   uint64_t* __restrict__ codes, int* status) {
  constexpr int NBT = NB / 16;   // bits per thread in the code product
  constexpr int WORDS = NB / 64;
  extern __shared__ __align__(16) unsigned char smem[];
  float* Kt = reinterpret_cast<float*>(smem + BuildSmem::kt);
  float* Rt = reinterpret_cast<float*>(smem + BuildSmem::rt);
  __nv_bfloat16* Ko = reinterpret_cast<__nv_bfloat16*>(smem + BuildSmem::ko);
  float* wn = reinterpret_cast<float*>(smem + BuildSmem::wn);
  float* kn = reinterpret_cast<float*>(smem + BuildSmem::kn);
  unsigned long long* cd = reinterpret_cast<unsigned long long*>(smem + BuildSmem::cd);
  __nv_bfloat16* Wt = reinterpret_cast<__nv_bfloat16*>(smem + BuildSmem::wt);

  const int h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int L = seq_len_of(dm, seq_lens, b);
  const int S0 = starts ? min(max(__ldg(starts + b), 0), L) : 0;  // first row (re)built
  const int row0 = (S0 & ~(BUILD_ROWS - 1)) + blockIdx.x * BUILD_TILES * BUILD_ROWS;
  if (row0 >= L || S0 >= L) return;

  // stage R_h^T and W_h^T, and the norms of the rows of W_h
  const float* Rh = R + (long long)h * D * D;
  for (int e = tid; e < D * D; e += BUILD_THREADS) {
    const int i = e / D, j = e % D;
    Rt[j * D + i] = __ldg(Rh + e);
  }
  const __nv_bfloat16* Wh = W + (long long)h * NB * D;
  for (int e = tid; e < NB * D; e += BUILD_THREADS) {
    const int bit = e / D, j = e % D;
    Wt[j * NB + bit] = Wh[e];
  }
  __syncthreads();
  for (int bit = tid; bit < NB; bit += BUILD_THREADS) {
    float s = 0.f;
    for (int j = 0; j < D; ++j) { const float w = __bfloat162float(Wt[j * NB + bit]); s = fmaf(w, w, s); }
    wn[bit] = sqrtf(s) * 1.0001f;  // a hair above |w_j| so the guard stays conservative
  }

  const int kg = tid >> 4, cg = tid & 15;
  for (int tile = 0; tile < BUILD_TILES; ++tile) {
    const int t0 = row0 + tile * BUILD_ROWS;
    if (t0 >= L) break;
    __syncthreads();
    // ---- load the K tile (transposed, fp32); rows >= L are zero ----
    for (int e = tid; e < BUILD_ROWS * (D / 8); e += BUILD_THREADS) {
      const int r = e / (D / 8), v = e % (D / 8);
      const int t = t0 + r;
      float f[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      if (t >= S0 && t < L) {
        const long long off = kv_row(dm, table, b, h, t, status);
        if (off >= 0) unpack8(*reinterpret_cast<const uint4*>(K + off + v * 8), f);
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) Kt[(v * 8 + c) * BUILD_ROWS + r] = f[c];
    }
    for (int e = tid; e < BUILD_ROWS * 4; e += BUILD_THREADS) cd[e] = 0ull;
    __syncthreads();
    if (tid < BUILD_ROWS) {
      float s = 0.f;
      for (int j = 0; j < D; ++j) { const float x = Kt[j * BUILD_ROWS + tid]; s = fmaf(x, x, s); }
      kn[tid] = sqrtf(s) * 1.0001f;
    }

    // ---- K' = K R^T: thread tile 4 rows x 8 channels ----
    {
      float acc[4][8];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[a][c] = 0.f;
#pragma unroll 4
      for (int j = 0; j < D; ++j) {
        const float4 kx = *reinterpret_cast<const float4*>(Kt + j * BUILD_ROWS + kg * 4);
        const float4 r0 = *reinterpret_cast<const float4*>(Rt + j * D + cg * 8);
        const float4 r1 = *reinterpret_cast<const float4*>(Rt + j * D + cg * 8 + 4);
        const float kr[4] = {kx.x, kx.y, kx.z, kx.w};
        const float rr[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int c = 0; c < 8; ++c) acc[a][c] = fmaf(kr[a], rr[c], acc[a][c]);
      }
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        __align__(16) __nv_bfloat16 ob[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) ob[c] = __float2bfloat16_rn(acc[a][c]);
        *reinterpret_cast<uint4*>(Ko + (kg * 4 + a) * D + cg * 8) = *reinterpret_cast<const uint4*>(ob);
      }
    }
    __syncthreads();

    // ---- code bits: thread tile 4 rows x NBT bits ----
    {
      float acc[4][NBT];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < NBT; ++c) acc[a][c] = 0.f;
#pragma unroll 2
      for (int j = 0; j < D; ++j) {
        const float4 kx = *reinterpret_cast<const float4*>(Kt + j * BUILD_ROWS + kg * 4);
        const float kr[4] = {kx.x, kx.y, kx.z, kx.w};
        float wf[NBT];
        const __nv_bfloat16* wrow = Wt + j * NB + cg * NBT;
        if constexpr (NBT % 8 == 0) {
#pragma unroll
          for (int u = 0; u < NBT / 8; ++u) unpack8(*reinterpret_cast<const uint4*>(wrow + 8 * u), wf + 8 * u);
        } else {
          const uint2 v = *reinterpret_cast<const uint2*>(wrow);
          wf[0] = bf_lo(v.x); wf[1] = bf_hi(v.x); wf[2] = bf_lo(v.y); wf[3] = bf_hi(v.y);
        }
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int c = 0; c < NBT; ++c) acc[a][c] = fmaf(kr[a], wf[c], acc[a][c]);
      }
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const int r = kg * 4 + a;
        unsigned long long bits = 0ull;
#pragma unroll
        for (int c = 0; c < NBT; ++c) {
          const int bit = cg * NBT + c;
          bool s;
          if (fabsf(acc[a][c]) <= ldexpf(wn[bit] * kn[r], -14)) {
            double x = 0.0;
            for (int j = 0; j < D; ++j)
              x += (double)Kt[j * BUILD_ROWS + r] * (double)__bfloat162float(Wt[j * NB + bit]);
            s = x > 0.0;
          } else {
            s = acc[a][c] > 0.f;
          }
          bits |= (unsigned long long)s << c;
        }
        const int bit0 = cg * NBT;
        atomicOr(&cd[r * 4 + bit0 / 64], bits << (bit0 % 64));
      }
    }
    __syncthreads();

    // ---- write K' (and copy V), codes and page min/max ----
    for (int e = tid; e < BUILD_ROWS * (D / 8); e += BUILD_THREADS) {
      const int r = e / (D / 8), v = e % (D / 8);
      const int t = t0 + r;
      if (t >= S0 && t < L) {
        const long long off = kv_row(dm, table, b, h, t, status);
        if (off >= 0) {
          *reinterpret_cast<uint4*>(Krot + off + v * 8) = *reinterpret_cast<const uint4*>(Ko + r * D + v * 8);
          if (Vcache != V) *reinterpret_cast<uint4*>(Vcache + off + v * 8) = ldg16(V + off + v * 8);
        }
      }
    }
    for (int e = tid; e < BUILD_ROWS * WORDS; e += BUILD_THREADS) {
      const int r = e / WORDS, w = e % WORDS;
      const int t = t0 + r;
      if (t >= S0 && t < L) {
        const long long off = code_row(dm, table, b, h, t, status);
        if (off >= 0) codes[off + w] = cd[r * 4 + w];
      }
    }
    const int pages = BUILD_ROWS / dm.P;
    for (int e = tid; e < pages * D; e += BUILD_THREADS) {
      const int pp = e / D, c = e % D;
      const int tp = t0 + pp * dm.P;
      const int r0 = max(0, S0 - tp), r1 = min(dm.P, L - tp);  // the page's rows built here
      if (r0 >= r1) continue;
      float lo = INFINITY, hi = -INFINITY;
      for (int r = r0; r < r1; ++r) {
        const float x = __bfloat162float(Ko[(pp * dm.P + r) * D + c]);
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
  }
}

}  // namespace hhr
