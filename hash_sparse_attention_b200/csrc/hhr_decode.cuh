// HHR decode step (sm_100a): one launch per layer, one group of S CTAs per
// unit (sequence b, KV head h), one CTA per SM, 512 threads.
//
// "HHR: Hierarchical Hash Retrieval for Efficient LLM Generation" (paper
// card, Abstract; rit.work explainer, section "Два уровня маршрутизации решают
// разные ошибки"): GKR bounds every page of keys and keeps the top-N pages,
// LHP ranks the keys of those pages by the Hamming distance of sign codes and
// keeps the top-k, then exact attention runs over the kept keys.
//
// Per unit, CTA r of the group:
//   1. issues cp.async copies of its share of the page metadata (pages
//      [p0, p1), 64 pages per stage, five stages in flight), then computes
//      q' = R_h q and the query sign codes (every CTA of the group; R_h and
//      W_h of the first unit are loaded before the previous kernel on the
//      stream has finished: programmatic dependent launch);
//   2. scans its pages: U = max over the group's query heads of the page
//      bound.  Every thread consumes exactly the 16-byte pieces it copied, so
//      the scan needs no CTA barrier;
//   3. group barrier; the page top-N on ALL the unit's bounds (read from L2),
//      the same in every CTA: a radix select on order-preserving keys, 11
//      bits per level starting from the keys' range, equal keys taken in page
//      order (ties go to the lower page);
//   4. when the key budget covers every candidate row, starts copying the K'/V
//      rows of its first gather chunks right away (the key select below then
//      keeps them all); scores its balanced share of the candidate rows
//      (Hamming distance summed over the group's heads, code words loaded
//      straight into registers) and publishes the score histogram;
//   5. group barrier; the S histograms give the threshold score T, the ties
//      taken at T and the CTA's place in the unit's kept-row list; it writes
//      its kept rows there (row + 1, polled by the readers) unless every
//      candidate is kept (then the list is implied by the kept pages);
//   6. gathers the K'/V rows of its share of the list's 128-row chunks
//      (cp.async, XOR-swizzled rows, three chunks in flight) and computes each
//      chunk's softmax partial on tensor cores (mma.sync: logits with q' as
//      bf16 hi + lo, P.V with P as bf16 hi + lo);
//   7. the last CTA of the group to arrive merges the chunk partials in chunk
//      order into the output and resets the unit's counters.
// A chunk's partial depends only on its rows and the merge order is fixed, so
// results do not depend on S, on the batch or on the cache layout.
#pragma once

#include <algorithm>

#include "hhr_dev.cuh"
#include "hhr_launch.h"

namespace hhr {

constexpr int SP_THREADS = 512;
constexpr int SP_WARPS = SP_THREADS / 32;
constexpr int SP_STAGE_PAGES = 64;                   // pages per metadata stage
constexpr int SP_META_STAGE = SP_STAGE_PAGES * 512;  // 64 rows of minima, then 64 rows of maxima
constexpr int SP_NST = 5;                            // metadata stages in flight
constexpr int SP_ROWS = 128;                         // rows per gather chunk
constexpr int SP_GSTAGE = SP_ROWS * 512;             // 128 K' rows, then 128 V rows
constexpr int SP_NGS = 3;                            // gather chunks in flight

// shared memory map (bytes).  Region A is reused by every phase.
constexpr int SP_A_BYTES = SP_NGS * SP_GSTAGE;                // 192 KB
constexpr int SP_PREP = SP_NST * SP_META_STAGE;               // q, q' (prep) and the page-select histograms
constexpr int SP_PSH = SP_PREP + 8192;                        // int [2][2048] page-select histograms
constexpr int SP_HISTS = 2 * SP_GSTAGE;                       // key select: S score histograms, then scores
constexpr int SP_QB = SP_A_BYTES;                             // bf16 [16][136] q' operand (hi, lo)
constexpr int SP_PB = SP_QB + 16 * 272;                       // bf16 [16][136] P operand (hi, lo)
constexpr int SP_MX = SP_PB + 16 * 272;                       // float [8 warps][8 heads] row-block maxima
constexpr int SP_LS = SP_MX + 256;                            // float [8][8] row-block weight sums
constexpr int SP_OB = SP_LS + 256;                            // float [128 ch][16 cols] P.V of a chunk
constexpr int SP_KP = SP_OB + 128 * 16 * 4;                   // int [MAX_KEEP_PAGES] kept pages
constexpr int SP_QC = SP_KP + MAX_KEEP_PAGES * 4;             // u32 [8 heads][8] query codes
constexpr int SP_RED = SP_QC + 256;                           // int: [0,64) scans, [64,128) min/max, [128,160) broadcasts
constexpr int SP_MISC = SP_RED + 640;                         // int [32] flags
constexpr int SP_SMEM = SP_MISC + 128;
static_assert(SP_SMEM <= 232448, "shared memory of the decode kernel");
static_assert(SP_PSH + 2 * 2048 * 4 <= SP_A_BYTES, "page-select scratch");
static_assert(SP_PREP >= 2 * SP_GSTAGE, "page-select scratch must not overlap the first two gather stages");

// misc flags
enum : int { MS_ABORT = 0, MS_LAST = 1 };

// per-unit words of the workspace exchange area, zero between calls
enum : int { GX_BAR = 0, GX_ARRIVE = 1 };

struct SpParams {
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
  long long wait_limit;  // SM clock cycles of every bounded wait
  int gsize;             // S: CTAs per group
  int ngroups;           // groups in the grid
};

struct SpUnit {
  int u, b, h, L, np;
};

__device__ __forceinline__ void share_of(int n, int S, int r, int& a, int& b) {
  a = (int)(((long long)n * r) / S);
  b = (int)(((long long)n * (r + 1)) / S);
}

__device__ __forceinline__ bool sp_aborted(const unsigned char* sm) {
  return *reinterpret_cast<const volatile int*>(sm + SP_MISC + 4 * MS_ABORT) != 0;
}
__device__ __forceinline__ void sp_abort(const SpParams& p, unsigned char* sm, int code) {
  set_status(p.status, code);
  *reinterpret_cast<volatile int*>(sm + SP_MISC + 4 * MS_ABORT) = 1;
}

// Group barrier: every write made before it by any thread of the group's S
// CTAs is visible after it (read such data with .cg loads: L1 is not
// coherent).  A release add and a bounded acquire poll on the unit's counter.
// False after a timeout or an abort (every thread of the CTA sees the same).
__device__ __forceinline__ bool sp_group_sync(const SpParams& p, unsigned char* sm, unsigned* gx, unsigned& epoch) {
  __syncthreads();
  if (p.gsize > 1) {
    epoch += (unsigned)p.gsize;
    if (threadIdx.x == 0) {
      red_release_add(gx + GX_BAR, 1u);
      if (ld_acquire(gx + GX_BAR) < epoch) {
        Spin sp(p.wait_limit);
        while (ld_acquire(gx + GX_BAR) < epoch) {
          if (sp_aborted(sm)) break;
          if (sp.expired()) {
            sp_abort(p, sm, HHR_ERR_TIMEOUT);
            break;
          }
        }
      }
    }
    __syncthreads();
  }
  return !sp_aborted(sm);
}

// ---------------------------------------------------------------------------
// prep: q' = R_h q and the query codes
// ---------------------------------------------------------------------------
// Warp w takes rows 8w .. 8w+7 of R_h and bits [w nb/16, (w+1) nb/16) of W_h
// in blocks of NBB rows; lane l holds channels 4l .. 4l+3 of each row.
template <int G>
struct Prep {
  static constexpr int GP = G <= 4 ? 4 : 8;  // heads padded to a power of two
  static constexpr int NBB = 32 / GP;        // code bits per block
  float4 rr[8];
  uint2 wv[NBB];
};

template <int G, bool CODES = true>
__device__ __forceinline__ void sp_prep_load(const SpParams& p, int h, Prep<G>& pr) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* Rh = p.R + (long long)h * D * D;
#pragma unroll
  for (int k = 0; k < 8; ++k) pr.rr[k] = __ldg(reinterpret_cast<const float4*>(Rh + (long long)(warp * 8 + k) * D) + lane);
  if constexpr (CODES) {
    const int bpw = p.dm.nb / SP_WARPS;
    const __nv_bfloat16* Wh = p.W + (long long)h * p.dm.nb * D;
#pragma unroll
    for (int bb = 0; bb < Prep<G>::NBB; ++bb)
      pr.wv[bb] = bb < bpw ? __ldg(reinterpret_cast<const uint2*>(Wh + (long long)(warp * bpw + bb) * D) + lane)
                           : make_uint2(0u, 0u);
  }
}

// Writes q' (fp32, natural order) to qs [G][128], the hi/lo bf16 operand of the
// logits (q' * sm_scale * log2 e) and the query codes (SP_QC).  The sign of a
// code bit is exact: the fp32 sum is trusted when |sum| > 2^-14 sum|w q|,
// otherwise it is recomputed in fp64.
template <int G, bool CODES = true>
__device__ void sp_prep(const SpParams& p, unsigned char* sm, const SpUnit& x, Prep<G>& pr, bool write_dbg) {
  constexpr int GP = Prep<G>::GP, NBB = Prep<G>::NBB;
  const Dims& dm = p.dm;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float* qf = reinterpret_cast<float*>(sm + SP_PREP);         // [G][128] q
  float* qs = reinterpret_cast<float*>(sm + SP_PREP + 4096);  // [G][128] q'
  unsigned* qc = reinterpret_cast<unsigned*>(sm + SP_QC);
  const __nv_bfloat16* qg = p.q + ((long long)x.b * dm.Hq + x.h * G) * D;
  for (int i = tid; i < G * D; i += SP_THREADS) qf[i] = __bfloat162float(qg[i]);
  if (tid < 64) qc[tid] = 0u;
  __syncthreads();
  float qv[GP][4];
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    if (g < G) {
      const float4 t = *reinterpret_cast<const float4*>(qf + g * D + 4 * lane);
      qv[g][0] = t.x; qv[g][1] = t.y; qv[g][2] = t.z; qv[g][3] = t.w;
    } else {
      qv[g][0] = qv[g][1] = qv[g][2] = qv[g][3] = 0.f;
    }
  }
  {
    // q' rows 8w + k for every head: 8 GP dot products per lane, reduced over the warp
    constexpr int NV = 8 * GP, KP = NV / 32;
    float v[NV];
#pragma unroll
    for (int k = 0; k < 8; ++k)
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        const float4 a = pr.rr[k];
        float s = a.x * qv[g][0];
        s = fmaf(a.y, qv[g][1], s);
        s = fmaf(a.z, qv[g][2], s);
        v[k * GP + g] = fmaf(a.w, qv[g][3], s);
      }
    group_reduce_scatter<NV, 32>(v, lane);
#pragma unroll
    for (int e = 0; e < KP; ++e) {
      const int vi = KP * lane + e, k = vi / GP, g = vi % GP;
      if (g < G) {
        const int i = warp * 8 + k;
        qs[g * D + i] = v[e];
        if (write_dbg && p.dbg.q_rot) p.dbg.q_rot[((long long)x.b * dm.Hq + x.h * G + g) * D + i] = v[e];
      }
    }
  }
  // query codes: warp w takes bits [w bpw, (w+1) bpw) in blocks of NBB
  const int bpw = CODES ? dm.nb / SP_WARPS : 0;
  const __nv_bfloat16* Wh = p.W + (long long)x.h * dm.nb * D;
  // (lane: channels 4l .. 4l+3 of a W row as two bf16 pairs, loaded as uint2)
  for (int jb = 0; jb < bpw; jb += NBB) {
    if (jb > 0) {
#pragma unroll
      for (int bb = 0; bb < NBB; ++bb)
        pr.wv[bb] = jb + bb < bpw ? __ldg(reinterpret_cast<const uint2*>(Wh + (long long)(warp * bpw + jb + bb) * D) + lane)
                                  : make_uint2(0u, 0u);
    }
    float v[2 * NBB * GP];
#pragma unroll
    for (int bb = 0; bb < NBB; ++bb) {
      const float w4[4] = {bf_lo(pr.wv[bb].x), bf_hi(pr.wv[bb].x), bf_lo(pr.wv[bb].y), bf_hi(pr.wv[bb].y)};
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        float a = 0.f, m = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float pe = w4[e] * qv[g][e];
          a += pe;
          m += fabsf(pe);
        }
        v[(bb * GP + g) * 2 + 0] = a;
        v[(bb * GP + g) * 2 + 1] = m;
      }
    }
    group_reduce_scatter<2 * NBB * GP, 32>(v, lane);
    const int bb = lane / GP, g = lane % GP;
    const int j = warp * bpw + jb + bb;
    if (g < G && jb + bb < bpw) {
      bool bit = v[0] > 0.f;
      if (fabsf(v[0]) <= ldexpf(v[1], -14)) {
        double ad = 0.0;
        const __nv_bfloat16* wrow = Wh + (long long)j * D;
        for (int c = 0; c < D; ++c) ad += (double)__bfloat162float(wrow[c]) * (double)qf[g * D + c];
        bit = ad > 0.0;
      }
      if (bit) atomicOr(&qc[g * 8 + j / 32], 1u << (j % 32));
    }
  }
  __syncthreads();
  // the logits operand: q' * sm_scale * log2(e) as bf16 hi (columns 0..HP-1) + lo (HP..2HP-1)
  {
    constexpr int HP = G <= 4 ? 4 : 8;
    const float qscale = p.sm_scale * 1.4426950408889634f;
    __nv_bfloat16* qb = reinterpret_cast<__nv_bfloat16*>(sm + SP_QB);
    for (int e = tid; e < HP * D; e += SP_THREADS) {
      const int hh = e / D, c = e - hh * D;
      const float val = hh < G ? qs[hh * D + c] * qscale : 0.f;
      __nv_bfloat16 hi, lo;
      split_bf16(val, hi, lo);
      qb[hh * 136 + c] = hi;
      qb[(HP + hh) * 136 + c] = lo;
    }
  }
  if (CODES && write_dbg && p.dbg.q_codes) {
    const int w32 = dm.words * 2;
    if (tid < G * w32) {
      const int g = tid / w32, k = tid - g * w32;
      reinterpret_cast<uint32_t*>(p.dbg.q_codes)[((long long)x.b * dm.Hq + x.h * G + g) * w32 + k] = qc[g * 8 + k];
    }
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------
// scan: page bounds of the CTA's pages
// ---------------------------------------------------------------------------
// Stage s holds pages p0 + 64 s + j (j < 64): minima rows at j*256, maxima at
// 64*256 + j*256.  Thread t copies and later reads the 16-byte piece (t & 15)
// (channels 8(t&15) .. +7) of pages j = t/16 and j = t/16 + 32, minima and maxima.
__device__ __forceinline__ void sp_issue_meta(const SpParams& p, unsigned char* stage, const SpUnit& x, int pg0,
                                              int p1) {
  const int tid = threadIdx.x, li = tid & 15;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int j = (tid >> 4) + 32 * half;
    const int pg = pg0 + j;
    unsigned char* dmin = stage + j * 256 + li * 16;
    // every thread issues both copies: a page past the share or with a bad
    // block id (the status records it) reads as zeros
    const long long off = pg < p1 ? meta_row(p.dm, p.table, x.b, x.h, pg, p.status) : -1;
    const bool ok = off >= 0;
    const long long e = ok ? off + li * 8 : 0;
    const unsigned nbytes = ok ? 16u : 0u;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dmin)), "l"(p.pmin + e), "r"(nbytes)
                 : "memory");
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dmin + SP_STAGE_PAGES * 256)),
                 "l"(p.pmax + e), "r"(nbytes)
                 : "memory");
  }
}

// Bounds of the (up to) 64 pages of one stage.  Half-warp hw = t/16 computes
// pages hw and hw + 32; lane li holds 8 channels; U = max over the heads.
template <int G>
__device__ __forceinline__ void sp_scan_stage(const SpParams& p, const unsigned char* stage, const SpUnit& x, int pg0,
                                              int p1, const float2 (&qa)[G][4], const float2 (&qb)[G][4]) {
  constexpr int GP = G <= 4 ? 4 : 8;
  constexpr bool SPLIT = G <= 4;  // q+ / q- kept apart (else q' with a select of min or max)
  constexpr int NV = 2 * GP;
  const int tid = threadIdx.x, lane = tid & 31, li = tid & 15;
  float v[NV];
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int j = (tid >> 4) + 32 * half;
    const uint4 mnv = *reinterpret_cast<const uint4*>(stage + j * 256 + li * 16);
    const uint4 mxv = *reinterpret_cast<const uint4*>(stage + SP_STAGE_PAGES * 256 + j * 256 + li * 16);
    const uint32_t mw[4] = {mnv.x, mnv.y, mnv.z, mnv.w};
    const uint32_t xw[4] = {mxv.x, mxv.y, mxv.z, mxv.w};
    float2 mn[4], mx[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      mn[k] = make_float2(bf_lo(mw[k]), bf_hi(mw[k]));
      mx[k] = make_float2(bf_lo(xw[k]), bf_hi(xw[k]));
    }
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      float s = 0.f;
      if (g < G) {
        float2 a0, a1;
        if constexpr (SPLIT) {
          a0 = __fmul2_rn(qa[g][0], mx[0]);
          a1 = __fmul2_rn(qb[g][0], mn[0]);
#pragma unroll
          for (int k = 1; k < 4; ++k) {
            a0 = __ffma2_rn(qa[g][k], mx[k], a0);
            a1 = __ffma2_rn(qb[g][k], mn[k], a1);
          }
        } else {
          float2 sel[4];
#pragma unroll
          for (int k = 0; k < 4; ++k)
            sel[k] = make_float2(qa[g][k].x >= 0.f ? mx[k].x : mn[k].x, qa[g][k].y >= 0.f ? mx[k].y : mn[k].y);
          a0 = __fmul2_rn(qa[g][0], sel[0]);
          a1 = __fmul2_rn(qa[g][1], sel[1]);
          a0 = __ffma2_rn(qa[g][2], sel[2], a0);
          a1 = __ffma2_rn(qa[g][3], sel[3], a1);
        }
        s = (a0.x + a0.y) + (a1.x + a1.y);
      }
      v[half * GP + g] = s;
    }
  }
  // lane li of the half-warp now holds quantity q = li * NV / 16: page half q / GP, head q % GP
  group_reduce_scatter<NV, 16>(v, lane);
  const int q = li * NV / 16;
  const int half = q / GP, g = q % GP;
  float U;
  if (!p.dm.page_sum) {  // max over the heads (lanes of a half hold its heads, some twice)
    U = g < G ? v[0] : -INFINITY;
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) U = fmaxf(U, __shfl_xor_sync(0xffffffffu, U, o));
  } else {  // sum over the heads: one lane per head (NV = 8: even and odd lanes hold copies)
    U = g < G ? v[0] : 0.f;
#pragma unroll
    for (int o = NV == 8 ? 2 : 1; o < 8; o <<= 1) U += __shfl_xor_sync(0xffffffffu, U, o);
  }
  const int j = (tid >> 4) + 32 * half;
  const int pg = pg0 + j;
  if (pg < p1) {
    const Dims& dm = p.dm;
    if ((li & 7) == 0) {
      p.wk.U[(long long)x.u * p.wk.Ustride + pg] = U;
      if (p.dbg.page_U) p.dbg.page_U[(long long)x.u * dm.np_max + pg] = U;
    }
    // the per-head bound (one writer per quantity)
    if (p.dbg.page_ub && g < G && (NV == 16 || (li & 1) == 0))
      p.dbg.page_ub[((long long)x.b * dm.Hq + x.h * G + g) * dm.np_max + pg] = v[0];
  }
}

// ---------------------------------------------------------------------------
// page top-N (larger bound first, ties to the lower page)
// ---------------------------------------------------------------------------
// Thread t holds pages [16t, 16t+16) of the unit as order-preserving keys (a
// larger bound gives a larger key; -0 folds into +0).  Each level bins the
// remaining candidates by (key - base) >> shift into at most 2048 bins, keeps
// every bin above the one holding the need-th largest and descends into that
// bin; the first level's shift comes from the keys' range, each next level
// resolves 11 more bits, and a bin of one key value (shift 0) is taken in
// page order.  Writes the kept pages (ascending) to SP_KP; returns their count.
static __device__ int sp_psel(const SpParams& p, unsigned char* sm, const SpUnit& x, int N, bool write_dbg) {
  const int tid = threadIdx.x;
  int* kp = reinterpret_cast<int*>(sm + SP_KP);
  int* red = reinterpret_cast<int*>(sm + SP_RED);
  int* bc = red + 128;
  int* hist0 = reinterpret_cast<int*>(sm + SP_PSH);
  const int np = x.np;
  const int i0 = tid * 16;
  const int cnt = max(0, min(16, np - i0));
  unsigned member = cnt >= 16 ? 0xffffu : ((1u << cnt) - 1u);
  unsigned keep = 0u;
  int par = 0;  // scan-buffer parity
  if (N >= np) {
    keep = member;
  } else {
    uint32_t key[16];
    const float* Ug = p.wk.U + (long long)x.u * p.wk.Ustride + i0;
#pragma unroll
    for (int k4 = 0; k4 < 4; ++k4) {
      float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
      if (i0 + 4 * k4 < np) t = __ldcg(reinterpret_cast<const float4*>(Ug) + k4);
      key[4 * k4 + 0] = order_key(t.x);
      key[4 * k4 + 1] = order_key(t.y);
      key[4 * k4 + 2] = order_key(t.z);
      key[4 * k4 + 3] = order_key(t.w);
    }
    for (int i = tid; i < 2 * 2048; i += SP_THREADS) hist0[i] = 0;
    unsigned lo = 0xffffffffu, hi = 0u;
#pragma unroll
    for (int k = 0; k < 16; ++k)
      if ((member >> k) & 1u) {
        lo = min(lo, key[k]);
        hi = max(hi, key[k]);
      }
    block_minmax_u32(lo, hi, reinterpret_cast<unsigned*>(red + 64));  // (its barrier also orders the clears)
    int need = N;
    unsigned base = lo;
    const unsigned width = hi - lo;
    int shift = width < 2048u ? 0 : (32 - __clz(width)) - 11;
#pragma unroll 1
    for (int level = 0;; ++level) {
      int* hist = hist0 + 2048 * (level & 1);
      int* hnext = hist0 + 2048 * ((level + 1) & 1);
#pragma unroll
      for (int k = 0; k < 16; ++k)
        if ((member >> k) & 1u) atomicAdd(&hist[(key[k] - base) >> shift], 1);
      __syncthreads();
      // thread t: bins 2047-4t .. 2044-4t, counted from the top
      int hv[4], c4 = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        hv[e] = hist[2047 - 4 * tid - e];
        c4 += hv[e];
      }
      int tot;
      const int before = block_scan_excl(c4, red, par++, &tot);
      if (before < need && before + c4 >= need) {
        int run = before;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (run < need && run + hv[e] >= need) {
            bc[0] = 2047 - 4 * tid - e;
            bc[1] = need - run;
            bc[2] = hv[e];
          }
          run += hv[e];
        }
      }
      for (int i = tid; i < 2048; i += SP_THREADS) hnext[i] = 0;
      __syncthreads();
      const int bstar = bc[0], need_in = bc[1], cnt_in = bc[2];
      unsigned m2 = 0u;
#pragma unroll
      for (int k = 0; k < 16; ++k)
        if ((member >> k) & 1u) {
          const int bn = (int)((key[k] - base) >> shift);
          if (bn > bstar) keep |= 1u << k;
          else if (bn == bstar) m2 |= 1u << k;
        }
      member = m2;
      need = need_in;
      if (cnt_in == need_in) {  // the whole bin is kept
        keep |= member;
        break;
      }
      if (shift == 0) {  // one key value: equal bounds, the first `need` in page order
        int tot2;
        const int mb = block_scan_excl(__popc(member), red, par++, &tot2);
        int take = max(0, min(__popc(member), need - mb));
#pragma unroll
        for (int k = 0; k < 16; ++k)
          if (((member >> k) & 1u) && take > 0) {
            keep |= 1u << k;
            --take;
          }
        break;
      }
      base += (unsigned)bstar << shift;
      shift = shift > 11 ? shift - 11 : 0;
    }
  }
  int nkp;
  int pos = block_scan_excl(__popc(keep), red, par++, &nkp);
  int* dsel = (write_dbg && p.dbg.sel_pages) ? p.dbg.sel_pages + (long long)x.u * p.wk.Nmax : nullptr;
#pragma unroll
  for (int k = 0; k < 16; ++k)
    if (((keep >> k) & 1u) && pos < MAX_KEEP_PAGES) {
      kp[pos] = i0 + k;
      if (dsel) dsel[pos] = i0 + k;
      ++pos;
    }
  if (write_dbg && tid == 0 && p.dbg.n_sel_pages) p.dbg.n_sel_pages[x.u] = nkp;
  __syncthreads();
  return nkp;
}

// ---------------------------------------------------------------------------
// gather: K'/V rows of a 128-row chunk, then its softmax partial
// ---------------------------------------------------------------------------
// Row j of the chunk, 16-byte piece c: K' at stage + j*256 + ((c ^ (j & 7)) * 16),
// V 32 KB further (eight consecutive rows' same piece fall in distinct banks
// for ldmatrix).  Warp w copies rows 8w .. 8w+7; lane l < 8 resolves row 8w + l
// (its element offset / 128, or -1 for a row past the chunk or a bad row).
__device__ __forceinline__ void sp_copy_rows(const SpParams& p, unsigned char* stage, int rowidx) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int c = lane & 15;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int jl = 2 * i + (lane >> 4);
    const int j = warp * 8 + jl;
    const int ri = __shfl_sync(0xffffffffu, rowidx, jl);
    unsigned char* dk = stage + j * 256 + ((c ^ (j & 7)) * 16);
    // a row past the chunk or a bad row reads as zeros (the tensor-core products stay finite)
    const long long e = ri >= 0 ? (long long)ri * D + c * 8 : 0;
    const unsigned nbytes = ri >= 0 ? 16u : 0u;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dk)), "l"(p.Kr + e), "r"(nbytes)
                 : "memory");
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dk + SP_ROWS * 256)),
                 "l"(p.Vc + e), "r"(nbytes)
                 : "memory");
  }
}

// Column layout of the two mma operands: NT = 1 (G <= 4): columns 0-3 the
// heads' hi parts, 4-7 their lo parts; NT = 2 (G <= 8): 0-7 hi, 8-15 lo.
template <int G>
struct GCols {
  static constexpr int NT = G <= 4 ? 1 : 2;
  static constexpr int HP = 4 * NT;
  __device__ static int hi(int h) { return h; }
  __device__ static int lo(int h) { return HP + h; }
};

// One chunk of up to 128 kept rows: logits S = K' (q' hi + lo)^T on tensor
// cores (warps 0-7, 16 rows each), the chunk's maximum and weights per head in
// fp32, then O^T = V^T (P hi + lo)^T (warps 0-7, 16 channels each over all 128
// rows).  The partial (unnormalised output, then per head the maximum and the
// sum of weights, in log2 units) goes to `part`; it depends only on the rows.
template <int G>
__device__ void sp_gather_step(unsigned char* sm, const unsigned char* stage, int n, float* part) {
  using C = GCols<G>;
  constexpr int NT = C::NT;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const unsigned char* qb = sm + SP_QB;
  __nv_bfloat16* pb = reinterpret_cast<__nv_bfloat16*>(sm + SP_PB);
  float* mx = reinterpret_cast<float*>(sm + SP_MX);
  float* ls = reinterpret_cast<float*>(sm + SP_LS);
  float* ob = reinterpret_cast<float*>(sm + SP_OB);
  float sv[2][2];
  int h0 = 0;
  if (warp < 8) {
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
    const int r0 = warp * 16;
    const int arow = r0 + (lane & 7) + ((lane >> 3) & 1) * 8;
    const unsigned char* krow = stage + arow * 256;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      uint32_t af[4];
      ldsm_x4(af, krow + (((2 * ks + (lane >> 4)) ^ (arow & 7)) * 16));
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        uint32_t bf[2];
        ldsm_x2(bf, qb + (nt * 8 + (lane & 7)) * 272 + (2 * ks + ((lane >> 3) & 1)) * 16);
        mma_bf16(acc[nt], af, bf);
      }
    }
    // hi + lo of the same heads: NT = 1 pairs columns 2t, 2t+1 with 2t+4, 2t+5
    // (lane t ^ 2); NT = 2 holds them in its two n-tiles
    float v0 = acc[0][0], v1 = acc[0][1], v2 = acc[0][2], v3 = acc[0][3];
    if constexpr (NT == 1) {
      v0 += __shfl_xor_sync(0xffffffffu, v0, 2);
      v1 += __shfl_xor_sync(0xffffffffu, v1, 2);
      v2 += __shfl_xor_sync(0xffffffffu, v2, 2);
      v3 += __shfl_xor_sync(0xffffffffu, v3, 2);
      h0 = 2 * (t & 1);
    } else {
      v0 += acc[NT - 1][0];
      v1 += acc[NT - 1][1];
      v2 += acc[NT - 1][2];
      v3 += acc[NT - 1][3];
      h0 = 2 * t;
    }
    const bool rg = r0 + g < n, rg8 = r0 + g + 8 < n;
    sv[0][0] = (rg && h0 < G) ? v0 : -INFINITY;
    sv[0][1] = (rg && h0 + 1 < G) ? v1 : -INFINITY;
    sv[1][0] = (rg8 && h0 < G) ? v2 : -INFINITY;
    sv[1][1] = (rg8 && h0 + 1 < G) ? v3 : -INFINITY;
    float m0 = fmaxf(sv[0][0], sv[1][0]), m1 = fmaxf(sv[0][1], sv[1][1]);
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, o));
      m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, o));
    }
    if (g == 0 && (NT == 2 || t < 2)) {
      mx[warp * 8 + h0] = m0;
      mx[warp * 8 + h0 + 1] = m1;
    }
  }
  __syncthreads();
  if (warp < 8) {
    const int r0 = warp * 16;
    float M0 = -INFINITY, M1 = -INFINITY;
#pragma unroll
    for (int w2 = 0; w2 < 8; ++w2) {
      M0 = fmaxf(M0, mx[w2 * 8 + h0]);
      M1 = fmaxf(M1, mx[w2 * 8 + h0 + 1]);
    }
    float pw[2][2];
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      pw[rr][0] = sv[rr][0] == -INFINITY ? 0.f : exp2f(sv[rr][0] - M0);
      pw[rr][1] = sv[rr][1] == -INFINITY ? 0.f : exp2f(sv[rr][1] - M1);
    }
    float l0 = pw[0][0] + pw[1][0], l1 = pw[0][1] + pw[1][1];
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, o);
      l1 += __shfl_xor_sync(0xffffffffu, l1, o);
    }
    if (NT == 2 || t < 2) {
      if (g == 0) {
        ls[warp * 8 + h0] = l0;
        ls[warp * 8 + h0 + 1] = l1;
      }
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        const int row = r0 + g + 8 * rr;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          __nv_bfloat16 hi, lo;
          split_bf16(pw[rr][e], hi, lo);
          pb[C::hi(h0 + e) * 136 + row] = hi;
          pb[C::lo(h0 + e) * 136 + row] = lo;
        }
      }
    }
  }
  __syncthreads();
  if (warp < 8) {  // O^T = V^T P^T: warp w: channels 16w .. 16w+15, all rows
    float oacc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) oacc[nt][0] = oacc[nt][1] = oacc[nt][2] = oacc[nt][3] = 0.f;
    const unsigned char* vbase = stage + SP_ROWS * 256;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const int k0 = ks * 16;
      const int vrow = k0 + (lane & 7) + 8 * (lane >> 4);  // matrices 2, 3: rows k0 + 8 ..
      const int vch = 2 * warp + ((lane >> 3) & 1);        // matrices 1, 3: channels + 8
      uint32_t af[4];
      ldsm_x4_t(af, vbase + vrow * 256 + ((vch ^ (vrow & 7)) * 16));
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        uint32_t bf[2];
        ldsm_x2(bf, reinterpret_cast<const unsigned char*>(pb) + (nt * 8 + (lane & 7)) * 272 +
                        (k0 / 8 + ((lane >> 3) & 1)) * 16);
        mma_bf16(oacc[nt], af, bf);
      }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int c0 = 16 * warp + g, col = 8 * nt + 2 * t;
      *reinterpret_cast<float2*>(ob + (c0 * 16 + col)) = make_float2(oacc[nt][0], oacc[nt][1]);
      *reinterpret_cast<float2*>(ob + ((c0 + 8) * 16 + col)) = make_float2(oacc[nt][2], oacc[nt][3]);
    }
  }
  __syncthreads();
  for (int e = tid; e < G * D; e += SP_THREADS) {
    const int h = e / D, c = e - h * D;
    const float* o0 = ob + c * 16;
    part[h * D + c] = o0[C::hi(h)] + o0[C::lo(h)];
  }
  if (tid < G) {
    float M = -INFINITY, Ls = 0.f;
#pragma unroll
    for (int w2 = 0; w2 < 8; ++w2) M = fmaxf(M, mx[w2 * 8 + tid]);
#pragma unroll
    for (int w2 = 0; w2 < 8; ++w2) Ls += ls[w2 * 8 + tid];
    part[G * D + tid] = M;
    part[G * D + 8 + tid] = Ls;
  }
  __syncthreads();  // the stage and the step's scratch are free
}

// Element offset / 128 of kept-list row j of the unit (the chunk's rows), or
// -1 for j >= n_rows.  all_kept: row j is candidate j (rows of the kept pages
// in page order); otherwise the list entry (row + 1, written by the key
// select of some CTA of the group) is polled, bounded, and cleared.
__device__ __forceinline__ int sp_row_of(const SpParams& p, unsigned char* sm, const SpUnit& x, int j, int n_rows,
                                         bool all_kept) {
  if (j >= n_rows) return -1;
  int t;
  if (all_kept) {
    const int* kp = reinterpret_cast<const int*>(sm + SP_KP);
    t = (kp[j >> p.dm.lgP] << p.dm.lgP) + (j & (p.dm.P - 1));
  } else {
    int* e = p.wk.sel_keys + (long long)x.u * p.wk.Kmax + j;
    int v = ld_relaxed_s32(e);
    if (v == 0) {
      Spin sp(p.wait_limit);
      while ((v = ld_relaxed_s32(e)) == 0) {
        if (sp_aborted(sm)) return -1;
        if (sp.expired()) {
          sp_abort(p, sm, HHR_ERR_TIMEOUT);
          return -1;
        }
      }
    }
    *e = 0;  // the list is zero again for the next call
    t = v - 1;
  }
  const long long off = kv_row(p.dm, p.table, x.b, x.h, t, p.status);
  return off >= 0 ? (int)(off / D) : -1;
}

// Issues the copies of chunk c into stage (c - c0) mod 3 (one commit group per
// thread, possibly empty).
__device__ __forceinline__ void sp_issue_chunk(const SpParams& p, unsigned char* sm, const SpUnit& x, int c, int c0,
                                               int c1, int keff, bool all_kept) {
  if (c < c1) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int j = c * SP_ROWS + warp * 8 + (lane & 7);
    const int ri = lane < 8 ? sp_row_of(p, sm, x, j, keff, all_kept) : -1;
    sp_copy_rows(p, sm + ((c - c0) % SP_NGS) * SP_GSTAGE, ri);
  }
  cp_async_commit();
}

// ---------------------------------------------------------------------------
// scores and key top-k (smaller score first, ties to the lower row)
// ---------------------------------------------------------------------------
// Candidates are the rows of the kept pages in page order (slot ci: page
// kp[ci / P], row ci % P; slots past the sequence end are not candidates).
// CTA r scores its balanced share [cs0, cs1) and publishes the histogram of
// its integer scores; after the group barrier the S histograms give the
// threshold T, the ties taken at T and the CTA's first place in the list.
// Returns k_eff (0 after an abort; `ok` then false).
template <int G, int WORDS>
__device__ int sp_keys(const SpParams& p, unsigned char* sm, const SpUnit& x, int r, int nkp, int n_cand_local,
                       int keff, bool all_kept, unsigned* gx, unsigned& epoch, bool& ok) {
  const Dims& dm = p.dm;
  const Work& wk = p.wk;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int S = p.gsize;
  const int nbins = G * dm.nb + 1, HB = wk.HB;
  int* hists = reinterpret_cast<int*>(sm + SP_HISTS);                          // [S][HB]
  uint16_t* sc = reinterpret_cast<uint16_t*>(sm + SP_HISTS + S * HB * 4);      // [share]
  int* hist = hists;                                                           // the CTA's own, first
  int* red = reinterpret_cast<int*>(sm + SP_RED);
  int* bc = red + 128;
  const int* kp = reinterpret_cast<const int*>(sm + SP_KP);
  const unsigned* qcw = reinterpret_cast<const unsigned*>(sm + SP_QC);
  const int ncs = nkp << dm.lgP;
  int cs0, cs1;
  share_of(ncs, S, r, cs0, cs1);
  const int nmy = cs1 - cs0;
  for (int i = tid; i < HB; i += SP_THREADS) hist[i] = 0;
  uint64_t cq[G][WORDS];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int w2 = 0; w2 < WORDS; ++w2)
      cq[g][w2] = (uint64_t)qcw[g * 8 + 2 * w2] | ((uint64_t)qcw[g * 8 + 2 * w2 + 1] << 32);
  __syncthreads();
  int* dsc = p.dbg.key_scores ? p.dbg.key_scores + (long long)x.u * wk.Nmax * dm.P + cs0 : nullptr;
#pragma unroll 1
  for (int j = tid; j < nmy; j += SP_THREADS) {
    const int ci = cs0 + j;
    const int t = (kp[ci >> dm.lgP] << dm.lgP) + (ci & (dm.P - 1));
    const long long woff = t < x.L ? code_row(dm, p.table, x.b, x.h, t, p.status) : -1;
    int sv = 0xFFFF;
    if (woff >= 0) {
      const uint64_t* src = p.codes + woff;
      uint64_t cw[WORDS];
      if constexpr (WORDS == 1) {
        cw[0] = __ldg(reinterpret_cast<const unsigned long long*>(src));
      } else {
#pragma unroll
        for (int w2 = 0; w2 < WORDS; w2 += 2) {
          const ulonglong2 v2 = __ldg(reinterpret_cast<const ulonglong2*>(src + w2));
          cw[w2] = v2.x;
          cw[w2 + 1] = v2.y;
        }
      }
      int sum = 0, mn = INT_MAX;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        int sg = 0;
#pragma unroll
        for (int w2 = 0; w2 < WORDS; ++w2) sg += __popcll(cw[w2] ^ cq[g][w2]);
        sum += sg;
        mn = min(mn, sg);
      }
      sv = dm.key_min ? mn : sum;
      atomicAdd(&hist[sv], 1);
    }
    sc[j] = (uint16_t)sv;
    if (dsc) dsc[j] = sv == 0xFFFF ? INT_MAX : sv;
  }
  __syncthreads();
  int* myh = wk.khist + (long long)blockIdx.x * HB;
  for (int i = tid; i < nbins; i += SP_THREADS) myh[i] = hist[i];
  if (!sp_group_sync(p, sm, gx, epoch)) {
    ok = false;
    return 0;
  }
  // ---- the group's S histograms (plain .cg loads: no cp.async group may be
  // waited here, the gather's chunk copies are in flight) ----
  {
    const int4* src = reinterpret_cast<const int4*>(wk.khist + (long long)(blockIdx.x - r) * HB);
    int4* dst = reinterpret_cast<int4*>(hists);
    const int n4 = S * HB / 4;
    for (int i = tid; i < n4; i += SP_THREADS) dst[i] = __ldcg(src + i);
  }
  __syncthreads();
  // sum per bin (thread t: bins [t bpt, t bpt + bpt)), threshold from below
  const int bpt = (nbins + SP_THREADS - 1) / SP_THREADS;  // <= 5
  int hv[5];
  int local = 0;
#pragma unroll
  for (int e = 0; e < 5; ++e) {
    const int bi = tid * bpt + e;
    int s = 0;
    if (e < bpt && bi < nbins)
      for (int rr = 0; rr < S; ++rr) s += hists[rr * HB + bi];
    hv[e] = s;
    local += s;
  }
  if (tid == 0) {
    bc[0] = -1;  // no candidate: nothing kept
    bc[1] = 0;
  }
  int n_cand;
  const int before = block_scan_excl(local, red, 0, &n_cand);
  if (n_cand != n_cand_local) {  // only a bad block id can make a candidate unreadable
    if (tid == 0) sp_abort(p, sm, HHR_ERR_BAD_BLOCK);
    __syncthreads();
    ok = false;
    return 0;
  }
  if (keff > 0 && before < keff && before + local >= keff) {
    int run = before;
#pragma unroll
    for (int e = 0; e < 5; ++e) {
      if (run < keff && run + hv[e] >= keff) {
        bc[0] = tid * bpt + e;
        bc[1] = keff - run;
      }
      run += hv[e];
    }
  }
  __syncthreads();
  const int T = bc[0], need_eq = bc[1];
  // rows below T and at T of the CTAs before r (warp w: CTAs w, w + 16, ...)
  int lt_before = 0, eq_before = 0;
  {
    int* acc = reinterpret_cast<int*>(sm + SP_HISTS + S * HB * 4 + 2 * ((nmy + 15) & ~15));  // [2][32]
    if (tid < 64) acc[tid] = 0;
    __syncthreads();
    for (int rr = warp; rr < r; rr += SP_WARPS) {
      int c = 0;
      for (int bb = lane; bb < T; bb += 32) c += hists[rr * HB + bb];
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
      if (lane == 0) {
        atomicAdd(&acc[0], c);
        atomicAdd(&acc[1], T >= 0 ? hists[rr * HB + T] : 0);
      }
    }
    __syncthreads();
    lt_before = acc[0];
    eq_before = acc[1];
  }
  const int off = lt_before + min(need_eq, eq_before);  // the CTA's first place in the list
  const int take = max(0, need_eq - eq_before);         // ties it may take
  if (r == 0 && tid == 0) {
    if (p.dbg.n_cand) p.dbg.n_cand[x.u] = n_cand;
    if (p.dbg.n_sel_keys) p.dbg.n_sel_keys[x.u] = keff;
  }
  // ---- kept rows in candidate order: thread t owns candidates [t m, (t+1) m) ----
  const int m = (nmy + SP_THREADS - 1) / SP_THREADS;
  const int j0 = tid * m, j1 = min(nmy, j0 + m);
  int lt_t = 0, eq_t = 0;
  for (int j = j0; j < j1; ++j) {
    const int sv = sc[j];
    lt_t += sv < T;
    eq_t += sv == T;
  }
  int tot2;
  const int pk = block_scan_excl((lt_t << 16) | eq_t, red, 1, &tot2);
  int lt_run = pk >> 16, eq_run = pk & 0xFFFF;
  const int room = keff - off;
  int* list = wk.sel_keys + (long long)x.u * wk.Kmax + off;
  int* dout = p.dbg.sel_keys ? p.dbg.sel_keys + (long long)x.u * wk.Kmax + off : nullptr;
  for (int j = j0; j < j1; ++j) {
    const int sv = sc[j];
    const bool l1 = sv < T, e1 = sv == T;
    if (l1 || (e1 && eq_run < take)) {
      const int pos = lt_run + min(eq_run, take);
      if (pos < room) {
        const int ci = cs0 + j;
        const int t = (kp[ci >> dm.lgP] << dm.lgP) + (ci & (dm.P - 1));
        if (!all_kept) list[pos] = t + 1;
        if (dout) dout[pos] = t;
      }
    }
    lt_run += l1;
    eq_run += e1;
  }
  return keff;
}

// ---------------------------------------------------------------------------
// final merge of a unit's chunk partials (the last CTA of the group)
// ---------------------------------------------------------------------------
// out[h][c] = sum_k w_k o_k[h][c] / sum_k w_k L_k[h], w_k = 2^(M_k[h] - M[h]),
// M[h] = max_k M_k[h]; every sum in chunk order.  The partials are copied to
// shared memory in passes (region A is free by now).
template <int G>
__device__ void sp_merge(const SpParams& p, unsigned char* sm, const SpUnit& x, int nch) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int PS = G * D + 16;
  const float* pt = p.wk.part + (long long)x.u * p.wk.C3 * PS;
  float* wbuf = reinterpret_cast<float*>(sm + SP_OB);  // [nch][8] chunk weights (nch <= 256)
  float* inv = reinterpret_cast<float*>(sm + SP_LS);   // [8] 1 / total weight
  // weights: warp h < G
  if (warp < G) {
    float M = -INFINITY;
    for (int k = lane; k < nch; k += 32) M = fmaxf(M, __ldcg(pt + (long long)k * PS + G * D + warp));
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    // sum of w_k L_k in chunk order: lanes take consecutive chunks, then a fixed tree
    float part_l = 0.f;
    for (int k0 = 0; k0 < nch; k0 += 32) {
      const int k = k0 + lane;
      float wl = 0.f;
      if (k < nch) {
        const float w = exp2f(__ldcg(pt + (long long)k * PS + G * D + warp) - M);
        wbuf[k * 8 + warp] = w;
        wl = w * __ldcg(pt + (long long)k * PS + G * D + 8 + warp);
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) wl += __shfl_xor_sync(0xffffffffu, wl, o);
      part_l += wl;
    }
    if (lane == 0) inv[warp] = 1.f / part_l;
  }
  // the partials, in passes of as many chunks as region A holds
  const int per = SP_A_BYTES / (PS * 4);
  float acc0 = 0.f, acc1 = 0.f;  // elements tid and tid + 512 (G * 128 <= 1024)
  float* sp = reinterpret_cast<float*>(sm);
  for (int k0 = 0; k0 < nch; k0 += per) {
    const int nk = min(per, nch - k0);
    const int n16 = nk * PS / 4;
    for (int i = tid; i < n16; i += SP_THREADS) cp_async16(sp + 4 * i, pt + (long long)k0 * PS + 4 * i);
    cp_async_commit();
    cp_async_wait_all();
    __syncthreads();
    for (int k = 0; k < nk; ++k) {
      const float* pk = sp + k * PS;
      if (tid < G * D) acc0 = fmaf(wbuf[(k0 + k) * 8 + (tid >> 7)], pk[tid], acc0);
      if (tid + SP_THREADS < G * D) acc1 = fmaf(wbuf[(k0 + k) * 8 + ((tid + SP_THREADS) >> 7)], pk[tid + SP_THREADS], acc1);
    }
    __syncthreads();
  }
  float* o = p.out + ((long long)x.b * p.dm.Hq + x.h * G) * D;
  if (tid < G * D) o[tid] = acc0 * inv[tid >> 7];
  if (tid + SP_THREADS < G * D) o[tid + SP_THREADS] = acc1 * inv[(tid + SP_THREADS) >> 7];
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------
template <int G, int WORDS>
__global__ void __launch_bounds__(SP_THREADS, 1) hhr_sparse_kernel(const __grid_constant__ SpParams p) {
  extern __shared__ __align__(128) unsigned char sm[];
  const Dims& dm = p.dm;
  const Work& wk = p.wk;
  const int tid = threadIdx.x;
  const int S = p.gsize;
  const int grp = blockIdx.x / S, r = blockIdx.x - grp * S;
  const int Units = dm.B * dm.Hkv;
  if (tid < 32) reinterpret_cast<volatile int*>(sm + SP_MISC)[tid] = 0;
  // weights of the first unit: read before the previous kernel on the stream
  // has finished (they are never written by a decode step)
  Prep<G> pr;
  if (grp < Units) sp_prep_load<G>(p, grp % dm.Hkv, pr);
  pdl_launch_dependents();
  pdl_wait();
  __syncthreads();
  bool first = true;
  for (int u = grp; u < Units; u += p.ngroups) {
    SpUnit x;
    x.u = u;
    x.b = u / dm.Hkv;
    x.h = u - x.b * dm.Hkv;
    x.L = seq_len_of(dm, p.seq_lens, x.b);
    x.np = (x.L + dm.P - 1) >> dm.lgP;
    unsigned* gx = wk.gx + (long long)u * wk.gx_stride;
    unsigned epoch = 0;
    const int nk_b = __ldg(p.n_keep + x.b), tk_b = __ldg(p.top_k + x.b);
    if (!first) sp_prep_load<G>(p, x.h, pr);
    first = false;
    // ---- metadata copies of the first stages, then the prep ----
    int p0, p1;
    share_of(x.np, S, r, p0, p1);
    const int nsteps = (p1 - p0 + SP_STAGE_PAGES - 1) / SP_STAGE_PAGES;
#pragma unroll 1
    for (int s = 0; s < SP_NST - 1; ++s) {
      if (s < nsteps) sp_issue_meta(p, sm + s * SP_META_STAGE, x, p0 + s * SP_STAGE_PAGES, p1);
      cp_async_commit();
    }
    sp_prep<G>(p, sm, x, pr, r == 0);
    if (x.L == 0) {  // empty sequence: zero output, no barrier (every CTA of the group skips alike)
      cp_async_wait_all();
      if (r == 0) {
        for (int e = tid; e < G * D; e += SP_THREADS) p.out[((long long)x.b * dm.Hq + x.h * G) * D + e] = 0.f;
        if (tid == 0) {
          if (p.dbg.n_sel_pages) p.dbg.n_sel_pages[x.u] = 0;
          if (p.dbg.n_sel_keys) p.dbg.n_sel_keys[x.u] = 0;
          if (p.dbg.n_cand) p.dbg.n_cand[x.u] = 0;
        }
      }
      __syncthreads();
      continue;
    }
    // ---- scan ----
    {
      float2 qa[G][4], qbn[G][4];
      const float* qs = reinterpret_cast<const float*>(sm + SP_PREP + 4096);
      const int li = tid & 15;
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 t = *reinterpret_cast<const float2*>(qs + g * D + 8 * li + 2 * k);
          if constexpr (G <= 4) {
            qa[g][k] = make_float2(fmaxf(t.x, 0.f), fmaxf(t.y, 0.f));
            qbn[g][k] = make_float2(fminf(t.x, 0.f), fminf(t.y, 0.f));
          } else {
            qa[g][k] = t;
            qbn[g][k] = t;
          }
        }
      __syncthreads();  // (qs is read; SP_PREP is free for the page select)
#pragma unroll 1
      for (int s = 0; s < nsteps; ++s) {
        const int sn = s + SP_NST - 1;
        if (sn < nsteps) sp_issue_meta(p, sm + (sn % SP_NST) * SP_META_STAGE, x, p0 + sn * SP_STAGE_PAGES, p1);
        cp_async_commit();
        cp_async_wait<SP_NST - 1>();
        sp_scan_stage<G>(p, sm + (s % SP_NST) * SP_META_STAGE, x, p0 + s * SP_STAGE_PAGES, p1, qa, qbn);
      }
      cp_async_wait_all();
    }
    // ---- the unit's bounds are complete ----
    if (!sp_group_sync(p, sm, gx, epoch)) break;
    const int N = min(min(max(nk_b, 1), wk.Nmax), x.np);
    const int nkp = sp_psel(p, sm, x, N, r == 0);
    // candidates: the valid rows of the kept pages (only the last page can be partial)
    const int* kp = reinterpret_cast<const int*>(sm + SP_KP);
    int n_cand = nkp << dm.lgP;
    if (nkp > 0 && kp[nkp - 1] == x.np - 1) n_cand -= (x.np << dm.lgP) - x.L;
    const int keff = min(min(max(tk_b, 1), wk.Kmax), n_cand);
    const bool all_kept = keff == n_cand;
    const int nch = (keff + SP_ROWS - 1) / SP_ROWS;
    int c0, c1;
    share_of(nch, S, r, c0, c1);
    if (all_kept) {  // the chunks' rows are known now: their copies start at once
      sp_issue_chunk(p, sm, x, c0, c0, c1, keff, true);
      sp_issue_chunk(p, sm, x, c0 + 1, c0, c1, keff, true);
    }
    bool ok = true;
    sp_keys<G, WORDS>(p, sm, x, r, nkp, n_cand, keff, all_kept, gx, epoch, ok);
    if (!ok) break;
    if (!all_kept) {
      sp_issue_chunk(p, sm, x, c0, c0, c1, keff, false);
      sp_issue_chunk(p, sm, x, c0 + 1, c0, c1, keff, false);
    }
    sp_issue_chunk(p, sm, x, c0 + 2, c0, c1, keff, all_kept);
    // ---- gather: three chunks in flight ----
    const int PS = G * D + 16;
    float* parts = wk.part + (long long)x.u * wk.C3 * PS;
#pragma unroll 1
    for (int c = c0; c < c1; ++c) {
      cp_async_wait<SP_NGS - 1>();
      __syncthreads();
      if (sp_aborted(sm)) break;
      sp_gather_step<G>(sm, sm + ((c - c0) % SP_NGS) * SP_GSTAGE, min(SP_ROWS, keff - c * SP_ROWS),
                        parts + (long long)c * PS);
      sp_issue_chunk(p, sm, x, c + SP_NGS, c0, c1, keff, all_kept);
    }
    cp_async_wait_all();
    __syncthreads();
    if (sp_aborted(sm)) break;
    // ---- the last CTA of the group merges ----
    if (tid == 0) {
      int last = 1;
      if (S > 1) last = atom_add_acq_rel(gx + GX_ARRIVE, 1u) == (unsigned)(S - 1);
      reinterpret_cast<volatile int*>(sm + SP_MISC)[MS_LAST] = last;
    }
    __syncthreads();
    if (reinterpret_cast<volatile int*>(sm + SP_MISC)[MS_LAST]) {
      sp_merge<G>(p, sm, x, nch);
      if (tid == 0) {
        gx[GX_BAR] = 0u;
        gx[GX_ARRIVE] = 0u;
      }
    }
    __syncthreads();
  }
  cp_async_wait_all();
}

// CTAs per group: the SMs shared out over the units, at most one CTA per 64
// pages of the longest sequence, and no more than the key select's scratch
// holds score histograms and scores of.
inline void sparse_group_shape(const Dims& dm, int sms, int Cmax, int HB, int* S, int* ngroups) {
  const int U = dm.B * dm.Hkv;
  sms = std::max(1, std::min(sms, MAX_GRID));
  int s = std::max(1, sms / U);
  s = std::min(s, std::max(1, dm.np_max / 64));
  while (s > 1 && (long long)s * HB * 4 + 2 * (((Cmax + s - 1) / s + 15) & ~15) + 256 > SP_A_BYTES - SP_HISTS) --s;
  *S = s;
  *ngroups = std::max(1, std::min(U, sms / s));
}

}  // namespace hhr
