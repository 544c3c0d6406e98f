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
//   1. starts the first two of its 64-page metadata stages (pages [p0, p1);
//      TMA bulk copies completing on one mbarrier per stage, five stages in
//      flight) and copies the query heads, then computes q' = R_h q and the
//      query sign codes on tensor cores (R_h and W_h of the first unit are
//      copied to shared memory before the previous kernel on the stream has
//      finished: programmatic dependent launch);
//   2. scans its pages: U = the page bound aggregated over the group's query
//      heads (max, or sum); a stage's slot is refilled once every thread is
//      done with it, and every wait on a stage's barrier is bounded;
//   3. group barrier; the page top-N on ALL the unit's bounds (read from
//      L2), the same in every CTA: order-preserving keys in registers, a level
//      over the keys' range, then the threshold bin's members refined 11 bits
//      at a time; equal keys are taken in page order (ties go to the lower
//      page);
//   4. when the key budget covers every candidate row, starts copying the K'/V
//      rows of its gather share right away; scores its balanced share of the
//      candidate rows (Hamming distance over the group's heads, summed or
//      minimised), adds its score histogram into the unit's and publishes
//      its cumulative form;
//   5. group barrier; the unit's histogram gives the threshold score T and the
//      ties taken at T (lower rows first); the CTA lists the kept rows of its
//      own scoring share, which it then gathers (with every candidate kept,
//      its balanced share of all candidates instead);
//   6. eight warps gather 16-row K'/V tiles (cp.async, XOR-swizzled rows, a
//      ring of three per warp) and run an online softmax on tensor cores
//      (mma.sync: logits with q' as bf16 hi + lo, P.V with P as bf16 hi + lo);
//      their partials are combined in warp order into the CTA's partial;
//   7. the last CTA of the group to arrive merges the S partials in CTA order
//      into the output and resets the unit's counters.
// Every order is fixed by the launch shape, so results are deterministic for
// a given S (they do not depend on the batch or on the cache layout).
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

// shared memory map (bytes).  Region A is reused by every phase:
//   prep     metadata stages 0-1 [0, 64K), R_h fp32 [64K, 128K), W_h bf16 [128K, 192K)
//   scan     five metadata stages [0, 160K)
//   psel     two refinement lists [0, 128K), histogram [128K, 136K), kept-page bitmap [136K, 137K)
//   keys     tile slots 0-1 of the gathering warps [0, 128K) (copies started early when every
//            candidate is kept), the CTA's score histogram and scores [128K, 192K)
//   gather   the warps' tile rings [0, 192K);  combine, merge: partials
constexpr int SP_A_BYTES = 192 * 1024;                        // region A
constexpr int SP_RS = 2 * SP_META_STAGE;                      // R_h during the prep (64 KB)
constexpr int SP_WS = SP_RS + D * D * 4;                      // W_h during the prep (<= 64 KB)
constexpr int SP_PLIST = MAX_SELECT_PAGES * 8;              // page select: one refinement list (keys, pages)
constexpr int SP_PSH = 2 * SP_PLIST;                          // int [2048] page-select histogram
constexpr int SP_BITS = SP_PSH + 2048 * 4;                    // u32 [256] kept-page bitmap
constexpr int SP_HISTS = 128 * 1024;                          // key select: the CTA's score histogram, then scores
constexpr int SP_QB = SP_A_BYTES;                             // bf16 [16][136] q' operand (hi, lo)
constexpr int SP_KLCAP = MAX_KEPT_PER_CTA;                    // kept rows a CTA gathers at most (see sparse_group_shape)
constexpr int SP_OB = SP_QB + 16 * 272;                       // prep: q, q' (fp32 [2][8][128]); keys/gather: kept list
                                                              // (u16 [SP_KLCAP]); merge: weights
constexpr int SP_LS = SP_OB + 2 * SP_KLCAP;                   // float [8] merge: 1 / total weight
constexpr int SP_KP = SP_LS + 256;                            // int [MAX_KEEP_PAGES] kept pages
constexpr int SP_QC = SP_KP + MAX_KEEP_PAGES * 4;             // u32 [8 heads][8] query codes
constexpr int SP_RED = SP_QC + 256;                           // int: [0,64) scans, [64,128) min/max, [128,160) broadcasts
constexpr int SP_MISC = SP_RED + 640;                         // int [16] flags
constexpr int SP_MBAR = SP_MISC + 64;                         // u64 [8] barriers of the metadata stages
constexpr int SP_SMEM = SP_MISC + 128;
static_assert(2 * SP_KLCAP >= 8192, "q and q' of the prep, merge weights");
static_assert(SP_SMEM <= 232448, "shared memory of the decode kernel");
static_assert(SP_WS + 256 * D * 2 <= SP_A_BYTES, "prep scratch");
static_assert(SP_BITS + 256 * 4 <= SP_A_BYTES, "page-select scratch");

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
// coherent).  A release add and a bounded acquire poll on the unit's counter,
// by the first thread of the CTA's participating warps (the whole CTA, or the
// warp group of named barrier `bar`).  False after a timeout or an abort
// (every participating thread sees the same).
__device__ __forceinline__ bool sp_group_sync(const SpParams& p, unsigned char* sm, unsigned* gx, unsigned& epoch,
                                              int tb = 0, int nthr = SP_THREADS, int bar = 0) {
  bar_sync(bar, nthr);
  if (p.gsize > 1) {
    epoch += (unsigned)p.gsize;
    if (threadIdx.x == tb) {
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
    bar_sync(bar, nthr);
  }
  return !sp_aborted(sm);
}

// ---------------------------------------------------------------------------
// prep: q' = R_h q and the query codes
// ---------------------------------------------------------------------------
// R_h (fp32) and W_h (bf16) are staged in shared memory with cp.async, their
// 16-byte pieces XOR-swizzled by row (piece c of row i at c ^ (i mod 32) for
// R, c ^ (i mod 16) for W) so that the fragment reads of a warp hit distinct
// banks.  They are weights, never written by a decode step: the first unit's
// are copied before the previous kernel on the stream has finished.  One
// commit group.
static __device__ __noinline__ void sp_issue_rw(const SpParams& p, unsigned char* sm, int h) {
  const float* Rh = p.R + (long long)h * D * D;
  #pragma unroll 1
  for (int q = threadIdx.x; q < D * 32; q += blockDim.x) {  // R: 128 rows x 32 pieces
    const int i = q >> 5, c = q & 31;
    cp_async16(sm + SP_RS + i * 512 + ((c ^ (i & 31)) * 16), Rh + i * D + c * 4);
  }
  const __nv_bfloat16* Wh = p.W + (long long)h * p.dm.nb * D;
  #pragma unroll 1
  for (int q = threadIdx.x; q < p.dm.nb * 16; q += blockDim.x) {  // W: nb rows x 16 pieces
    const int j = q >> 4, c = q & 15;
    cp_async16(sm + SP_WS + j * 256 + ((c ^ (j & 15)) * 16), Wh + j * D + c * 8);
  }
  cp_async_commit();
}

// Copies the unit's query heads (bf16, G rows of 256 bytes) to rows 0..G-1 of
// the [8][136] bf16 buffer at SP_OB (rows G..7 are zeroed by the caller).
// One commit group.
static __device__ __noinline__ void sp_issue_q(const SpParams& p, unsigned char* sm, const SpUnit& x, int G) {
  const int tid = threadIdx.x;
  if (tid < G * 16) {
    const int g = tid >> 4, c = tid & 15;
    cp_async16(sm + SP_OB + g * 272 + c * 16, p.q + ((long long)x.b * p.dm.Hq + x.h * G + g) * D + c * 8);
  }
  cp_async_commit();
}

// On tensor cores (mma.sync m16n8k16, bf16 in, fp32 accumulate), with the
// query heads as the 8 columns of B (q is bf16: exact; heads >= G are zero):
//   warps 0-7   q' = R_h q, rows 16w .. 16w+15: R_h as bf16 hi + lo (two
//               products into one accumulator; |R - hi - lo| <= 2^-17 |R|).
//               q' goes to qs (fp32 [8][128] at SP_OB + 4096) and the Q
//               operand of the logits (q' * sm_scale * log2 e as bf16 hi in
//               row g and lo in row 8 + g of SP_QB);
//   warps 8-15  the query codes: bit j of head g is [(W_h q_g)_j > 0] for bit
//               tiles m = w - 8 and w (rows 16 m .. +15, while < nb / 16); the
//               products are exact and the fp32 sum is trusted when |sum| >
//               2^-14 sum|w q| (a second product, of the magnitudes), else the
//               sign comes from fp64.
// The caller has issued sp_issue_rw and sp_issue_q (cp.async).
template <int G>
__device__ void sp_prep(const SpParams& p, unsigned char* sm, const SpUnit& x, bool write_dbg) {
  const Dims& dm = p.dm;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g = lane >> 2, t = lane & 3;
  float* qs = reinterpret_cast<float*>(sm + SP_OB + 4096);
  unsigned* qc = reinterpret_cast<unsigned*>(sm + SP_QC);
  // B fragments q[g][16 ks + 2t, +1] and q[g][16 ks + 8 + 2t, +1]
  const uint32_t* qrow = reinterpret_cast<const uint32_t*>(sm + SP_OB + g * 272) + t;
  if (tid < 64) qc[tid] = 0u;
  cp_async_wait_all();  // R, W and q
  __syncthreads();
  if (warp < 8) {
    const int i0 = 16 * warp + g, i1 = i0 + 8;  // the lane's two rows of R_h
    const unsigned char* R0 = sm + SP_RS + i0 * 512;
    const unsigned char* R1 = sm + SP_RS + i1 * 512;
    float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 2
    for (int ks = 0; ks < 8; ++ks) {
      // A: R[i][16 ks + 2t, +1] and R[i][16 ks + 8 + 2t, +1] (piece 4 ks + t/2, +2; swizzled)
      const int pa = 4 * ks + (t >> 1), off = 8 * (t & 1);
      const float2 rr[4] = {*reinterpret_cast<const float2*>(R0 + ((pa ^ (i0 & 31)) * 16) + off),
                            *reinterpret_cast<const float2*>(R1 + ((pa ^ (i1 & 31)) * 16) + off),
                            *reinterpret_cast<const float2*>(R0 + (((pa + 2) ^ (i0 & 31)) * 16) + off),
                            *reinterpret_cast<const float2*>(R1 + (((pa + 2) ^ (i1 & 31)) * 16) + off)};
      uint32_t ah[4], al[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(rr[e].x, rr[e].y);
        const float2 hf = __bfloat1622float2(h);
        const __nv_bfloat162 l = __floats2bfloat162_rn(rr[e].x - hf.x, rr[e].y - hf.y);
        ah[e] = *reinterpret_cast<const uint32_t*>(&h);
        al[e] = *reinterpret_cast<const uint32_t*>(&l);
      }
      const uint32_t b[2] = {qrow[8 * ks], qrow[8 * ks + 4]};
      mma_bf16(c, ah, b);
      mma_bf16(c, al, b);
    }
    // c0, c1: q'[2t][i0], q'[2t+1][i0]; c2, c3: the same at i1
    const float qscale = p.sm_scale * 1.4426950408889634f;
    __nv_bfloat16* qo = reinterpret_cast<__nv_bfloat16*>(sm + SP_QB);
    float* dq = (write_dbg && p.dbg.q_rot) ? p.dbg.q_rot + ((long long)x.b * dm.Hq + x.h * G) * D : nullptr;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int n = 2 * t + (e & 1), i = (e < 2) ? i0 : i1;
      const float v = n < G ? c[e] : 0.f;
      qs[n * D + i] = v;
      __nv_bfloat16 hi, lo;
      split_bf16(v * qscale, hi, lo);
      qo[n * 136 + i] = hi;
      qo[(8 + n) * 136 + i] = lo;
      if (dq && n < G) dq[n * D + i] = v;
    }
  } else {
#pragma unroll 1
    for (int m = warp - 8; m < (dm.nb >> 4); m += 8) {
      float cs[4] = {0.f, 0.f, 0.f, 0.f}, cm[4] = {0.f, 0.f, 0.f, 0.f};
      const int j = 16 * m + (lane & 15);  // the ldmatrix row of this lane
      const unsigned char* Wj = sm + SP_WS + j * 256;
#pragma unroll 2
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t a[4];
        ldsm_x4(a, Wj + (((2 * ks + (lane >> 4)) ^ (j & 15)) * 16));
        const uint32_t am[4] = {a[0] & 0x7fff7fffu, a[1] & 0x7fff7fffu, a[2] & 0x7fff7fffu, a[3] & 0x7fff7fffu};
        const uint32_t b[2] = {qrow[8 * ks], qrow[8 * ks + 4]};
        const uint32_t bm[2] = {b[0] & 0x7fff7fffu, b[1] & 0x7fff7fffu};
        mma_bf16(cs, a, b);
        mma_bf16(cm, am, bm);
      }
      // cs[e]: bit row jj = 16 m + g (+8 for e >= 2), head n = 2t + (e & 1).
      // A sum too close to zero for fp32 is recomputed by the whole warp in
      // fp64, one flagged (bit, head) at a time (the products are exact, so the
      // sign is exact up to fp64 rounding of the sum).
      unsigned bits = 0u, flag = 0u;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        bits |= (unsigned)(cs[e] > 0.f) << e;
        if (2 * t + (e & 1) < G && fabsf(cs[e]) <= ldexpf(cm[e], -14)) flag |= 1u << e;
      }
      unsigned lanes = __ballot_sync(0xffffffffu, flag != 0u);
      while (lanes) {
        const int src = __ffs(lanes) - 1;
        lanes &= lanes - 1u;
        unsigned fe = __shfl_sync(0xffffffffu, flag, src);
        while (fe) {
          const int e = __ffs(fe) - 1;
          fe &= fe - 1u;
          const int jf = 16 * m + (src >> 2) + (e >= 2 ? 8 : 0), nf = 2 * (src & 3) + (e & 1);
          const unsigned char* Wr = sm + SP_WS + jf * 256;
          const __nv_bfloat16* qr = reinterpret_cast<const __nv_bfloat16*>(sm + SP_OB + nf * 272);
          double ad = 0.0;
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            const int cc = lane + 32 * c4;
            const int pc = ((cc >> 3) ^ (jf & 15)) * 8 + (cc & 7);
            ad += (double)__bfloat162float(reinterpret_cast<const __nv_bfloat16*>(Wr)[pc]) *
                  (double)__bfloat162float(qr[cc]);
          }
#pragma unroll
          for (int o = 16; o >= 1; o >>= 1) ad += __shfl_xor_sync(0xffffffffu, ad, o);
          if (lane == src) bits = (bits & ~(1u << e)) | ((unsigned)(ad > 0.0) << e);
        }
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int n = 2 * t + (e & 1), jj = 16 * m + g + (e >= 2 ? 8 : 0);
        if (n < G && ((bits >> e) & 1u)) atomicOr(&qc[n * 8 + (jj >> 5)], 1u << (jj & 31));
      }
    }
  }
  fence_proxy_async();  // (R_h and W_h's room is refilled by TMA copies next)
  __syncthreads();
  if (write_dbg && p.dbg.q_codes) {
    const int w32 = dm.words * 2;
    if (tid < G * w32) {
      const int gg = tid / w32, k = tid - gg * w32;
      reinterpret_cast<uint32_t*>(p.dbg.q_codes)[((long long)x.b * dm.Hq + x.h * G + gg) * w32 + k] = qc[gg * 8 + k];
    }
  }
}

// ---------------------------------------------------------------------------
// scan: page bounds of the CTA's pages
// ---------------------------------------------------------------------------
// Stage s holds pages p0 + 64 s + j (j < 64, clipped to p1): minima rows at
// j*256, maxima at 64*256 + j*256, copied by TMA bulk copies that complete on
// the stage's barrier: two copies of n rows (contiguous cache; thread 0), or
// one 256-byte copy per row (paged cache; threads 0..2n-1; a bad block id
// copies row 0 of the pool instead and is recorded in the status).  Thread 0
// arms the barrier with the stage's byte count.  Thread t later reads the
// 16-byte piece (t & 15) (channels 8(t&15) .. +7) of pages j = t/16 and
// j = t/16 + 32, minima and maxima.
static __device__ __noinline__ void sp_issue_meta(const SpParams& p, unsigned char* stage, uint64_t* bar,
                                                  const SpUnit& x, int pg0, int p1) {
  const int tid = threadIdx.x;
  const int n = min(SP_STAGE_PAGES, p1 - pg0);  // >= 1
  if (tid == 0) mbar_arrive_expect_tx(bar, 2u * n * 256u);
  if (!p.dm.paged) {
    if (tid == 0) {
      const long long off = meta_row(p.dm, p.table, x.b, x.h, pg0, p.status);
      bulk_g2s(stage, p.pmin + off, n * 256, bar);
      bulk_g2s(stage + SP_STAGE_PAGES * 256, p.pmax + off, n * 256, bar);
    }
  } else if (tid < 2 * n) {
    const int j = tid >> 1, mx = tid & 1;
    const long long off = meta_row(p.dm, p.table, x.b, x.h, pg0 + j, p.status);
    bulk_g2s(stage + mx * SP_STAGE_PAGES * 256 + j * 256, (mx ? p.pmax : p.pmin) + (off >= 0 ? off : 0), 256, bar);
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
// Every CTA of the group runs the same select on the unit's bounds (read
// from L2), so all of them know every kept page without another exchange.
// Bounds become order-preserving keys (a larger bound gives a larger key; -0
// folds into +0).  Thread t holds the keys of pages [16t, 16t + 16) in
// registers (np <= 8192).  Level 0 bins them by (key - min) >> shift into at
// most 2048 bins (shift from the keys' range), keeps every page above the bin
// holding the N-th largest and, unless that bin is kept whole or holds one key
// value, moves its members (in page order) to a list in shared memory, where
// each further level resolves 11 more bits the same way.  A bin of one key
// value is taken in page order (ties go to the lower page).  Writes the kept
// pages (ascending) to SP_KP; returns their count.

// One refinement level over the list at `lst` (cnt keys, then pages, in page
// order), binned by (key - base) >> shift; marks the kept pages in `keep`.
// Returns the number of bin members moved (in order) to `nxt` for the next
// level, 0 when the select is complete.
static __device__ __noinline__ int psel_level(unsigned char* sm, const unsigned char* lst, unsigned char* nxt, int cnt,
                                              int& need, unsigned& base, int& shift, int par) {
  const int tid = threadIdx.x;
  int* red = reinterpret_cast<int*>(sm + SP_RED);
  int* bc = red + 128;
  int* hist = reinterpret_cast<int*>(sm + SP_PSH);
  unsigned* keep = reinterpret_cast<unsigned*>(sm + SP_BITS);
  const uint32_t* lk = reinterpret_cast<const uint32_t*>(lst);
  const int* lp = reinterpret_cast<const int*>(lst + SP_PLIST / 2);
  // thread t: list elements [t c, t c + c)
  const int c = (cnt + SP_THREADS - 1) / SP_THREADS;
  const int e0 = min(cnt, tid * c), e1 = min(cnt, e0 + c);
  #pragma unroll 1
  for (int e = e0; e < e1; ++e) atomicAdd(&hist[(lk[e] - base) >> shift], 1);
  __syncthreads();
  int hv[4], c4 = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    hv[q] = hist[2047 - 4 * tid - q];
    c4 += hv[q];
  }
  int tot;
  const int before = block_scan_excl(c4, red, par, &tot);
  if (before < need && before + c4 >= need) {
    int run = before;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (run < need && run + hv[q] >= need) {
        bc[0] = 2047 - 4 * tid - q;
        bc[1] = need - run;
        bc[2] = hv[q];
      }
      run += hv[q];
    }
  }
  __syncthreads();
  const int bstar = bc[0], need_in = bc[1], cnt_in = bc[2];
  #pragma unroll 1
  for (int i = tid; i < 512; i += SP_THREADS) hist[4 * i] = hist[4 * i + 1] = hist[4 * i + 2] = hist[4 * i + 3] = 0;
  // members above the bin are kept; the bin's members are counted per thread
  int nb = 0;
  #pragma unroll 1
  for (int e = e0; e < e1; ++e) {
    const int bn = (int)((lk[e] - base) >> shift);
    if (bn > bstar) atomicOr(&keep[lp[e] >> 5], 1u << (lp[e] & 31));
    nb += bn == bstar;
  }
  const bool whole = cnt_in == need_in, ties = shift == 0;
  int nt;
  const int pre = block_scan_excl(nb, red, par + 1, &nt);  // (its barrier also orders the clears above)
  int* nk = reinterpret_cast<int*>(nxt);
  int* np2 = reinterpret_cast<int*>(nxt + SP_PLIST / 2);
  int q = pre;
  #pragma unroll 1
  for (int e = e0; e < e1; ++e) {
    if ((int)((lk[e] - base) >> shift) != bstar) continue;
    if (whole || (ties && q < need_in)) {
      atomicOr(&keep[lp[e] >> 5], 1u << (lp[e] & 31));
    } else if (!ties) {
      nk[q] = lk[e];
      np2[q] = lp[e];
    }
    ++q;
  }
  __syncthreads();
  if (whole || ties) return 0;
  need = need_in;
  base += (unsigned)bstar << shift;
  shift = shift > 11 ? shift - 11 : 0;
  return cnt_in;
}

static __device__ __noinline__ int sp_psel(const SpParams& p, unsigned char* sm, const SpUnit& x, int N, bool write_dbg) {
  const int tid = threadIdx.x;
  int* kp = reinterpret_cast<int*>(sm + SP_KP);
  int* red = reinterpret_cast<int*>(sm + SP_RED);
  int* bc = red + 128;
  int* hist = reinterpret_cast<int*>(sm + SP_PSH);
  unsigned* keep = reinterpret_cast<unsigned*>(sm + SP_BITS);
  const int np = x.np, i0 = tid * 16;
  const int nv = min(16, max(0, np - i0));  // the thread's pages
  unsigned sel = 0u;                        // bit e: page i0 + e is kept
  int par = 0;
  if (N >= np) {
    sel = nv >= 16 ? 0xffffu : ((1u << nv) - 1u);
  } else {
    // the thread's 16 bounds: four 16-byte loads, all in flight at once (a U
    // row is padded to a multiple of 32 pages, so they stay inside it)
    uint32_t k[16];
    {
      const float4* Ug = reinterpret_cast<const float4*>(p.wk.U + (long long)x.u * p.wk.Ustride + i0);
      float4 v[4];
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4) v[k4] = i0 + 4 * k4 < np ? __ldcg(Ug + k4) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4) {
        k[4 * k4] = order_key(v[k4].x);
        k[4 * k4 + 1] = order_key(v[k4].y);
        k[4 * k4 + 2] = order_key(v[k4].z);
        k[4 * k4 + 3] = order_key(v[k4].w);
      }
    }
    unsigned lo = 0xffffffffu, hi = 0u;
#pragma unroll
    for (int e = 0; e < 16; ++e)
      if (e < nv) {
        lo = min(lo, k[e]);
        hi = max(hi, k[e]);
      }
    reinterpret_cast<int4*>(hist)[tid] = make_int4(0, 0, 0, 0);  // 2048 bins
    if (tid < 256) keep[tid] = 0u;
    block_minmax_u32(lo, hi, reinterpret_cast<unsigned*>(red + 64));  // (its barrier orders the clears)
    unsigned base = lo;
    const unsigned width = hi - lo;
    int shift = width < 2048u ? 0 : (32 - __clz(width)) - 11;
#pragma unroll
    for (int e = 0; e < 16; ++e)
      if (e < nv) atomicAdd(&hist[(k[e] - base) >> shift], 1);
    __syncthreads();
    int hv[4], c4 = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      hv[q] = hist[2047 - 4 * tid - q];
      c4 += hv[q];
    }
    int tot;
    const int before = block_scan_excl(c4, red, par++, &tot);
    if (before < N && before + c4 >= N) {
      int run = before;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (run < N && run + hv[q] >= N) {
          bc[0] = 2047 - 4 * tid - q;
          bc[1] = N - run;
          bc[2] = hv[q];
        }
        run += hv[q];
      }
    }
    __syncthreads();
    const int bstar = bc[0], need_in = bc[1], cnt_in = bc[2];
    reinterpret_cast<int4*>(hist)[tid] = make_int4(0, 0, 0, 0);
    unsigned at = 0u;
#pragma unroll
    for (int e = 0; e < 16; ++e)
      if (e < nv) {
        const int bn = (int)((k[e] - base) >> shift);
        sel |= (unsigned)(bn > bstar) << e;
        at |= (unsigned)(bn == bstar) << e;
      }
    if (cnt_in == need_in) {
      sel |= at;
    } else {
      // the bin's members in page order: the first need_in when they are one
      // key value, else the list of the next level
      int nt;
      const int pre = block_scan_excl(__popc(at), red, par++, &nt);
      if (shift == 0) {
        int take = max(0, min(__popc(at), need_in - pre));
        unsigned t = at;
        while (take-- > 0) {
          sel |= t & (0u - t);
          t &= t - 1u;
        }
      } else {
        uint32_t* lk = reinterpret_cast<uint32_t*>(sm);
        int* lp = reinterpret_cast<int*>(sm + SP_PLIST / 2);
        int q = pre;
#pragma unroll
        for (int e = 0; e < 16; ++e)
          if ((at >> e) & 1u) {
            lk[q] = k[e];
            lp[q] = i0 + e;
            ++q;
          }
        __syncthreads();
        int need = need_in, cnt = cnt_in, lv = 0;
        base += (unsigned)bstar << shift;
        shift = shift > 11 ? shift - 11 : 0;
        #pragma unroll 1
        for (; cnt > 32; ++lv)
          cnt = psel_level(sm, sm + (lv & 1) * SP_PLIST, sm + ((lv + 1) & 1) * SP_PLIST, cnt, need, base, shift, 2 * lv + 2);
        if (cnt > 0) {
          // at most 32 members left: warp 0 ranks them directly (larger key
          // first, then lower page) and keeps the first `need`
          if (tid < 32) {
            const uint32_t* lk2 = reinterpret_cast<const uint32_t*>(sm + (lv & 1) * SP_PLIST);
            const int* lp2 = reinterpret_cast<const int*>(sm + (lv & 1) * SP_PLIST + SP_PLIST / 2);
            const bool v = tid < cnt;
            const uint32_t key = v ? lk2[tid] : 0u;
            const int pg = v ? lp2[tid] : INT_MAX;
            int rank = 0;
            #pragma unroll 1
            for (int o = 0; o < cnt; ++o) {  // (cnt is the same in every lane)
              const uint32_t k2 = __shfl_sync(0xffffffffu, key, o);
              const int p2 = __shfl_sync(0xffffffffu, pg, o);
              rank += (k2 > key || (k2 == key && p2 < pg));
            }
            if (v && rank < need) atomicOr(&keep[pg >> 5], 1u << (pg & 31));
          }
          __syncthreads();
        }
        // (the keep bitmap is complete: psel_level and the rank step end with a barrier)
        sel |= (keep[i0 >> 5] >> (i0 & 16)) & 0xffffu;
      }
    }
  }
  // kept pages in ascending order
  int nkp;
  int pos = block_scan_excl(__popc(sel), red, par & 1, &nkp);
  int* dsel = (write_dbg && p.dbg.sel_pages) ? p.dbg.sel_pages + (long long)x.u * p.wk.Nmax : nullptr;
  unsigned t = sel;
  while (t) {
    const int pg = i0 + __ffs(t) - 1;
    t &= t - 1u;
    if (pos < MAX_KEEP_PAGES) {
      kp[pos] = pg;
      if (dsel) dsel[pos] = pg;
    }
    ++pos;
  }
  if (write_dbg && tid == 0 && p.dbg.n_sel_pages) p.dbg.n_sel_pages[x.u] = nkp;
  __syncthreads();
  return nkp;
}

// ---------------------------------------------------------------------------
// attention over 16-row tiles (the gather of the decode step and the dense
// kernel): eight warps work independently, each streaming its tiles through a
// ring of three in shared memory, with its online-softmax state in registers
// ---------------------------------------------------------------------------
constexpr int TL_ROWS = 16;
constexpr int TL_BYTES = TL_ROWS * 512;  // 16 K' rows, then 16 V rows
constexpr int TL_WARPS = 8;
constexpr int TL_NBUF = 3;
static_assert(TL_NBUF * TL_WARPS * TL_BYTES == SP_A_BYTES, "tile rings fill region A");

// Slot s of warp w: the three slots of all warps are interleaved so that
// slots 0 and 1 of every warp lie in [0, 128K) and slot 2 in [128K, 192K).
__device__ __forceinline__ unsigned char* tile_slot(unsigned char* sm, int warp, int s) {
  return sm + (s * TL_WARPS + warp) * TL_BYTES;
}

// Copies one tile: lane l < 16 passes rowidx = element offset / 128 of the
// tile's row l (or -1: past the end, or a bad row, which then reads as zeros).
// Piece c of row j goes to piece c ^ (j mod 8) of its 256-byte row, so that
// eight consecutive rows' same piece fall in distinct banks for ldmatrix.
// One commit group per lane.
__device__ __forceinline__ void tile_copy(const __nv_bfloat16* K, const __nv_bfloat16* V, unsigned char* slot,
                                          int rowidx, bool live) {
  const int lane = threadIdx.x & 31;
  if (live) {
#pragma unroll 1
    for (int i = 0; i < 8; ++i) {
      const int q = lane + 32 * i, j = q >> 4, c = q & 15;
      const int ri = __shfl_sync(0xffffffffu, rowidx, j);
      const long long e = ri >= 0 ? (long long)ri * D + c * 8 : 0;
      const unsigned nbytes = ri >= 0 ? 16u : 0u;
      unsigned char* dk = slot + j * 256 + ((c ^ (j & 7)) * 16);
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dk)), "l"(K + e), "r"(nbytes)
                   : "memory");
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dk + TL_ROWS * 256)), "l"(V + e),
                   "r"(nbytes)
                   : "memory");
    }
  }
  cp_async_commit();
}

// The Q operand of the logits (all eight k-steps) from the [16][136] bf16
// layout at qb: head g's q' * sm_scale * log2 e, hi in row g, lo in row 8 + g.
__device__ __forceinline__ void load_q_operand(const unsigned char* qb, uint32_t (&aq)[8][4]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks)
    ldsm_x4(aq[ks], qb + ((lane & 7) + ((lane >> 3) & 1) * 8) * 272 + (2 * ks + (lane >> 4)) * 16);
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// One tile of `rows` (1..16) valid rows: on tensor cores (mma.sync m16n8k16,
// bf16 in, fp32 accumulate) S = Q K'^T, where the 16 rows of Q are the heads'
// hi and lo parts, so head g = lane / 4's logit is the sum of two rows held by
// the same lane; the online softmax of head g in registers; then
// O += P V, with P's hi and lo parts as the 16 rows of the A operand, built
// from the lane's own logits.  O[nt] holds channels 8 nt + 2 (lane mod 4), +1
// of head g: rows 0 (hi) and 2 (lo) of the accumulator, summed at the end.
__device__ __forceinline__ void tile_attend(const uint32_t (&aq)[8][4], float (&o)[16][4], float& m_run,
                                            float& l_run, const unsigned char* kt, int rows) {
  const int lane = threadIdx.x & 31, t = lane & 3;
  const unsigned char* vt = kt + TL_ROWS * 256;
  float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
  {
    const int krow = (lane & 7) + 8 * (lane >> 4);  // matrices 0,1: rows 0-7; 2,3: rows 8-15
    const int kp = (lane >> 3) & 1;                 // matrices 1,3: channels + 8
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      uint32_t b[4];
      ldsm_x4(b, kt + krow * 256 + (((2 * ks + kp) ^ (krow & 7)) * 16));
      const uint32_t b0[2] = {b[0], b[1]}, b1[2] = {b[2], b[3]};
      mma_bf16(s0, aq[ks], b0);
      mma_bf16(s1, aq[ks], b1);
    }
  }
  float sv[4] = {s0[0] + s0[2], s0[1] + s0[3], s1[0] + s1[2], s1[1] + s1[3]};  // rows 2t, 2t+1, 8+2t, 9+2t
  if (2 * t >= rows) sv[0] = -INFINITY;
  if (2 * t + 1 >= rows) sv[1] = -INFINITY;
  if (8 + 2 * t >= rows) sv[2] = -INFINITY;
  if (9 + 2 * t >= rows) sv[3] = -INFINITY;
  float mt = fmaxf(fmaxf(sv[0], sv[1]), fmaxf(sv[2], sv[3]));
  mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
  mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
  const float mn = fmaxf(m_run, mt);  // finite: row 0 of a tile is always valid
  const float alpha = exp2f(m_run - mn);
  float pw[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) pw[e] = exp2f(sv[e] - mn);
  l_run = l_run * alpha + ((pw[0] + pw[1]) + (pw[2] + pw[3]));
  m_run = mn;
  if (__any_sync(0xffffffffu, alpha != 1.f)) {  // (no head's maximum moved: nothing to rescale)
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      o[nt][0] *= alpha;
      o[nt][1] *= alpha;
      o[nt][2] *= alpha;
      o[nt][3] *= alpha;
    }
  }
  uint32_t ap[4];
  {
    const float h0 = __bfloat162float(__float2bfloat16_rn(pw[0])), h1 = __bfloat162float(__float2bfloat16_rn(pw[1]));
    const float h2 = __bfloat162float(__float2bfloat16_rn(pw[2])), h3 = __bfloat162float(__float2bfloat16_rn(pw[3]));
    ap[0] = pack_bf16(h0, h1);
    ap[1] = pack_bf16(pw[0] - h0, pw[1] - h1);
    ap[2] = pack_bf16(h2, h3);
    ap[3] = pack_bf16(pw[2] - h2, pw[3] - h3);
  }
  {
    const int vrow = (lane & 7) + 8 * ((lane >> 3) & 1);  // matrices 1,3: rows 8-15
    const int vp = lane >> 4;                             // matrices 2,3: channels + 8
#pragma unroll
    for (int cp = 0; cp < 8; ++cp) {
      uint32_t b[4];
      ldsm_x4_t(b, vt + vrow * 256 + (((2 * cp + vp) ^ (vrow & 7)) * 16));
      const uint32_t b0[2] = {b[0], b[1]}, b1[2] = {b[2], b[3]};
      mma_bf16(o[2 * cp], ap, b0);
      mma_bf16(o[2 * cp + 1], ap, b1);
    }
  }
}

// The gathering warps' partials (head g: max, sum, O) combined in warp order
// into `part` (G*128 outputs, then per head the max and the sum of weights, in
// log2 units).  Region A is the scratch; every thread of the CTA calls it.
template <int G>
__device__ void tile_combine(unsigned char* sm, const float (&o)[16][4], float m_run, float l_run, bool had, float* part,
                             bool write) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g = lane >> 2, t = lane & 3;
  constexpr int WS = D + 2;
  float* wsm = reinterpret_cast<float*>(sm);  // [8 warps][8 heads][130]
  __syncthreads();  // every warp is done with its ring
  if (warp < TL_WARPS) {
    float l4 = l_run;
    l4 += __shfl_xor_sync(0xffffffffu, l4, 1);
    l4 += __shfl_xor_sync(0xffffffffu, l4, 2);
    float* wr = wsm + (warp * 8 + g) * WS;
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      wr[8 * nt + 2 * t] = o[nt][0] + o[nt][2];
      wr[8 * nt + 2 * t + 1] = o[nt][1] + o[nt][3];
    }
    if (t == 0) {
      wr[D] = had ? m_run : -INFINITY;
      wr[D + 1] = had ? l4 : 0.f;
    }
  }
  __syncthreads();
  // the warps' scale factors: thread 8 hh + w (hh < 8 heads, w < 8 warps)
  float* scl = wsm + TL_WARPS * 8 * WS;  // [8 heads][8 warps]
  if (tid < 64) {
    const int hh = tid >> 3, w = tid & 7;
    const float m = wsm[(w * 8 + hh) * WS + D];
    float M = m;
    M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, 1));
    M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, 2));
    M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, 4));
    const float sc = M == -INFINITY ? 0.f : exp2f(m - M);  // 0 for a warp without rows
    scl[tid] = sc;
    const float lw = sc * wsm[(w * 8 + hh) * WS + D + 1];
    float Ls = 0.f;  // in warp order
#pragma unroll
    for (int v = 0; v < TL_WARPS; ++v) Ls += __shfl_sync(0xffffffffu, lw, (lane & ~7) + v);
    if (write && w == 0 && hh < G) {
      part[G * D + hh] = M;
      part[G * D + 8 + hh] = Ls;
    }
  }
  __syncthreads();
  if (write) {
#pragma unroll 1
    for (int e = tid; e < G * D; e += blockDim.x) {
      const int hh = e >> 7, c = e & (D - 1);
      float acc = 0.f;
#pragma unroll
      for (int w = 0; w < TL_WARPS; ++w) acc = fmaf(scl[hh * 8 + w], wsm[(w * 8 + hh) * WS + c], acc);
      part[e] = acc;
    }
  }
  __syncthreads();
}

// Element offset / 128 (row index into K', V) of gather row j of the CTA, or
// -1 for j >= n_rows.  all_kept: j is a candidate slot of the unit (rows of the
// kept pages in page order); otherwise j indexes the CTA's own kept list
// (u16 slots relative to its candidate share, which starts at cs0).
__device__ __forceinline__ int sp_row_of(const SpParams& p, const unsigned char* sm, const SpUnit& x, int j,
                                         int n_rows, bool all_kept, int cs0) {
  if (j >= n_rows) return -1;
  const int* kp = reinterpret_cast<const int*>(sm + SP_KP);
  const int ci = all_kept ? j : cs0 + reinterpret_cast<const uint16_t*>(sm + SP_OB)[j];
  const int t = (kp[ci >> p.dm.lgP] << p.dm.lgP) + (ci & (p.dm.P - 1));
  const long long off = kv_row(p.dm, p.table, x.b, x.h, t, p.status);
  return off >= 0 ? (int)(off / D) : -1;
}

// Issues tile k of gathering warp `warp` (gather rows j0 + 16 (warp + 8 k) ..
// +15, clipped to j1) into its slot k mod 3.
static __device__ __noinline__ void sp_issue_tile(const SpParams& p, unsigned char* sm, const SpUnit& x, int warp, int k,
                                                  int j0, int j1, bool all_kept, int cs0, bool live) {
  const int lane = threadIdx.x & 31;
  const int j = j0 + TL_ROWS * (warp + TL_WARPS * k) + lane;
  const int ri = (live && lane < TL_ROWS) ? sp_row_of(p, sm, x, j, j1, all_kept, cs0) : -1;
  tile_copy(p.Kr, p.Vc, tile_slot(sm, warp, k % TL_NBUF), ri, live);
}

// ---------------------------------------------------------------------------
// scores and key top-k (smaller score first, ties to the lower row)
// ---------------------------------------------------------------------------
// Candidates are the rows of the kept pages in page order (slot ci: page
// kp[ci / P], row ci % P; slots past the sequence end are not candidates).
// CTA r scores its balanced share [cs0, cs1) of the slots and publishes the
// histogram of its integer scores (added into the unit's histogram, and in
// cumulative form); after the group barrier the unit's histogram gives the
// threshold score T, the cumulative histograms of the CTAs before r the rows
// below and at T that precede the CTA's (ties are taken lower slots, i.e.
// lower rows, first), and the CTA lists its own kept slots (u16, relative to cs0,
// in slot order) at SP_OB: the rows it gathers.  Returns how many it keeps
// (`ok` false after an abort).

// Code row of slot ci (or -1: past the sequence end or a bad block).
__device__ __forceinline__ long long sp_code_of(const SpParams& p, const int* kp, const SpUnit& x, int ci) {
  const int t = (kp[ci >> p.dm.lgP] << p.dm.lgP) + (ci & (p.dm.P - 1));
  return t < x.L ? code_row(p.dm, p.table, x.b, x.h, t, p.status) : -1;
}

template <int WORDS>
__device__ __forceinline__ void sp_load_code(const uint64_t* src, uint64_t (&cw)[WORDS]) {
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
}

// The key's score: Hamming distance to the query codes summed (or, with
// key_min, minimised) over the group's heads.
template <int G, int WORDS>
__device__ __forceinline__ int sp_score(const uint64_t (&cw)[WORDS], const uint64_t (&cq)[G][WORDS], bool key_min) {
  int sum = 0, mn = INT_MAX;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    int sg = 0;
#pragma unroll
    for (int w2 = 0; w2 < WORDS; ++w2) sg += __popcll(cw[w2] ^ cq[g][w2]);
    sum += sg;
    mn = min(mn, sg);
  }
  return key_min ? mn : sum;
}

// The key select runs on the warp group [tb / 32, (tb + nthr) / 32) with named
// barrier `bar` (the whole CTA: tb = 0, nthr = 512, bar = 0), its histogram
// and scores at `scr`; with make_list it writes the kept list at SP_OB.
template <int G, int WORDS>
__device__ __noinline__ int sp_keys(const SpParams& p, unsigned char* sm, const SpUnit& x, int r, int nkp, int n_cand_local,
                       int keff, unsigned* gx, unsigned& epoch, int& cs0, bool& ok, int tb, int nthr, int bar,
                       unsigned char* scr, bool make_list) {
  const Dims& dm = p.dm;
  const Work& wk = p.wk;
  const int tid = threadIdx.x - tb, lane = tid & 31, warp = tid >> 5, nw = nthr >> 5;
  const int S = p.gsize;
  const int nbins = G * dm.nb + 1, HB = wk.HB;
  int* hist = reinterpret_cast<int*>(scr);                            // [HB] the CTA's histogram
  uint16_t* sc = reinterpret_cast<uint16_t*>(scr + HB * 4);           // [share] scores
  uint16_t* klist = reinterpret_cast<uint16_t*>(sm + SP_OB);          // [kept]
  int* red = reinterpret_cast<int*>(sm + SP_RED);
  int* bc = red + 128;
  const int* kp = reinterpret_cast<const int*>(sm + SP_KP);
  const unsigned* qcw = reinterpret_cast<const unsigned*>(sm + SP_QC);
  const int ncs = nkp << dm.lgP;
  int cs1;
  share_of(ncs, S, r, cs0, cs1);
  const int nmy = cs1 - cs0;
  #pragma unroll 1
  for (int i = tid; i < HB; i += nthr) hist[i] = 0;
  uint64_t cq[G][WORDS];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int w2 = 0; w2 < WORDS; ++w2)
      cq[g][w2] = (uint64_t)qcw[g * 8 + 2 * w2] | ((uint64_t)qcw[g * 8 + 2 * w2 + 1] << 32);
  bar_sync(bar, nthr);
  int* dsc = p.dbg.key_scores ? p.dbg.key_scores + (long long)x.u * wk.Nmax * dm.P + cs0 : nullptr;
  // two slots per thread and pass, both code loads in flight together
#pragma unroll 1
  for (int j = tid; j < nmy; j += 2 * nthr) {
    const int j2 = j + nthr;
    const long long w1 = sp_code_of(p, kp, x, cs0 + j);
    const long long w2 = j2 < nmy ? sp_code_of(p, kp, x, cs0 + j2) : -1;
    uint64_t c1[WORDS], c2[WORDS];
    if (w1 >= 0) sp_load_code<WORDS>(p.codes + w1, c1);
    if (w2 >= 0) sp_load_code<WORDS>(p.codes + w2, c2);
    int s1 = 0xFFFF, s2 = 0xFFFF;
    if (w1 >= 0) {
      s1 = sp_score<G, WORDS>(c1, cq, dm.key_min);
      atomicAdd(&hist[s1], 1);
    }
    if (w2 >= 0) {
      s2 = sp_score<G, WORDS>(c2, cq, dm.key_min);
      atomicAdd(&hist[s2], 1);
    }
    sc[j] = (uint16_t)s1;
    if (dsc) dsc[j] = s1 == 0xFFFF ? INT_MAX : s1;
    if (j2 < nmy) {
      sc[j2] = (uint16_t)s2;
      if (dsc) dsc[j2] = s2 == 0xFFFF ? INT_MAX : s2;
    }
  }
  bar_sync(bar, nthr);
  // publish: the CTA's histogram added into the unit's, and its cumulative
  // form (thread t: bins [t bpt, t bpt + bpt))
  const int bpt = (nbins + nthr - 1) / nthr;  // <= 9
  int* tot_h = wk.ktot + (long long)x.u * HB;
  {
    int hv[9], loc = 0;
#pragma unroll
    for (int e = 0; e < 9; ++e) {
      const int bi = tid * bpt + e;
      hv[e] = (e < bpt && bi < nbins) ? hist[bi] : 0;
      if (hv[e]) atomicAdd(tot_h + bi, hv[e]);
      loc += hv[e];
    }
    int tot0;
    int run = block_scan_excl(loc, red, 0, &tot0, tb >> 5, nw, bar);
    int* myh = wk.khist + (long long)blockIdx.x * HB;
#pragma unroll
    for (int e = 0; e < 9; ++e) {
      const int bi = tid * bpt + e;
      run += hv[e];
      if (e < bpt && bi < nbins) myh[bi] = run;
    }
  }
  if (!sp_group_sync(p, sm, gx, epoch, tb, nthr, bar)) {
    ok = false;
    return 0;
  }
  // ---- the unit's histogram: the threshold from below ----
  int hv[9];
  int local = 0;
#pragma unroll
  for (int e = 0; e < 9; ++e) {
    const int bi = tid * bpt + e;
    hv[e] = (e < bpt && bi < nbins) ? __ldcg(tot_h + bi) : 0;
    local += hv[e];
  }
  if (tid == 0) {
    bc[0] = -1;  // no candidate: nothing kept
    bc[1] = 0;
  }
  int n_cand;
  const int before = block_scan_excl(local, red, 1, &n_cand, tb >> 5, nw, bar);
  if (n_cand != n_cand_local) {  // only a bad block id can make a candidate unreadable
    if (tid == 0) sp_abort(p, sm, HHR_ERR_BAD_BLOCK);
    bar_sync(bar, nthr);
    ok = false;
    return 0;
  }
  if (keff > 0 && before < keff && before + local >= keff) {
    int run = before;
#pragma unroll
    for (int e = 0; e < 9; ++e) {
      if (run < keff && run + hv[e] >= keff) {
        bc[0] = tid * bpt + e;
        bc[1] = keff - run;
      }
      run += hv[e];
    }
  }
  bar_sync(bar, nthr);
  const int T = bc[0], need_eq = bc[1];
  // rows below T and at T of the CTAs before r, from their cumulative histograms
  int lt_before = 0, eq_before = 0;
  {
    int* acc = red + 136;  // [2]
    if (tid < 2) acc[tid] = 0;
    bar_sync(bar, nthr);
    int lt = 0, eq = 0;
    if (tid < r && T >= 0) {
      const int* ch = wk.khist + (long long)(blockIdx.x - r + tid) * HB;
      const int cT = __ldcg(ch + T), cB = T > 0 ? __ldcg(ch + T - 1) : 0;
      lt = cB;
      eq = cT - cB;
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      lt += __shfl_xor_sync(0xffffffffu, lt, o);
      eq += __shfl_xor_sync(0xffffffffu, eq, o);
    }
    if (lane == 0 && warp * 32 < r) {
      atomicAdd(&acc[0], lt);
      atomicAdd(&acc[1], eq);
    }
    bar_sync(bar, nthr);
    lt_before = acc[0];
    eq_before = acc[1];
  }
  const int off = lt_before + min(need_eq, eq_before);  // the CTA's first place in the unit's kept order
  const int take = max(0, need_eq - eq_before);         // ties it may take
  if (r == 0 && tid == 0) {
    if (p.dbg.n_cand) p.dbg.n_cand[x.u] = n_cand;
    if (p.dbg.n_sel_keys) p.dbg.n_sel_keys[x.u] = keff;
  }
  // ---- kept slots in slot order: thread t owns slots [t m, (t+1) m) ----
  const int m = (nmy + nthr - 1) / nthr;
  const int j0 = min(nmy, tid * m), j1 = min(nmy, j0 + m);
  int lt_t = 0, eq_t = 0;
  #pragma unroll 1
  for (int j = j0; j < j1; ++j) {
    const int sv = sc[j];
    lt_t += sv < T;
    eq_t += sv == T;
  }
  int tot2;
  const int pk = block_scan_excl((lt_t << 16) | eq_t, red, 0, &tot2, tb >> 5, nw, bar);
  int lt_run = pk >> 16, eq_run = pk & 0xFFFF;
  const int n_loc = min(SP_KLCAP, (tot2 >> 16) + min(tot2 & 0xFFFF, take));
  int* dout = p.dbg.sel_keys ? p.dbg.sel_keys + (long long)x.u * wk.Kmax + off : nullptr;
  #pragma unroll 1
  for (int j = j0; j < j1; ++j) {
    const int sv = sc[j];
    const bool l1 = sv < T, e1 = sv == T;
    if (l1 || (e1 && eq_run < take)) {
      const int pos = lt_run + min(eq_run, take);
      if (pos < n_loc) {
        if (make_list) klist[pos] = (uint16_t)j;
        if (dout) {
          const int ci = cs0 + j;
          dout[pos] = (kp[ci >> dm.lgP] << dm.lgP) + (ci & (dm.P - 1));
        }
      }
    }
    lt_run += l1;
    eq_run += e1;
  }
  bar_sync(bar, nthr);
  return n_loc;
}

// ---------------------------------------------------------------------------
// final merge of a unit's partials (the last CTA of the group to arrive)
// ---------------------------------------------------------------------------
// out[h][c] = sum_k w_k o_k[h][c] / sum_k w_k L_k[h], w_k = 2^(M_k[h] - M[h]),
// M[h] = max_k M_k[h], over the n partials in order (a partial without rows
// has M = -inf and weight 0).  The partials are copied to shared memory in
// passes (region A is free by now).
template <int G>
__device__ void sp_merge(const SpParams& p, unsigned char* sm, const SpUnit& x, int n) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int PS = G * D + 16;
  const float* pt = p.wk.part + (long long)x.u * p.wk.C3 * PS;
  float* wbuf = reinterpret_cast<float*>(sm + SP_OB);  // [n][8] weights (n <= 256)
  float* inv = reinterpret_cast<float*>(sm + SP_LS);   // [8] 1 / total weight
  const int per = SP_A_BYTES / (PS * 4);              // partials per pass through region A
  float* sp = reinterpret_cast<float*>(sm);
  // the first pass's copies are in flight while the weights are computed
  {
    const int n16 = min(per, n) * PS / 4;
#pragma unroll 1
    for (int i = tid; i < n16; i += SP_THREADS) cp_async16(sp + 4 * i, pt + 4 * i);
    cp_async_commit();
  }
  // warp h: the weights of head h, from the partials' (max, sum) pairs: in
  // shared memory when every partial fits one pass, else read through L2
  // (written by the other CTAs of the group)
  auto weights = [&](const float* src, bool l2) {
    auto ld = [&](long long i) { return l2 ? __ldcg(src + i) : src[i]; };
    float M = -INFINITY;
#pragma unroll 1
    for (int k = lane; k < n; k += 32) M = fmaxf(M, ld((long long)k * PS + G * D + warp));
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float tot = 0.f;
#pragma unroll 1
    for (int k0 = 0; k0 < n; k0 += 32) {
      const int k = k0 + lane;
      float wl = 0.f;
      if (k < n) {
        const float mk = ld((long long)k * PS + G * D + warp);
        const float w = mk == -INFINITY ? 0.f : exp2f(mk - M);
        wbuf[k * 8 + warp] = w;
        wl = w * ld((long long)k * PS + G * D + 8 + warp);
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) wl += __shfl_xor_sync(0xffffffffu, wl, o);
      tot += wl;
    }
    if (lane == 0) inv[warp] = 1.f / tot;
  };
  const bool one_pass = n <= per;
  if (!one_pass && warp < G) weights(pt, true);
  float acc0 = 0.f, acc1 = 0.f;  // elements tid and tid + 512 (G * 128 <= 1024)
#pragma unroll 1
  for (int k0 = 0; k0 < n; k0 += per) {
    const int nk = min(per, n - k0);
    if (k0 > 0) {
      const int n16 = nk * PS / 4;
#pragma unroll 1
      for (int i = tid; i < n16; i += SP_THREADS) cp_async16(sp + 4 * i, pt + (long long)k0 * PS + 4 * i);
      cp_async_commit();
    }
    cp_async_wait_all();
    __syncthreads();
    if (one_pass) {
      if (warp < G) weights(sp, false);
      __syncthreads();
    }
#pragma unroll 1
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
  const int tid = threadIdx.x, warp = tid >> 5;
  const int S = p.gsize;
  const int grp = blockIdx.x / S, r = blockIdx.x - grp * S;
  const int Units = dm.B * dm.Hkv;
  if (tid < 16) reinterpret_cast<volatile int*>(sm + SP_MISC)[tid] = 0;
  // one barrier per metadata stage slot; bit i of `ph` is the parity of slot
  // i's next phase, bit i of `pend` marks a phase armed and not yet waited for
  uint64_t* mbar = reinterpret_cast<uint64_t*>(sm + SP_MBAR);
  if (tid == 0) {
    for (int i = 0; i < SP_NST; ++i) mbar_init(mbar + i, 1);
    mbar_fence_init();
  }
  unsigned ph = 0u, pend = 0u;
  // the prep's weights of the first unit: copied before the previous kernel on
  // the stream has finished (they are never written by a decode step)
  if (grp < Units) sp_issue_rw(p, sm, grp % dm.Hkv);
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
    if (!first) sp_issue_rw(p, sm, x.h);
    first = false;
    // ---- the query heads, metadata copies of the first two stages, the prep, two more stages ----
    #pragma unroll 1
    for (int e = tid; e < (8 - G) * 68; e += SP_THREADS) reinterpret_cast<uint32_t*>(sm + SP_OB + G * 272)[e] = 0u;
    sp_issue_q(p, sm, x, G);
    int p0, p1;
    share_of(x.np, S, r, p0, p1);
    const int nsteps = (p1 - p0 + SP_STAGE_PAGES - 1) / SP_STAGE_PAGES;
    auto issue_stage = [&](int st) {  // (every thread calls it alike)
      if (st < nsteps) {
        const int slot = st % SP_NST;
        sp_issue_meta(p, sm + slot * SP_META_STAGE, mbar + slot, x, p0 + st * SP_STAGE_PAGES, p1);
        pend |= 1u << slot;
      }
    };
    issue_stage(0);
    issue_stage(1);
    sp_prep<G>(p, sm, x, r == 0);
    issue_stage(2);
    issue_stage(3);
    if (x.L == 0) {  // empty sequence: zero output, no barrier (every CTA of the group skips alike)
      cp_async_wait_all();
      if (r == 0) {
        #pragma unroll 1
        for (int e = tid; e < G * D; e += SP_THREADS) p.out[((long long)x.b * dm.Hq + x.h * G) * D + e] = 0.f;
        if (tid == 0) {
          if (p.dbg.n_sel_pages) p.dbg.n_sel_pages[x.u] = 0;
          if (p.dbg.n_sel_keys) p.dbg.n_sel_keys[x.u] = 0;
          if (p.dbg.n_cand) p.dbg.n_cand[x.u] = 0;
        }
      }
      fence_proxy_async();
      __syncthreads();
      continue;
    }
    // ---- scan ----
    {
      float2 qa[G][4], qbn[G][4];
      const float* qs = reinterpret_cast<const float*>(sm + SP_OB + 4096);
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
#pragma unroll 1
      for (int s = 0; s < nsteps; ++s) {
        if (s + SP_NST - 1 < nsteps) {
          __syncthreads();  // every thread is done with stage s - 1, whose slot is refilled
          issue_stage(s + SP_NST - 1);
        }
        const int slot = s % SP_NST;
        if (!mbar_wait(mbar + slot, (ph >> slot) & 1u, p.wait_limit)) sp_abort(p, sm, HHR_ERR_TIMEOUT);
        ph ^= 1u << slot;
        pend &= ~(1u << slot);
        sp_scan_stage<G>(p, sm + slot * SP_META_STAGE, x, p0 + s * SP_STAGE_PAGES, p1, qa, qbn);
      }
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
    // gather rows of the CTA, in 16-row tiles (gathering warp w < 8 takes tiles
    // w, w + 8, ...): with every candidate kept, its balanced share of the
    // candidate slots, known now; else the kept slots of its own scoring share
    // (after the key select).  With every candidate kept and the key select's
    // scratch small enough for region B, warps 8-15 run the key select while
    // warps 0-7 gather (the key select then keeps every candidate).
    const bool gw = warp < TL_WARPS;
    const int ncs = nkp << dm.lgP;
    const bool conc = all_kept && wk.HB * 4 + 2 * ((ncs + S - 1) / S) <= 2 * SP_KLCAP;
    int j0 = 0, j1 = 0, mine = 0;
    if (conc) {  // the scoring share's code rows go out ahead of the tile copies
      if (!gw) {
        int c0, c1;
        share_of(ncs, S, r, c0, c1);
        const int pa = c0 >> dm.lgP, pb = c1 > c0 ? ((c1 - 1) >> dm.lgP) + 1 : pa;
        const int lines = (dm.P * WORDS * 8 + 127) >> 7;  // 128-byte lines of a page's code rows
        #pragma unroll 1
        for (int e = tid - TL_WARPS * 32; e < (pb - pa) * lines; e += SP_THREADS - TL_WARPS * 32) {
          const int pg = kp[pa + e / lines];
          const long long off = pg * dm.P < x.L ? code_row(dm, p.table, x.b, x.h, pg * dm.P, p.status) : -1;
          if (off >= 0) prefetch_l2(p.codes + off + (e % lines) * 16);
        }
        bar_arrive(3, SP_THREADS);
      } else {
        bar_sync(3, SP_THREADS);
      }
    }
    if (all_kept) {
      share_of(keff, S, r, j0, j1);
      const int ntile = (j1 - j0 + TL_ROWS - 1) / TL_ROWS;
      mine = (gw && ntile > warp) ? (ntile - warp + TL_WARPS - 1) / TL_WARPS : 0;
      if (gw) {  // (their copies start at once)
        sp_issue_tile(p, sm, x, warp, 0, j0, j1, true, 0, mine > 0);
        sp_issue_tile(p, sm, x, warp, 1, j0, j1, true, 0, mine > 1);
        if (conc) sp_issue_tile(p, sm, x, warp, 2, j0, j1, true, 0, mine > 2);
      }
    }
    bool ok = true;
    int cs0 = 0;
    if (conc) {
      if (!gw) sp_keys<G, WORDS>(p, sm, x, r, nkp, n_cand, keff, gx, epoch, cs0, ok, TL_WARPS * 32, SP_THREADS - TL_WARPS * 32, 1, sm + SP_OB, false);
    } else {
      const int n_loc = sp_keys<G, WORDS>(p, sm, x, r, nkp, n_cand, keff, gx, epoch, cs0, ok, 0, SP_THREADS, 0, sm + SP_HISTS, true);
      if (!ok) break;
      if (!all_kept) {
        j1 = n_loc;
        const int ntile = (j1 + TL_ROWS - 1) / TL_ROWS;
        mine = (gw && ntile > warp) ? (ntile - warp + TL_WARPS - 1) / TL_WARPS : 0;
      }
    }
    // ---- gather: the warps' tiles, three in flight ----
    float o[16][4];
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;
    if (gw) {
      if (!all_kept) {
        sp_issue_tile(p, sm, x, warp, 0, j0, j1, false, cs0, mine > 0);
        sp_issue_tile(p, sm, x, warp, 1, j0, j1, false, cs0, mine > 1);
      }
      if (!conc) sp_issue_tile(p, sm, x, warp, 2, j0, j1, all_kept, cs0, mine > 2);
      uint32_t aq[8][4];
      load_q_operand(sm + SP_QB, aq);
#pragma unroll 1
      for (int k = 0; k < mine; ++k) {
        cp_async_wait<TL_NBUF - 1>();
        __syncwarp();
        const int tl = warp + TL_WARPS * k;
        tile_attend(aq, o, m_run, l_run, tile_slot(sm, warp, k % TL_NBUF), min(TL_ROWS, j1 - j0 - TL_ROWS * tl));
        __syncwarp();
        sp_issue_tile(p, sm, x, warp, k + TL_NBUF, j0, j1, all_kept, cs0, k + TL_NBUF < mine);
      }
    }
    cp_async_wait_all();
    __syncthreads();  // (the key select of warps 8-15 may have raised the abort flag)
    if (sp_aborted(sm)) break;
    const int PS = G * D + 16;
    tile_combine<G>(sm, o, m_run, l_run, mine > 0, wk.part + ((long long)x.u * wk.C3 + r) * PS, true);
    if (sp_aborted(sm)) break;
    // ---- the last CTA of the group merges ----
    if (tid == 0) {
      int last = 1;
      if (S > 1) last = atom_add_acq_rel(gx + GX_ARRIVE, 1u) == (unsigned)(S - 1);
      reinterpret_cast<volatile int*>(sm + SP_MISC)[MS_LAST] = last;
    }
    __syncthreads();
    if (reinterpret_cast<volatile int*>(sm + SP_MISC)[MS_LAST]) {
      sp_merge<G>(p, sm, x, S);
      // the unit's counters and score histogram are zero again for the next call
      #pragma unroll 1
      for (int i = tid; i < G * dm.nb + 1; i += SP_THREADS) wk.ktot[(long long)x.u * wk.HB + i] = 0;
      if (tid == 0) {
        gx[GX_BAR] = 0u;
        gx[GX_ARRIVE] = 0u;
      }
    }
    fence_proxy_async();  // (region A is refilled by TMA copies in the next unit)
    __syncthreads();
  }
  cp_async_wait_all();
  // an abort can leave metadata copies in flight: they land before the CTA exits
  #pragma unroll 1
  for (int i = 0; i < SP_NST; ++i)
    if ((pend >> i) & 1u) mbar_wait(mbar + i, (ph >> i) & 1u, p.wait_limit);
}

// CTAs per group: the SMs shared out over the units, at most one CTA per 64
// pages of the longest sequence, few enough that the key select's scratch
// holds a CTA's scores, and at least enough that a CTA's kept rows
// (at most its share of the candidates, and at most the key budget) fit its
// kept list.  Groups take units in a grid-stride loop.
inline void sparse_group_shape(const Dims& dm, int sms, int Cmax, int Kmax, int HB, int* S, int* ngroups) {
  const int U = dm.B * dm.Hkv;
  sms = std::max(1, std::min(sms, MAX_GRID));
  int s = std::max(1, sms / U);
  s = std::min(s, std::max(1, dm.np_max / 64));
  while (s > 1 && (long long)HB * 4 + 2 * ((Cmax + s - 1) / s) > SP_A_BYTES - SP_HISTS) --s;
  const int kcap = std::min(Kmax, Cmax);
  s = std::max(s, (kcap + SP_KLCAP - 1) / SP_KLCAP);
  *S = s;
  *ngroups = std::max(1, std::min(U, sms / s));
}

}  // namespace hhr
