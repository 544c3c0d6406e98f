// HHR decode step with CTA groups: one group of S CTAs per unit (sequence b,
// KV head h), every CTA of a group owning a contiguous share of the unit's
// pages and, after the selects, a share of the chunks of its kept rows (sm_100a).
//
// Per unit, CTA r of the group:
//   1. computes q' = R_h q and the query sign codes itself (R_h, W_h and q are
//      read by every CTA of the group; the copies after the first hit L2),
//      while its producer warp already streams the page metadata of its share
//      into the shared-memory ring;
//   2. scans its pages: U = max over the group's heads of the page bound,
//      written to the workspace; one group barrier;
//   3. runs the page top-N on all the unit's bounds (read from L2), the same
//      in every CTA of the group: value-bin histograms, refined while the
//      threshold bin is crowded, then an exact ranking (larger bound first,
//      then the lower page), so every CTA knows every kept page;
//   4. scores its balanced share of the candidate rows (the rows of the kept
//      pages in page order; Hamming distance summed over the group's heads)
//      and publishes the histogram of its scores; one group barrier; the S
//      histograms give the threshold, the ties taken and the CTA's place in
//      the unit's row list (CTA order is row order);
//   5. writes its kept rows there (row + 1; readers poll the entries) and
//      gathers the K'/V rows of its share of that list's chunks of 128 rows
//      (cp.async by the consumer warps, one chunk ahead; logits and P.V on
//      tensor cores), one softmax partial per chunk;
//   6. the last CTA of the group to arrive merges the chunk partials in chunk
//      order into the output and clears the unit's counters (the result does
//      not depend on the number of CTAs per group).
// A group barrier is an acquire-release counter in the workspace: every CTA
// adds 1 after a CTA barrier, then waits (bounded) for S per barrier passed.
// All of a group's CTAs are resident at once (one CTA per SM, grid <= SMs).
#pragma once

#include "hhr_fused.cuh"

namespace hhr {

constexpr int GP_WORK = 90112;                 // consumer scratch
constexpr int GP_SMAX = MAX_GRID;              // CTAs per group at most
constexpr int GP_LEVELS = 4;                   // page select levels
constexpr int SEL_RANK_SMALL = 32;             // threshold-bin size ranked without another level
constexpr int GP_PAGES_PER_SLOT = 32;          // a ring slot: 32 pages of minima, then their maxima
constexpr size_t GP_OFF_RING = 0;
constexpr size_t GP_OFF_WORK = GP_OFF_RING + (size_t)FZ_NSLOT * FZ_SLOT;
constexpr size_t GP_OFF_QS = GP_OFF_WORK + GP_WORK;   // q' fp32 [8][128] (quad-permuted)
constexpr size_t GP_OFF_QC = GP_OFF_QS + 8 * D * 4;   // query codes u32 [8][8]
constexpr size_t GP_OFF_RIDX = GP_OFF_QC + 256;       // row numbers of two gather steps [2][128]
constexpr int GP_PF_MAX = 512;                 // pages in the producer's prefetch list
constexpr size_t GP_OFF_PF = GP_OFF_RIDX + 2 * FZ_ROWS * 4;  // int [GP_PF_MAX]
constexpr size_t GP_OFF_BAR = GP_OFF_PF + GP_PF_MAX * 4;
constexpr size_t GP_OFF_MISC = GP_OFF_BAR + 8 * (2 * FZ_NSLOT);
constexpr size_t GP_SMEM = GP_OFF_MISC + 256;
static_assert(GP_SMEM <= 232448, "shared memory of the group kernel");

// consumer scratch during the scan and the selects (the gather reuses it all)
constexpr int GW_US = 0;                       // float [8192] bounds of the CTA's pages
constexpr int GW_HIST = 32768;                 // int [2056] value bins / score histogram
constexpr int GW_CAND = GW_HIST + 8448;        // int2 [512] members of the threshold bin
constexpr int GW_FLAG = GW_CAND + 4096;        // u32 [256] kept members (bitmap over local pages)
constexpr int GW_RED = GW_FLAG + 1024;         // int [256] scan scratch and broadcasts
constexpr int GW_KP = GW_RED + 1024;           // int [2048] kept pages (ascending)
constexpr int GW_SC = GW_KP + 8192;            // uint16 [16384] scores of the candidate rows
static_assert(GW_SC + 2 * MAX_CANDIDATES <= GP_WORK, "group kernel scratch");
static_assert(MAX_SELECT_PAGES * 4 <= GW_HIST && FZ_HIST_BINS * 4 <= 8448, "group kernel scratch");
static_assert(GA_LB + 512 <= GP_WORK, "gather scratch");

// Per-unit counters in the workspace (32-bit words), zero between calls (the
// merging CTA resets them).
enum : int {
  GX_BAR = 0,     // group barrier arrivals
  GX_ARRIVE = 1,  // CTAs done with the unit (the last one merges)
  GX_WORDS = 4,
};

__device__ __forceinline__ int ld_relaxed32(const int* w) {
  int v;
  asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(w) : "memory");
  return v;
}
__device__ __forceinline__ void prefetch_l2(const void* p, unsigned bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

struct GpShared {
  unsigned char* ring;
  unsigned char* work;
  float* qs;
  unsigned* qc;
  int* ridx;
  int* pf;          // pages whose code (then K'/V) rows the producer prefetches to L2
  const int* kpw;   // kept pages of the unit (consumer scratch)
  uint64_t* full;
  uint64_t* empty;
  int* misc;        // [0] abort, [1] slots consumed, [2] slots armed, [17], [18] broadcasts,
                    // [20] units whose ring use the consumers have finished, [21] units whose
                    // prefetch list is ready, [22], [23] its code and K'/V page counts
};

__device__ __forceinline__ GpShared gp_shared(unsigned char* base) {
  GpShared s;
  s.ring = base + GP_OFF_RING;
  s.work = base + GP_OFF_WORK;
  s.qs = reinterpret_cast<float*>(base + GP_OFF_QS);
  s.qc = reinterpret_cast<unsigned*>(base + GP_OFF_QC);
  s.ridx = reinterpret_cast<int*>(base + GP_OFF_RIDX);
  s.pf = reinterpret_cast<int*>(base + GP_OFF_PF);
  s.kpw = reinterpret_cast<const int*>(base + GP_OFF_WORK + GW_KP);
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + GP_OFF_BAR);
  s.full = bars;
  s.empty = bars + FZ_NSLOT;
  s.misc = reinterpret_cast<int*>(base + GP_OFF_MISC);
  return s;
}

// Bounded mbarrier wait for the group kernel (abort flag in misc[0]).
__device__ __forceinline__ bool gp_wait(const GpShared& s, uint64_t* bar, uint32_t parity, int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*reinterpret_cast<volatile int*>(s.misc)) return false;
    if (clock64() - t0 > FZ_WAIT_CYCLES) {
      set_status(status, HHR_ERR_TIMEOUT);
      *reinterpret_cast<volatile int*>(s.misc) = 1;
      return false;
    }
  }
}

__device__ __forceinline__ void red_release_add(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Group of unit u's CTAs: the unit's exchange area.
__device__ __forceinline__ unsigned* gx_of(const FzParams& p, int u) { return p.wk.gx + (long long)u * p.wk.gx_stride; }

// Pages [p0, p1) of CTA r among S for a unit of np pages.
__device__ __forceinline__ void share_of(int n, int S, int r, int& a, int& b) {
  a = (int)(((long long)n * r) / S);
  b = (int)(((long long)n * (r + 1)) / S);
}


// Group barrier among the consumer threads of the group's S CTAs.  Every
// consumer thread calls it; writes made before it by any thread of the group
// are visible after it (read them with ld.global.cg: L1 is not coherent).
// False after a timeout or an abort (then every thread of the CTA sees false).
__device__ __forceinline__ bool gp_sync(const FzParams& p, const GpShared& s, unsigned* gx, unsigned& epoch) {
  cons_sync();
  if (p.gsize == 1) return *reinterpret_cast<volatile int*>(s.misc) == 0;  // a CTA barrier suffices
  epoch += (unsigned)p.gsize;
  if (threadIdx.x == 0) {
    volatile int* ab = s.misc;
    red_release_add(gx + GX_BAR, 1u);
    if (ld_acquire(gx + GX_BAR) < epoch) {
      const long long t0 = clock64();
      while (ld_acquire(gx + GX_BAR) < epoch) {
        if (*ab) break;
        if (clock64() - t0 > FZ_WAIT_CYCLES) {
          set_status(p.status, HHR_ERR_TIMEOUT);
          *ab = 1;
          break;
        }
      }
    }
  }
  cons_sync();
  return *reinterpret_cast<volatile int*>(s.misc) == 0;
}

// ---------------------------------------------------------------------------
// producer (warp 16): streams the page metadata of the CTA's share of every
// unit of its group into the ring, 32 pages per slot (minima, then maxima)
// ---------------------------------------------------------------------------
static __device__ void gp_producer(const FzParams& p, const GpShared& s, int g, int r) {
  const int lane = threadIdx.x & 31;
  const Dims& dm = p.dm;
  const int U = dm.B * dm.Hkv, S = p.gsize;
  const uint64_t ef = evict_first_policy();
  unsigned nslot = 0, nunit = 0;
  for (int u = g; u < U; u += p.ngroups, ++nunit) {
    if (nunit > 0) {  // the consumers are done with the ring (gather of the previous unit)
      bool ok = true;
      if (lane == 0) {
        volatile int* rel = s.misc + 20;  // units the consumers have released
        if (*rel < (int)nunit) {
          const long long t0 = clock64();
          while (*rel < (int)nunit) {
            __nanosleep(256);  // (a tight spin would take issue slots from the consumer warps)
            if (*reinterpret_cast<volatile int*>(s.misc)) {
              ok = false;
              break;
            }
            if (clock64() - t0 > FZ_WAIT_CYCLES) {
              set_status(p.status, HHR_ERR_TIMEOUT);
              *reinterpret_cast<volatile int*>(s.misc) = 1;
              ok = false;
              break;
            }
          }
        }
      }
      if (__shfl_sync(0xffffffffu, (int)ok, 0) == 0) break;
    }
    const int b = u / dm.Hkv, h = u - b * dm.Hkv;
    const int L = seq_len_of(dm, p.seq_lens, b);
    const int np = (L + dm.P - 1) >> dm.lgP;
    int p0, p1;
    share_of(np, S, r, p0, p1);
    bool aborted = false;
    for (int j0 = p0; j0 < p1; j0 += GP_PAGES_PER_SLOT) {
      const int n = min(GP_PAGES_PER_SLOT, p1 - j0);
      const int slot = (int)(nslot % FZ_NSLOT);
      if (nslot >= FZ_NSLOT) {
        bool ok = true;
        if (lane == 0) ok = gp_wait(s, &s.empty[slot], ((nslot / FZ_NSLOT) - 1) & 1, p.status);
        if (__shfl_sync(0xffffffffu, (int)ok, 0) == 0) {
          aborted = true;
          break;
        }
      }
      unsigned char* dst = s.ring + (size_t)slot * FZ_SLOT;
      if (!dm.paged) {
        if (lane == 0) {
          const long long off = ((long long)(b * dm.Hkv + h) * dm.np_max + j0) * D;
          mbar_arrive_expect_tx(&s.full[slot], (uint32_t)(2 * n * 256));
          bulk_g2s_stream(dst, p.pmin + off, (uint32_t)(n * 256), &s.full[slot], ef);
          bulk_g2s_stream(dst + FZ_SLOT / 2, p.pmax + off, (uint32_t)(n * 256), &s.full[slot], ef);
        }
      } else {
        // one page per lane; a bad block id reads as zero rows
        int blk = -1;
        bool ok = false;
        if (lane < n) {
          blk = __ldg(p.table + (long long)b * dm.max_blocks + j0 + lane);
          ok = (unsigned)blk < (unsigned)dm.num_blocks;
          if (!ok) {
            set_status(p.status, HHR_ERR_BAD_BLOCK);
            uint4* z0 = reinterpret_cast<uint4*>(dst + lane * 256);
            uint4* z1 = reinterpret_cast<uint4*>(dst + FZ_SLOT / 2 + lane * 256);
#pragma unroll
            for (int i = 0; i < 16; ++i) z0[i] = z1[i] = make_uint4(0u, 0u, 0u, 0u);
          }
        }
        const unsigned okm = __ballot_sync(0xffffffffu, ok);
        if (lane == 0) mbar_arrive_expect_tx(&s.full[slot], (uint32_t)(__popc(okm) * 512));
        __syncwarp();
        if (ok) {
          const long long off = ((long long)blk * dm.Hkv + h) * D;
          bulk_g2s_stream(dst + lane * 256, p.pmin + off, 256u, &s.full[slot], ef);
          bulk_g2s_stream(dst + FZ_SLOT / 2 + lane * 256, p.pmax + off, 256u, &s.full[slot], ef);
        }
      }
      __syncwarp();
      ++nslot;
      if (lane == 0) s.misc[2] = (int)nslot;  // slots armed (drained at exit after an abort)
    }
    if (aborted) break;
    if (L > 0) {
      // L2 prefetches from the consumers' list, once the kept pages are known:
      // code rows (trimmed to 16-byte boundaries), then K'/V rows of pages
      bool ok = true;
      if (lane == 0) {
        volatile int* rdy = s.misc + 21;
        if (*rdy < (int)nunit + 1) {
          const long long t0 = clock64();
          while (*rdy < (int)nunit + 1) {
            __nanosleep(128);
            if (*reinterpret_cast<volatile int*>(s.misc)) {
              ok = false;
              break;
            }
            if (clock64() - t0 > FZ_WAIT_CYCLES) {
              set_status(p.status, HHR_ERR_TIMEOUT);
              *reinterpret_cast<volatile int*>(s.misc) = 1;
              ok = false;
              break;
            }
          }
        }
      }
      if (__shfl_sync(0xffffffffu, (int)ok, 0) == 0) break;
      const int n1 = reinterpret_cast<volatile int*>(s.misc)[22], n2 = reinterpret_cast<volatile int*>(s.misc)[23];
      for (int i = lane; i < n1 + n2; i += 32) {
        const int pg = reinterpret_cast<volatile int*>(s.pf)[i];
        const int t0 = pg << dm.lgP;
        if (i < n1) {
          const long long co = code_row(dm, p.table, b, h, t0, p.status);
          if (co >= 0) {
            const uintptr_t a0 = reinterpret_cast<uintptr_t>(p.codes + co);
            const uintptr_t a1 = a0 + (uintptr_t)(dm.P * dm.words * 8);
            const uintptr_t c0 = (a0 + 15) & ~(uintptr_t)15, c1 = a1 & ~(uintptr_t)15;
            if (c1 > c0) prefetch_l2(reinterpret_cast<const void*>(c0), (unsigned)(c1 - c0));
          }
        } else {
          const long long ro = kv_row(dm, p.table, b, h, t0, p.status);
          if (ro >= 0) {
            prefetch_l2(p.Kr + ro, (unsigned)(dm.P * D * 2));
            prefetch_l2(p.Vc + ro, (unsigned)(dm.P * D * 2));
          }
        }
      }
      __syncwarp();
    }
  }
}

// ---- PREP: q' = R_h q and the query codes, read straight from global memory ----
// Same arithmetic as the fused kernel's query preparation: q' rows reduced by
// a transposed butterfly; code bits from fp32 sums with an fp64 recompute
// whenever |sum| <= 2^-14 sum |w q| (the sign is then exact).
template <int G>
__device__ void gp_prep(const FzParams& p, const GpShared& s, const Unit& x, bool write_dbg) {
  constexpr int GP = G <= 4 ? 4 : 8;
  const Dims& dm = p.dm;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float* qf = reinterpret_cast<float*>(s.work);  // [G][128] q in natural order
  const __nv_bfloat16* qg = p.q + ((long long)x.b * dm.Hq + x.h * G) * D;
  // R_h rows 8w .. 8w+7 of this warp (lane: channels 4l .. 4l+3), issued first
  const float* Rh = p.R + (long long)x.h * D * D;
  constexpr int NBB = 32 / GP;  // code bits per block (see below)
  const int bpw = dm.nb / FZ_CWARPS;
  const __nv_bfloat16* Wh = p.W + (long long)x.h * dm.nb * D;
  // every load of the first round is issued before any is used: R_h rows, the
  // first block of W_h rows, q
  float4 rr[8];
  uint2 wv[NBB];
#pragma unroll
  for (int k = 0; k < 8; ++k) rr[k] = __ldg(reinterpret_cast<const float4*>(Rh + (long long)(warp * 8 + k) * D) + lane);
#pragma unroll
  for (int bb = 0; bb < NBB; ++bb)
    wv[bb] = bb < bpw ? __ldg(reinterpret_cast<const uint2*>(Wh + (long long)(warp * bpw + bb) * D) + lane)
                      : make_uint2(0u, 0u);
  for (int i = tid; i < G * D; i += FZ_CONS) qf[i] = __bfloat162float(qg[i]);
  if (tid < 64) s.qc[tid] = 0u;
  cons_sync();
  float qv[G][4];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float4 t = *reinterpret_cast<const float4*>(qf + g * D + 4 * lane);
    qv[g][0] = t.x; qv[g][1] = t.y; qv[g][2] = t.z; qv[g][3] = t.w;
  }
  {
    constexpr int NV = 8 * GP, KP = NV / 32;
    float v[NV];
#pragma unroll
    for (int k = 0; k < 8; ++k)
#pragma unroll
      for (int g = 0; g < GP; ++g) v[k * GP + g] = (g < G) ? dot4(rr[k], qv[g]) : 0.f;
    warp_reduce_t<NV>(v, lane);
#pragma unroll
    for (int e = 0; e < KP; ++e) {
      const int vi = KP * lane + e;
      const int k = vi / GP, g = vi % GP;
      if (g < G) {
        const int i = warp * 8 + k;
        s.qs[g * D + qpos(i)] = v[e];
        if (write_dbg && p.dbg.q_rot) p.dbg.q_rot[((long long)x.b * dm.Hq + x.h * G + g) * D + i] = v[e];
      }
    }
  }
  // query codes: warp w takes bits [w nb/16, (w+1) nb/16) in blocks of NBB
  for (int jb = 0; jb < bpw; jb += NBB) {
    float v[2 * NBB * GP];
    if (jb > 0) {
#pragma unroll
      for (int bb = 0; bb < NBB; ++bb) {
        const int j = warp * bpw + jb + bb;
        wv[bb] = (jb + bb < bpw) ? __ldg(reinterpret_cast<const uint2*>(Wh + (long long)j * D) + lane)
                                 : make_uint2(0u, 0u);
      }
    }
#pragma unroll
    for (int bb = 0; bb < NBB; ++bb) {
      const float w4[4] = {bf_lo(wv[bb].x), bf_hi(wv[bb].x), bf_lo(wv[bb].y), bf_hi(wv[bb].y)};
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        float a = 0.f, m = 0.f;
        if (g < G) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float pe = w4[e] * qv[g][e];
            a += pe;
            m += fabsf(pe);
          }
        }
        v[(bb * GP + g) * 2 + 0] = a;
        v[(bb * GP + g) * 2 + 1] = m;
      }
    }
    warp_reduce_t<2 * NBB * GP>(v, lane);
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
      if (bit) atomicOr(&s.qc[g * 8 + j / 32], 1u << (j % 32));
    }
  }
  cons_sync();
  if (write_dbg && p.dbg.q_codes) {
    const int w32 = dm.words * 2;
    if (tid < G * w32) {
      const int g = tid / w32, k = tid - g * w32;
      reinterpret_cast<uint32_t*>(p.dbg.q_codes)[((long long)x.b * dm.Hq + x.h * G + g) * w32 + k] = s.qc[g * 8 + k];
    }
  }
}

// ---- SCAN: bounds of up to 128 pages of the CTA's share ----
// As the fused kernel's scan (half a warp per page, lane: 8 channels), with
// the ring layout of the group kernel: page j of the step in slot
// sb + j / 32, its minima at row j % 32 and its maxima half a slot further.
template <int G>
__device__ void gp_scan(const FzParams& p, const GpShared& s, const Unit& x, int pg0, int n, int sb) {
  constexpr int GP = G <= 4 ? 4 : 8;
  constexpr bool SPLIT = G <= 4;
  constexpr int PB = GP == 4 ? 4 : 2;
  constexpr int NBT = 4 / PB;
  constexpr int NV = PB * GP;
  const Dims& dm = p.dm;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int hw = lane >> 4, li = lane & 15;
  float2 qa[G][4], qb[G][4];
#pragma unroll
  for (int g = 0; g < G; ++g) {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const float4 t = *reinterpret_cast<const float4*>(s.qs + g * D + 4 * (li + 16 * k));
      if constexpr (SPLIT) {
        qa[g][2 * k] = make_float2(fmaxf(t.x, 0.f), fmaxf(t.y, 0.f));
        qa[g][2 * k + 1] = make_float2(fmaxf(t.z, 0.f), fmaxf(t.w, 0.f));
        qb[g][2 * k] = make_float2(fminf(t.x, 0.f), fminf(t.y, 0.f));
        qb[g][2 * k + 1] = make_float2(fminf(t.z, 0.f), fminf(t.w, 0.f));
      } else {
        qa[g][2 * k] = make_float2(t.x, t.y);
        qa[g][2 * k + 1] = make_float2(t.z, t.w);
      }
    }
  }
  const int pl = li / GP, hidx = li % GP;
#pragma unroll
  for (int bt = 0; bt < NBT; ++bt) {
    float v[NV];
#pragma unroll
    for (int pp = 0; pp < PB; ++pp) {
      const int j = warp * 8 + hw * 4 + bt * PB + pp;
      const unsigned char* slot = s.ring + (size_t)((sb + j / GP_PAGES_PER_SLOT) % FZ_NSLOT) * FZ_SLOT;
      const size_t off = (size_t)(j % GP_PAGES_PER_SLOT) * 256 + li * 16;
      const uint4 mnv = *reinterpret_cast<const uint4*>(slot + off);
      const uint4 mxv = *reinterpret_cast<const uint4*>(slot + FZ_SLOT / 2 + off);
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
        float sum = 0.f;
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
          sum = (a0.x + a0.y) + (a1.x + a1.y);
        }
        v[pp * GP + g] = sum;
      }
    }
    group_reduce_t<NV, 16>(v, lane);
    float U = hidx < G ? v[0] : -INFINITY;
#pragma unroll
    for (int o = 1; o < GP; o <<= 1) U = fmaxf(U, __shfl_xor_sync(0xffffffffu, U, o));
    const int j = warp * 8 + hw * 4 + bt * PB + pl;
    if (j < n) {
      const int pg = pg0 + j;
      if (hidx == 0) {
        p.wk.U[(long long)x.u * p.wk.Ustride + pg] = U;
        if (p.dbg.page_U) p.dbg.page_U[(long long)x.u * dm.np_max + pg] = U;
      }
      if (p.dbg.page_ub && hidx < G)
        p.dbg.page_ub[((long long)x.b * dm.Hq + x.h * G + hidx) * dm.np_max + pg] = v[0];
    }
  }
}


// ---- page top-N of the unit (larger bound first, ties to the lower page) ----
// Every CTA of the group runs the same select on the unit's bounds (written
// by the group's scans, read from L2), so all of them know every kept page
// without another exchange.  Thread t holds the bounds of pages
// [16 t, 16 t + 16) in registers.  A level bins the undecided pages over
// their value range into 2048 bins (monotone bin), keeps every bin above the
// one holding the need-th largest and descends into that bin; a bin of at
// most 512 pages is ranked exactly (larger bound first, then the lower page),
// a bin of equal bounds (or one still crowded after four levels) is taken in
// page order.  Writes the kept pages (ascending) to GW_KP; returns N.
static __device__ int gp_psel_all(const FzParams& p, const GpShared& s, const Unit& x, int N, bool write_dbg) {
  const Work& wk = p.wk;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  unsigned char* w = s.work;
  int* hist = reinterpret_cast<int*>(w + GW_HIST);
  int* cand = reinterpret_cast<int*>(w + GW_CAND);              // int [512]
  float* candv = reinterpret_cast<float*>(w + GW_CAND + 2048);  // float [512]
  unsigned* flag = reinterpret_cast<unsigned*>(w + GW_FLAG);
  int* red = reinterpret_cast<int*>(w + GW_RED);  // scan buffers of 16 at 0, 16, 32, 48, 64; broadcasts at 128
  int* bc = red + 128;
  float* wr = reinterpret_cast<float*>(red + 160);
  int* kp = reinterpret_cast<int*>(w + GW_KP);
  const int np = x.np;
  const int i0 = tid * PS_PER;
  const int cnt = max(0, min(PS_PER, np - i0));
  unsigned member = (1u << cnt) - 1u;
  unsigned keep = 0u;
  if (N >= np) {
    keep = member;
  } else {
    const float* Ug = wk.U + (long long)x.u * wk.Ustride;
    float v[PS_PER];
#pragma unroll
    for (int k4 = 0; k4 < PS_PER / 4; ++k4) {
      const float4 t = i0 + 4 * k4 < np ? __ldcg(reinterpret_cast<const float4*>(Ug + i0) + k4)
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
      v[4 * k4 + 0] = t.x; v[4 * k4 + 1] = t.y; v[4 * k4 + 2] = t.z; v[4 * k4 + 3] = t.w;
    }
    for (int i = tid; i < SEL_NBIN; i += FZ_CONS) hist[i] = 0;
    if (tid < MAX_SELECT_PAGES / 32) flag[tid] = 0u;
    if (tid == 0) bc[4] = 0;
    float lo = INFINITY, hi = -INFINITY;
#pragma unroll
    for (int k = 0; k < PS_PER; ++k)
      if ((member >> k) & 1u) {
        lo = fminf(lo, v[k]);
        hi = fmaxf(hi, v[k]);
      }
    cons_minmax(lo, hi, wr);
    int need = N, nbin = 0;
    bool tie = false;
#pragma unroll 1
    for (int level = 0; level < GP_LEVELS; ++level) {
      tie = !(hi > lo);
      if (tie) break;
      const float scale = (float)SEL_NBIN / (hi - lo);
      if (level > 0) {
        for (int i = tid; i < SEL_NBIN; i += FZ_CONS) hist[i] = 0;
        cons_sync();
      }
      int bn[PS_PER];
#pragma unroll
      for (int k = 0; k < PS_PER; ++k) {
        bn[k] = value_bin(v[k], lo, scale);
        if ((member >> k) & 1u) atomicAdd(&hist[bn[k]], 1);
      }
      cons_sync();
      {
        constexpr int BPT = SEL_NBIN / FZ_CONS;  // 4 bins per thread, counted from the top
        int hv[BPT];
        int c4 = 0;
#pragma unroll
        for (int e = 0; e < BPT; ++e) {
          hv[e] = hist[SEL_NBIN - 1 - (tid * BPT + e)];
          c4 += hv[e];
        }
        int tot;
        const int before = cons_scan1(c4, red + 16 * (level & 1), &tot);
        if (before < need && before + c4 >= need) {
          int run = before;
#pragma unroll
          for (int e = 0; e < BPT; ++e) {
            if (run < need && run + hv[e] >= need) {
              bc[0] = SEL_NBIN - 1 - (tid * BPT + e);
              bc[1] = need - run;
              bc[2] = hv[e];
            }
            run += hv[e];
          }
        }
        cons_sync();
      }
      const int bstar = bc[0];
      need = bc[1];
      nbin = bc[2];
      float nlo = INFINITY, nhi = -INFINITY;
#pragma unroll
      for (int k = 0; k < PS_PER; ++k) {
        const bool m = (member >> k) & 1u;
        const bool at = m && bn[k] == bstar;
        keep |= (m && bn[k] > bstar) ? 1u << k : 0u;
        member &= at ? ~0u : ~(1u << k);
        nlo = at ? fminf(nlo, v[k]) : nlo;
        nhi = at ? fmaxf(nhi, v[k]) : nhi;
      }
      // a small bin is ranked exactly; a larger one is refined (ranking costs nbin^2)
      if (nbin <= SEL_RANK_SMALL || (nbin <= SEL_MAX_CAND && level == GP_LEVELS - 1)) break;
      cons_minmax(nlo, nhi, wr);
      lo = nlo;
      hi = nhi;
    }
    if (tie || nbin > SEL_MAX_CAND) {
      // equal bounds (or still crowded): members in page order, the first `need`
      const int m = __popc(member);
      int tot;
      const int mb = cons_scan1(m, red + 32, &tot);
      int take = max(0, min(m, need - mb));
#pragma unroll
      for (int k = 0; k < PS_PER; ++k) {
        if (((member >> k) & 1u) && take > 0) {
          keep |= 1u << k;
          --take;
        }
      }
    } else {
      // exact ranking of the (few) members: larger bound first, then lower page
#pragma unroll
      for (int k = 0; k < PS_PER; ++k)
        if ((member >> k) & 1u) {
          const int at = atomicAdd(&bc[4], 1);
          cand[at] = i0 + k;
          candv[at] = v[k];
        }
      cons_sync();
      for (int a = tid; a < nbin; a += FZ_CONS) {
        const int ia = cand[a];
        const float va = candv[a];
        int rank = 0;
        for (int b2 = 0; b2 < nbin; ++b2) {
          const float vb = candv[b2];
          rank += (vb > va) || (vb == va && cand[b2] < ia);
        }
        if (rank < need) atomicOr(&flag[ia >> 5], 1u << (ia & 31));
      }
      cons_sync();
      const unsigned fw = flag[i0 >> 5] >> (i0 & 31);  // the thread's 16 pages share one flag word
      keep |= member & fw & 0xffffu;
    }
  }
  int nkp;
  int pos = cons_scan1(__popc(keep), red + 64, &nkp);
  int* dsel = (write_dbg && p.dbg.sel_pages) ? p.dbg.sel_pages + (long long)x.u * wk.Nmax : nullptr;
#pragma unroll
  for (int k = 0; k < PS_PER; ++k)
    if ((keep >> k) & 1u) {
      kp[pos] = i0 + k;
      if (dsel) dsel[pos] = i0 + k;
      ++pos;
    }
  if (write_dbg && tid == 0 && p.dbg.n_sel_pages) p.dbg.n_sel_pages[x.u] = nkp;
  (void)lane;
  (void)warp;
  cons_sync();
  return nkp;
}

// ---- Hamming scores and key top-k of the unit (smaller score first, ties
// to the lower row), one group barrier ----
// Candidates are the rows of the kept pages in page order; CTA r scores the
// balanced share [cs0, cs1) and publishes the histogram of its integer scores
// (G nb + 1 bins).  After the barrier every CTA reads the S histograms: their
// sum gives the threshold T and the ties taken at T; the histograms of the
// CTAs before r give r's place in the row list (rows below T of lower CTAs,
// plus their ties, which go to the lower rows first).  The CTA writes its kept
// rows there as row + 1 (0 = not yet written), so that the gather of a chunk
// polls only the entries it needs.  Returns k_eff.
template <int G, int WORDS>
__device__ int gp_ksel(const FzParams& p, const GpShared& s, const Unit& x, int r, int nkp, unsigned* gx,
                       unsigned& epoch, bool& ok) {
  const Dims& dm = p.dm;
  const Work& wk = p.wk;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int S = p.gsize;
  unsigned char* w = s.work;
  int* hist = reinterpret_cast<int*>(w + GW_HIST);
  int* red = reinterpret_cast<int*>(w + GW_RED);
  int* bc = red + 128;
  const int* kp = reinterpret_cast<const int*>(w + GW_KP);
  uint16_t* sc = reinterpret_cast<uint16_t*>(w + GW_SC);
  int* hm = reinterpret_cast<int*>(s.ring);         // the S histograms [S][HB] (the ring is idle here)
  int* ltc = reinterpret_cast<int*>(w + GW_CAND);   // [S] rows below T per CTA
  const int nbins = G * dm.nb + 1;
  const int HB = wk.HB;
  const int ncs = nkp << dm.lgP;
  int cs0, cs1;
  share_of(ncs, S, r, cs0, cs1);
  const int nmy = cs1 - cs0;
  for (int i = tid; i < nbins; i += FZ_CONS) hist[i] = 0;
  uint64_t cq[G][WORDS];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int w2 = 0; w2 < WORDS; ++w2)
      cq[g][w2] = (uint64_t)s.qc[g * 8 + 2 * w2] | ((uint64_t)s.qc[g * 8 + 2 * w2 + 1] << 32);
  // ---- scores of the CTA's share: the code rows are staged in the (idle)
  // ring by cp.async, all in flight at once, then scored from shared memory ----
  const int cap = (FZ_NSLOT * FZ_SLOT) / (WORDS * 8);
  unsigned char* cstage = s.ring;
  for (int jb = 0; jb < nmy; jb += cap) {
    const int nbt = min(cap, nmy - jb);
    for (int j = tid; j < nbt; j += FZ_CONS) {
      const int ci = cs0 + jb + j;
      const int t = (kp[ci >> dm.lgP] << dm.lgP) + (ci & (dm.P - 1));
      const long long woff = t < x.L ? code_row(dm, p.table, x.b, x.h, t, p.status) : -1;
      sc[jb + j] = woff >= 0 ? 0 : 0xFFFF;
      if (woff >= 0) {
        const uint64_t* src = p.codes + woff;
        if constexpr (WORDS == 1) {
          asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(cstage + j * 8)), "l"(src) : "memory");
        } else {
#pragma unroll
          for (int w2 = 0; w2 < WORDS; w2 += 2) cp_async16(cstage + (j * WORDS + w2) * 8, src + w2);
        }
      }
    }
    cp_async_commit();
    cp_async_wait<0>();
    cons_sync();
    for (int j = tid; j < nbt; j += FZ_CONS) {
      if (sc[jb + j] == 0xFFFF) continue;
      const uint64_t* cw = reinterpret_cast<const uint64_t*>(cstage + j * WORDS * 8);
      int sv = 0;
#pragma unroll
      for (int w2 = 0; w2 < WORDS; ++w2) {
        const uint64_t c = cw[w2];
#pragma unroll
        for (int g = 0; g < G; ++g) sv += __popcll(c ^ cq[g][w2]);
      }
      sc[jb + j] = (uint16_t)sv;
    }
    cons_sync();
  }
  cons_sync();  // scores complete, histogram zero
  for (int j = tid; j < nmy; j += FZ_CONS) {
    const int sv = sc[j];
    if (sv != 0xFFFF) atomicAdd(&hist[sv], 1);
  }
  cons_sync();
  // publish the CTA's histogram (one slot per CTA of the grid)
  int* myh = wk.khist + (long long)blockIdx.x * HB;
  for (int i = tid; i < nbins; i += FZ_CONS) myh[i] = hist[i];
  if (p.dbg.key_scores) {
    int* dsc = p.dbg.key_scores + (long long)x.u * wk.Nmax * dm.P + cs0;
    for (int j = tid; j < nmy; j += FZ_CONS) {
      const int sv = sc[j];
      dsc[j] = sv == 0xFFFF ? INT_MAX : sv;
    }
  }
  if (!gp_sync(p, s, gx, epoch)) {
    ok = false;
    return 0;
  }
  // ---- the group's histograms: sum, threshold T, ties ----
  const int* gh0 = wk.khist + (long long)(blockIdx.x - r) * HB;
  for (int i = tid; i < S * HB / 4; i += FZ_CONS) cp_async16(hm + 4 * i, gh0 + 4 * i);  // all in flight
  cp_async_commit();
  cp_async_wait<0>();
  cons_sync();
  for (int b = tid; b < nbins; b += FZ_CONS) {
    int t = 0;
    for (int rr = 0; rr < S; ++rr) t += hm[rr * HB + b];
    hist[b] = t;
  }
  if (tid == 0) {
    bc[0] = -1;  // no candidate: nothing is kept
    bc[1] = 0;
  }
  cons_sync();
  const int bpt = (nbins + FZ_CONS - 1) / FZ_CONS;  // <= 5
  int hv[5];
  int local = 0;
#pragma unroll
  for (int e = 0; e < 5; ++e) {
    const int bi = tid * bpt + e;
    hv[e] = (e < bpt && bi < nbins) ? hist[bi] : 0;
    local += hv[e];
  }
  int n_cand;
  const int before = cons_scan1(local, red + 16, &n_cand);
  const int tk = __ldg(p.top_k + x.b);
  const int keff = min(min(max(tk, 1), wk.Kmax), n_cand);
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
  cons_sync();
  const int T = bc[0], need_eq = bc[1];
  // rows below T of each CTA (warp w: CTAs w, w + 16, ...)
  for (int rr = warp; rr < S; rr += FZ_CWARPS) {
    int c = 0;
    for (int b = lane; b < T; b += 32) c += hm[rr * HB + b];
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    if (lane == 0) ltc[rr] = c;
  }
  cons_sync();
  if (tid == 0) {
    int lt_before = 0, eq_before = 0;
    for (int rr = 0; rr < r; ++rr) {
      lt_before += ltc[rr];
      eq_before += T >= 0 ? hm[rr * HB + T] : 0;
    }
    bc[3] = lt_before + min(need_eq, eq_before);     // the CTA's first place in the list
    bc[4] = max(0, need_eq - eq_before);             // ties it may take
  }
  if (r == 0 && tid == 0) {
    if (p.dbg.n_sel_pages) p.dbg.n_sel_pages[x.u] = nkp;
    if (p.dbg.n_cand) p.dbg.n_cand[x.u] = n_cand;
    if (p.dbg.n_sel_keys) p.dbg.n_sel_keys[x.u] = keff;
  }
  cons_sync();
  const int off = bc[3], take = bc[4];
  // ---- the CTA's kept rows in candidate order: warp w owns candidates
  // [w nbw, (w+1) nbw) of the share in rounds of 32; counts per warp, one
  // scan, then ballots place the rows ----
  const int rounds = (nmy + 32 * FZ_CWARPS - 1) / (32 * FZ_CWARPS);
  const int cw0 = warp * rounds * 32;
  const unsigned lanemask_lt = (1u << lane) - 1u;
  int lt_w = 0, eq_w = 0;
  for (int rr = 0; rr < rounds; ++rr) {
    const int j = cw0 + 32 * rr + lane;
    const int sv = j < nmy ? (int)sc[j] : 0xFFFF;
    lt_w += __popc(__ballot_sync(0xffffffffu, sv < T));
    eq_w += __popc(__ballot_sync(0xffffffffu, sv == T));
  }
  int totw;
  const int pk = cons_scan1(lane == 0 ? (lt_w << 16) | eq_w : 0, red + 96, &totw);
  int lt_b = __shfl_sync(0xffffffffu, pk, 0) >> 16, eq_b = __shfl_sync(0xffffffffu, pk, 0) & 0xFFFF;
  int* out = wk.sel_keys + (long long)x.u * wk.Kmax + off;
  int* dout = p.dbg.sel_keys ? p.dbg.sel_keys + (long long)x.u * wk.Kmax + off : nullptr;
  const int room = keff - off;
  for (int rr = 0; rr < rounds; ++rr) {
    const int j = cw0 + 32 * rr + lane;
    const int sv = j < nmy ? (int)sc[j] : 0xFFFF;
    const bool l1 = sv < T, e1 = sv == T;
    const unsigned blt = __ballot_sync(0xffffffffu, l1), beq = __ballot_sync(0xffffffffu, e1);
    const int eq_before = eq_b + __popc(beq & lanemask_lt);
    const bool tk1 = l1 || (e1 && eq_before < take);
    const int pos = lt_b + __popc(blt & lanemask_lt) + min(eq_before, take);
    if (tk1 && pos < room) {
      const int ci = cs0 + j;
      const int t = (kp[ci >> dm.lgP] << dm.lgP) + (ci & (dm.P - 1));
      out[pos] = t + 1;
      if (dout) dout[pos] = t;
    }
    lt_b += __popc(blt);
    eq_b += __popc(beq);
  }
  return keff;
}

// Consumers copy the K'/V rows of one gather step into four ring slots:
// warp w the rows 8w .. 8w+7 (K' row j in slot sb + j / 64, V row j two
// slots further).  The 16-byte chunk q of row j goes to chunk q ^ (j & 7) of
// its 256-byte row, so that eight consecutive rows' same chunk fall in
// distinct banks for ldmatrix.  Rows at or past n and bad rows read as zeros
// (the tensor-core products then stay finite).  One cp.async group.
__device__ __forceinline__ void gp_gather_rows(unsigned char* ring, const int* ridx, int n, int sb,
                                               const __nv_bfloat16* K, const __nv_bfloat16* V) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int q = lane & 15;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int j = warp * 8 + 2 * i + (lane >> 4);
    const int off = (j % 64) * 256 + ((q ^ (j & 7)) * 16);
    unsigned char* d1 = ring + (size_t)(sb + j / 64) * FZ_SLOT + off;
    unsigned char* d2 = ring + (size_t)(sb + 2 + j / 64) * FZ_SLOT + off;
    const int r = j < n ? ridx[j] : -1;
    if (r >= 0) {
      cp_async16(d1, K + (long long)r * D + q * 8);
      cp_async16(d2, V + (long long)r * D + q * 8);
    } else {
      *reinterpret_cast<uint4*>(d1) = make_uint4(0u, 0u, 0u, 0u);
      *reinterpret_cast<uint4*>(d2) = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  cp_async_commit();
}

// ---- tensor-core helpers (mma.sync m16n8k16, bf16 in, fp32 accumulate) ----
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x2(uint32_t (&r)[2], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r[0]), "=r"(r[1]) : "r"(smem_u32(p)));
}
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
               "{%0,%1,%2,%3};"
               : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
               : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// x as bf16 hi + lo (hi = RNE(x), lo = RNE(x - hi)): |x - hi - lo| <= 2^-17 |x|
__device__ __forceinline__ void split_bf16(float x, __nv_bfloat16& hi, __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(x);
  lo = __float2bfloat16_rn(x - __bfloat162float(hi));
}

// gather scratch (consumer work area)
constexpr int GM_QB = 0;                 // bf16 [16 cols][136] q'^T operand (hi, lo), rows 272 B apart
constexpr int GM_PB = GM_QB + 16 * 272;  // bf16 [16 cols][136] P^T operand (hi, lo)
constexpr int GM_MX = GM_PB + 16 * 272;  // float [8 warps][8 heads] row-block maxima
constexpr int GM_LS = GM_MX + 256;       // float [8][8] row-block sums of weights
constexpr int GM_OB = GM_LS + 256;       // float [2 row halves][128 ch][16 cols] P.V partials
static_assert(GM_OB + 2 * 128 * 16 * 4 <= GP_WORK, "gather scratch");

// Column layout of the two operands: NT = 1 (G <= 4): columns 0-3 the heads'
// hi parts, 4-7 their lo parts; NT = 2 (G <= 8): 0-7 hi, 8-15 lo.
template <int G>
struct GCols {
  static constexpr int NT = G <= 4 ? 1 : 2;
  static constexpr int HP = 4 * NT;  // heads padded
  __device__ static int hi(int h) { return h; }
  __device__ static int lo(int h) { return HP + h; }
};

// q' of the unit, scaled to log2 units, as the hi/lo bf16 operand of the logits.
template <int G>
__device__ void gp_build_qb(const FzParams& p, const GpShared& s) {
  using C = GCols<G>;
  const float qscale = p.sm_scale * 1.4426950408889634f;
  __nv_bfloat16* qb = reinterpret_cast<__nv_bfloat16*>(s.work + GM_QB);
  for (int e = threadIdx.x; e < C::HP * D; e += FZ_CONS) {
    const int h = e / D, c = e - h * D;
    const float v = h < G ? s.qs[h * D + qpos(c)] * qscale : 0.f;
    __nv_bfloat16 hi, lo;
    split_bf16(v, hi, lo);
    qb[C::hi(h) * 136 + c] = hi;
    qb[C::lo(h) * 136 + c] = lo;
  }
}

// ---- one gather step: softmax attention over one chunk of up to 128 kept rows ----
// Logits S = K' (q' hi + lo)^T on tensor cores (warps 0-7, 16 rows each),
// the chunk's maximum and weights per head in fp32, then O^T = V^T (P hi + lo)^T
// on tensor cores (warp w: channels 16 (w & 7) .. +15 over rows 64 (w >> 3) .. +63),
// the two row halves added in order.  The chunk's partial (unnormalised output,
// maximum and sum of weights per head, in log2 units) goes to `part`; it depends
// only on the chunk's rows.
template <int G>
__device__ void gp_gather_step(const FzParams& p, const GpShared& s, int n, int sb, float* part) {
  using C = GCols<G>;
  constexpr int NT = C::NT, HP = C::HP;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  unsigned char* w = s.work;
  const unsigned char* qb = w + GM_QB;
  __nv_bfloat16* pb = reinterpret_cast<__nv_bfloat16*>(w + GM_PB);
  float* mx = reinterpret_cast<float*>(w + GM_MX);
  float* ls = reinterpret_cast<float*>(w + GM_LS);
  float* ob = reinterpret_cast<float*>(w + GM_OB);
  cons_sync();  // every warp's rows have landed (each thread waited for its own copies)
  // ---- logits: warp w < 8 takes rows 16w .. 16w+15 ----
  float sv[2][2];  // [row g / g+8][head pair element]
  int h0 = 0;      // first head of this thread's pair
  if (warp < 8) {
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
    const int r0 = warp * 16;
    const int arow = r0 + (lane & 7) + ((lane >> 3) & 1) * 8;  // A: this lane's row address
    const unsigned char* krow = s.ring + (size_t)(sb + arow / 64) * FZ_SLOT + (arow % 64) * 256;
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
  cons_sync();
  // ---- weights p = 2^(s - M) per head, their sums, P^T as hi / lo ----
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
  cons_sync();
  // ---- O^T = V^T P^T: warp w: channels 16 (w & 7) .., rows 64 (w >> 3) .. ----
  {
    const int mt = warp & 7, kh = warp >> 3;
    float oacc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) oacc[nt][0] = oacc[nt][1] = oacc[nt][2] = oacc[nt][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      const int k0 = kh * 64 + ks * 16;
      const int vrow = k0 + (lane & 7) + 8 * (lane >> 4);  // matrices 2, 3: rows k0 + 8 ..
      const int vch = 2 * mt + ((lane >> 3) & 1);           // matrices 1, 3: channels + 8
      uint32_t af[4];
      ldsm_x4_t(af, s.ring + (size_t)(sb + 2 + vrow / 64) * FZ_SLOT + (vrow % 64) * 256 + ((vch ^ (vrow & 7)) * 16));
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        uint32_t bf[2];
        ldsm_x2(bf, reinterpret_cast<const unsigned char*>(pb) + (nt * 8 + (lane & 7)) * 272 +
                        (k0 / 8 + ((lane >> 3) & 1)) * 16);
        mma_bf16(oacc[nt], af, bf);
      }
    }
    // rows 16 mt + g (+8) are channels; columns 8 nt + 2t, +1
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int c0 = 16 * mt + g, col = 8 * nt + 2 * t;
      *reinterpret_cast<float2*>(ob + ((kh * 128 + c0) * 16 + col)) = make_float2(oacc[nt][0], oacc[nt][1]);
      *reinterpret_cast<float2*>(ob + ((kh * 128 + c0 + 8) * 16 + col)) = make_float2(oacc[nt][2], oacc[nt][3]);
    }
  }
  cons_sync();
  // ---- the chunk's partial: o[h][c] = sum over the row halves of hi + lo columns ----
  for (int e = tid; e < G * D; e += FZ_CONS) {
    const int h = e / D, c = e - h * D;
    const float* o0 = ob + c * 16;
    const float* o1 = ob + (128 + c) * 16;
    part[h * D + c] = (o0[C::hi(h)] + o0[C::lo(h)]) + (o1[C::hi(h)] + o1[C::lo(h)]);
  }
  if (tid < G) {
    float M = -INFINITY, L = 0.f;
#pragma unroll
    for (int w2 = 0; w2 < 8; ++w2) M = fmaxf(M, mx[w2 * 8 + tid]);
#pragma unroll
    for (int w2 = 0; w2 < 8; ++w2) L += ls[w2 * 8 + tid];
    part[G * D + tid] = M;
    part[G * D + 8 + tid] = L;
  }
  (void)HP;
  cons_sync();  // the step's scratch and slots are free
}

// ---------------------------------------------------------------------------
// consumer warps 0-15: the units of the group, one after another
// ---------------------------------------------------------------------------
template <int G, int WORDS>
__device__ void gp_consumer(const FzParams& p, const GpShared& s, int g, int r) {
  const Dims& dm = p.dm;
  const Work& wk = p.wk;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int U = dm.B * dm.Hkv, S = p.gsize;
  const int PS = G * D + 16;
  volatile int* misc = s.misc;
  unsigned nslot = 0, nunit = 0;
  for (int u = g; u < U; u += p.ngroups) {
    Unit x;
    x.u = u;
    x.b = u / dm.Hkv;
    x.h = u - x.b * dm.Hkv;
    x.L = seq_len_of(dm, p.seq_lens, x.b);
    x.np = (x.L + dm.P - 1) >> dm.lgP;
    unsigned* gx = gx_of(p, u);
    unsigned epoch = 0;
    bool ok = true;
    // the unit's budgets, loaded now (their latency hides behind the prep and the scan)
    const int nk_b = __ldg(p.n_keep + x.b), tk_b = __ldg(p.top_k + x.b);
    gp_prep<G>(p, s, x, r == 0);  // (q' and the query codes are stage outputs even for an empty sequence)
    if (x.L == 0) {
      if (r == 0) {
        for (int e = tid; e < G * D; e += FZ_CONS) p.out[((long long)x.b * dm.Hq + x.h * G) * D + e] = 0.f;
        if (tid == 0) {
          if (p.dbg.n_sel_pages) p.dbg.n_sel_pages[x.u] = 0;
          if (p.dbg.n_sel_keys) p.dbg.n_sel_keys[x.u] = 0;
          if (p.dbg.n_cand) p.dbg.n_cand[x.u] = 0;
        }
      }
    } else {
      // ---- scan of the CTA's pages, 128 per step ----
      int p0, p1;
      share_of(x.np, S, r, p0, p1);
      const int nr = p1 - p0;
      for (int j = 0; j < nr; j += FZ_ROWS) {
        const int n = min(FZ_ROWS, nr - j), nsl = (n + GP_PAGES_PER_SLOT - 1) / GP_PAGES_PER_SLOT;
        if (tid == 0) {
          int good = 1;
          for (int k = 0; k < nsl && good; ++k) {
            const unsigned gs = nslot + k;
            if (!gp_wait(s, &s.full[gs % FZ_NSLOT], (gs / FZ_NSLOT) & 1, p.status)) good = 0;
          }
          misc[17] = good;
        }
        cons_sync();
        if (!misc[17]) {
          ok = false;
          break;
        }
        gp_scan<G>(p, s, x, p0 + j, n, (int)(nslot % FZ_NSLOT));
        cons_sync();
        if (tid == 0)
          for (int k = 0; k < nsl; ++k) mbar_arrive(&s.empty[(nslot + k) % FZ_NSLOT]);
        nslot += nsl;
      }
      // ---- the group's bounds are complete: one group barrier ----
      if (ok) ok = gp_sync(p, s, gx, epoch);
      // ---- selects, the same in every CTA of the group ----
      int nkp = 0, keff = 0, k0 = 0, k1 = 0;
      if (ok) {
        const int N = min(min(max(nk_b, 1), wk.Nmax), x.np);
        nkp = gp_psel_all(p, s, x, N, r == 0);
        // L2 prefetches for the producer warp: this CTA's share of the kept
        // pages' code rows, and (when every candidate row will be kept) the
        // K'/V rows of the pages its own chunks will gather
        const bool pf_kv = min(max(tk_b, 1), wk.Kmax) >= nkp * dm.P;
        if (tid == 0) {
          int a0, a1;
          share_of(nkp, S, r, a0, a1);
          const int n1 = min(a1 - a0, GP_PF_MAX);
          int n2 = 0, b0 = 0;
          if (pf_kv) {
            const int nch = (nkp * dm.P + FZ_ROWS - 1) / FZ_ROWS;
            int c0, c1;
            share_of(nch, S, r, c0, c1);
            b0 = (c0 * FZ_ROWS) >> dm.lgP;
            n2 = min(min(nkp, (c1 * FZ_ROWS) >> dm.lgP) - b0, GP_PF_MAX - n1);
            n2 = max(n2, 0);
          }
          misc[22] = n1;
          misc[23] = n2;
          misc[24] = a0;
          misc[25] = b0;
        }
        cons_sync();
        {
          const int n1 = misc[22], n2 = misc[23], a0 = misc[24], b0 = misc[25];
          for (int i = tid; i < n1 + n2; i += FZ_CONS) s.pf[i] = i < n1 ? s.kpw[a0 + i] : s.kpw[b0 + i - n1];
        }
        cons_sync();
        if (tid == 0) {
          __threadfence_block();
          misc[21] = (int)nunit + 1;
        }
        keff = gp_ksel<G, WORDS>(p, s, x, r, nkp, gx, epoch, ok);
        const int nch = (keff + FZ_ROWS - 1) / FZ_ROWS;
        int c0, c1;
        share_of(nch, S, r, c0, c1);
        k0 = c0 * FZ_ROWS;
        k1 = min(keff, c1 * FZ_ROWS);
      }
      if (ok) {
        // ---- attention over the CTA's chunks of 128 kept rows ----
        const int nch = (keff + FZ_ROWS - 1) / FZ_ROWS;
        const int c0 = k0 / FZ_ROWS;
        const int nrow = k1 - k0, nst = (nrow + FZ_ROWS - 1) / FZ_ROWS;
        const int* keys = wk.sel_keys + (long long)x.u * wk.Kmax + k0;
        float* parts = wk.part + (long long)x.u * wk.C3 * PS;
        // row numbers of step i, warp w: rows 8w .. 8w+7 (the rows it copies).
        // A list entry holds row + 1 once written (polled, bounded); it is
        // cleared after reading for the next call.
        // (with two steps, lanes 8-15 poll the entries of step i + 1 into rx + FZ_ROWS at once)
        auto rows_of = [&](int i, int* rx, bool two) {
          if (lane < (two ? 16 : 8)) {
            const int st = lane >> 3;
            const int j = warp * 8 + (lane & 7), jj = (i + st) * FZ_ROWS + j;
            if (st) rx = s.ridx + ((i + 1) & 1) * FZ_ROWS;
            if (jj < nrow) {
              int* e = const_cast<int*>(keys) + jj;
              int t1 = ld_relaxed32(e);
              if (t1 == 0) {
                const long long w0 = clock64();
                while ((t1 = ld_relaxed32(e)) == 0) {
                  if (misc[0]) break;
                  if (clock64() - w0 > FZ_WAIT_CYCLES) {
                    set_status(p.status, HHR_ERR_TIMEOUT);
                    misc[0] = 1;
                    break;
                  }
                }
              }
              *e = 0;
              const long long off = t1 > 0 ? kv_row(dm, p.table, x.b, x.h, t1 - 1, p.status) : -1;
              rx[j] = off >= 0 ? (int)(off / D) : -1;
            }
          }
          __syncwarp();
        };
        gp_build_qb<G>(p, s);  // (ordered before the first step by its barrier)
        if (nst > 0) {  // the first two steps' row lists are polled together
          rows_of(0, s.ridx, nst > 1);
          gp_gather_rows(s.ring, s.ridx, min(FZ_ROWS, nrow), 0, p.Kr, p.Vc);
          if (nst > 1) gp_gather_rows(s.ring, s.ridx + FZ_ROWS, min(FZ_ROWS, nrow - FZ_ROWS), 4, p.Kr, p.Vc);
        }
        for (int i = 0; i < nst; ++i) {
          const int n = min(FZ_ROWS, nrow - i * FZ_ROWS);
          if (i + 1 < nst) {
            if (i >= 1) {
              int* rx = s.ridx + ((i + 1) & 1) * FZ_ROWS;
              rows_of(i + 1, rx, false);
              gp_gather_rows(s.ring, rx, min(FZ_ROWS, nrow - (i + 1) * FZ_ROWS), 4 * ((i + 1) & 1), p.Kr, p.Vc);
            }
            cp_async_wait<1>();
          } else {
            cp_async_wait<0>();
          }
          __syncwarp();
          gp_gather_step<G>(p, s, n, 4 * (i & 1), parts + (long long)(c0 + i) * PS);
        }
        // ---- the last CTA of the group merges the unit's chunk partials in chunk order ----
        if (tid == 0) {
          int last = 1;
          if (S > 1) last = atom_add_acq_rel(gx + GX_ARRIVE, 1u) == (unsigned)(S - 1);
          misc[18] = last;
        }
        cons_sync();
        if (misc[18]) {
          merge_partials<G>(s.work, parts, nch, nullptr, p.out + ((long long)x.b * dm.Hq + x.h * G) * D);
          // the unit's counters are zero again for the next call
          if (tid == 0) {
            gx[GX_BAR] = 0u;
            gx[GX_ARRIVE] = 0u;
          }
        }
      }
    }
    if (!ok) break;
    // the ring is free for the producer's next unit
    cons_sync();
    ++nunit;
    if (tid == 0) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      misc[20] = (int)nunit;
    }
  }
  cp_async_wait<0>();
  if (tid == 0) misc[1] = (int)nslot;
}

template <int G, int WORDS>
__global__ void __launch_bounds__(FZ_THREADS, 1) hhr_group_kernel(FzParams p) {
  extern __shared__ __align__(128) unsigned char gp_smem[];
  const GpShared s = gp_shared(gp_smem);
  const int tid = threadIdx.x;
  if (tid == 0) {
    for (int i = 0; i < FZ_NSLOT; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < 32; ++i) s.misc[i] = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const int g = blockIdx.x / p.gsize, r = blockIdx.x - g * p.gsize;
  const int warp = tid >> 5;
  if (warp >= FZ_CWARPS) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(FZ_REGS_AUX));
    if (warp == FZ_PRODUCER_WARP) gp_producer(p, s, g, r);
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(FZ_REGS_CONS));
    gp_consumer<G, WORDS>(p, s, g, r);
  }
  __syncthreads();
  // drain metadata copies that were armed but never consumed (only after an abort)
  if (tid == 0) {
    const unsigned armed = (unsigned)s.misc[2], consumed = (unsigned)s.misc[1];
    for (unsigned gs = consumed; gs < armed; ++gs) {
      const long long t0 = clock64();
      while (!mbar_try_wait(&s.full[gs % FZ_NSLOT], (gs / FZ_NSLOT) & 1)) {
        if (clock64() - t0 > FZ_WAIT_CYCLES) break;
      }
    }
  }
}

template <int G, int WORDS>
static cudaError_t launch_group_t(const FzParams& prm, int grid, cudaStream_t st) {
  static bool configured[64] = {false};  // the attribute is per function and device
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    const cudaError_t e =
        cudaFuncSetAttribute(hhr_group_kernel<G, WORDS>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)GP_SMEM);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  hhr_group_kernel<G, WORDS><<<grid, FZ_THREADS, GP_SMEM, st>>>(prm);
  return cudaGetLastError();
}

// CTAs per group: the SMs shared out over the units, at most one CTA per 64
// pages of the longest sequence (a short unit gains nothing from more), and
// no more than the ring holds score histograms of.
inline void group_shape(const Dims& dm, int sms, int* S, int* ngroups) {
  const int U = dm.B * dm.Hkv;
  sms = std::max(1, std::min(sms, (int)GP_SMAX));
  int s = std::max(1, sms / U);
  s = std::min(s, std::max(1, dm.np_max / 64));
  // the key select holds the group's S score histograms in the ring
  const int HB = (dm.G * dm.nb + 1 + 7) / 8 * 8;
  s = std::min(s, std::max(1, (FZ_NSLOT * FZ_SLOT / 4) / HB));
  *S = s;
  *ngroups = std::max(1, std::min(U, sms / s));
}


static_assert(GX_WORDS == GROUP_GX_WORDS, "exchange area layout");

template <int G>
cudaError_t launch_decode(const DecodeArgs& a) {
  FzParams prm = make_params(a, false);
  int S = 1, ngroups = 1;
  group_shape(a.dm, a.num_sms, &S, &ngroups);
  prm.gsize = S;
  prm.ngroups = ngroups;
  const int grid = S * ngroups;
  switch (a.dm.words) {
    case 1: return launch_group_t<G, 1>(prm, grid, a.stream);
    case 2: return launch_group_t<G, 2>(prm, grid, a.stream);
    case 4: return launch_group_t<G, 4>(prm, grid, a.stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace hhr
