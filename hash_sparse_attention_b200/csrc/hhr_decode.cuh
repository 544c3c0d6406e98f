// HHR decode-step kernels (sm_100a).
//
// One decode step of one layer runs four kernels chained with programmatic
// dependent launch (each waits on its predecessor with griddepcontrol.wait
// only where it first reads the predecessor's output):
//   prep_query       q' = R_h q and the query sign codes          (GKR, LHP)
//   gkr_scan_select  page bounds over all pages, then the top-N pages;
//                    the last CTA of each (b, KV head) performs the select
//   lhp_score_select group Hamming distance of every candidate row, then
//                    the top-k rows; the last CTA of each (b, KV head) selects
//   attn_split       softmax attention split over the kept rows; the last
//                    CTA of each (b, KV head) merges the split partials
// "Last CTA" is decided by an atomic arrival ticket; nothing ever waits on
// another CTA, so no kernel can hang on a missing arrival.
#pragma once

#include <climits>

#include "hhr_common.cuh"
#include "hhr_launch.h"

namespace hhr {

// ============================================================================
// prep_query: q' = R_h q (fp32) and the query sign codes of W_h q.
// grid (Hkv, B); one CTA per KV head and sequence handles its G query heads.
// ============================================================================
template <int G>
__global__ void __launch_bounds__(PREP_THREADS)
prep_query_kernel(Dims dm, const __nv_bfloat16* __restrict__ q, const float* __restrict__ R,
                  const __nv_bfloat16* __restrict__ W, Work wk, float* dbg_qrot,
                  uint64_t* dbg_qcodes, int do_hash) {
  pdl_trigger();  // the scan kernel may start prefetching page metadata now
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int hq0 = h * G;
  __shared__ float qs[G][D];
  for (int i = tid; i < G * D; i += blockDim.x)
    qs[i / D][i % D] = __bfloat162float(q[((long long)b * dm.Hq + hq0 + i / D) * D + i % D]);
  __syncthreads();

  // q'_i = sum_j R_h[i][j] q_j
  const float* Rh = R + (long long)h * D * D;
  for (int o = tid; o < G * D; o += blockDim.x) {
    const int g = o / D, i = o % D;
    const float4* row = reinterpret_cast<const float4*>(Rh + (long long)i * D);
    float acc = 0.f;
#pragma unroll 8
    for (int j = 0; j < D / 4; ++j) {
      const float4 r = __ldg(row + j);
      acc = fmaf(r.x, qs[g][4 * j + 0], acc);
      acc = fmaf(r.y, qs[g][4 * j + 1], acc);
      acc = fmaf(r.z, qs[g][4 * j + 2], acc);
      acc = fmaf(r.w, qs[g][4 * j + 3], acc);
    }
    const long long idx = ((long long)b * dm.Hq + hq0 + g) * D + i;
    wk.qrot[idx] = acc;
    if (dbg_qrot) dbg_qrot[idx] = acc;
  }
  if (!do_hash) return;

  // bit j of query head g = [ (W_h q_g)_j > 0 ].  Each product of two bf16
  // values is exact in fp32, so the fp32 sum is off by at most
  // 127 * 2^-24 * sum|w q|; below 2^-14 * sum|w q| the sign is decided by
  // an fp64 recompute instead.  G * nb is a multiple of 32, so every warp
  // covers 32 consecutive bits of one query head.
  const __nv_bfloat16* Wh = W + (long long)h * dm.nb * D;
  for (int o = tid; o < G * dm.nb; o += blockDim.x) {
    const int g = o / dm.nb, j = o % dm.nb;
    const uint4* row = reinterpret_cast<const uint4*>(Wh + (long long)j * D);
    float acc = 0.f, mag = 0.f;
#pragma unroll 4
    for (int u = 0; u < D / 8; ++u) {
      float wf[8];
      unpack8(__ldg(row + u), wf);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float p = wf[e] * qs[g][8 * u + e];
        acc += p;
        mag += fabsf(p);
      }
    }
    bool bit;
    if (fabsf(acc) <= ldexpf(mag, -14)) {
      double a = 0.0;
      for (int u = 0; u < D / 8; ++u) {
        float wf[8];
        unpack8(__ldg(row + u), wf);
        for (int e = 0; e < 8; ++e) a += (double)wf[e] * (double)qs[g][8 * u + e];
      }
      bit = a > 0.0;
    } else {
      bit = acc > 0.f;
    }
    const unsigned m = __ballot_sync(0xffffffffu, bit);
    if ((tid & 31) == 0) {
      const long long w32 = ((long long)b * dm.Hq + hq0 + g) * dm.words * 2 + j / 32;
      reinterpret_cast<uint32_t*>(wk.qcodes)[w32] = m;
      if (dbg_qcodes) reinterpret_cast<uint32_t*>(dbg_qcodes)[w32] = m;
    }
  }
}

// ============================================================================
// Page select: keep the N largest of U[0, n) (equal values -> lower index),
// write the kept ids in ascending order.  Whole CTA; exact radix select on
// order-preserving keys (four 8-bit digits, most significant first), then
// one compaction pass in index order.
// ============================================================================
__device__ __forceinline__ void select_top_pages(const float* U, int n, int N, int* out,
                                                 int* dbg_out, int* s_hist, int* s_red,
                                                 int* s_bcast) {
  const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5;
  if (N >= n) {
    for (int i = tid; i < n; i += nt) {
      out[i] = i;
      if (dbg_out) dbg_out[i] = i;
    }
    return;
  }
  const int kpt = (n + nt - 1) / nt;  // <= SEL_KPT (checked by the host)
  uint32_t key[SEL_KPT];
#pragma unroll
  for (int i = 0; i < SEL_KPT; ++i) {
    const int idx = tid * kpt + i;
    key[i] = (i < kpt && idx < n) ? order_key(__ldcg(U + idx)) : 0u;
  }
  uint32_t prefix = 0u, pmask = 0u;
  int need = N;
#pragma unroll 1
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += nt) s_hist[i] = 0;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < SEL_KPT; ++i) {
      if (i < kpt) {  // kpt is uniform: every lane takes the same path
        const int idx = tid * kpt + i;
        const bool m = idx < n && (key[i] & pmask) == prefix;
        const unsigned dg = (key[i] >> shift) & 255u;
        const unsigned bin = m ? dg : (256u + lane);
        const unsigned peers = __match_any_sync(0xffffffffu, bin);
        if (m && lane == __ffs(peers) - 1) atomicAdd(&s_hist[dg], __popc(peers));
      }
    }
    __syncthreads();
    if (warp == 0) {
      // lane L covers digits 255-8L down to 248-8L (descending), so an
      // inclusive scan over lanes counts keys from the largest digit down
      int c[8], tot = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) { c[e] = s_hist[255 - 8 * lane - e]; tot += c[e]; }
      int incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const unsigned ball = __ballot_sync(0xffffffffu, incl >= need);
      if (lane == __ffs(ball) - 1) {
        int run = incl - tot;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if (run + c[e] >= need) {
            s_bcast[0] = 255 - 8 * lane - e;
            s_bcast[1] = need - run;
            break;
          }
          run += c[e];
        }
      }
    }
    __syncthreads();
    prefix |= (uint32_t)s_bcast[0] << shift;
    pmask |= 255u << shift;
    need = s_bcast[1];
    __syncthreads();
  }
  // prefix is now the N-th largest key; `need` keys equal to it are kept,
  // the first ones in index order.
  int gt = 0, eq = 0;
#pragma unroll
  for (int i = 0; i < SEL_KPT; ++i) {
    const int idx = tid * kpt + i;
    if (i < kpt && idx < n) { gt += key[i] > prefix; eq += key[i] == prefix; }
  }
  int tot;
  const int eq_before = block_excl_scan(eq, s_red, &tot);
  const int take_eq = max(0, min(eq, need - eq_before));
  int pos = block_excl_scan(gt + take_eq, s_red, &tot);
  int taken = 0;
#pragma unroll
  for (int i = 0; i < SEL_KPT; ++i) {
    const int idx = tid * kpt + i;
    if (i < kpt && idx < n) {
      const bool is_eq = key[i] == prefix;
      if (key[i] > prefix || (is_eq && taken < take_eq)) {
        out[pos] = idx;
        if (dbg_out) dbg_out[pos] = idx;
        ++pos;
        taken += is_eq;
      }
    }
  }
}

// ============================================================================
// gkr_scan_select: U_p = max_g sum_i max(q'_gi mn_pi, q'_gi mx_pi).
// grid (ceil(np_max / SCAN_PAGES), Hkv, B).  A half-warp handles one page per
// step: lane l owns channels 8l..8l+7 (one 16-byte load of min, one of max).
// ============================================================================
template <int G>
__global__ void __launch_bounds__(SCAN_THREADS)
gkr_scan_select_kernel(Dims dm, const __nv_bfloat16* __restrict__ pmin,
                       const __nv_bfloat16* __restrict__ pmax, const int* __restrict__ seq_lens,
                       const int* __restrict__ table, const int* __restrict__ n_keep, Work wk,
                       float* dbg_ub, float* dbg_U, int* dbg_sel, int* dbg_nsel, int* status) {
  constexpr int HW = SCAN_THREADS / 16;      // half-warps per CTA
  constexpr int PPH = SCAN_PAGES / HW;       // pages per half-warp
  __shared__ int s_hist[256];
  __shared__ int s_red[33];
  __shared__ int s_bcast[2];
  __shared__ int s_last;

  const int chunk = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int hw = tid >> 4, ln = tid & 15;
  const int bh = b * dm.Hkv + h;
  const int L = seq_len_of(dm, seq_lens, b);
  const int np = (L + dm.P - 1) / dm.P;

  // prefetch this CTA's metadata before waiting for q'
  uint4 vmn[PPH], vmx[PPH];
#pragma unroll
  for (int r = 0; r < PPH; ++r) {
    const int p = chunk * SCAN_PAGES + r * HW + hw;
    vmn[r] = make_uint4(0, 0, 0, 0);
    vmx[r] = make_uint4(0, 0, 0, 0);
    if (p < np) {
      const long long off = meta_row(dm, table, b, h, p, status);
      if (off >= 0) {
        vmn[r] = ld_stream16(pmin + off + ln * 8);
        vmx[r] = ld_stream16(pmax + off + ln * 8);
      }
    }
  }
  pdl_wait();

  float qv[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float4* qp = reinterpret_cast<const float4*>(wk.qrot + ((long long)b * dm.Hq + h * G + g) * D + ln * 8);
    const float4 a = __ldcg(qp), c = __ldcg(qp + 1);
    qv[g][0] = a.x; qv[g][1] = a.y; qv[g][2] = a.z; qv[g][3] = a.w;
    qv[g][4] = c.x; qv[g][5] = c.y; qv[g][6] = c.z; qv[g][7] = c.w;
  }

#pragma unroll
  for (int r = 0; r < PPH; ++r) {
    const int p = chunk * SCAN_PAGES + r * HW + hw;
    float mn[8], mx[8];
    unpack8(vmn[r], mn);
    unpack8(vmx[r], mx);
    float acc[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float a = 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) a = fmaf(qv[g][c], qv[g][c] >= 0.f ? mx[c] : mn[c], a);
      acc[g] = a;
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
      for (int o = 8; o >= 1; o >>= 1) acc[g] += __shfl_xor_sync(0xffffffffu, acc[g], o, 16);
    }
    if (p < np) {
      float U = acc[0];
#pragma unroll
      for (int g = 1; g < G; ++g) U = fmaxf(U, acc[g]);
      if (ln == 0) {
        wk.U[(long long)bh * dm.np_max + p] = U;
        if (dbg_U) dbg_U[(long long)bh * dm.np_max + p] = U;
      }
      if (dbg_ub) {
#pragma unroll
        for (int g = 0; g < G; ++g)
          if (ln == g) dbg_ub[((long long)b * dm.Hq + h * G + g) * dm.np_max + p] = acc[g];
      }
    }
  }
  __threadfence();
  pdl_trigger();
  __syncthreads();
  if (tid == 0) {
    const unsigned t = atomicAdd(wk.tickets + bh * 4 + 0, 1u);
    s_last = (t == gridDim.x - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  const int N = min(max(__ldg(n_keep + b), 1), wk.Nmax);
  const int Neff = min(N, np);
  select_top_pages(wk.U + (long long)bh * dm.np_max, np, Neff, wk.sel_pages + (long long)bh * wk.Nmax,
                   dbg_sel ? dbg_sel + (long long)bh * wk.Nmax : nullptr, s_hist, s_red, s_bcast);
  if (tid == 0) {
    wk.n_sel[bh] = Neff;
    if (dbg_nsel) dbg_nsel[bh] = Neff;
    wk.tickets[bh * 4 + 0] = 0u;  // ready for the next call
  }
}

// ============================================================================
// lhp_score_select: S = sum_g popcount(cq_g ^ code) for each valid row of
// the kept pages, then keep the k smallest (equal -> lower token id).
// grid (ceil(Nmax * P / LHP_THREADS), Hkv, B); one candidate row per thread.
// Scores are small integers (0 .. G * nb), so the select is an exact
// counting select on a histogram built with warp-aggregated atomics.
// ============================================================================
template <int G, int WORDS>
__global__ void __launch_bounds__(LHP_THREADS)
lhp_score_select_kernel(Dims dm, const uint64_t* __restrict__ codes,
                        const int* __restrict__ seq_lens, const int* __restrict__ table,
                        const int* __restrict__ top_k, Work wk, int* dbg_scores, int* dbg_ncand,
                        int* dbg_sel, int* dbg_nsel, int* status) {
  __shared__ uint64_t s_cq[G * WORDS];
  __shared__ int s_red[33];
  __shared__ int s_bcast[3];
  __shared__ int s_last;
  const int chunk = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x, lane = tid & 31;
  const int bh = b * dm.Hkv + h;
  const int L = seq_len_of(dm, seq_lens, b);
  int* hist = wk.hist + (long long)bh * wk.hist_stride;
  const long long cand_base = (long long)bh * wk.Nmax * dm.P;

  pdl_wait();
  if (tid < G * WORDS) s_cq[tid] = __ldcg(wk.qcodes + ((long long)b * dm.Hq + h * G) * WORDS + tid);
  const int nsel = __ldcg(wk.n_sel + bh);
  __syncthreads();

  const int ci = chunk * LHP_THREADS + tid;  // candidate index = kept-page slot * P + row
  const int slot = ci / dm.P, row = ci - slot * dm.P;
  int S = INT_MAX;
  bool valid = false;
  if (slot < nsel) {
    const int t = __ldcg(wk.sel_pages + (long long)bh * wk.Nmax + slot) * dm.P + row;
    if (t < L) {
      const long long off = code_row(dm, table, b, h, t, status);
      if (off >= 0) {
        uint64_t c[WORDS];
        if constexpr (WORDS == 1) {
          c[0] = __ldg(codes + off);
        } else {
#pragma unroll
          for (int w2 = 0; w2 < WORDS; w2 += 2) {
            const ulonglong2 v = __ldg(reinterpret_cast<const ulonglong2*>(codes + off + w2));
            c[w2] = v.x;
            c[w2 + 1] = v.y;
          }
        }
        int s = 0;
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
          for (int w2 = 0; w2 < WORDS; ++w2) s += __popcll(s_cq[g * WORDS + w2] ^ c[w2]);
        S = s;
        valid = true;
      }
    }
    wk.scores[cand_base + ci] = S;
    if (dbg_scores) dbg_scores[cand_base + ci] = S;
  }
  {
    const unsigned bin = valid ? (unsigned)S : (0x80000000u | lane);
    const unsigned peers = __match_any_sync(0xffffffffu, bin);
    if (valid && lane == __ffs(peers) - 1) atomicAdd(hist + S, __popc(peers));
  }
  __threadfence();
  pdl_trigger();
  __syncthreads();
  if (tid == 0) {
    const unsigned t = atomicAdd(wk.tickets + bh * 4 + 1, 1u);
    s_last = (t == gridDim.x - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // ---- threshold from the histogram ----
  const int nbins = G * dm.nb + 1;
  const int bpt = (nbins + LHP_THREADS - 1) / LHP_THREADS;
  int local = 0;
  for (int i = 0; i < bpt; ++i) {
    const int bi = tid * bpt + i;
    if (bi < nbins) local += __ldcg(hist + bi);
  }
  int n_cand;
  const int before = block_excl_scan(local, s_red, &n_cand);
  const int kreq = min(max(__ldg(top_k + b), 1), wk.Kmax);
  const int keff = min(kreq, n_cand);
  if (keff > 0 && before < keff && before + local >= keff) {
    int run = before;
    for (int i = 0; i < bpt; ++i) {
      const int bi = tid * bpt + i;
      const int c = bi < nbins ? __ldcg(hist + bi) : 0;
      if (run + c >= keff) { s_bcast[0] = bi; s_bcast[1] = keff - run; break; }
      run += c;
    }
  }
  __syncthreads();
  // the histogram has been read: clear it for the next call
  for (int i = 0; i < bpt; ++i) {
    const int bi = tid * bpt + i;
    if (bi < nbins) hist[bi] = 0;
  }
  if (keff == 0) {
    if (tid == 0) {
      wk.n_keys[bh] = 0;
      if (dbg_nsel) dbg_nsel[bh] = 0;
      if (dbg_ncand) dbg_ncand[bh] = n_cand;
      wk.tickets[bh * 4 + 1] = 0u;
    }
    return;
  }
  const int T = s_bcast[0];
  const int need_eq = s_bcast[1];

  // ---- compaction in candidate order (= ascending token id) ----
  const int ncand_slots = nsel * dm.P;
  int carry_eq = 0, carry_pos = 0;
  int* out = wk.sel_keys + (long long)bh * wk.Kmax;
  int* dout = dbg_sel ? dbg_sel + (long long)bh * wk.Kmax : nullptr;
  const int* sel_pages = wk.sel_pages + (long long)bh * wk.Nmax;
  for (int base = 0; base < ncand_slots; base += LHP_THREADS * LHP_KPT) {
    int sc[LHP_KPT];
    int lt = 0, eq = 0;
#pragma unroll
    for (int i = 0; i < LHP_KPT; ++i) {
      const int c = base + tid * LHP_KPT + i;
      sc[i] = c < ncand_slots ? __ldcg(wk.scores + cand_base + c) : INT_MAX;
      lt += sc[i] < T;
      eq += sc[i] == T;
    }
    int tot_eq, tot_cnt;
    const int eq_before = carry_eq + block_excl_scan(eq, s_red, &tot_eq);
    const int take_eq = max(0, min(eq, need_eq - eq_before));
    int pos = carry_pos + block_excl_scan(lt + take_eq, s_red, &tot_cnt);
    int taken = 0;
#pragma unroll
    for (int i = 0; i < LHP_KPT; ++i) {
      const int c = base + tid * LHP_KPT + i;
      const bool is_eq = sc[i] == T;
      if (sc[i] < T || (is_eq && taken < take_eq)) {
        const int slot_c = c / dm.P;
        const int t = __ldcg(sel_pages + slot_c) * dm.P + (c - slot_c * dm.P);
        out[pos] = t;
        if (dout) dout[pos] = t;
        ++pos;
        taken += is_eq;
      }
    }
    carry_eq += tot_eq;
    carry_pos += tot_cnt;
  }
  if (tid == 0) {
    wk.n_keys[bh] = keff;
    if (dbg_nsel) dbg_nsel[bh] = keff;
    if (dbg_ncand) dbg_ncand[bh] = n_cand;
    wk.tickets[bh * 4 + 1] = 0u;
  }
}

// ============================================================================
// attn_split: softmax attention of the G query heads of one KV head over a
// range of rows (the kept rows, or all rows when DENSE), fp32 throughout.
// grid (nsplit, Hkv, B), ATT_THREADS threads.  A half-warp takes CH rows per
// step; lane l owns channels 8l..8l+7 of K' and V (16-byte loads).  The
// G x CH partial logits are summed over the 16 lanes by a transposed
// butterfly (each round halves the values a lane keeps), after which lane l
// holds KPL logits of head l / LPH.  Weights go through shared memory to
// every lane for the V accumulation.  Each CTA writes an unnormalised
// partial (o, running max m, sum l); the last CTA merges them.
// ============================================================================
template <int GP, int CH, int N>
struct HalvingReduce {
  // values v[0..N) -> after the round lane keeps N/2 values
  static __device__ __forceinline__ void round(float* v, int ln, int o, unsigned hmask) {
    const bool up = (ln & o) != 0;
#pragma unroll
    for (int i = 0; i < N / 2; ++i) {
      const float send = up ? v[i] : v[i + N / 2];
      const float keep = up ? v[i + N / 2] : v[i];
      v[i] = keep + __shfl_xor_sync(hmask, send, o, 16);
    }
  }
};

template <int G, bool DENSE>
__global__ void __launch_bounds__(ATT_THREADS)
attn_split_kernel(Dims dm, const __nv_bfloat16* __restrict__ Kr, const __nv_bfloat16* __restrict__ Vc,
                  const int* __restrict__ seq_lens, const int* __restrict__ table, Work wk,
                  float sm_scale, float* __restrict__ out, int* status) {
  constexpr int GP = G <= 2 ? 2 : (G <= 4 ? 4 : 8);  // heads padded to a power of two
  constexpr int CH = GP <= 4 ? 8 : 4;                // rows per half-warp step
  constexpr int NV = GP * CH;                        // partial logits per lane
  constexpr int KPL = NV / 16;                       // logits a lane keeps
  constexpr int LPH = CH / KPL;                      // lanes per head afterwards
  constexpr int NHW = ATT_THREADS / 16;
  __shared__ __align__(16) float s_p[NHW][CH * GP];
  __shared__ float s_m[NHW][G], s_l[NHW][G];
  __shared__ __align__(16) float s_o[NHW][G][D];
  __shared__ int s_last;

  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int hw = tid >> 4, ln = tid & 15, lane = tid & 31;
  const unsigned hmask = 0xffffu << (lane & 16);
  const int bh = b * dm.Hkv + h;

  pdl_wait();
  const int nk = DENSE ? seq_len_of(dm, seq_lens, b) : __ldcg(wk.n_keys + bh);
  const int KS = wk.keys_per_split;
  const int k0 = split * KS, k1 = min(k0 + KS, nk);

  // q' slice scaled so that exp2 of a logit is the softmax weight
  const float qscale = sm_scale * 1.4426950408889634f;
  float qv[GP][8];
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    if (g < G) {
      const float4* qp = reinterpret_cast<const float4*>(wk.qrot + ((long long)b * dm.Hq + h * G + g) * D + ln * 8);
      const float4 a = __ldcg(qp), c = __ldcg(qp + 1);
      qv[g][0] = a.x * qscale; qv[g][1] = a.y * qscale; qv[g][2] = a.z * qscale; qv[g][3] = a.w * qscale;
      qv[g][4] = c.x * qscale; qv[g][5] = c.y * qscale; qv[g][6] = c.z * qscale; qv[g][7] = c.w * qscale;
    } else {
#pragma unroll
      for (int c = 0; c < 8; ++c) qv[g][c] = 0.f;
    }
  }
  float m[G], o[G][8];
  float l_own = 0.f;  // sum of weights of head g_own over this lane's rows
  const int g_own = ln / LPH;
  const int kk0 = (ln % LPH) * KPL;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -INFINITY;
#pragma unroll
    for (int c = 0; c < 8; ++c) o[g][c] = 0.f;
  }
  const int* sel = wk.sel_keys + (long long)bh * wk.Kmax;

  for (int kb = k0 + hw * CH; kb < k1; kb += NHW * CH) {
    const int nvalid = min(CH, k1 - kb);
    uint4 kv[CH], vv[CH];
#pragma unroll
    for (int kk = 0; kk < CH; ++kk) {
      kv[kk] = make_uint4(0, 0, 0, 0);
      vv[kk] = make_uint4(0, 0, 0, 0);
      if (kk < nvalid) {
        const int t = DENSE ? kb + kk : __ldcg(sel + kb + kk);
        const long long off = kv_row(dm, table, b, h, t, status);
        if (off >= 0) {
          kv[kk] = ld_stream16(Kr + off + ln * 8);
          vv[kk] = ld_stream16(Vc + off + ln * 8);
        }
      }
    }
    // partial logits, value index g * CH + kk
    float val[NV];
#pragma unroll
    for (int kk = 0; kk < CH; ++kk) {
      float kf[8];
      unpack8(kv[kk], kf);
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        float a = 0.f;
        if (g < G) {
#pragma unroll
          for (int c = 0; c < 8; ++c) a = fmaf(qv[g][c], kf[c], a);
        }
        val[g * CH + kk] = a;
      }
    }
    HalvingReduce<GP, CH, NV>::round(val, ln, 8, hmask);
    HalvingReduce<GP, CH, NV / 2>::round(val, ln, 4, hmask);
    HalvingReduce<GP, CH, NV / 4>::round(val, ln, 2, hmask);
    HalvingReduce<GP, CH, NV / 8>::round(val, ln, 1, hmask);
    // lane holds logits of head g_own for rows kk0 .. kk0 + KPL - 1
    float cmax = -INFINITY;
#pragma unroll
    for (int i = 0; i < KPL; ++i) {
      if (kk0 + i >= nvalid) val[i] = -INFINITY;
      cmax = fmaxf(cmax, val[i]);
    }
#pragma unroll
    for (int o2 = 1; o2 < LPH; o2 <<= 1) cmax = fmaxf(cmax, __shfl_xor_sync(hmask, cmax, o2, 16));
    float alpha[G];
    float m_own = -INFINITY, a_own = 1.f;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float cm = __shfl_sync(hmask, cmax, g * LPH, 16);
      const float mn = fmaxf(m[g], cm);
      alpha[g] = (mn == -INFINITY) ? 1.f : exp2f(m[g] - mn);
      m[g] = mn;
      if (g == g_own) { m_own = mn; a_own = alpha[g]; }
    }
    float psum = 0.f;
#pragma unroll
    for (int i = 0; i < KPL; ++i) {
      const float p = (g_own >= G || val[i] == -INFINITY) ? 0.f : exp2f(val[i] - m_own);
      psum += p;
      s_p[hw][(kk0 + i) * GP + g_own] = p;
    }
    l_own = l_own * a_own + psum;
    __syncwarp(hmask);
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int c = 0; c < 8; ++c) o[g][c] *= alpha[g];
#pragma unroll
    for (int kk = 0; kk < CH; ++kk) {
      if (kk < nvalid) {
        float vf[8];
        unpack8(vv[kk], vf);
        float pk[GP];
        if constexpr (GP >= 4) {
#pragma unroll
          for (int g4 = 0; g4 < GP; g4 += 4) {
            const float4 t4 = *reinterpret_cast<const float4*>(&s_p[hw][kk * GP + g4]);
            pk[g4] = t4.x; pk[g4 + 1] = t4.y; pk[g4 + 2] = t4.z; pk[g4 + 3] = t4.w;
          }
        } else {
          const float2 t2 = *reinterpret_cast<const float2*>(&s_p[hw][kk * GP]);
          pk[0] = t2.x; pk[1] = t2.y;
        }
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
          for (int c = 0; c < 8; ++c) o[g][c] = fmaf(pk[g], vf[c], o[g][c]);
      }
    }
    __syncwarp(hmask);
  }

  // ---- merge the half-warps of this CTA ----
#pragma unroll
  for (int o2 = 1; o2 < LPH; o2 <<= 1) l_own += __shfl_xor_sync(hmask, l_own, o2, 16);
  if (g_own < G && (ln % LPH) == 0) s_l[hw][g_own] = l_own;
  if (ln == 0) {
#pragma unroll
    for (int g = 0; g < G; ++g) s_m[hw][g] = m[g];
  }
#pragma unroll
  for (int g = 0; g < G; ++g) {
    *reinterpret_cast<float4*>(&s_o[hw][g][ln * 8]) = make_float4(o[g][0], o[g][1], o[g][2], o[g][3]);
    *reinterpret_cast<float4*>(&s_o[hw][g][ln * 8 + 4]) = make_float4(o[g][4], o[g][5], o[g][6], o[g][7]);
  }
  __syncthreads();
  const int nsplit_used = (nk + KS - 1) / KS;
  float* part = wk.part + ((long long)bh * wk.nsplit + split) * (G * (D + 2));
  if (split < nsplit_used) {
    for (int e = tid; e < G * D; e += ATT_THREADS) {
      const int g = e / D, c = e % D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < NHW; ++w) M = fmaxf(M, s_m[w][g]);
      float Ls = 0.f, Os = 0.f;
#pragma unroll
      for (int w = 0; w < NHW; ++w) {
        const float sc = (s_m[w][g] == -INFINITY) ? 0.f : exp2f(s_m[w][g] - M);
        Ls = fmaf(s_l[w][g], sc, Ls);
        Os = fmaf(s_o[w][g][c], sc, Os);
      }
      part[g * (D + 2) + c] = Os;
      if (c == 0) { part[g * (D + 2) + D] = M; part[g * (D + 2) + D + 1] = Ls; }
    }
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const unsigned t = atomicAdd(wk.tickets + bh * 4 + (DENSE ? 3 : 2), 1u);
    s_last = (t == gridDim.x - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // ---- last CTA: merge the split partials into the output ----
  const float* pb = wk.part + (long long)bh * wk.nsplit * (G * (D + 2));
  for (int e = tid; e < G * D; e += ATT_THREADS) {
    const int g = e / D, c = e % D;
    float M = -INFINITY;
    for (int s = 0; s < nsplit_used; ++s) M = fmaxf(M, __ldcg(pb + (long long)s * G * (D + 2) + g * (D + 2) + D));
    float Ls = 0.f, Os = 0.f;
    for (int s = 0; s < nsplit_used; ++s) {
      const float* ps = pb + (long long)s * G * (D + 2) + g * (D + 2);
      const float ms = __ldcg(ps + D);
      const float sc = (ms == -INFINITY) ? 0.f : exp2f(ms - M);
      Ls = fmaf(__ldcg(ps + D + 1), sc, Ls);
      Os = fmaf(__ldcg(ps + c), sc, Os);
    }
    out[((long long)b * dm.Hq + h * G + g) * D + c] = (Ls > 0.f) ? Os / Ls : 0.f;
  }
  if (tid == 0) wk.tickets[bh * 4 + (DENSE ? 3 : 2)] = 0u;
}


// ============================================================================
// launchers (explicitly instantiated per group size in hhr_decode_g*.cu)
// ============================================================================
template <typename Kern, typename... Args>
static cudaError_t launch_ex(Kern kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
                             Args... args) {
  cudaLaunchConfig_t lc = {};
  lc.gridDim = grid;
  lc.blockDim = block;
  lc.dynamicSmemBytes = smem;
  lc.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&lc, kernel, args...);
}

template <int G, int WORDS>
static cudaError_t launch_lhp(const DecodeArgs& a) {
  const Dims& dm = a.dm;
  return launch_ex(lhp_score_select_kernel<G, WORDS>,
                   dim3((a.wk.Nmax * dm.P + LHP_THREADS - 1) / LHP_THREADS, dm.Hkv, dm.B), dim3(LHP_THREADS), 0,
                   a.stream, true, dm, a.codes, a.seq_lens, a.table, a.top_k, a.wk, a.dbg.key_scores,
                   a.dbg.n_cand, a.dbg.sel_keys, a.dbg.n_sel_keys, a.status);
}

template <int G>
cudaError_t launch_decode(const DecodeArgs& a) {
  const Dims& dm = a.dm;
  cudaError_t e = launch_ex(prep_query_kernel<G>, dim3(dm.Hkv, dm.B), dim3(PREP_THREADS), 0, a.stream, false, dm,
                            a.q, a.R, a.W, a.wk, a.dbg.q_rot, a.dbg.q_codes, 1);
  if (e != cudaSuccess) return e;
  e = launch_ex(gkr_scan_select_kernel<G>, dim3((dm.np_max + SCAN_PAGES - 1) / SCAN_PAGES, dm.Hkv, dm.B),
                dim3(SCAN_THREADS), 0, a.stream, true, dm, a.pmin, a.pmax, a.seq_lens, a.table, a.n_keep, a.wk,
                a.dbg.page_ub, a.dbg.page_U, a.dbg.sel_pages, a.dbg.n_sel_pages, a.status);
  if (e != cudaSuccess) return e;
  switch (dm.words) {
    case 1: e = launch_lhp<G, 1>(a); break;
    case 2: e = launch_lhp<G, 2>(a); break;
    case 4: e = launch_lhp<G, 4>(a); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  return launch_ex(attn_split_kernel<G, false>, dim3(a.wk.nsplit, dm.Hkv, dm.B), dim3(ATT_THREADS), 0, a.stream,
                   true, dm, a.Kr, a.Vc, a.seq_lens, a.table, a.wk, a.sm_scale, a.out, a.status);
}

template <int G>
cudaError_t launch_dense(const DecodeArgs& a) {
  const Dims& dm = a.dm;
  cudaError_t e = launch_ex(prep_query_kernel<G>, dim3(dm.Hkv, dm.B), dim3(PREP_THREADS), 0, a.stream, false, dm,
                            a.q, a.R, a.W, a.wk, static_cast<float*>(nullptr), static_cast<uint64_t*>(nullptr), 0);
  if (e != cudaSuccess) return e;
  return launch_ex(attn_split_kernel<G, true>, dim3(a.wk.nsplit, dm.Hkv, dm.B), dim3(ATT_THREADS), 0, a.stream,
                   true, dm, a.Kr, a.Vc, a.seq_lens, a.table, a.wk, a.sm_scale, a.out, a.status);
}

#define HHR_INSTANTIATE_DECODE(G)                                \
  template cudaError_t launch_decode<G>(const DecodeArgs&);      \
  template cudaError_t launch_dense<G>(const DecodeArgs&);

}  // namespace hhr
