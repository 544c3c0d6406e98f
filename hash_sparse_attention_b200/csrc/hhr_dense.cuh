// Dense decode attention over every cached row (sm_100a): the "Full
// Attention" comparison row of the paper's tables ("HHR: Hierarchical Hash
// Retrieval for Efficient LLM Generation", thelatestinai.com page, Tables 1-2).
//
// out[b, hq] = sum_{t < L} softmax_t(sm_scale * (R_h q) . K'_t) V_t.
//
// Work items are (unit, split) pairs: split i of unit u covers rows
// [i R, (i+1) R), one item per CTA at a time (one CTA per SM, items in a
// grid-stride loop).  The CTA's 8 warps work independently on 16-row tiles
// (warp w: tiles w, w + 8, ...), each streaming its tiles through a private
// ring of three (cp.async into XOR-swizzled rows, two tiles in flight), with
// no CTA barrier in the loop.  Per tile and warp, on tensor cores (mma.sync
// m16n8k16, bf16 in, fp32 accumulate):
//   S = Q K'^T    Q's 16 rows are the heads' q' * sm_scale * log2 e as bf16
//                 hi (rows 0-7) and lo (rows 8-15); a head's logit is the sum
//                 of its two rows, both held by the same lane;
//   online softmax per head in registers (running maximum and sum);
//   O += P V      P (the weights) as bf16 hi (rows 0-7) and lo (rows 8-15),
//                 built from the lane's own logits (the accumulator layout of
//                 S is the operand layout of P), O in registers.
// The warps' (max, sum, O) are combined in warp order into the item's
// partial; the last item of a unit to finish merges the unit's partials in
// split order.  Deterministic: every order is fixed by the split.
#pragma once

#include "hhr_decode.cuh"

namespace hhr {

constexpr int DN_THREADS = TL_WARPS * 32;
constexpr int DN_QB = SP_A_BYTES;                   // bf16 [16][136] Q operand
constexpr int DN_QF = DN_QB + 16 * 272;             // fp32 [8][128] q, then q'
constexpr int DN_MISC = DN_QF + 2 * 8 * D * 4;      // int [32]
constexpr int DN_SMEM = DN_MISC + 128;
constexpr int DN_RS = TL_NBUF > 2 ? 2 * TL_WARPS * TL_BYTES : 0;  // R_h in the slot-2 room during the prep
static_assert(DN_SMEM <= 232448 && DN_RS + D * D * 4 <= SP_A_BYTES, "shared memory of the dense kernel");

struct DnParams {
  SpParams sp;   // shared fields (q, R, K', V, lengths, table, scale, out, status)
  int nsplit;    // splits per unit
  int rows;      // R: rows per split (multiple of 16)
};

// R_h (fp32) is staged in shared memory with cp.async, its 16-byte pieces
// XOR-swizzled by row (piece c of row i at c ^ (i mod 32)) so that a warp
// reading the same piece of 32 consecutive rows hits distinct banks.  One
// commit group.
static __device__ __noinline__ void dn_issue_r(const SpParams& p, unsigned char* sm, int h, int r_off) {
  const float* Rh = p.R + (long long)h * D * D;
  #pragma unroll 1
  for (int q = threadIdx.x; q < D * 32; q += blockDim.x) {  // 128 rows x 32 pieces
    const int i = q >> 5, c = q & 31;
    cp_async16(sm + r_off + i * 512 + ((c ^ (i & 31)) * 16), Rh + i * D + c * 4);
  }
  cp_async_commit();
}

// Copies tile k of warp `warp` of the item (rows t0 + 16 (warp + 8 k) .. +15,
// clipped to tend) into its slot k mod 3.
__device__ __forceinline__ void dn_issue_tile(const SpParams& p, unsigned char* sm, const SpUnit& x, int warp, int k,
                                              int t0, int tend, bool live) {
  const int lane = threadIdx.x & 31;
  const int t = t0 + TL_ROWS * (warp + TL_WARPS * k) + lane;
  int ri = -1;
  if (live && lane < TL_ROWS && t < tend) {
    const long long off = kv_row(p.dm, p.table, x.b, x.h, t, p.status);
    ri = off >= 0 ? (int)(off / D) : -1;
  }
  tile_copy(p.Kr, p.Vc, tile_slot(sm, warp, k % TL_NBUF), ri, live);
}

// q' = R_h q (fp32, channel order) and the Q operand (head g's q' * sm_scale *
// log2 e as bf16 hi in row g, lo in row 8 + g).  R_h sits XOR-swizzled at
// DN_RS (dn_issue_r), issued before the two first tiles.
template <int G>
__device__ void dn_prep(const SpParams& p, unsigned char* sm, const SpUnit& x) {
  const int tid = threadIdx.x;
  float* qf = reinterpret_cast<float*>(sm + DN_QF);   // [8][128] q
  float* qs = qf + 8 * D;                             // [8][128] q'
  const __nv_bfloat16* qg = p.q + ((long long)x.b * p.dm.Hq + x.h * G) * D;
#pragma unroll 1
  for (int i = tid; i < G * D; i += DN_THREADS) qf[i] = __bfloat162float(qg[i]);
  cp_async_wait<2>();
  __syncthreads();
  {
    const int i = tid & (D - 1);
    const unsigned char* Ri = sm + DN_RS + i * 512;
#pragma unroll 1
    for (int g = tid >> 7; g < G; g += DN_THREADS / D) {
      float a = 0.f;
#pragma unroll 4
      for (int c = 0; c < 32; ++c) {
        const float4 r = *reinterpret_cast<const float4*>(Ri + ((c ^ (i & 31)) * 16));
        const float4 v = *reinterpret_cast<const float4*>(qf + g * D + 4 * c);
        a = fmaf(r.x, v.x, a); a = fmaf(r.y, v.y, a); a = fmaf(r.z, v.z, a); a = fmaf(r.w, v.w, a);
      }
      qs[g * D + i] = a;
    }
  }
  __syncthreads();
  const float qscale = p.sm_scale * 1.4426950408889634f;
  __nv_bfloat16* qb = reinterpret_cast<__nv_bfloat16*>(sm + DN_QB);
#pragma unroll 1
  for (int e = tid; e < 8 * D; e += DN_THREADS) {
    const int hh = e / D, c = e - hh * D;
    const float v = hh < G ? qs[hh * D + c] * qscale : 0.f;
    __nv_bfloat16 hi, lo;
    split_bf16(v, hi, lo);
    qb[hh * 136 + c] = hi;
    qb[(8 + hh) * 136 + c] = lo;
  }
  __syncthreads();
}

template <int G>
__global__ void __launch_bounds__(DN_THREADS, 1) hhr_dense_kernel(const __grid_constant__ DnParams dp) {
  extern __shared__ __align__(128) unsigned char sm[];
  const SpParams& p = dp.sp;
  const Dims& dm = p.dm;
  const Work& wk = p.wk;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int Units = dm.B * dm.Hkv;
  const int items = Units * dp.nsplit;
  const int PS = G * D + 16;
  volatile int* misc = reinterpret_cast<volatile int*>(sm + DN_MISC);
  if (tid < 32) misc[tid] = 0;
  int it = blockIdx.x;
  const int pre_h = it < items ? (it / dp.nsplit) % dm.Hkv : -1;  // the head whose R_h is copied first
  if (it < items) dn_issue_r(p, sm, pre_h, DN_RS);
  pdl_launch_dependents();
  pdl_wait();
  __syncthreads();
  bool first = true;
#pragma unroll 1
  for (; it < items; it += gridDim.x) {
    SpUnit x;
    x.u = it / dp.nsplit;
    const int i = it - x.u * dp.nsplit;
    x.b = x.u / dm.Hkv;
    x.h = x.u - x.b * dm.Hkv;
    x.L = seq_len_of(dm, p.seq_lens, x.b);
    x.np = (x.L + dm.P - 1) >> dm.lgP;
    const int nsp = x.L == 0 ? 1 : (x.L + dp.rows - 1) / dp.rows;  // splits this unit uses
    unsigned* gx = wk.gx + (long long)x.u * wk.gx_stride;
    if (i >= nsp) continue;
    if (!first || x.h != pre_h) {
      // (an R_h copy of a skipped first item may still be in flight: it lands
      // first, so the copy of this head's R_h is the one that stays)
      cp_async_wait_all();
      dn_issue_r(p, sm, x.h, DN_RS);
    }
    first = false;
    const int t0 = i * dp.rows, tend = min(x.L, t0 + dp.rows);
    const int ntile = (max(tend - t0, 0) + TL_ROWS - 1) / TL_ROWS;
    const int mine = ntile > warp ? (ntile - warp + TL_WARPS - 1) / TL_WARPS : 0;
    dn_issue_tile(p, sm, x, warp, 0, t0, tend, mine > 0);
    dn_issue_tile(p, sm, x, warp, 1, t0, tend, mine > 1);
    dn_prep<G>(p, sm, x);
    dn_issue_tile(p, sm, x, warp, 2, t0, tend, mine > 2);
    uint32_t aq[8][4];
    load_q_operand(sm + DN_QB, aq);
    float o[16][4];
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;
#pragma unroll 1
    for (int k = 0; k < mine; ++k) {
      cp_async_wait<TL_NBUF - 1>();
      __syncwarp();
      const int tl = warp + TL_WARPS * k;
      tile_attend(aq, o, m_run, l_run, tile_slot(sm, warp, k % TL_NBUF), min(TL_ROWS, tend - t0 - TL_ROWS * tl));
      __syncwarp();
      dn_issue_tile(p, sm, x, warp, k + TL_NBUF, t0, tend, k + TL_NBUF < mine);
    }
    cp_async_wait_all();
    tile_combine<G>(sm, o, m_run, l_run, mine > 0, wk.part + ((long long)x.u * wk.C3 + i) * PS, ntile > 0);
    if (x.L == 0) {  // empty sequence: zero output
#pragma unroll 1
      for (int e = tid; e < G * D; e += DN_THREADS) p.out[((long long)x.b * dm.Hq + x.h * G) * D + e] = 0.f;
    } else {
      if (tid == 0) {
        int last = 1;
        if (nsp > 1) last = atom_add_acq_rel(gx + GX_ARRIVE, 1u) == (unsigned)(nsp - 1);
        misc[MS_LAST] = last;
      }
      __syncthreads();
      if (misc[MS_LAST]) {
        // the unit's split partials, merged in split order
        const float* pt = wk.part + (long long)x.u * wk.C3 * PS;
#pragma unroll 1
        for (int e = tid; e < G * D; e += DN_THREADS) {
          const int hh = e >> 7;
          float M = -INFINITY;
#pragma unroll 1
          for (int k = 0; k < nsp; ++k) M = fmaxf(M, __ldcg(pt + (long long)k * PS + G * D + hh));
          float acc = 0.f, Ls = 0.f;
#pragma unroll 1
          for (int k = 0; k < nsp; ++k) {
            const float* pk = pt + (long long)k * PS;
            const float sc = exp2f(__ldcg(pk + G * D + hh) - M);
            acc = fmaf(sc, __ldcg(pk + e), acc);
            Ls = fmaf(sc, __ldcg(pk + G * D + 8 + hh), Ls);
          }
          p.out[((long long)x.b * dm.Hq + x.h * G) * D + e] = acc / Ls;
        }
        if (tid == 0) gx[GX_ARRIVE] = 0u;
      }
    }
    __syncthreads();
  }
  cp_async_wait_all();
}

}  // namespace hhr

// ---------------------------------------------------------------------------
// launches (programmatic dependent launch; co-residency checked on the host)
// ---------------------------------------------------------------------------
#include <algorithm>

namespace hhr {

// Sets the kernel's shared-memory attribute once per device and checks that
// a CTA of it fits on an SM (a launch of at most one CTA per SM then has all
// of its CTAs resident at once, which the CTA groups need: they wait for one
// another).
template <typename K>
inline cudaError_t prepare_kernel(K kernel, bool* configured, int threads = SP_THREADS, int smem = SP_SMEM) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorCooperativeLaunchTooLarge;
    configured[dev] = true;
  }
  return cudaSuccess;
}

template <typename P>
inline cudaError_t launch_pdl(void (*kernel)(P), const P& prm, int grid, cudaStream_t st, int threads = SP_THREADS,
                              int smem = SP_SMEM) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, prm);
}

inline SpParams sp_params(const DecodeArgs& a) {
  SpParams p = {};
  p.dm = a.dm;
  p.wk = a.wk;
  p.q = a.q;
  p.R = a.R;
  p.W = a.W;
  p.Kr = a.Kr;
  p.Vc = a.Vc;
  p.pmin = a.pmin;
  p.pmax = a.pmax;
  p.codes = a.codes;
  p.seq_lens = a.seq_lens;
  p.table = a.table;
  p.n_keep = a.n_keep;
  p.top_k = a.top_k;
  p.sm_scale = a.sm_scale;
  p.out = a.out;
  p.dbg = a.dbg;
  p.status = a.status;
  p.wait_limit = a.wait_limit;
  return p;
}

template <int G, int WORDS>
inline cudaError_t launch_sparse_t(const DecodeArgs& a) {
  static bool configured[64] = {false};
  SpParams p = sp_params(a);
  int S = 1, ng = 1;
  sparse_group_shape(a.dm, a.num_sms, a.wk.Nmax * a.dm.P, a.wk.Kmax, a.wk.HB, &S, &ng);
  p.gsize = S;
  p.ngroups = ng;
  const int grid = S * ng;
  cudaError_t e = prepare_kernel(hhr_sparse_kernel<G, WORDS>, configured);
  if (e != cudaSuccess) return e;
  if (grid > a.num_sms) return cudaErrorCooperativeLaunchTooLarge;
  return launch_pdl(hhr_sparse_kernel<G, WORDS>, p, grid, a.stream);
}

template <int G>
cudaError_t launch_decode(const DecodeArgs& a) {
  switch (a.dm.words) {
    case 1: return launch_sparse_t<G, 1>(a);
    case 2: return launch_sparse_t<G, 2>(a);
    case 4: return launch_sparse_t<G, 4>(a);
  }
  return cudaErrorInvalidValue;
}

template <int G>
cudaError_t launch_dense(const DecodeArgs& a) {
  static bool configured[64] = {false};
  DnParams dp = {};
  dp.sp = sp_params(a);
  dp.nsplit = a.dense_nsplit;
  dp.rows = a.dense_rows;
  const int items = a.dm.B * a.dm.Hkv * dp.nsplit;
  const int grid = std::max(1, std::min(items, a.num_sms));
  cudaError_t e = prepare_kernel(hhr_dense_kernel<G>, configured, DN_THREADS, DN_SMEM);
  if (e != cudaSuccess) return e;
  return launch_pdl(hhr_dense_kernel<G>, dp, grid, a.stream, DN_THREADS, DN_SMEM);
}

}  // namespace hhr

#define HHR_INSTANTIATE_DECODE(G_)                                   \
  template cudaError_t launch_decode<G_>(const DecodeArgs& a);       \
  template cudaError_t launch_dense<G_>(const DecodeArgs& a);
