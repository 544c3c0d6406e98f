// Dense decode attention over every cached row (sm_100a): the "Full
// Attention" comparison row of the paper's tables ("HHR: Hierarchical Hash
// Retrieval for Efficient LLM Generation", thelatestinai.com page, Tables 1-2).
//
// out[b, hq] = sum_{t < L} softmax_t(sm_scale * (R_h q) . K'_t) V_t.
//
// Work items are (unit, split) pairs: split i of unit u covers rows
// [i R, (i+1) R) (R a multiple of 128), one item per CTA at a time (one CTA
// per SM, items in a grid-stride loop).  A CTA streams its rows in 128-row
// chunks (cp.async, three chunks in flight, XOR-swizzled for ldmatrix),
// computes each chunk's softmax partial on tensor cores with the decode
// kernel's gather step, and folds it into a running (max, sum, output) in
// registers; the item's partial goes to the workspace and the last item of a
// unit to finish merges the unit's partials in split order.  Deterministic:
// the fold and the merge orders are fixed by the split.
#pragma once

#include "hhr_decode.cuh"

namespace hhr {

struct DnParams {
  SpParams sp;   // shared fields (q, R, K', V, lengths, table, scale, out, status)
  int nsplit;    // splits per unit
  int rows;      // R: rows per split (multiple of 128)
};

// Element offset / 128 of row t of the unit, or -1 (past the end or a bad block).
__device__ __forceinline__ int dn_row_of(const SpParams& p, const SpUnit& x, int t, int tend) {
  if (t >= tend) return -1;
  const long long off = kv_row(p.dm, p.table, x.b, x.h, t, p.status);
  return off >= 0 ? (int)(off / D) : -1;
}

__device__ __forceinline__ void dn_issue_chunk(const SpParams& p, unsigned char* sm, const SpUnit& x, int k, int nk,
                                               int t0, int tend) {
  if (k < nk) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int ri = lane < 8 ? dn_row_of(p, x, t0 + k * SP_ROWS + warp * 8 + lane, tend) : -1;
    sp_copy_rows(p, sm + (k % SP_NGS) * SP_GSTAGE, ri);
  }
  cp_async_commit();
}

template <int G>
__global__ void __launch_bounds__(SP_THREADS, 1) hhr_dense_kernel(const __grid_constant__ DnParams dp) {
  extern __shared__ __align__(128) unsigned char sm[];
  const SpParams& p = dp.sp;
  const Dims& dm = p.dm;
  const Work& wk = p.wk;
  const int tid = threadIdx.x;
  const int Units = dm.B * dm.Hkv;
  const int items = Units * dp.nsplit;
  const int PS = G * D + 16;
  float* pc = reinterpret_cast<float*>(sm + SP_KP);  // the current chunk's partial [PS]
  if (tid < 32) reinterpret_cast<volatile int*>(sm + SP_MISC)[tid] = 0;
  Prep<G> pr;
  int it = blockIdx.x;
  if (it < items) sp_prep_load<G, false>(p, (it / dp.nsplit) % dm.Hkv, pr);
  pdl_launch_dependents();
  pdl_wait();
  __syncthreads();
  bool first = true;
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
    if (i < nsp) {
      if (!first) sp_prep_load<G, false>(p, x.h, pr);
      first = false;
      const int t0 = i * dp.rows, tend = min(x.L, t0 + dp.rows);
      const int nk = (max(tend - t0, 0) + SP_ROWS - 1) / SP_ROWS;
      dn_issue_chunk(p, sm, x, 0, nk, t0, tend);
      dn_issue_chunk(p, sm, x, 1, nk, t0, tend);
      sp_prep<G, false>(p, sm, x, pr, false);
      dn_issue_chunk(p, sm, x, 2, nk, t0, tend);
      // running state of elements tid and tid + 512 (G * 128 <= 1024)
      float o0 = 0.f, o1 = 0.f, M0 = -INFINITY, M1 = -INFINITY, L0 = 0.f, L1 = 0.f;
      const int e0 = tid, e1 = tid + SP_THREADS;
      const int h0 = e0 >> 7, h1 = e1 >> 7;
#pragma unroll 1
      for (int k = 0; k < nk; ++k) {
        cp_async_wait<SP_NGS - 1>();
        __syncthreads();
        sp_gather_step<G>(sm, sm + (k % SP_NGS) * SP_GSTAGE, min(SP_ROWS, tend - t0 - k * SP_ROWS), pc);
        dn_issue_chunk(p, sm, x, k + SP_NGS, nk, t0, tend);
        if (e0 < G * D) {
          const float Mc = pc[G * D + h0], Lc = pc[G * D + 8 + h0];
          const float Mn = fmaxf(M0, Mc);
          const float a = exp2f(M0 - Mn), c = exp2f(Mc - Mn);
          o0 = o0 * a + pc[e0] * c;
          L0 = L0 * a + Lc * c;
          M0 = Mn;
        }
        if (e1 < G * D) {
          const float Mc = pc[G * D + h1], Lc = pc[G * D + 8 + h1];
          const float Mn = fmaxf(M1, Mc);
          const float a = exp2f(M1 - Mn), c = exp2f(Mc - Mn);
          o1 = o1 * a + pc[e1] * c;
          L1 = L1 * a + Lc * c;
          M1 = Mn;
        }
      }
      cp_async_wait_all();
      // the item's partial
      float* part = wk.part + ((long long)x.u * wk.C3 + i) * PS;
      if (nk > 0) {
        if (e0 < G * D) {
          part[e0] = o0;
          if ((e0 & (D - 1)) == 0) {
            part[G * D + h0] = M0;
            part[G * D + 8 + h0] = L0;
          }
        }
        if (e1 < G * D) {
          part[e1] = o1;
          if ((e1 & (D - 1)) == 0) {
            part[G * D + h1] = M1;
            part[G * D + 8 + h1] = L1;
          }
        }
      }
      __syncthreads();
      if (x.L == 0) {  // empty sequence: zero output
        for (int e = tid; e < G * D; e += SP_THREADS) p.out[((long long)x.b * dm.Hq + x.h * G) * D + e] = 0.f;
      } else {
        if (tid == 0) {
          int last = 1;
          if (nsp > 1) last = atom_add_acq_rel(gx + GX_ARRIVE, 1u) == (unsigned)(nsp - 1);
          reinterpret_cast<volatile int*>(sm + SP_MISC)[MS_LAST] = last;
        }
        __syncthreads();
        if (reinterpret_cast<volatile int*>(sm + SP_MISC)[MS_LAST]) {
          sp_merge<G>(p, sm, x, nsp);
          if (tid == 0) gx[GX_ARRIVE] = 0u;
        }
      }
      __syncthreads();
    }
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
inline cudaError_t prepare_kernel(K kernel, bool* configured) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SP_SMEM);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, SP_THREADS, SP_SMEM);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorCooperativeLaunchTooLarge;
    configured[dev] = true;
  }
  return cudaSuccess;
}

template <typename P>
inline cudaError_t launch_pdl(void (*kernel)(P), const P& prm, int grid, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(SP_THREADS);
  cfg.dynamicSmemBytes = SP_SMEM;
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
  sparse_group_shape(a.dm, a.num_sms, a.wk.Nmax * a.dm.P, a.wk.HB, &S, &ng);
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
  cudaError_t e = prepare_kernel(hhr_dense_kernel<G>, configured);
  if (e != cudaSuccess) return e;
  return launch_pdl(hhr_dense_kernel<G>, dp, grid, a.stream);
}

}  // namespace hhr

#define HHR_INSTANTIATE_DECODE(G_)                                   \
  template cudaError_t launch_decode<G_>(const DecodeArgs& a);       \
  template cudaError_t launch_dense<G_>(const DecodeArgs& a);
