// Exact top-k keys and the recall of a selection against them (sm_100a).
//
// The fidelity measure of the HHR paper ("HHR: Hierarchical Hash Retrieval
// for Efficient LLM Generation", thelatestinai.com page, Figure 4 caption:
// "Top-10% key recall"): the share of the truly highest-scoring keys that a
// retrieval keeps.  Per (sequence b, KV head h) the score of key t is the
// largest logit of the group's query heads, z_t = max_g q'_g . k'_t (q' = R_h q,
// k' the stored rotated key; a key matters if any head of the group attends
// to it, the same aggregation as the page bound's), the exact top-k keeps the
// k largest z (equal scores to the lower token) and the recall of a selection
// S is |S n top-k| / k.
//
// Three kernels: logits (one thread per key, q' in shared memory, fp32 dot
// products in channel order), the top-k (one CTA per unit: an order-key
// radix select over the unit's scores, read from L2 once per level), and the
// recall (a bitmap of the exact top-k in shared memory).
#include <algorithm>

#include "hhr_api_internal.h"
#include "hhr_dev.cuh"

namespace hhr {
namespace {

constexpr int TK_THREADS = 512;

// q' = R_h q for the G query heads of (b, h) into shared memory qs[G][128].
__device__ void tk_rotate_query(const Dims& dm, const __nv_bfloat16* q, const float* R, int b, int h, float* qs,
                                float* qf) {
  const int G = dm.G;
  const __nv_bfloat16* qg = q + ((long long)b * dm.Hq + h * G) * D;
  for (int i = threadIdx.x; i < G * D; i += blockDim.x) qf[i] = __bfloat162float(qg[i]);
  __syncthreads();
  const float* Rh = R + (long long)h * D * D;
  for (int e = threadIdx.x; e < G * D; e += blockDim.x) {
    const int g = e / D, i = e - g * D;
    float s = 0.f;
    for (int j = 0; j < D; ++j) s = fmaf(__ldg(Rh + i * D + j), qf[g * D + j], s);
    qs[g * D + i] = s;
  }
  __syncthreads();
}

// z[b, h, t] = max_g q'_g . k'_t for t < L (fp32, channel order); -inf past L.
__global__ void __launch_bounds__(TK_THREADS) topk_logits_kernel(Dims dm, const __nv_bfloat16* q, const float* R,
                                                                 const __nv_bfloat16* Kr, const int* seq_lens,
                                                                 const int* table, float* z, int* status) {
  __shared__ float qs[8 * D], qf[8 * D];
  const int h = blockIdx.y, b = blockIdx.z;
  const int L = seq_len_of(dm, seq_lens, b);
  const int t = blockIdx.x * TK_THREADS + threadIdx.x;
  if (blockIdx.x * TK_THREADS >= dm.T) return;
  tk_rotate_query(dm, q, R, b, h, qs, qf);
  if (t >= dm.T) return;
  float out = -INFINITY;
  if (t < L) {
    const long long off = kv_row(dm, table, b, h, t, status);
    if (off >= 0) {
      float acc[8];
#pragma unroll
      for (int g = 0; g < 8; ++g) acc[g] = 0.f;
      for (int v = 0; v < D / 8; ++v) {
        float k8[8];
        unpack8(ldg16(Kr + off + v * 8), k8);
#pragma unroll
        for (int g = 0; g < 8; ++g)
          if (g < dm.G) {
#pragma unroll
            for (int c = 0; c < 8; ++c) acc[g] = fmaf(qs[g * D + v * 8 + c], k8[c], acc[g]);
          }
      }
      for (int g = 0; g < dm.G; ++g) out = fmaxf(out, acc[g]);
    }
  }
  z[((long long)b * dm.Hkv + h) * dm.T + t] = out;
}

// Exact top-k of one unit's scores: thread t owns positions [t m, (t+1) m)
// (m = ceil(L / 512)), levels of a radix select on order keys (11 bits per
// level from the keys' range, as the page select), equal keys in index order;
// the kept positions are written ascending.
__global__ void __launch_bounds__(TK_THREADS) topk_select_kernel(Dims dm, const float* z, const int* seq_lens,
                                                                 const int* top_k, int kmax, int* sel, int* n_sel) {
  __shared__ int hist[2][2048];
  __shared__ int red[160];
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int L = seq_len_of(dm, seq_lens, b);
  const float* zu = z + ((long long)b * dm.Hkv + h) * dm.T;
  const int k = min(min(max(__ldg(top_k + b), 1), kmax), L);
  const int m = (L + TK_THREADS - 1) / TK_THREADS;
  const int j0 = min(L, tid * m), j1 = min(L, j0 + m);
  int* bc = red + 128;
  unsigned lo = 0xffffffffu, hi = 0u;
  for (int j = j0; j < j1; ++j) {
    const unsigned kk = order_key(__ldcg(zu + j));
    lo = min(lo, kk);
    hi = max(hi, kk);
  }
  for (int i = tid; i < 4096; i += TK_THREADS) (&hist[0][0])[i] = 0;
  block_minmax_u32(lo, hi, reinterpret_cast<unsigned*>(red + 64));
  // level state: the candidates are the keys in [base, base + span]; every
  // key above that range is kept
  unsigned base = lo, span = hi - lo;
  int need = k, par = 0;
  unsigned thr_hi = 0u;  // keys >= thr_hi are kept ...
  unsigned tie = 0u;     // ... and, when all_ties, the first take_ties keys equal to `tie`
  int take_ties = 0;
  bool all_ties = false;
  if (k < L) {
#pragma unroll 1
    for (int level = 0;; ++level) {
      const int shift = span < 2048u ? 0 : (32 - __clz(span)) - 11;
      int* hc = hist[level & 1];
      int* hn = hist[(level + 1) & 1];
      for (int j = j0; j < j1; ++j) {
        const unsigned kk = order_key(__ldcg(zu + j));
        if (kk >= base && kk - base <= span) atomicAdd(&hc[(kk - base) >> shift], 1);
      }
      __syncthreads();
      int hv[4], c4 = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        hv[e] = hc[2047 - 4 * tid - e];
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
      for (int i = tid; i < 2048; i += TK_THREADS) hn[i] = 0;
      __syncthreads();
      const int bstar = bc[0], need_in = bc[1], cnt_in = bc[2];
      const unsigned bin_lo = base + ((unsigned)bstar << shift);
      if (cnt_in == need_in) {  // the whole bin is kept: every key >= bin_lo
        thr_hi = bin_lo;
        break;
      }
      if (shift == 0) {  // one key value: the keys above it, then the first need_in equal ones
        thr_hi = bin_lo + 1u;
        tie = bin_lo;
        take_ties = need_in;
        all_ties = true;
        break;
      }
      need = need_in;
      span = min(span - ((unsigned)bstar << shift), (1u << shift) - 1u);
      base = bin_lo;
    }
  }
  // keep: key >= thr_hi, or key == tie among the first take_ties (index order)
  int cgt = 0, ceq = 0;
  for (int j = j0; j < j1; ++j) {
    const unsigned kk = order_key(__ldcg(zu + j));
    cgt += kk >= thr_hi;
    ceq += (all_ties && kk == tie) ? 1 : 0;
  }
  int tot;
  const int pg = block_scan_excl(cgt, red, par++, &tot);
  const int pe = block_scan_excl(ceq, red, par++, &tot);
  int run_g = pg, run_e = pe;
  int* out = sel + ((long long)b * dm.Hkv + h) * kmax;
  for (int j = j0; j < j1; ++j) {
    const unsigned kk = order_key(__ldcg(zu + j));
    const bool gt = kk >= thr_hi, eq = all_ties && kk == tie;
    if (gt || (eq && run_e < take_ties)) {
      // position = kept keys before j: those above the threshold, plus the ties taken
      const int pos = run_g + min(run_e, take_ties);
      if (pos < kmax) out[pos] = j;
    }
    run_g += gt;
    run_e += eq;
  }
  if (tid == 0) n_sel[b * dm.Hkv + h] = k;
}

// recall[b, h] = |A n B| / |B| for ascending index lists A (a selection) and
// B (the exact top-k) of one unit: B is marked in a shared-memory bitmap.
__global__ void __launch_bounds__(TK_THREADS) recall_kernel(Dims dm, const int* sel_a, const int* n_a, int stride_a,
                                                            const int* sel_b, const int* n_b, int stride_b,
                                                            float* recall) {
  extern __shared__ unsigned bits[];
  const int u = blockIdx.x, tid = threadIdx.x;
  const int nw = (dm.T + 31) / 32;
  for (int i = tid; i < nw; i += TK_THREADS) bits[i] = 0u;
  __syncthreads();
  const int nb = n_b[u], na = n_a[u];
  for (int i = tid; i < nb; i += TK_THREADS) {
    const int t = sel_b[(long long)u * stride_b + i];
    if (t >= 0 && t < dm.T) atomicOr(&bits[t >> 5], 1u << (t & 31));
  }
  __syncthreads();
  int hit = 0;
  for (int i = tid; i < na; i += TK_THREADS) {
    const int t = sel_a[(long long)u * stride_a + i];
    hit += (t >= 0 && t < dm.T) ? (bits[t >> 5] >> (t & 31)) & 1 : 0;
  }
  int tot;
  __shared__ int red[64];
  block_scan_excl(hit, red, 0, &tot);
  if (tid == 0) recall[u] = nb > 0 ? (float)tot / (float)nb : 0.f;
}

}  // namespace
}  // namespace hhr

using namespace hhr;

extern "C" {

hhr_status hhr_exact_topk(const hhr_config* cfg, const void* q, const float* R, const void* Krot,
                          const int32_t* seq_lens, const int32_t* block_table, const int32_t* top_k,
                          int32_t max_top_k, float* logits, int32_t* sel, int32_t* n_sel, int32_t* device_status,
                          hhr_stream_t stream) {
  Dims dm;
  hhr_status s = make_dims(cfg, &dm);
  if (s != HHR_OK) return s;
  if (!q || !R || !Krot || !seq_lens || !top_k || !logits || !sel || !n_sel)
    return record_error(HHR_ERR_INVALID_ARG, "hhr_exact_topk: NULL pointer");
  if (dm.paged && !block_table) return record_error(HHR_ERR_INVALID_ARG, "hhr_exact_topk: paged needs block_table");
  if (((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(Krot) | reinterpret_cast<uintptr_t>(R)) & 15u) != 0)
    return record_error(HHR_ERR_INVALID_ARG, "hhr_exact_topk: tensor not 16-byte aligned");
  if (max_top_k < 1) return record_error(HHR_ERR_INVALID_ARG, "hhr_exact_topk: max_top_k must be >= 1");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const dim3 g1((dm.T + TK_THREADS - 1) / TK_THREADS, dm.Hkv, dm.B);
  topk_logits_kernel<<<g1, TK_THREADS, 0, st>>>(dm, static_cast<const __nv_bfloat16*>(q), R,
                                                static_cast<const __nv_bfloat16*>(Krot), seq_lens, block_table, logits,
                                                device_status);
  topk_select_kernel<<<dim3(dm.Hkv, dm.B), TK_THREADS, 0, st>>>(dm, logits, seq_lens, top_k, max_top_k, sel, n_sel);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return record_error(HHR_ERR_CUDA, cudaGetErrorString(e));
  return record_error(HHR_OK, "");
}

hhr_status hhr_recall(const hhr_config* cfg, const int32_t* sel_a, const int32_t* n_a, int32_t stride_a,
                      const int32_t* sel_b, const int32_t* n_b, int32_t stride_b, float* recall, hhr_stream_t stream) {
  Dims dm;
  hhr_status s = make_dims(cfg, &dm);
  if (s != HHR_OK) return s;
  if (!sel_a || !n_a || !sel_b || !n_b || !recall) return record_error(HHR_ERR_INVALID_ARG, "hhr_recall: NULL pointer");
  if (stride_a < 1 || stride_b < 1) return record_error(HHR_ERR_INVALID_ARG, "hhr_recall: strides must be >= 1");
  const size_t smem = sizeof(unsigned) * ((dm.T + 31) / 32);
  if (smem > 200 * 1024) return record_error(HHR_ERR_UNSUPPORTED, "hhr_recall: max_seq_len too long");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(recall_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return record_error(HHR_ERR_CUDA, "hhr_recall: shared memory attribute");
  recall_kernel<<<dm.B * dm.Hkv, TK_THREADS, smem, st>>>(dm, sel_a, n_a, stride_a, sel_b, n_b, stride_b, recall);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return record_error(HHR_ERR_CUDA, cudaGetErrorString(e));
  return record_error(HHR_OK, "");
}

}  // extern "C"
