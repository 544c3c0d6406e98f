/*
 * hhr.h -- C ABI of the HHR decode-path library (libhhr.so), sm_100a.
 *
 * HHR ("HHR: Hierarchical Hash Retrieval for Efficient LLM Generation",
 * paper card, Abstract) retrieves keys for one decode step in two stages
 * before attention (rit.work explainer, section "Два уровня маршрутизации
 * решают разные ошибки"):
 *   GKR  keys are stored rotated by a per-KV-head orthogonal R_h (q.k is
 *        unchanged); pages of P neighbouring keys keep channel min/max; each
 *        page gets a logit upper bound and only the top-N pages survive.
 *   LHP  keys of surviving pages are ranked by the Hamming distance between
 *        sign codes of W_h k and W_h q; the top-k keys are kept.
 *   Then exact softmax attention runs over the kept keys only.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The
 *     library never allocates or frees device memory and never synchronises;
 *     every call is enqueued on `stream` and returns immediately.
 *   - The return value reports host-side validation and launch errors only.
 *     Device-side problems (a block-table entry outside the pool, a bounded
 *     wait that ran out) are written to `device_status` (an int32 the caller
 *     zeroes and reads after synchronising); kernels never trap.
 *   - bf16 tensors and uint64 codes must be 16-byte aligned (vector loads).
 *   - head_dim must be 128; num_q_heads must be a multiple of num_kv_heads
 *     with a group size G = num_q_heads / num_kv_heads of 1..8; page_size 16
 *     or 32; hash_bits 64, 128 or 256.
 *   - No C++ exception crosses this boundary.
 *
 * Layouts (row-major, innermost last).  d = head_dim, T = max_seq_len,
 * np = ceil(T / page_size), w = hash_bits / 64, Bk = num_blocks.
 *   contiguous (paged == 0)        paged (paged == 1, block = one page)
 *   K, Krot, V : [B, Hkv, T, d]    [Bk, Hkv, P, d]
 *   page_min/max: [B, Hkv, np, d]  [Bk, Hkv, d]
 *   codes       : [B, Hkv, T, w]   [Bk, Hkv, P, w]
 *   block_table : unused (NULL)    int32 [B, max_blocks_per_seq]; logical
 *                                  page p of sequence b lives in block
 *                                  block_table[b * max_blocks_per_seq + p]
 *   q : bf16 [B, Hq, d];  R : fp32 [Hkv, d, d] with k' = R_h k (row i of
 *   R_h gives channel i);  W : bf16 [Hkv, hash_bits, d];  out : fp32 [B, Hq, d].
 *   Query head hq belongs to KV head hq / G.
 */
#ifndef HHR_H_
#define HHR_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define HHR_API __attribute__((visibility("default")))
#else
#define HHR_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL means the legacy default stream. */
typedef struct CUstream_st* hhr_stream_t;

typedef enum {
  HHR_OK = 0,
  HHR_ERR_INVALID_ARG = 1,  /* null / misaligned pointer, bad size or shape  */
  HHR_ERR_UNSUPPORTED = 2,  /* head_dim, group size, bits or page size       */
  HHR_ERR_WORKSPACE = 3,    /* workspace too small for the requested budgets */
  HHR_ERR_CUDA = 4,         /* a CUDA launch or copy failed                  */
  HHR_ERR_TIMEOUT = 5,      /* (device_status only) a bounded wait ran out   */
  HHR_ERR_BAD_BLOCK = 6     /* (device_status only) block id outside the pool */
} hhr_status;

typedef struct {
  int32_t batch;              /* B                                            */
  int32_t num_q_heads;        /* Hq                                           */
  int32_t num_kv_heads;       /* Hkv                                          */
  int32_t head_dim;           /* d, must be 128                               */
  int32_t page_size;          /* P: 16 or 32 (the block size when paged)      */
  int32_t hash_bits;          /* 64, 128 or 256                               */
  int32_t max_seq_len;        /* T: capacity of one sequence                  */
  int32_t paged;              /* 0 contiguous, 1 block pool + block table     */
  int32_t num_blocks;         /* Bk: blocks in the pool (paged only)          */
  int32_t max_blocks_per_seq; /* row length of block_table (paged only)       */
  /* How the G query heads of a KV head are combined (the paper is silent on
   * grouped query heads; 0 selects the library's readings):                 */
  int32_t page_group_agg;     /* page bound U_p: 0 max over the heads, 1 sum  */
  int32_t key_group_agg;      /* key score S_j: 0 sum over the heads, 1 min   */
} hhr_config;

/* Optional stage outputs of hhr_decode_step (any pointer may be NULL). They
 * expose each stage's result so that it can be checked on its own.
 * np_max = ceil(T / P), Nmax = max_keep_pages, Kmax = max_top_k.            */
typedef struct {
  float* q_rot;          /* [B, Hq, d]        q' = R_h q                        */
  float* page_ub;        /* [B, Hq, np_max]   per query head page bound          */
  float* page_U;         /* [B, Hkv, np_max]  max of page_ub over the group      */
  int32_t* sel_pages;    /* [B, Hkv, Nmax]    kept pages, ascending              */
  int32_t* n_sel_pages;  /* [B, Hkv]                                             */
  uint64_t* q_codes;     /* [B, Hq, w]        query sign codes                   */
  int32_t* key_scores;   /* [B, Hkv, Nmax*P]  group Hamming distance per candidate
                                              (candidate order: kept pages
                                              ascending, rows ascending; rows past
                                              the sequence end hold INT32_MAX)   */
  int32_t* n_cand;       /* [B, Hkv]          valid candidates                   */
  int32_t* sel_keys;     /* [B, Hkv, Kmax]    kept token ids, ascending          */
  int32_t* n_sel_keys;   /* [B, Hkv]                                             */
} hhr_debug;

/* Human-readable name of a status code (static storage). */
HHR_API const char* hhr_status_string(hhr_status s);

/* Message describing the last host-side validation failure on this thread
 * (static thread-local storage; empty when the last call succeeded). */
HHR_API const char* hhr_last_error(void);

/* Bound of every device-side wait of the launches that follow (a CTA waiting
 * for the other CTAs of its group, a reader polling the kept-row list), in SM
 * clock cycles; cycles <= 0 restores the default of 4e9 (about 2 s).  On
 * expiry a launch records HHR_ERR_TIMEOUT in its device_status and returns
 * (see hhr_decode_step).  The paper has no counterpart: this is a testing and
 * watchdog aid.  Process-wide; takes effect at the next launch. */
HHR_API void hhr_set_wait_limit(int64_t cycles);

/*
 * hhr_build_cache -- cache build for one layer (prefill side of HHR).
 *
 * GKR stores keys in the basis of the head-wise orthogonal transform, which
 * leaves every query-key product unchanged (paper card, Abstract; rit.work,
 * two-level routing section); pages keep what their bound needs; LHP keys
 * get sign codes (paper page, Figure 2 caption: projection then sign).
 * For every sequence b, KV head h and row t < seq_lens[b]:
 *   Krot[t] = bf16_rne(R_h K[t])                 (the exact product rounded
 *                                                 once: tensor-core fp32
 *                                                 accumulation, elements near
 *                                                 a rounding midpoint
 *                                                 recomputed in fp64)
 *   codes[t] bit j = [ (W_h K[t])_j > 0 ]        (unrotated K; bit j in word
 *                                                 j/64 at position j%64; the
 *                                                 sign is exact: near-zero
 *                                                 projections are recomputed
 *                                                 in fp64)
 *   page_min/max[p] = channel min/max of the stored Krot rows of page p that
 *                     lie below seq_lens[b]
 *   Vcache = V (copied unless Vcache == V).
 * Rows at or past seq_lens[b] and pages past the last valid one are left
 * untouched (V rows are copied for t < seq_lens[b] only).  Krot may alias K
 * (in place).  seq_lens is a device array [B].
 */
HHR_API hhr_status hhr_build_cache(const hhr_config* cfg, const void* K, const void* V,
                           const float* R, const void* W, const int32_t* seq_lens,
                           const int32_t* block_table, void* Krot, void* Vcache,
                           void* page_min, void* page_max, uint64_t* codes,
                           hhr_stream_t stream);

/*
 * hhr_append_cache -- extends the cache as tokens are generated.
 *
 * A decode loop adds one key and value per step; GKR keeps a bound per page
 * of neighbouring keys, so the new key must be rotated and hashed and its
 * page's stored min/max kept current (rit.work explainer, sections "Два
 * уровня маршрутизации решают разные ошибки": pages of neighbouring keys with
 * a bound each, and "Когда HHR меняет планы запуска модели": the page bounds
 * are stored with the cache).  For every sequence b, rows t in
 * [old_lens[b], new_lens[b]) are built exactly as hhr_build_cache builds them
 * (K'[t], codes[t], V copied unless Vcache == V), and the min/max of every page
 * they touch is merged with that page's rows below old_lens[b] (a page that
 * starts at t is opened).  The cache then equals, bit for bit, a
 * hhr_build_cache over [0, new_lens[b]).
 *   - K and V hold the new rows at their cache positions (same layouts as
 *     hhr_build_cache); only rows >= old_lens[b] are read, so K may alias
 *     Krot (write the raw key into Krot's row, then append).
 *   - old_lens and new_lens are device arrays [B]; lengths are clamped to
 *     [0, max_seq_len] and a sequence with new_lens[b] <= old_lens[b] is left
 *     untouched.  max_new (host) bounds new_lens[b] - old_lens[b]; it sizes
 *     the launch (rows beyond it are not built).
 *   - Paged: the blocks of the new rows must already be in block_table.
 */
HHR_API hhr_status hhr_append_cache(const hhr_config* cfg, const void* K, const void* V, const float* R,
                                    const void* W, const int32_t* old_lens, const int32_t* new_lens,
                                    int32_t max_new, const int32_t* block_table, void* Krot, void* Vcache,
                                    void* page_min, void* page_max, uint64_t* codes, hhr_stream_t stream);

/* Bytes of workspace hhr_decode_step needs for these budgets. */
HHR_API size_t hhr_decode_workspace_size(const hhr_config* cfg, int32_t max_keep_pages,
                                 int32_t max_top_k);

/* Zero a workspace before its first use (the decode step keeps its arrival
 * counters and per-unit score histograms at zero between calls).  Enqueued
 * on `stream`. */
HHR_API hhr_status hhr_workspace_init(void* workspace, size_t workspace_bytes, hhr_stream_t stream);

/*
 * hhr_decode_step -- one HHR decode step of one layer for all sequences.
 *
 * For each sequence b with L = seq_lens[b], np = ceil(L / P), each KV head h
 * and its query heads g (hq = h*G + g):
 *  1. q'_g = R_h q_g (fp32).                      GKR rotation (Abstract)
 *  2. ub[g,p] = sum_i max(q'_gi mn_pi, q'_gi mx_pi); U_p = max_g ub[g,p]
 *     (sum_g with cfg->page_group_agg = 1).       page logit bound (Abstract)
 *  3. keep N = min(clamp(n_keep_pages[b], 1, max_keep_pages), np) pages with
 *     the largest U_p; equal bounds go to the lower page index.  Coarse
 *     pruning of whole pages (rit.work, two-level routing section).
 *  4. query codes: bit j = [ (W_h q_g)_j > 0 ] (exact sign, fp64 fallback).
 *  5. for the valid rows of kept pages: S = sum_g popcount(code_g ^ code_row)
 *     (min_g with cfg->key_group_agg = 1).
 *  6. keep k = min(clamp(top_k[b], 1, max_top_k), #candidates) rows with the
 *     smallest S; equal scores go to the lower token index.
 *  7. out[b, hq] = sum_j softmax_j(sm_scale * q'_g . Krot_j) V_j over the kept
 *     rows (fp32 accumulation, fp32 output).  L == 0 gives a zero output.
 * n_keep_pages and top_k are device arrays [B]; max_keep_pages and max_top_k
 * are their host-side upper bounds and size the workspace.  `dbg` may be
 * NULL.  `workspace` must be at least hhr_decode_workspace_size() bytes,
 * 256-byte aligned, zeroed once with hhr_workspace_init(), and not shared by
 * calls that may run concurrently.  `device_status` may be NULL.
 *
 * One kernel launch of at most one CTA per SM (the library checks on the host
 * that a CTA fits on an SM); the CTAs of a group that shares a (sequence, KV
 * head) wait for one another, so the launch expects the SMs it was sized for
 * (a kernel occupying SMs on another stream delays it; one that holds them
 * past the wait limit makes it end with HHR_ERR_TIMEOUT).  Every
 * device-side wait is bounded (hhr_set_wait_limit): on expiry the launch
 * records HHR_ERR_TIMEOUT in `device_status` and returns.  After any call
 * whose device status is not HHR_OK, zero the workspace again
 * (hhr_workspace_init) before the next call: its counters and histograms
 * may be left mid-use.  Results are deterministic for a given launch shape
 * (the CTAs per unit follow from the SM count, the number of (sequence, KV
 * head) units and the budgets) and do not depend on the layout (contiguous or
 * paged); selections do not depend on the shape at all.
 *
 * The launch is a programmatic dependent launch: it may start while the
 * previous kernel on `stream` is still running and then reads R and W (the
 * learned per-head transforms) before that kernel has finished; everything
 * else (q, the cache, lengths, budgets, the workspace, out) is read or written
 * only after it has finished.  Do not write R or W in the kernel launched just
 * before.
 */
HHR_API hhr_status hhr_decode_step(const hhr_config* cfg, const void* q, const float* R, const void* W,
                           const void* Krot, const void* Vcache, const void* page_min,
                           const void* page_max, const uint64_t* codes,
                           const int32_t* seq_lens, const int32_t* block_table,
                           const int32_t* n_keep_pages, const int32_t* top_k,
                           int32_t max_keep_pages, int32_t max_top_k, float sm_scale,
                           float* out, const hhr_debug* dbg, void* workspace,
                           size_t workspace_bytes, int32_t* device_status,
                           hhr_stream_t stream);

/* Size of the scratch array behind hhr_decode_step_noalloc (16 MiB). */
#define HHR_NOALLOC_SCRATCH_BYTES (16u << 20)

/*
 * hhr_decode_step_noalloc -- hhr_decode_step without a caller workspace.
 *
 * (The paper has no counterpart; this is a library convenience.)  Some
 * callers cannot call cudaMalloc at all: plugins of inference runtimes that
 * must draw every byte of device memory from the host runtime's own pool
 * (and may not allocate behind its back), and latency-critical serving loops
 * in which an allocation, with the device synchronisation it can bring, is
 * not allowed.  Such callers still pass every input and output, but the
 * scratch comes from a fixed HHR_NOALLOC_SCRATCH_BYTES array in the
 * library's device memory, which every GPU that loads the library holds
 * until the process exits.
 *   - Same arguments, checks, status codes and results as hhr_decode_step,
 *     minus the workspace.  Every host-side check runs before anything is
 *     enqueued on `stream`.
 *   - Sizes whose workspace (hhr_decode_workspace_size) exceeds the array are
 *     rejected with HHR_ERR_WORKSPACE and a message; nothing is enqueued.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *   - The first call on a device looks up the array's device address with
 *     that device current (cudaGetSymbolAddress) and caches it; make that
 *     first call before any stream capture.
 *   - Every call clears the part of the array it uses (one cudaMemsetAsync on
 *     `stream`) and then runs the decode step in it.  All calls share the one
 *     array, so calls that may overlap on the GPU (other streams, other host
 *     threads) race with each other: serialise them.
 */
HHR_API hhr_status hhr_decode_step_noalloc(const hhr_config* cfg, const void* q, const float* R,
                                           const void* W, const void* Krot, const void* Vcache,
                                           const void* page_min, const void* page_max,
                                           const uint64_t* codes, const int32_t* seq_lens,
                                           const int32_t* block_table, const int32_t* n_keep_pages,
                                           const int32_t* top_k, int32_t max_keep_pages,
                                           int32_t max_top_k, float sm_scale, float* out,
                                           const hhr_debug* dbg, int32_t* device_status,
                                           hhr_stream_t stream);

/*
 * hhr_exact_topk -- the exact top-k keys, the reference of the recall metric
 * ("HHR: Hierarchical Hash Retrieval for Efficient LLM Generation",
 * thelatestinai.com page, Figure 4 caption: "Top-10% key recall").
 *
 * For every sequence b (L = seq_lens[b]) and KV head h, the score of key t < L
 * is the largest logit of the group's query heads,
 *   logits[b, h, t] = max_g (R_h q_g) . Krot[t]       (fp32, channel order),
 * and -inf for t >= L (layout [B, Hkv, max_seq_len]).  sel[b, h, :n] holds the
 * k = min(clamp(top_k[b], 1, max_top_k), L) keys with the largest scores,
 * ascending (equal scores go to the lower token); n_sel[b, h] = k.
 * top_k is a device array [B]; sel is [B, Hkv, max_top_k].  Same layouts and
 * alignment rules as hhr_decode_step; no workspace (logits is the scratch).
 * The paper has no kernel for this: it is the measuring stick of Figure 4.
 */
HHR_API hhr_status hhr_exact_topk(const hhr_config* cfg, const void* q, const float* R, const void* Krot,
                                  const int32_t* seq_lens, const int32_t* block_table, const int32_t* top_k,
                                  int32_t max_top_k, float* logits, int32_t* sel, int32_t* n_sel,
                                  int32_t* device_status, hhr_stream_t stream);

/*
 * hhr_recall -- recall[u] = |A_u n B_u| / |B_u| for every unit u = b*Hkv + h,
 * where A_u = sel_a[u*stride_a .. +n_a[u]) (e.g. the keys a decode step kept:
 * hhr_debug.sel_keys) and B_u = sel_b[u*stride_b .. +n_b[u]) (e.g. the exact
 * top-k of hhr_exact_topk).  Token ids outside [0, max_seq_len) are ignored.
 * Device arrays; recall is float [B*Hkv] (0 where B_u is empty).
 */
HHR_API hhr_status hhr_recall(const hhr_config* cfg, const int32_t* sel_a, const int32_t* n_a, int32_t stride_a,
                              const int32_t* sel_b, const int32_t* n_b, int32_t stride_b, float* recall,
                              hhr_stream_t stream);

/* Bytes of workspace hhr_dense_decode needs. */
HHR_API size_t hhr_dense_workspace_size(const hhr_config* cfg);

/*
 * hhr_dense_decode -- full decode attention over all L = seq_lens[b] keys of
 * the same cache (the "Full Attention" comparison row of the paper's tables):
 *   out[b, hq] = sum_{t<L} softmax_t(sm_scale * (R_h q) . Krot_t) V_t
 * Same layouts, workspace and status rules as hhr_decode_step.
 */
HHR_API hhr_status hhr_dense_decode(const hhr_config* cfg, const void* q, const float* R,
                            const void* Krot, const void* Vcache, const int32_t* seq_lens,
                            const int32_t* block_table, float sm_scale, float* out,
                            void* workspace, size_t workspace_bytes, int32_t* device_status,
                            hhr_stream_t stream);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* HHR_H_ */
