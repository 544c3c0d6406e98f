// HHR decode step as one persistent, warp-specialised kernel per layer (sm_100a).
// The library launches it for the dense comparison (DENSE = 1: every row, no
// selects); the sparse decode step runs in hhr_group.cuh, which also uses the
// device helpers of this file (mbarriers, bulk copies, scans, reductions, the
// partial merge).  The sparse items below are not instantiated.
//
// Work is a queue of items claimed in order by the CTAs (one CTA per SM).
// For units u = (sequence b, KV head h) the queue holds, in this order:
//   PREP(u)        for every unit: q' = R_h q, then the query sign codes
//   SCAN(u, c)     page bounds of pages [128c, 128c + 128)
//   SCORE(u, c)    Hamming scores of candidates [1024c, 1024c + 1024) (the
//                  rows of the kept pages, in page order) and their histogram
//   GATHER(u, c)   softmax attention over kept rows [128c, 128c + 128),
//                  written as a partial per chunk
// Four more steps are tasks, made by the CTA whose counter increment completes
// their inputs.  Group merges stay in that CTA; the others join a grid-wide
// queue and the first CTA whose consumers are free (they look at the queue
// before every item) runs them:
//   PSEL(u)        after the last scan chunk of u: page top-N
//   KSEL(u)        after the last score chunk of u: key top-k from the
//                  score histogram, kept rows compacted in index order
//   GMERGE(u, g)   after the 16 gather chunks of group g: their partials merged
//   MERGE(u)       after the last group: the groups merged into the output
// No CTA ever waits for another CTA's consumers; only the producer waits, for
// q' (scan), the kept pages and query codes (score) or the kept rows (gather)
// of a unit claimed before.
//
// Warps 0-15 consume; warp 16 (producer) claims items, moves contiguous
// blocks (R_h, W_h, q or q', page metadata, dense K'/V) into a ring of shared
// memory slots with cp.async.bulk, each slot completing on an mbarrier, and
// lists the rows at scattered addresses (kept or paged K'/V rows, paged
// metadata, code pages), which the consumer warps copy themselves one item
// ahead; warp 17 (finisher) publishes completions (a gpu-scope fence, then an
// acquire-release counter increment) and queues the tasks that become ready.
// In the scan and the gather a group of 8 or 16 lanes shares a 128-channel
// row, each lane holding 16 or 8 channels, so a dot product is reduced over
// that group only; the rest of the warp's work is warp-local.
//
// Every wait (mbarrier, shared flag or global counter) is bounded by a clock
// budget; on expiry the kernel records HHR_ERR_TIMEOUT in the status word,
// drains its own copies in flight and returns.  Results do not depend on the
// schedule: every partial and every merge has a fixed place and order.
#pragma once

#include <climits>

#include "hhr_common.cuh"
#include "hhr_launch.h"

namespace hhr {

// ---------------------------------------------------------------------------
// PTX helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// 1-D bulk copy global -> shared (16-byte aligned, size a multiple of 16)
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}
// the same for bytes read once: marked first to leave L2 (code, queue words and
// partials stay resident while the cache streams through)
__device__ __forceinline__ void bulk_g2s_stream(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                                uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}
__device__ __forceinline__ uint64_t evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
// 16-byte asynchronous copy global -> shared through L2 only (the rows that
// consumer threads gather themselves), and its group bookkeeping
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ void st_release(unsigned* p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ unsigned ld_relaxed(const unsigned* p) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ unsigned atom_add_acq_rel(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// ---------------------------------------------------------------------------
// parameters
// ---------------------------------------------------------------------------
constexpr int FZ_CONS = 512;                 // consumer threads (warps 0-15)
constexpr int FZ_CWARPS = FZ_CONS / 32;
constexpr int FZ_PRODUCER_WARP = FZ_CWARPS;
constexpr int FZ_FINISHER_WARP = FZ_CWARPS + 1;
constexpr int FZ_THREADS = FZ_CONS + 128;    // + one warpgroup: producer, finisher, two idle warps
// Registers: the block starts with 96 per thread (20 warps); the last
// warpgroup gives most of its share to the consumers.
constexpr int FZ_REGS_CONS = 104, FZ_REGS_AUX = 64;
static_assert(FZ_CONS * FZ_REGS_CONS + 128 * FZ_REGS_AUX <= FZ_THREADS * 96, "register split");
constexpr int FZ_NSLOT = 8;                  // ring slots
constexpr int FZ_SLOT = 16384;               // bytes per slot (64 rows of 256 B)
constexpr int FZ_NDESC = 4;                  // descriptor ring
constexpr int FZ_NFIN = 8;                   // finisher ring
constexpr int FZ_NTASK = 16;                 // local task ring (group merges)
constexpr int FZ_QBUF = 4096;                // q (bf16) or q' (fp32) of one unit
constexpr int FZ_ROWS = FUSED_ROWS;          // pages per SCAN item, rows per GATHER item
constexpr int FZ_CS = FUSED_SCORE;           // candidates per SCORE item
constexpr int FZ_GROUP = FUSED_GROUP;        // gather chunks per group merge
constexpr int FZ_WORK = 74752;               // consumer scratch
constexpr int FZ_SEQ = 256;                  // sequences whose length, n_keep and top_k sit in shared memory
constexpr int FZ_HIST_BINS = 2052;           // >= 8 heads x 256 bits + 1
constexpr long long FZ_WAIT_CYCLES = 4000000000ll;  // ~2 s at 1.9 GHz

constexpr size_t FZ_OFF_RING = 0;
constexpr size_t FZ_OFF_QBUF = FZ_OFF_RING + (size_t)FZ_NSLOT * FZ_SLOT;
constexpr size_t FZ_OFF_WORK = FZ_OFF_QBUF + (size_t)FZ_NDESC * FZ_QBUF;
constexpr size_t FZ_OFF_SEQP = FZ_OFF_WORK + FZ_WORK;
constexpr size_t FZ_OFF_RIDX = FZ_OFF_SEQP + 3 * FZ_SEQ * 4;
constexpr int FZ_UCACHE = 512;               // units whose readiness the producer remembers
constexpr size_t FZ_OFF_UCACHE = FZ_OFF_RIDX + FZ_NDESC * FZ_ROWS * 4;
constexpr size_t FZ_OFF_DESC = FZ_OFF_UCACHE + FZ_UCACHE * 4;
constexpr size_t FZ_OFF_FINQ = FZ_OFF_DESC + FZ_NDESC * 32;
constexpr size_t FZ_OFF_TASK = FZ_OFF_FINQ + FZ_NFIN * 32;
constexpr size_t FZ_OFF_BAR = FZ_OFF_TASK + FZ_NTASK * 16;
constexpr size_t FZ_OFF_MISC = FZ_OFF_BAR + 8 * (2 * FZ_NSLOT + 2 * FZ_NDESC + 2 * FZ_NFIN);
constexpr size_t FZ_SMEM = FZ_OFF_MISC + 256;
static_assert(FZ_SMEM <= 232448, "shared memory of the fused kernel");
static_assert(4 * FZ_HIST_BINS <= FZ_WORK, "score histogram");

enum : int { IT_PREP = 0, IT_SCAN = 1, IT_SCORE = 2, IT_GATHER = 3, IT_END = 4 };
enum : int { TK_PSEL = 10, TK_KSEL = 11, TK_GMERGE = 12, TK_MERGE = 13 };

// A descriptor with `gather` set names rows that the consumer threads copy
// themselves (16-byte cp.async): ridx[j] is the 256-byte row number of row j
// in the item's first tensor and second tensor alike (K' and V, or the page
// minima and maxima), -1 for a row whose block id is bad.
struct __align__(16) FzDesc {
  int kind, unit, chunk, n;
  int nslots, pad0, gather, pad2;
};

// finisher request: after a gpu-scope fence add `value` to `counter`; if the
// counter then reaches `target`, post task (kind, unit, arg) to this CTA
struct __align__(16) FzFin {
  unsigned* counter;
  unsigned value;
  unsigned target;  // 0: no task
  int kind, unit, arg, pad;
};


struct __align__(16) FzTask {
  int kind, unit, arg, pad;
};

// per-unit control words (kept at zero between calls; the last CTA resets them)
enum : int {
  CU_PREP = 0,    // q' published
  CU_CODES = 1,   // query codes published
  CU_SEL = 2,     // kept rows published (sel_keys, CU_NKEYS)
  CU_SCAN = 3,    // scan chunks finished
  CU_MERGED = 4,  // groups merged
  CU_NKEYS = 5,   // kept rows
  CU_PSEL = 6,    // kept pages published
  CU_SCORE = 7,   // score chunks finished
  CU_STRIDE = 8
};

struct FzParams {
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
  int items_per_unit_scan;    // C1 (sparse) or 0 (dense)
  int items_per_unit_score;   // C2 (sparse) or 0 (dense)
  int items_per_unit_gather;  // C3
  int total_items;
  int gsize, ngroups;         // group kernel: CTAs per group, groups
};

struct FzShared {
  unsigned char* ring;
  unsigned char* qbuf;
  unsigned char* work;
  FzDesc* desc;
  FzFin* finq;
  FzTask* tasks;
  uint64_t* full;
  uint64_t* empty;
  uint64_t* dfull;
  uint64_t* dempty;
  uint64_t* ffull;
  uint64_t* fempty;
  int* seqp;  // [3][FZ_SEQ]: clamped sequence length, n_keep, top_k of the first FZ_SEQ sequences
  int* ridx;  // [FZ_NDESC][FZ_ROWS]: row numbers of a descriptor (see FzDesc)
  unsigned* ucache;  // [FZ_UCACHE] producer only: readiness flags seen (UC_*) and the kept rows
  int* misc;  // [0] abort, [1] consumed slots, [2] local tasks posted, [3] local tasks taken,
              // [4] armed slots, [5] finisher requests done, [6] consumers finished,
              // [16..23] consumer broadcasts
};

__device__ __forceinline__ FzShared fz_shared(unsigned char* base) {
  FzShared s;
  s.ring = base + FZ_OFF_RING;
  s.qbuf = base + FZ_OFF_QBUF;
  s.work = base + FZ_OFF_WORK;
  s.seqp = reinterpret_cast<int*>(base + FZ_OFF_SEQP);
  s.ridx = reinterpret_cast<int*>(base + FZ_OFF_RIDX);
  s.ucache = reinterpret_cast<unsigned*>(base + FZ_OFF_UCACHE);
  s.desc = reinterpret_cast<FzDesc*>(base + FZ_OFF_DESC);
  s.finq = reinterpret_cast<FzFin*>(base + FZ_OFF_FINQ);
  s.tasks = reinterpret_cast<FzTask*>(base + FZ_OFF_TASK);
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + FZ_OFF_BAR);
  s.full = bars;
  s.empty = bars + FZ_NSLOT;
  s.dfull = bars + 2 * FZ_NSLOT;
  s.dempty = s.dfull + FZ_NDESC;
  s.ffull = s.dempty + FZ_NDESC;
  s.fempty = s.ffull + FZ_NFIN;
  s.misc = reinterpret_cast<int*>(base + FZ_OFF_MISC);
  return s;
}

__device__ __forceinline__ volatile int* abort_flag(const FzShared& s) { return s.misc; }

// barrier among the consumer threads only
__device__ __forceinline__ void cons_sync() { asm volatile("bar.sync 1, %0;" ::"n"(FZ_CONS) : "memory"); }

// Bounded wait on an mbarrier phase; false (and the abort flag) on expiry.
__device__ __forceinline__ bool fz_wait(const FzShared& s, uint64_t* bar, uint32_t parity, int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag(s)) return false;
    if (clock64() - t0 > FZ_WAIT_CYCLES) {
      set_status(status, HHR_ERR_TIMEOUT);
      *abort_flag(s) = 1;
      return false;
    }
  }
}

// Bounded wait until a global counter reaches `target` (acquire).
__device__ __forceinline__ bool fz_wait_count(const FzShared& s, const unsigned* ctr, unsigned target, int* status) {
  if (ld_acquire(ctr) >= target) return true;
  const long long t0 = clock64();
  while (true) {
    __nanosleep(64);
    if (ld_acquire(ctr) >= target) return true;
    if (*abort_flag(s)) return false;
    if (clock64() - t0 > FZ_WAIT_CYCLES) {
      set_status(status, HHR_ERR_TIMEOUT);
      *abort_flag(s) = 1;
      return false;
    }
  }
}

struct Unit {
  int u, b, h, L, np;
};
__device__ __forceinline__ Unit unit_of(const FzParams& p, const FzShared& s, int u) {
  Unit x;
  x.u = u;
  x.b = u / p.dm.Hkv;
  x.h = u - x.b * p.dm.Hkv;
  x.L = x.b < FZ_SEQ ? s.seqp[x.b] : seq_len_of(p.dm, p.seq_lens, x.b);
  x.np = (x.L + p.dm.P - 1) >> p.dm.lgP;
  return x;
}

// kept pages N of a unit: n_keep clamped to [1, Nmax] and to the page count
__device__ __forceinline__ int keep_pages(const FzParams& p, const FzShared& s, const Unit& x) {
  if (x.np == 0) return 0;
  const int nk = x.b < FZ_SEQ ? s.seqp[FZ_SEQ + x.b] : __ldg(p.n_keep + x.b);
  return min(min(max(nk, 1), p.wk.Nmax), x.np);
}
__device__ __forceinline__ int score_items(const FzParams& p, const FzShared& s, const Unit& x) {
  return (keep_pages(p, s, x) * p.dm.P + FZ_CS - 1) / FZ_CS;
}

__device__ __forceinline__ unsigned* unit_ctrl(const FzParams& p, int u) { return p.wk.ctrl + 4 + u * CU_STRIDE; }
__device__ __forceinline__ unsigned* group_ctrl(const FzParams& p, int u, int g) {
  return p.wk.ctrl + 4 + p.dm.B * p.dm.Hkv * CU_STRIDE + u * p.wk.max_groups + g;
}
__device__ __forceinline__ int nchunks_of(unsigned nk) { return (int)((nk + FZ_ROWS - 1) / FZ_ROWS); }

// item index -> (kind, unit, chunk)
__device__ __forceinline__ void decode_item(const FzParams& p, int item, int& kind, int& u, int& c) {
  const int U = p.dm.B * p.dm.Hkv;
  u = 0;
  c = 0;
  if (item < U) {
    kind = IT_PREP;
    u = item;
    return;
  }
  item -= U;
  const int per[3] = {p.items_per_unit_scan, p.items_per_unit_score, p.items_per_unit_gather};
  const int kinds[3] = {IT_SCAN, IT_SCORE, IT_GATHER};
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    if (item < U * per[k]) {
      kind = kinds[k];
      u = item / per[k];
      c = item - u * per[k];
      return;
    }
    item -= U * per[k];
  }
  kind = IT_END;
}

// producer-side memory of a unit's readiness: flags seen and the kept rows
enum : unsigned { UC_PREP = 1u << 31, UC_SEL = 1u << 30, UC_SCORE = 1u << 29, UC_NKEYS = (1u << 24) - 1u };

// The producer warp waits (bounded) until unit u is ready for an item kind:
// q' published (UC_PREP), kept rows published (UC_SEL; their count is
// remembered), or kept pages and query codes published (UC_SCORE).  The
// first time, every lane acquires what the publishing CTA wrote and orders
// later bulk copies (async proxy) after it; later items of the unit reuse
// that.  False after a timeout or an abort.
__device__ __forceinline__ bool fz_unit_ready(const FzParams& p, const FzShared& s, int u, unsigned flag, int lane) {
  if (u < FZ_UCACHE && (s.ucache[u] & flag)) return true;
  unsigned* uc = unit_ctrl(p, u);
  bool ok = true;
  if (lane == 0) {
    if (flag == UC_PREP) ok = fz_wait_count(s, uc + CU_PREP, 1u, p.status);
    else if (flag == UC_SEL) ok = fz_wait_count(s, uc + CU_SEL, 1u, p.status);
    else ok = fz_wait_count(s, uc + CU_PSEL, 1u, p.status) && fz_wait_count(s, uc + CU_CODES, 1u, p.status);
  }
  if (__shfl_sync(0xffffffffu, (int)ok, 0) == 0) return false;
  (void)ld_acquire(uc + (flag == UC_PREP ? CU_PREP : flag == UC_SEL ? CU_SEL : CU_PSEL));
  if (flag == UC_SCORE) (void)ld_acquire(uc + CU_CODES);
  fence_proxy_async_global();  // q' was written by another CTA with ordinary stores
  if (u < FZ_UCACHE) {
    unsigned v = 0;
    if (flag == UC_SEL) v = min(__ldcg(uc + CU_NKEYS), UC_NKEYS);
    __syncwarp();
    if (lane == 0) s.ucache[u] |= flag | v;
    __syncwarp();
  }
  return true;
}

// ---------------------------------------------------------------------------
// producer (warp 16): claims items, moves contiguous blocks with bulk copies
// and lists the rows that the consumers gather themselves
// ---------------------------------------------------------------------------
template <int G, int WORDS, bool DENSE>
__device__ void fz_producer(const FzParams& p, const FzShared& s) {
  const int lane = threadIdx.x & 31;
  const Dims& dm = p.dm;
  const int prep_slots = DENSE ? 4 : 4 + dm.nb / 64;  // R_h, then W_h (not needed without hashing)
  const uint64_t ef = evict_first_policy();
  unsigned nslot = 0, ndesc = 0, armed = 0;
  // The next item is claimed one item ahead (the atomic's round trip overlaps
  // the current item); a unit's readiness, once seen, is remembered.
  int next = 0;
  if (lane == 0) next = (int)atomicAdd(p.wk.ctrl + 0, 1u);
  while (true) {
    const int item = __shfl_sync(0xffffffffu, next, 0);
    if (lane == 0) next = (int)atomicAdd(p.wk.ctrl + 0, 1u);
    int kind, u, c;
    decode_item(p, item, kind, u, c);
    const Unit x = unit_of(p, s, u);
    int n = 0;
    unsigned nk = 0;
    if (kind == IT_SCAN) {
      n = min(FZ_ROWS, x.np - c * FZ_ROWS);
      if (n <= 0) continue;
    } else if (kind == IT_SCORE) {
      n = min(FZ_CS, keep_pages(p, s, x) * dm.P - c * FZ_CS);
      if (n <= 0) continue;
      if (!fz_unit_ready(p, s, u, UC_SCORE, lane)) break;
    } else if (kind == IT_GATHER) {
      if (!fz_unit_ready(p, s, u, UC_SEL, lane)) break;
      nk = u < FZ_UCACHE ? (s.ucache[u] & UC_NKEYS) : __ldcg(unit_ctrl(p, u) + CU_NKEYS);
      n = min(FZ_ROWS, (int)nk - c * FZ_ROWS);
      if (n <= 0) continue;
    } else if (kind == IT_PREP) {
      n = x.L;
    }
    const int d = (int)(ndesc % FZ_NDESC);
    if (ndesc >= FZ_NDESC) {
      bool ok = true;
      if (lane == 0) ok = fz_wait(s, &s.dempty[d], ((ndesc / FZ_NDESC) - 1) & 1, p.status);
      if (__shfl_sync(0xffffffffu, (int)ok, 0) == 0) break;
    }
    // rows at scattered addresses (paged metadata, kept or paged K'/V rows)
    // are gathered by the consumers: here only their row numbers
    const bool gather = (kind == IT_SCAN && dm.paged) || (kind == IT_GATHER && !(DENSE && !dm.paged));
    const int nslots = kind == IT_PREP ? prep_slots : (kind == IT_SCAN || kind == IT_GATHER) ? 4 : 0;
    int* ridx = s.ridx + d * FZ_ROWS;
    if (gather) {
#pragma unroll
      for (int i = 0; i < FZ_ROWS / 32; ++i) {
        const int j = lane + 32 * i;
        if (j < n) {
          int r = -1;
          if (kind == IT_SCAN) {
            const int blk = __ldg(p.table + (long long)x.b * dm.max_blocks + c * FZ_ROWS + j);
            if ((unsigned)blk < (unsigned)dm.num_blocks) r = blk * dm.Hkv + x.h;
            else set_status(p.status, HHR_ERR_BAD_BLOCK);
          } else {
            const int t = DENSE ? c * FZ_ROWS + j
                                : __ldcg(p.wk.sel_keys + (long long)u * p.wk.Kmax + (long long)c * FZ_ROWS + j);
            const long long off = kv_row(dm, p.table, x.b, x.h, t, p.status);
            if (off >= 0) r = (int)(off / D);
          }
          ridx[j] = r;
        }
      }
    } else if (kind == IT_SCORE) {
      // pages of the item: code word offset, then the page's rows inside the sequence
      const int npg = (n + dm.P - 1) / dm.P;
      const int pfirst = c * (FZ_CS / dm.P);
      for (int jp = lane; jp < npg; jp += 32) {
        const int pg = __ldcg(p.wk.sel_pages + (long long)u * p.wk.Nmax + pfirst + jp);
        const long long off = code_row(dm, p.table, x.b, x.h, pg * dm.P, p.status);
        ridx[jp] = off >= 0 ? (int)off : -1;
        ridx[FZ_ROWS / 2 + jp] = min(dm.P, x.L - pg * dm.P);
      }
    }
    // the unit's q or q' goes to the descriptor's q buffer, completing on the first slot
    uint32_t qbytes = 0;
    const void* qsrc = nullptr;
    if (kind == IT_PREP) {
      qbytes = G * D * 2;
      qsrc = p.q + ((long long)x.b * dm.Hq + x.h * G) * D;
    } else if (kind == IT_SCAN || kind == IT_GATHER) {
      if (kind == IT_SCAN && !fz_unit_ready(p, s, u, UC_PREP, lane)) break;
      qbytes = G * D * 4;
      qsrc = p.wk.qrot + ((long long)x.b * dm.Hq + x.h * G) * D;
    }
    unsigned char* qdst = s.qbuf + d * FZ_QBUF;
    bool aborted = false;
    for (int k = 0; k < nslots; ++k) {
      const unsigned gs = nslot + k;
      const int slot = (int)(gs % FZ_NSLOT);
      if (gs >= FZ_NSLOT) {
        bool ok = true;
        if (lane == 0) ok = fz_wait(s, &s.empty[slot], ((gs / FZ_NSLOT) - 1) & 1, p.status);
        if (__shfl_sync(0xffffffffu, (int)ok, 0) == 0) {
          aborted = true;
          break;
        }
      }
      if (lane == 0) {
        unsigned char* dst = s.ring + (size_t)slot * FZ_SLOT;
        uint32_t bytes = 0;
        if (kind == IT_PREP) {
          const void* src = (k < 4) ? (const void*)(p.R + (long long)x.h * D * D + (long long)k * 32 * D)
                                    : (const void*)(p.W + ((long long)x.h * dm.nb + (long long)(k - 4) * 64) * D);
          bulk_g2s(dst, src, FZ_SLOT, &s.full[slot]);
          bytes = FZ_SLOT;
        } else if (!gather) {
          // contiguous rows: page minima / maxima of the scan, or K'/V of dense attention
          const __nv_bfloat16* base = kind == IT_SCAN ? ((k < 2) ? p.pmin : p.pmax) : ((k < 2) ? p.Kr : p.Vc);
          const long long rows_per_head = kind == IT_SCAN ? dm.np_max : dm.T;
          const int j0 = (k & 1) * 64;
          const int rows = max(0, min(64, n - j0));
          if (rows > 0) {
            bulk_g2s_stream(dst, base + ((long long)(x.b * dm.Hkv + x.h) * rows_per_head + (long long)c * FZ_ROWS + j0) * D,
                            rows * 256, &s.full[slot], ef);
            bytes = rows * 256;
          }
        }
        if (k == 0 && qbytes) {
          bulk_g2s(qdst, qsrc, qbytes, &s.full[slot]);
          bytes += qbytes;
        }
        mbar_arrive_expect_tx(&s.full[slot], bytes);
      }
      __syncwarp();
      armed = gs + 1;
    }
    if (aborted) break;
    __syncwarp();  // the row lists are written before the descriptor is published
    if (lane == 0) {
      FzDesc& ds = s.desc[d];
      ds.kind = kind;
      ds.unit = u;
      ds.chunk = c;
      ds.n = n;
      ds.nslots = nslots;
      ds.pad0 = (int)nk;  // gather: the unit's kept rows
      ds.gather = gather ? 1 : 0;
      mbar_arrive(&s.dfull[d]);
    }
    __syncwarp();
    nslot += nslots;
    ++ndesc;
    if (kind == IT_END) break;
  }
  if (lane == 0) {
    s.misc[4] = (int)armed;  // slots armed with copies (drained at exit)
    // the claim issued ahead has returned before the CTA reports its exit
    // (the last CTA then resets the queue counter)
    asm volatile("" ::"r"(next));
  }
}

// Consumers copy the rows of a gathering descriptor into its slots: warp w
// takes rows 8w .. 8w+7 (the rows it computes on), two rows per instruction,
// 16 bytes per lane, from both tensors; a bad row reads as zeros.  One
// cp.async group per call.
__device__ __forceinline__ void gather_rows(const FzShared& s, const int* ridx, int n, int sbase,
                                            const __nv_bfloat16* first, const __nv_bfloat16* second) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int q = lane & 15;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int j = warp * 8 + 2 * i + (lane >> 4);
    if (j < n) {
      const int r = ridx[j];
      unsigned char* d1 = s.ring + (size_t)((sbase + j / 64) % FZ_NSLOT) * FZ_SLOT + (j % 64) * 256 + q * 16;
      unsigned char* d2 = s.ring + (size_t)((sbase + 2 + j / 64) % FZ_NSLOT) * FZ_SLOT + (j % 64) * 256 + q * 16;
      if (r >= 0) {
        cp_async16(d1, first + (long long)r * D + q * 8);
        cp_async16(d2, second + (long long)r * D + q * 8);
      } else {
        *reinterpret_cast<uint4*>(d1) = make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(d2) = make_uint4(0u, 0u, 0u, 0u);
      }
    }
  }
  cp_async_commit();
}

// ---------------------------------------------------------------------------
// finisher (warp 17): gpu-scope fence, the counter increment, task posting
// ---------------------------------------------------------------------------
static __device__ void fz_finisher(const FzParams& p, const FzShared& s) {
  const int lane = threadIdx.x & 31;
  if (lane != 0) return;
  volatile int* misc = s.misc;
  for (unsigned k = 0;; ++k) {
    const int f = (int)(k % FZ_NFIN);
    // wait for a request, or for the consumers to finish (bounded)
    const long long t0 = clock64();
    bool have = false;
    while (true) {
      if (mbar_try_wait(&s.ffull[f], (k / FZ_NFIN) & 1)) { have = true; break; }
      if (misc[6] || misc[0]) break;
      if (clock64() - t0 > FZ_WAIT_CYCLES) {
        set_status(p.status, HHR_ERR_TIMEOUT);
        misc[0] = 1;
        break;
      }
    }
    if (!have) break;
    const FzFin r = s.finq[f];
    mbar_arrive(&s.fempty[f]);  // the request has been read
    __threadfence();  // the consumers' writes (ordered before by their barrier) become visible first
    const unsigned old = atom_add_acq_rel(r.counter, r.value);
    if (r.target != 0u && old + r.value == r.target && r.kind == TK_GMERGE) {
      // group merges (many, off the critical path) stay in this CTA
      const long long t1 = clock64();
      while (misc[2] - misc[3] >= FZ_NTASK) {  // ring full: wait for the consumers (bounded)
        if (misc[0] || clock64() - t1 > FZ_WAIT_CYCLES) {
          set_status(p.status, HHR_ERR_TIMEOUT);
          misc[0] = 1;
          break;
        }
      }
      const int t = misc[2];
      FzTask& tk = s.tasks[t % FZ_NTASK];
      tk.kind = r.kind;
      tk.unit = r.unit;
      tk.arg = r.arg;
      __threadfence_block();
      misc[2] = t + 1;
    } else if (r.target != 0u && old + r.value == r.target) {
      // selects and final merges join the grid-wide queue: whichever CTA is free first runs them
      const unsigned t = atomicAdd(p.wk.ctrl + 3, 1u);
      if (t < (unsigned)p.wk.tq_cap) {
        int4* e = p.wk.tq + t;
        e->x = r.kind;
        e->y = r.unit;
        e->z = r.arg;
        st_release(reinterpret_cast<unsigned*>(&e->w), t + 1u);
      } else {
        set_status(p.status, HHR_ERR_WORKSPACE);  // cannot happen: the queue holds every task of a call
        misc[0] = 1;
      }
    }
    __threadfence_block();
    misc[5] = misc[5] + 1;
  }
}

// Consumers hand a completion to the finisher (call after a consumer barrier).
__device__ __forceinline__ bool fz_finish(const FzShared& s, unsigned& nfin, unsigned* counter, unsigned value,
                                          unsigned target, int kind, int unit, int arg, int* status) {
  bool ok = true;
  if (threadIdx.x == 0) {
    const int f = (int)(nfin % FZ_NFIN);
    if (nfin >= FZ_NFIN) ok = fz_wait(s, &s.fempty[f], ((nfin / FZ_NFIN) - 1) & 1, status);
    if (ok) {
      FzFin& r = s.finq[f];
      r.counter = counter;
      r.value = value;
      r.target = target;
      r.kind = kind;
      r.unit = unit;
      r.arg = arg;
      mbar_arrive(&s.ffull[f]);
    }
  }
  ++nfin;
  return ok;
}

// ---------------------------------------------------------------------------
// consumer helpers
// ---------------------------------------------------------------------------

// One halving round of a transposed butterfly over the 32 lanes: the lane
// keeps the half of its N values selected by bit `o` of its lane index and
// adds the partner's copy of that half.
template <int N>
__device__ __forceinline__ void halving_round(float* v, int lane, int o) {
  const bool up = (lane & o) != 0;
#pragma unroll
  for (int i = 0; i < N / 2; ++i) {
    const float send = up ? v[i] : v[i + N / 2];
    const float keep = up ? v[i + N / 2] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
  }
}

// Sums NV (>= 32) per-lane values over the 32 lanes of a warp; lane l ends
// with the sums of values [ (NV/32) l, (NV/32)(l+1) ) in v[0 .. NV/32).
template <int NV>
__device__ __forceinline__ void warp_reduce_t(float* v, int lane) {
  halving_round<NV>(v, lane, 16);
  halving_round<NV / 2>(v, lane, 8);
  halving_round<NV / 4>(v, lane, 4);
  halving_round<NV / 8>(v, lane, 2);
  halving_round<NV / 16>(v, lane, 1);
}

// Exclusive scan of one int over the consumer threads; `red` holds 33 ints.
__device__ __forceinline__ int cons_excl_scan(int v, int* red, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) red[warp] = x;
  cons_sync();
  if (warp == 0) {
    int t = lane < FZ_CWARPS ? red[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    red[lane] = t;
  }
  cons_sync();
  const int before = (warp > 0 ? red[warp - 1] : 0) + x - v;
  *total = red[FZ_CWARPS - 1];
  cons_sync();
  return before;
}

// Exclusive scan of one int over the consumer threads with one barrier:
// `red` holds FZ_CWARPS ints and must not be reused before the next barrier.
__device__ __forceinline__ int cons_scan1(int v, int* red, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) red[warp] = x;
  cons_sync();
  int before = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < FZ_CWARPS; ++w) {
    const int r = red[w];
    before += w < warp ? r : 0;
    tot += r;
  }
  *total = tot;
  return before + x - v;
}

// Block-wide min and max of one value per consumer thread (scratch: 32 floats).
__device__ __forceinline__ void cons_minmax(float& lo, float& hi, float* wr) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if (lane == 0) {
    wr[warp * 2 + 0] = lo;
    wr[warp * 2 + 1] = hi;
  }
  cons_sync();
  lo = wr[0];
  hi = wr[1];
#pragma unroll
  for (int w = 1; w < FZ_CWARPS; ++w) {
    lo = fminf(lo, wr[w * 2 + 0]);
    hi = fmaxf(hi, wr[w * 2 + 1]);
  }
  cons_sync();
}

// q' of a head is stored with its channel quads (4 channels) reordered:
// quad 2m + b at position m + 16 b.  The scan's and the gather's lanes then
// read 8 consecutive 16-byte vectors per wavefront (no bank conflicts).
__device__ __forceinline__ int qpos(int c) {
  const int q = c >> 2;
  return 4 * ((q >> 1) + ((q & 1) << 4)) + (c & 3);
}

__device__ __forceinline__ float dot4(const float4& a, const float* b) {
  float r = a.x * b[0];
  r = fmaf(a.y, b[1], r);
  r = fmaf(a.z, b[2], r);
  return fmaf(a.w, b[3], r);
}

// ---- PREP: q' = R_h q, then the query codes --------------------------------
template <int G, bool DENSE>
__device__ void fz_prep(const FzParams& p, const FzShared& s, const Unit& x, int d, int s0) {
  constexpr int GP = G <= 4 ? 4 : 8;
  const Dims& dm = p.dm;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float* qf = reinterpret_cast<float*>(s.work);               // [G][128]
  unsigned* qc = reinterpret_cast<unsigned*>(s.work + 4096);  // [G][8] 32-bit code words
  const __nv_bfloat16* qb = reinterpret_cast<const __nv_bfloat16*>(s.qbuf + d * FZ_QBUF);
  for (int i = tid; i < G * D; i += FZ_CONS) qf[i] = __bfloat162float(qb[i]);
  if (tid < 64) qc[tid] = 0u;
  cons_sync();
  // lane owns channels 4l .. 4l+3
  float qv[G][4];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float4 t = *reinterpret_cast<const float4*>(qf + g * D + 4 * lane);
    qv[g][0] = t.x; qv[g][1] = t.y; qv[g][2] = t.z; qv[g][3] = t.w;
  }
  // q'_i = sum_j R_h[i][j] q_j: warp w takes rows 8w .. 8w+7; the 8 x GP
  // partial sums are reduced together (transposed)
  {
    constexpr int NV = 8 * GP, KP = NV / 32;
    float v[NV];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int i = warp * 8 + r;
      const float4 rr = *reinterpret_cast<const float4*>(
          s.ring + (size_t)((s0 + i / 32) % FZ_NSLOT) * FZ_SLOT + (i % 32) * 512 + lane * 16);
#pragma unroll
      for (int g = 0; g < GP; ++g) v[r * GP + g] = (g < G) ? dot4(rr, qv[g]) : 0.f;
    }
    warp_reduce_t<NV>(v, lane);
#pragma unroll
    for (int e = 0; e < KP; ++e) {
      const int vi = KP * lane + e;
      const int r = vi / GP, g = vi % GP;
      if (g < G) {
        const int i = warp * 8 + r;
        const long long idx = ((long long)x.b * dm.Hq + x.h * G + g) * D;
        p.wk.qrot[idx + qpos(i)] = v[e];
        if (p.dbg.q_rot) p.dbg.q_rot[idx + i] = v[e];
      }
    }
  }
  // publish q' now: the scans of this unit need only q'.  (The barrier orders
  // every consumer's writes before thread 0's gpu-scope fence and release.)
  cons_sync();
  if (tid == 0) {
    __threadfence();
    st_release(unit_ctrl(p, x.u) + CU_PREP, 1u);
  }
  if constexpr (DENSE) return;  // full attention needs no codes (and has no W_h)
  // Query codes: bit j = [ (W_h q)_j > 0 ].  Products of bf16 values are exact
  // in fp32; the 128-term fp32 sum errs by at most 127 * 2^-24 * sum|w q|, so
  // below 2^-14 * sum|w q| the sign is taken from an fp64 recompute.  Warp w
  // takes bits [w nb/16, (w+1) nb/16) in blocks of NBB bits; after the
  // transposed reduction lane l holds (sum, magnitude) of bit l / GP of the
  // block and head l % GP.
  constexpr int NBB = 32 / GP;  // 8 (GP 4) or 4 (GP 8) bits per block
  const int bpw = dm.nb / FZ_CWARPS;
  for (int jb = 0; jb < bpw; jb += NBB) {
    float v[2 * NBB * GP];  // [bit][head][sum, magnitude]
#pragma unroll
    for (int bb = 0; bb < NBB; ++bb) {
      const int j = warp * bpw + jb + bb;
      const bool live = jb + bb < bpw;
      float w4[4] = {0.f, 0.f, 0.f, 0.f};
      if (live) {
        const uint2 wv = *reinterpret_cast<const uint2*>(s.ring + (size_t)((s0 + 4 + j / 64) % FZ_NSLOT) * FZ_SLOT +
                                                         (j % 64) * 256 + lane * 8);
        w4[0] = bf_lo(wv.x); w4[1] = bf_hi(wv.x); w4[2] = bf_lo(wv.y); w4[3] = bf_hi(wv.y);
      }
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
        const unsigned char* wrow = s.ring + (size_t)((s0 + 4 + j / 64) % FZ_NSLOT) * FZ_SLOT + (j % 64) * 256;
        for (int c = 0; c < D; c += 2) {
          const uint32_t w2 = *reinterpret_cast<const uint32_t*>(wrow + c * 2);
          ad += (double)bf_lo(w2) * (double)qf[g * D + c];
          ad += (double)bf_hi(w2) * (double)qf[g * D + c + 1];
        }
        bit = ad > 0.0;
      }
      if (bit) atomicOr(&qc[g * 8 + j / 32], 1u << (j % 32));
    }
  }
  cons_sync();
  const int w32 = dm.words * 2;
  if (tid < G * w32) {
    const int g = tid / w32, k = tid - g * w32;
    const long long o = ((long long)x.b * dm.Hq + x.h * G + g) * w32 + k;
    reinterpret_cast<uint32_t*>(p.wk.qcodes)[o] = qc[g * 8 + k];
    if (p.dbg.q_codes) reinterpret_cast<uint32_t*>(p.dbg.q_codes)[o] = qc[g * 8 + k];
  }
  cons_sync();
  if (tid == 0) {
    __threadfence();
    st_release(unit_ctrl(p, x.u) + CU_CODES, 1u);
  }
}

// ---- SCAN: page bounds of one chunk ------------------------------------------
// ub_g(page) = sum_i max(q'_gi mn_i, q'_gi mx_i) = q'+_g . mx + q'-_g . mn with
// q'+ = max(q', 0) and q'- = min(q', 0) (the same products, summed); the
// unit's page score is U = max_g ub_g.  Warp w takes pages 8w .. 8w+7, half
// a warp per page (lane: channels 8l .. 8l+7 of the half-warp's pages).

// One halving round of a transposed butterfly among the lanes that differ in
// bit `o`: the lane keeps the half of its N values selected by that bit and
// adds the partner's copy of that half.
template <int N>
__device__ __forceinline__ void halving_round_o(float* v, int lane, int o) {
  const bool up = (lane & o) != 0;
#pragma unroll
  for (int i = 0; i < N / 2; ++i) {
    const float send = up ? v[i] : v[i + N / 2];
    const float keep = up ? v[i + N / 2] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
  }
}
// Sums NV per-lane values over groups of W lanes (W = 8 or 16, NV >= W);
// lane l of a group ends with the sums of values [(NV/W) l, (NV/W)(l+1)).
template <int NV, int W>
__device__ __forceinline__ void group_reduce_t(float* v, int lane) {
  if constexpr (W == 16) halving_round_o<NV>(v, lane, 8);
  halving_round_o<(W == 16 ? NV / 2 : NV)>(v, lane, 4);
  halving_round_o<(W == 16 ? NV / 4 : NV / 2)>(v, lane, 2);
  halving_round_o<(W == 16 ? NV / 8 : NV / 4)>(v, lane, 1);
}

template <int G>
__device__ void fz_scan(const FzParams& p, const FzShared& s, const Unit& x, int c, int n, int d, int s0) {
  constexpr int GP = G <= 4 ? 4 : 8;
  constexpr bool SPLIT = G <= 4;          // q'+ and q'- in registers (else q' and a select)
  constexpr int PB = GP == 4 ? 4 : 2;     // pages per half-warp per batch
  constexpr int NBT = 4 / PB;             // batches (4 pages per half-warp)
  constexpr int NV = PB * GP;             // 16 partial bounds per lane
  const Dims& dm = p.dm;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int hw = lane >> 4, li = lane & 15;
  const float* qs = reinterpret_cast<const float*>(s.qbuf + d * FZ_QBUF);
  float2 qa[G][4], qb[G][4];
#pragma unroll
  for (int g = 0; g < G; ++g) {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const float4 t = *reinterpret_cast<const float4*>(qs + g * D + 4 * (li + 16 * k));  // channels 8 li + 4 k ..
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
  // after the reduction lane l of a half-warp holds page l / GP of the batch, head l % GP
  const int pl = li / GP, hidx = li % GP;
#pragma unroll
  for (int bt = 0; bt < NBT; ++bt) {
    float v[NV];
#pragma unroll
    for (int pp = 0; pp < PB; ++pp) {
      const int j = warp * 8 + hw * 4 + bt * PB + pp;  // page within the chunk
      const size_t off = (size_t)(j % 64) * 256 + li * 16;
      const uint4 mnv = *reinterpret_cast<const uint4*>(s.ring + (size_t)((s0 + j / 64) % FZ_NSLOT) * FZ_SLOT + off);
      const uint4 mxv = *reinterpret_cast<const uint4*>(s.ring + (size_t)((s0 + 2 + j / 64) % FZ_NSLOT) * FZ_SLOT + off);
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
    // U = max over the real heads of the lane's page (GP adjacent lanes)
    float U = hidx < G ? v[0] : -INFINITY;
#pragma unroll
    for (int o = 1; o < GP; o <<= 1) U = fmaxf(U, __shfl_xor_sync(0xffffffffu, U, o));
    const int j = warp * 8 + hw * 4 + bt * PB + pl;
    if (j < n) {
      const int pg = c * FZ_ROWS + j;
      if (hidx == 0) {
        p.wk.U[(long long)x.u * p.wk.Ustride + pg] = U;
        if (p.dbg.page_U) p.dbg.page_U[(long long)x.u * dm.np_max + pg] = U;
      }
      if (p.dbg.page_ub && hidx < G)
        p.dbg.page_ub[((long long)x.b * dm.Hq + x.h * G + hidx) * dm.np_max + pg] = v[0];
    }
  }
}

// ---- PSEL: page top-N (larger bound first, ties to the lower page) ------------
constexpr int PS_HIST = 0;                // int [2048] value bins
constexpr int PS_CAND = 8192;             // int [512] members of the threshold bin
constexpr int PS_CANDV = PS_CAND + 2048;  // float [512] their bounds
constexpr int PS_FLAG = PS_CANDV + 2048;  // u32 [256] bitmap of kept members
constexpr int PS_RED = PS_FLAG + 1024;    // int [128]: four scan buffers of 16 and broadcasts
constexpr int PS_WR = PS_RED + 512;       // float [32] min / max scratch
constexpr int SEL_NBIN = 2048;
constexpr int SEL_MAX_CAND = 512;
constexpr int PS_PER = MAX_SELECT_PAGES / FZ_CONS;  // 16 pages per thread
static_assert(PS_PER == 16, "page select layout");

// Bin of a bound: monotone non-decreasing in the value, so the N-th largest
// lies in one bin and every larger bin is kept whole.
__device__ __forceinline__ int value_bin(float v, float lo, float scale) {
  // nearest integer by the 1.5 * 2^23 addition (monotone, and cheaper than a
  // conversion instruction; members lie in [0, SEL_NBIN])
  const float t = fminf(fmaxf((v - lo) * scale, 0.f), (float)(SEL_NBIN - 1));
  return __float_as_int(t + 12582912.0f) - 0x4B400000;
}

static __device__ void fz_psel(const FzParams& p, const FzShared& s, const Unit& x) {
  const Work& wk = p.wk;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int* hist = reinterpret_cast<int*>(s.work + PS_HIST);
  int* cand = reinterpret_cast<int*>(s.work + PS_CAND);
  float* candv = reinterpret_cast<float*>(s.work + PS_CANDV);
  unsigned* flag = reinterpret_cast<unsigned*>(s.work + PS_FLAG);
  int* red = reinterpret_cast<int*>(s.work + PS_RED);  // scans: [0, 32) levels, [64, 80) ties, [80, 96) kept pages
  int* bc = red + 48;                                  // broadcasts [0..11]
  float* wr = reinterpret_cast<float*>(s.work + PS_WR);
  const int np = x.np;
  const int N = keep_pages(p, s, x);
  int* gsel = wk.sel_pages + (long long)x.u * wk.Nmax;
  int* dsel = p.dbg.sel_pages ? p.dbg.sel_pages + (long long)x.u * wk.Nmax : nullptr;
  if (N >= np) {
    for (int i = tid; i < np; i += FZ_CONS) {
      gsel[i] = i;
      if (dsel) dsel[i] = i;
    }
  } else {
    // ---- the bounds of pages [16 t, 16 t + 16) into registers; hist zeroed meanwhile ----
    const float* Ug = wk.U + (long long)x.u * wk.Ustride;
    const int i0 = tid * PS_PER;
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
    const int cnt = max(0, min(PS_PER, np - i0));
    unsigned member = (1u << cnt) - 1u;
    float lo = INFINITY, hi = -INFINITY;
#pragma unroll
    for (int k = 0; k < PS_PER; ++k)
      if ((member >> k) & 1u) {
        lo = fminf(lo, v[k]);
        hi = fmaxf(hi, v[k]);
      }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if (lane == 0) {
      wr[2 * warp] = lo;
      wr[2 * warp + 1] = hi;
    }
    cons_sync();
#pragma unroll
    for (int w = 0; w < FZ_CWARPS; ++w) {
      lo = fminf(lo, wr[2 * w]);
      hi = fmaxf(hi, wr[2 * w + 1]);
    }
    // ---- threshold by value bins.  `member` marks pages still undecided,
    // `keep` the kept.  A level bins the members over their value range,
    // keeps every bin above the one holding the need-th largest member and
    // descends into that bin; a small bin is then ranked exactly, a bin of
    // equal values is taken in index order. ----
    unsigned keep = 0u;
    int need = N, nbin = 0;
    bool tie = false;
#pragma unroll 1
    for (int level = 0; level < 4; ++level) {
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
        const bool above = m && bn[k] > bstar, at = m && bn[k] == bstar;
        keep |= above ? 1u << k : 0u;
        member &= at ? ~0u : ~(1u << k);
        nlo = at ? fminf(nlo, v[k]) : nlo;
        nhi = at ? fmaxf(nhi, v[k]) : nhi;
      }
      if (nbin <= SEL_MAX_CAND) break;
      cons_minmax(nlo, nhi, wr);
      lo = nlo;
      hi = nhi;
    }
    if (tie || nbin > SEL_MAX_CAND) {
      // equal values (or still crowded): members in index order, the first `need`
      const int m = __popc(member);
      int tot;
      const int mb = cons_scan1(m, red + 64, &tot);
      int take = max(0, min(m, need - mb));
#pragma unroll
      for (int k = 0; k < PS_PER; ++k) {
        if (((member >> k) & 1u) && take > 0) {
          keep |= 1u << k;
          --take;
        }
      }
    } else {
      // exact ranking of the (few) members: larger value first, then lower index
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
          const int ib = cand[b2];
          const float vb = candv[b2];
          rank += (vb > va) || (vb == va && ib < ia);
        }
        if (rank < need) atomicOr(&flag[ia >> 5], 1u << (ia & 31));
      }
      cons_sync();
      const unsigned fw = flag[i0 >> 5] >> (i0 & 31);  // the thread's 16 pages share one flag word
      keep |= member & fw & 0xffffu;
    }
    // ---- kept pages in index order ----
    int tot;
    int pos = cons_scan1(__popc(keep), red + 80, &tot);
#pragma unroll
    for (int k = 0; k < PS_PER; ++k) {
      if ((keep >> k) & 1u) {
        gsel[pos] = i0 + k;
        if (dsel) dsel[pos] = i0 + k;
        ++pos;
      }
    }
  }
  if (tid == 0 && p.dbg.n_sel_pages) p.dbg.n_sel_pages[x.u] = N;
}

// ---- SCORE: Hamming scores of one chunk of candidates ------------------------
// S = sum over the group's heads g of popcount(code(q_g) XOR code(k)); the
// chunk's scores go to kscore (uint16, 0xFFFF for rows past the sequence end)
// and their histogram is added to the unit's global histogram.
template <int G, int WORDS>
__device__ void fz_score(const FzParams& p, const FzShared& s, const Unit& x, int c, int n, int d) {
  const Dims& dm = p.dm;
  const Work& wk = p.wk;
  const int tid = threadIdx.x;
  int* hist = reinterpret_cast<int*>(s.work);
  const int nbins = G * dm.nb + 1;
  for (int b = tid; b < nbins; b += FZ_CONS) hist[b] = 0;
  const int* ridx = s.ridx + d * FZ_ROWS;  // per page: code word offset, then rows inside the sequence
  // the candidates' code words (two per thread), straight from global memory
  constexpr int NR = FZ_CS / FZ_CONS;
  uint64_t cw[NR][WORDS];
  bool valid[NR];
#pragma unroll
  for (int r = 0; r < NR; ++r) {
    const int j = r * FZ_CONS + tid;
    const int jp = j >> dm.lgP, jr = j & (dm.P - 1);
    const int woff = j < n ? ridx[jp] : -1;
    valid[r] = woff >= 0 && jr < ridx[FZ_ROWS / 2 + jp];
#pragma unroll
    for (int w2 = 0; w2 < WORDS; ++w2) cw[r][w2] = 0ull;
    if (valid[r]) {
      const uint64_t* src = p.codes + (long long)woff + (long long)jr * WORDS;
      if constexpr (WORDS == 1) {
        cw[r][0] = __ldg(src);
      } else {
#pragma unroll
        for (int w2 = 0; w2 < WORDS; w2 += 2) {
          const ulonglong2 t = __ldg(reinterpret_cast<const ulonglong2*>(src + w2));
          cw[r][w2] = t.x;
          cw[r][w2 + 1] = t.y;
        }
      }
    }
  }
  (void)ld_acquire(unit_ctrl(p, x.u) + CU_CODES);
  uint64_t cq[G][WORDS];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int w2 = 0; w2 < WORDS; ++w2) cq[g][w2] = __ldcg(wk.qcodes + ((long long)x.b * dm.Hq + x.h * G + g) * WORDS + w2);
  cons_sync();  // the histogram is zero
  int* dsc = p.dbg.key_scores ? p.dbg.key_scores + (long long)x.u * wk.Nmax * dm.P : nullptr;
  uint16_t* ks = wk.kscore + (long long)x.u * wk.Cmax;
#pragma unroll
  for (int r = 0; r < NR; ++r) {
    const int j = r * FZ_CONS + tid;
    if (j < n) {
      int S = 0;
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int w2 = 0; w2 < WORDS; ++w2) S += __popcll(cq[g][w2] ^ cw[r][w2]);
      const int ci = c * FZ_CS + j;
      ks[ci] = valid[r] ? (uint16_t)S : (uint16_t)0xFFFFu;
      if (dsc) dsc[ci] = valid[r] ? S : INT_MAX;
      if (valid[r]) atomicAdd(&hist[S], 1);
    }
  }
  cons_sync();
  int* gh = wk.khist + (long long)x.u * wk.HB;
  for (int b = tid; b < nbins; b += FZ_CONS) {
    const int h = hist[b];
    if (h) atomicAdd(gh + b, h);
  }
}

// ---- KSEL: key top-k (smaller score first, ties to the lower row) ------------
constexpr int KS_SPAGE = 0;      // int [2048] kept pages
constexpr int KS_RED = 8192;     // int [64] scan scratch and broadcasts
constexpr int KS_SC = 8448;      // uint16 [32 rounds x 512] staged candidate scores
static_assert(MAX_KEEP_PAGES <= 2048 && MAX_CANDIDATES <= 32 * FZ_CONS && KS_SC + 2 * 32 * FZ_CONS <= FZ_WORK,
              "key select layout");

template <int G>
__device__ void fz_ksel(const FzParams& p, const FzShared& s, const Unit& x) {
  const Dims& dm = p.dm;
  const Work& wk = p.wk;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int* spage = reinterpret_cast<int*>(s.work + KS_SPAGE);
  int* red = reinterpret_cast<int*>(s.work + KS_RED);
  int* bc = red + 48;
  uint16_t* scs = reinterpret_cast<uint16_t*>(s.work + KS_SC);
  const int N = keep_pages(p, s, x);
  const int ncs = N * dm.P;
  const int nbins = G * dm.nb + 1;
  for (int i = tid; i < N; i += FZ_CONS) spage[i] = __ldcg(wk.sel_pages + (long long)x.u * wk.Nmax + i);
  // ---- histogram (blocked bins per thread) -> threshold T and the ties taken ----
  int* gh = wk.khist + (long long)x.u * wk.HB;
  const int bpt = (nbins + FZ_CONS - 1) / FZ_CONS;  // <= 5
  int hv[5];
  int local = 0;
#pragma unroll
  for (int e = 0; e < 5; ++e) {
    const int bi = tid * bpt + e;
    hv[e] = (e < bpt && bi < nbins) ? __ldcg(gh + bi) : 0;
    local += hv[e];
  }
  int n_cand;
  const int before = cons_scan1(local, red, &n_cand);
  const int tk = x.b < FZ_SEQ ? s.seqp[2 * FZ_SEQ + x.b] : __ldg(p.top_k + x.b);
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
  // the histogram is kept at zero between calls
#pragma unroll
  for (int e = 0; e < 5; ++e) {
    const int bi = tid * bpt + e;
    if (e < bpt && bi < nbins && hv[e]) gh[bi] = 0;
  }
  cons_sync();  // bc, spage
  if (keff > 0) {
    // Kept rows in candidate order: count S < T and S == T over this
    // thread's run, one scan, then each thread writes its kept rows.
    // Kept rows in candidate order.  Warp w owns candidates
    // [w nbw, (w + 1) nbw) in rounds of 32 (lane l: candidate 32 r + l).
    // Pass 1 stages the scores and counts S < T and S == T per warp; one
    // scan over the warp totals; pass 2 places the kept rows with ballots
    // (coalesced stores).
    const int T = bc[0], need_eq = bc[1];
    const int rounds = (ncs + 32 * FZ_CWARPS - 1) / (32 * FZ_CWARPS);  // <= 32
    const int cw0 = warp * rounds * 32;
    const uint16_t* ks = wk.kscore + (long long)x.u * wk.Cmax;
    const unsigned lanemask_lt = (1u << lane) - 1u;
    int lt_w = 0, eq_w = 0;
#pragma unroll 8
    for (int r = 0; r < rounds; ++r) {
      const int ci = cw0 + 32 * r + lane;
      const int S = ci < ncs ? (int)__ldcg(ks + ci) : 0xFFFF;
      scs[ci] = (uint16_t)S;
      lt_w += __popc(__ballot_sync(0xffffffffu, S < T));
      eq_w += __popc(__ballot_sync(0xffffffffu, S == T));
    }
    int tot;
    const int pk = cons_scan1(lane == 0 ? (lt_w << 16) | eq_w : 0, red + 16, &tot);
    int lt_b = __shfl_sync(0xffffffffu, pk, 0) >> 16, eq_b = __shfl_sync(0xffffffffu, pk, 0) & 0xFFFF;
    __syncwarp();  // the warp's staged scores
    int* out = wk.sel_keys + (long long)x.u * wk.Kmax;
    int* dout = p.dbg.sel_keys ? p.dbg.sel_keys + (long long)x.u * wk.Kmax : nullptr;
#pragma unroll 4
    for (int r = 0; r < rounds; ++r) {
      const int ci = cw0 + 32 * r + lane;
      const int S = scs[ci];
      const bool lt = S < T, eq = S == T;
      const unsigned blt = __ballot_sync(0xffffffffu, lt), beq = __ballot_sync(0xffffffffu, eq);
      const int eq_before = eq_b + __popc(beq & lanemask_lt);
      const bool take = lt || (eq && eq_before < need_eq);
      const int pos = lt_b + __popc(blt & lanemask_lt) + min(eq_before, need_eq);
      if (take && pos < keff) {  // (pos < keff always holds; keeps the stores inside the list)
        const int t = (spage[ci >> dm.lgP] << dm.lgP) + (ci & (dm.P - 1));
        out[pos] = t;
        if (dout) dout[pos] = t;
      }
      lt_b += __popc(blt);
      eq_b += __popc(beq);
    }
  }
  if (tid == 0) {
    unit_ctrl(p, x.u)[CU_NKEYS] = (unsigned)keff;
    if (p.dbg.n_sel_keys) p.dbg.n_sel_keys[x.u] = keff;
    if (p.dbg.n_cand) p.dbg.n_cand[x.u] = n_cand;
  }
}

// ---- GATHER: softmax attention over one chunk of kept rows ---------------------
// Warp w takes rows 8w .. 8w+7.  Logits: groups of LPR lanes share a row (a
// lane holds 16 or 8 of its channels), so a dot product is reduced over LPR
// lanes only.  Then the warp's max and weights per head, and the weighted V
// sum of its rows (lane: channels 4l .. 4l+3).  One barrier later the 16 warp
// partials are combined in warp order into the chunk's partial (unnormalised
// output, max and sum of weights per head, in log2 units) at part[u][c].
constexpr int GA_OB = 0;                  // float [16 warps][G][128] warp outputs
constexpr int GA_PB = 65536;              // float2 [16 warps][8 rows][GP] weights as (p, p)
constexpr int GA_MB = GA_PB + 8192;       // float [16][8] warp maxima
constexpr int GA_LB = GA_MB + 512;        // float [16][8] warp sums
static_assert(GA_LB + 512 <= FZ_WORK, "gather scratch");

template <int G>
__device__ void fz_gather(const FzParams& p, const FzShared& s, const Unit& x, int c, int n, int d, int s0) {
  constexpr int GP = G <= 4 ? 4 : 8;     // heads padded to a power of two
  constexpr int LPR = GP == 4 ? 8 : 16;  // lanes per row in the logits
  constexpr int NCK = 128 / LPR / 8;     // 16-byte chunks per lane and row (2 or 1)
  constexpr int RPG = LPR / 4;           // rows per lane group (2 or 4; 8 rows per warp)
  constexpr int NV = RPG * GP;           // partial logits per lane (8 or 32)
  constexpr int KP = NV / LPR;           // logits per lane after the reduction (1 or 2)
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int grp = lane / LPR, li = lane % LPR;
  float* OB = reinterpret_cast<float*>(s.work + GA_OB);
  float2* PB = reinterpret_cast<float2*>(s.work + GA_PB) + warp * 8 * GP;
  float* MB = reinterpret_cast<float*>(s.work + GA_MB);
  float* LB = reinterpret_cast<float*>(s.work + GA_LB);
  const float* qs = reinterpret_cast<const float*>(s.qbuf + d * FZ_QBUF);
  const float qscale = p.sm_scale * 1.4426950408889634f;
  // ---- logits: lane holds channels 8 (LPR k + li) .. +7 for chunks k < NCK ----
  float sv[KP];
  {
    float2 q2[G][4 * NCK];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int k = 0; k < NCK; ++k)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          // channels 8 (LPR k + li) + 4 h .. (stored in quad order, see qpos)
          const float4 t = *reinterpret_cast<const float4*>(qs + g * D + 4 * (LPR * k + li + 16 * h));
          q2[g][4 * k + 2 * h] = make_float2(t.x * qscale, t.y * qscale);
          q2[g][4 * k + 2 * h + 1] = make_float2(t.z * qscale, t.w * qscale);
        }
    float v[NV];  // [head][row of the group]
#pragma unroll
    for (int r = 0; r < RPG; ++r) {
      const int j = warp * 8 + grp * RPG + r;
      const unsigned char* row = s.ring + (size_t)((s0 + j / 64) % FZ_NSLOT) * FZ_SLOT + (j % 64) * 256;
      float2 kf[4 * NCK];
#pragma unroll
      for (int k = 0; k < NCK; ++k) {
        const uint4 kv = *reinterpret_cast<const uint4*>(row + 16 * (LPR * k + li));
        kf[4 * k] = make_float2(bf_lo(kv.x), bf_hi(kv.x));
        kf[4 * k + 1] = make_float2(bf_lo(kv.y), bf_hi(kv.y));
        kf[4 * k + 2] = make_float2(bf_lo(kv.z), bf_hi(kv.z));
        kf[4 * k + 3] = make_float2(bf_lo(kv.w), bf_hi(kv.w));
      }
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        float a = 0.f;
        if (g < G) {
          float2 a0 = __fmul2_rn(q2[g][0], kf[0]);
#pragma unroll
          for (int k = 1; k < 4 * NCK; ++k) a0 = __ffma2_rn(q2[g][k], kf[k], a0);
          a = a0.x + a0.y;
        }
        v[g * RPG + r] = a;
      }
    }
    group_reduce_t<NV, LPR>(v, lane);
    // lane li holds values [KP li, KP li + KP): head (KP li) / RPG = li / 2, rows KP li % RPG + e
#pragma unroll
    for (int e = 0; e < KP; ++e) {
      const int r = (KP * li + e) % RPG;
      const int j = warp * 8 + grp * RPG + r;
      sv[e] = ((li >> 1) < G && j < n) ? v[e] : -INFINITY;
    }
  }
  const int gl = li >> 1;  // the lane's head
  // ---- the warp's max and weights per head: lanes 2 gl, 2 gl + 1 of every group ----
  float m = sv[0];
#pragma unroll
  for (int e = 1; e < KP; ++e) m = fmaxf(m, sv[e]);
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
#pragma unroll
  for (int o = LPR; o < 32; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float l = 0.f;
#pragma unroll
  for (int e = 0; e < KP; ++e) {
    const float pv = (sv[e] == -INFINITY) ? 0.f : exp2f(sv[e] - m);
    const int r = (KP * li + e) % RPG;
    PB[(grp * RPG + r) * GP + gl] = make_float2(pv, pv);
    l += pv;
  }
  l += __shfl_xor_sync(0xffffffffu, l, 1);
#pragma unroll
  for (int o = LPR; o < 32; o <<= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
  if (lane < LPR && (li & 1) == 0 && gl < G) {
    MB[warp * 8 + gl] = m;
    LB[warp * 8 + gl] = l;
  }
  __syncwarp();
  // ---- weighted V sum of the warp's rows ----
  float2 o2[G][2];
#pragma unroll
  for (int g = 0; g < G; ++g) o2[g][0] = o2[g][1] = make_float2(0.f, 0.f);
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const int j = warp * 8 + r;
    if (j < n) {
      const uint2 vv = *reinterpret_cast<const uint2*>(s.ring + (size_t)((s0 + 2 + j / 64) % FZ_NSLOT) * FZ_SLOT +
                                                       (j % 64) * 256 + lane * 8);
      const float2 v0 = make_float2(bf_lo(vv.x), bf_hi(vv.x)), v1 = make_float2(bf_lo(vv.y), bf_hi(vv.y));
      float2 pr[GP];
#pragma unroll
      for (int g2 = 0; g2 < G; g2 += 2) {
        const float4 t = *reinterpret_cast<const float4*>(PB + r * GP + g2);
        pr[g2] = make_float2(t.x, t.y);
        pr[g2 + 1] = make_float2(t.z, t.w);
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        o2[g][0] = __ffma2_rn(pr[g], v0, o2[g][0]);
        o2[g][1] = __ffma2_rn(pr[g], v1, o2[g][1]);
      }
    }
  }
#pragma unroll
  for (int g = 0; g < G; ++g)
    *reinterpret_cast<float4*>(OB + (warp * G + g) * D + 4 * lane) =
        make_float4(o2[g][0].x, o2[g][0].y, o2[g][1].x, o2[g][1].y);
  cons_sync();
  // ---- the chunk's partial: warps combined in order (thread: head g, channels 4 c4 ..) ----
  if (tid < G * 32) {
    const int g = warp, c4 = lane;  // warp-uniform head
    const float mw = MB[(lane & 15) * 8 + g];
    float M = mw;
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float sc = (mw == -INFINITY) ? 0.f : exp2f(mw - M);  // lane l: scale of warp l & 15
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float L = 0.f;
#pragma unroll
    for (int w = 0; w < FZ_CWARPS; ++w) {
      const float scw = __shfl_sync(0xffffffffu, sc, w);
      const float4 a = *reinterpret_cast<const float4*>(OB + (w * G + g) * D + 4 * c4);
      acc.x = fmaf(scw, a.x, acc.x);
      acc.y = fmaf(scw, a.y, acc.y);
      acc.z = fmaf(scw, a.z, acc.z);
      acc.w = fmaf(scw, a.w, acc.w);
      L = fmaf(scw, LB[w * 8 + g], L);
    }
    const int PS = G * D + 16;  // partial: o[G][D], m at G D, l at G D + 8 (16-byte rows)
    float* part = p.wk.part + ((long long)x.u * p.wk.C3 + c) * PS;
    *reinterpret_cast<float4*>(part + g * D + 4 * c4) = acc;
    if (c4 == 0) {
      part[G * D + g] = M;
      part[G * D + 8 + g] = L;
    }
  }
}

// Merges K partials src[0 .. K) (stride G D + 16 floats) in index order:
// M = max m_k, w_k = 2^(m_k - M), L = sum w_k l_k, O = sum w_k o_k.  With
// dst, the merged partial (O, M, L) is written there; otherwise out = O / L.
// K <= 256.  The output float4s are split over NPART groups of threads, each
// taking every NPART-th partial (loads issued before the weights are known);
// the group sums are then added in group order.
template <int G>
__device__ void merge_partials(unsigned char* work, const float* src, int K, float* dst, float* out) {
  constexpr int NOUT = G * 32;  // float4 outputs
  constexpr int NPART = FZ_CONS / NOUT >= 4 ? 4 : FZ_CONS / NOUT;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int PS = G * D + 16;
  float* wsm = reinterpret_cast<float*>(work);            // [256][G] weights
  float* MH = reinterpret_cast<float*>(work + 8192);      // [8]
  float* LH = MH + 8;                                      // [8]
  float4* psum = reinterpret_cast<float4*>(work + 16384);  // [NPART][NOUT]
  cons_sync();  // the work area's previous readers are done
  const int f = tid % NOUT, part = tid / NOUT;
  const int g = f >> 5, c4 = f & 31;
  const bool active = part < NPART;
  // prefetch the first batch of this thread's partials
  constexpr int PF = G <= 4 ? 16 : 8;  // (G <= 4: up to 64 partials in one round of loads)
  float4 pv[PF];
#pragma unroll
  for (int i = 0; i < PF; ++i) {
    const int k = part + NPART * i;
    pv[i] = (active && k < K) ? __ldcg(reinterpret_cast<const float4*>(src + (long long)k * PS + g * D) + c4)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  if (warp < G) {
    const int gg = warp;
    float mk[8], lk[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int k = lane + 32 * i;
      mk[i] = (k < K) ? __ldcg(src + (long long)k * PS + G * D + gg) : -INFINITY;
      lk[i] = (k < K) ? __ldcg(src + (long long)k * PS + G * D + 8 + gg) : 0.f;
    }
    float M = mk[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) M = fmaxf(M, mk[i]);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float L = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int k = lane + 32 * i;
      const float w = (mk[i] == -INFINITY) ? 0.f : exp2f(mk[i] - M);
      if (k < K) wsm[k * G + gg] = w;
      L = fmaf(lk[i], w, L);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    if (lane == 0) {
      MH[gg] = M;
      LH[gg] = L;
    }
  }
  cons_sync();
  if (active) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int k0 = 0; k0 < K; k0 += NPART * PF) {
      if (k0 > 0) {
#pragma unroll
        for (int i = 0; i < PF; ++i) {
          const int k = k0 + part + NPART * i;
          pv[i] = (k < K) ? __ldcg(reinterpret_cast<const float4*>(src + (long long)k * PS + g * D) + c4)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
#pragma unroll
      for (int i = 0; i < PF; ++i) {
        const int k = k0 + part + NPART * i;
        const float w = (k < K) ? wsm[k * G + g] : 0.f;
        acc.x = fmaf(pv[i].x, w, acc.x);
        acc.y = fmaf(pv[i].y, w, acc.y);
        acc.z = fmaf(pv[i].z, w, acc.z);
        acc.w = fmaf(pv[i].w, w, acc.w);
      }
    }
    psum[part * NOUT + f] = acc;
  }
  cons_sync();
  if (tid < NOUT) {
    float4 a = psum[tid];
#pragma unroll
    for (int q = 1; q < NPART; ++q) {
      const float4 b = psum[q * NOUT + tid];
      a.x += b.x;
      a.y += b.y;
      a.z += b.z;
      a.w += b.w;
    }
    if (dst) {
      *reinterpret_cast<float4*>(dst + g * D + 4 * c4) = a;
    } else {
      const float L = LH[g];
      const float r = L > 0.f ? 1.f / L : 0.f;
      *reinterpret_cast<float4*>(out + g * D + 4 * c4) = make_float4(a.x * r, a.y * r, a.z * r, a.w * r);
    }
  }
  if (dst && tid < G) {
    dst[G * D + tid] = MH[tid];
    dst[G * D + 8 + tid] = LH[tid];
  }
}
template <int G>
__device__ __forceinline__ void fz_merge(const FzShared& s, const float* src, int K, float* dst, float* out) {
  merge_partials<G>(s.work, src, K, dst, out);
}

// ---------------------------------------------------------------------------
// consumer loop (warps 0-15)
// ---------------------------------------------------------------------------
template <int G, int WORDS, bool DENSE>
__device__ void fz_run_task(const FzParams& p, const FzShared& s, int kind, int u, int arg, unsigned& nfin) {
  const int tid = threadIdx.x;
  const int PS = G * D + 16;
  const Unit x = unit_of(p, s, u);
  // every thread acquires what the counted CTAs wrote before reading it
  if (kind == TK_PSEL) (void)ld_acquire(unit_ctrl(p, u) + CU_SCAN);
  else if (kind == TK_KSEL) (void)ld_acquire(unit_ctrl(p, u) + CU_SCORE);
  else if (kind == TK_GMERGE) (void)ld_acquire(group_ctrl(p, u, arg));
  else (void)ld_acquire(unit_ctrl(p, u) + CU_MERGED);
  if (kind == TK_PSEL || kind == TK_KSEL) {
    if constexpr (!DENSE) {
      if (kind == TK_PSEL) fz_psel(p, s, x);
      else fz_ksel<G>(p, s, x);
      cons_sync();
      if (tid == 0) {
        __threadfence();
        st_release(unit_ctrl(p, u) + (kind == TK_PSEL ? CU_PSEL : CU_SEL), 1u);
      }
    }
    return;
  }
  const unsigned nk = __ldcg(unit_ctrl(p, u) + CU_NKEYS);
  const int nch = nchunks_of(nk);
  const int ngroups = (nch + FZ_GROUP - 1) / FZ_GROUP;
  if (kind == TK_GMERGE) {
    const int gsize = min(FZ_GROUP, nch - arg * FZ_GROUP);
    const float* src = p.wk.part + ((long long)u * p.wk.C3 + (long long)arg * FZ_GROUP) * PS;
    float* gp = p.wk.gpart + ((long long)u * p.wk.max_groups + arg) * PS;
    fz_merge<G>(s, src, gsize, gp, nullptr);
    cons_sync();
    fz_finish(s, nfin, unit_ctrl(p, u) + CU_MERGED, 1u, (unsigned)ngroups, TK_MERGE, u, 0, p.status);
  } else if (kind == TK_MERGE) {
    fz_merge<G>(s, p.wk.gpart + (long long)u * p.wk.max_groups * PS, ngroups, nullptr,
                p.out + ((long long)x.b * p.dm.Hq + x.h * G) * D);
    cons_sync();
  }
}

template <int G, int WORDS, bool DENSE>
__device__ void fz_consumer(const FzParams& p, const FzShared& s) {
  const Dims& dm = p.dm;
  const int tid = threadIdx.x, lane = tid & 31;
  volatile int* misc = s.misc;
  unsigned nslot = 0, ndesc = 0, nfin = 0;
  bool ended = false;
  bool pref = false;  // the rows of the next descriptor were gathered during the previous item
  int* dec = s.misc + 16;  // decisions broadcast by thread 0 (outside every scratch area)
  unsigned qhead = 0, qtail = 0;  // thread 0: the task queue as last read
  while (true) {
    const int d = (int)(ndesc % FZ_NDESC);
    const uint32_t dpar = (ndesc / FZ_NDESC) & 1;
    // Thread 0 alone waits (bounded) for the next thing to do and broadcasts
    // it, so all consumer threads act together: 1 = a local task, 2 = the
    // next descriptor, 0 = stop.  Tasks come first.
    if (tid == 0) {
      int res = 0;
      const long long t0 = clock64();
      unsigned spins = 0;
      while (true) {
        if (misc[3] != misc[2]) {  // a group merge of this CTA
          __threadfence_block();
          const FzTask tk = s.tasks[misc[3] % FZ_NTASK];
          dec[4] = tk.kind;
          dec[5] = tk.unit;
          dec[6] = tk.arg;
          misc[3] = misc[3] + 1;
          res = 1;
          break;
        }
        // the grid-wide task queue (head and tail read before the last release, then fresh)
        if (spins++ > 0) {
          qhead = ld_relaxed(p.wk.ctrl + 2);
          qtail = ld_relaxed(p.wk.ctrl + 3);
        }
        if (qhead < qtail) {
          if (atomicCAS(p.wk.ctrl + 2, qhead, qhead + 1u) == qhead) {
            int4* e = p.wk.tq + qhead;
            const long long t1 = clock64();
            while (ld_acquire(reinterpret_cast<const unsigned*>(&e->w)) != qhead + 1u) {
              if (misc[0] || clock64() - t1 > FZ_WAIT_CYCLES) {
                set_status(p.status, HHR_ERR_TIMEOUT);
                misc[0] = 1;
                break;
              }
            }
            dec[4] = e->x;
            dec[5] = e->y;
            dec[6] = e->z;
            e->w = 0;  // the queue is clean for the next call
            res = misc[0] ? 0 : 1;
            break;
          }
          continue;
        }
        if (!ended) {
          if (mbar_test_wait(&s.dfull[d], dpar)) {
            // the descriptor's bulk copies (bounded wait), then: is the
            // descriptor after it published already, with rows to gather?
            res = 2;
            const int ns = s.desc[d].nslots;
            for (int k = 0; k < ns && res; ++k) {
              const unsigned gs = nslot + k;
              if (!fz_wait(s, &s.full[gs % FZ_NSLOT], (gs / FZ_NSLOT) & 1, p.status)) res = 0;
            }
            const unsigned n1 = ndesc + 1;
            const int d1 = (int)(n1 % FZ_NDESC);
            dec[3] = (mbar_test_wait(&s.dfull[d1], (n1 / FZ_NDESC) & 1) && s.desc[d1].gather) ? 1 : 0;
            break;
          }
        } else if (misc[5] == (int)nfin) {
          // Every request of this CTA is handled (tasks it made are in the
          // queue).  Done when the queue is empty; a task posted later by
          // another CTA is run there, at the latest by that CTA itself.
          __threadfence_block();
          if (misc[3] != misc[2]) continue;
          const unsigned h2 = ld_acquire(p.wk.ctrl + 2), t2 = ld_acquire(p.wk.ctrl + 3);
          if (h2 >= t2) break;
          continue;
        }
        if (misc[0]) break;
        if (clock64() - t0 > FZ_WAIT_CYCLES) {
          set_status(p.status, HHR_ERR_TIMEOUT);
          misc[0] = 1;
          break;
        }
      }
      dec[1] = res;
    }
    cons_sync();
    const int res = dec[1];
    if (res == 0) break;
    if (res == 1) {
      const int kind = dec[4], u = dec[5], arg = dec[6];
      cons_sync();  // dec is free again
      fz_run_task<G, WORDS, DENSE>(p, s, kind, u, arg, nfin);
      continue;
    }
    // Thread 0 saw the descriptor's phase and its slots' phases complete; the
    // consumer barrier above orders every other thread after it.  (The
    // descriptor stays put until this item releases it.)
    const FzDesc ds = s.desc[d];
    if (ds.kind == IT_END) {
      ended = true;
      if (tid == 0) mbar_arrive(&s.dempty[d]);
      ++ndesc;
      continue;
    }
    const int nslots = ds.nslots;
    const int s0 = (int)(nslot % FZ_NSLOT);
    // Rows this item gathers (unless already requested during the previous
    // item), then the rows of the next descriptor, so that its copies run
    // while this item computes.
    const bool pn = dec[3] != 0;
    if (ds.gather && !pref)
      gather_rows(s, s.ridx + d * FZ_ROWS, ds.n, s0, ds.kind == IT_SCAN ? p.pmin : p.Kr,
                  ds.kind == IT_SCAN ? p.pmax : p.Vc);
    if (pn) {
      const int d1 = (int)((ndesc + 1) % FZ_NDESC);
      const FzDesc nx = s.desc[d1];
      gather_rows(s, s.ridx + d1 * FZ_ROWS, nx.n, (int)((nslot + nslots) % FZ_NSLOT), nx.kind == IT_SCAN ? p.pmin : p.Kr,
                  nx.kind == IT_SCAN ? p.pmax : p.Vc);
    }
    pref = pn;
    if (ds.gather) {
      // this thread's copies of this item have landed (the next item's may still fly);
      // every warp computes on the rows it copied itself
      if (pn) cp_async_wait<1>();
      else cp_async_wait<0>();
      __syncwarp();
    }
    const Unit x = unit_of(p, s, ds.unit);
    if (ds.kind == IT_PREP) {
      fz_prep<G, DENSE>(p, s, x, d, s0);
    } else if (ds.kind == IT_SCAN) {
      if constexpr (!DENSE) fz_scan<G>(p, s, x, ds.chunk, ds.n, d, s0);
    } else if (ds.kind == IT_SCORE) {
      if constexpr (!DENSE) fz_score<G, WORDS>(p, s, x, ds.chunk, ds.n, d);
    } else if (ds.kind == IT_GATHER) {
      fz_gather<G>(p, s, x, ds.chunk, ds.n, d, s0);
    }
    // every consumer thread is done with the slots: release them and the descriptor
    if (tid == 0) {  // the task queue's state, read now so the next poll need not wait for it
      qhead = ld_relaxed(p.wk.ctrl + 2);
      qtail = ld_relaxed(p.wk.ctrl + 3);
    }
    cons_sync();
    if (tid == 0) {
      if (ds.gather) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // before later bulk copies into the slots
      for (int k = 0; k < nslots; ++k) mbar_arrive(&s.empty[(nslot + k) % FZ_NSLOT]);
      mbar_arrive(&s.dempty[d]);
    }
    nslot += nslots;
    ++ndesc;
    // ---- completion ----
    if (ds.kind == IT_PREP) {
      if (x.L == 0) {
        for (int e = tid; e < G * D; e += FZ_CONS) p.out[((long long)x.b * dm.Hq + x.h * G) * D + e] = 0.f;
        if (tid == 0) {
          if (p.dbg.n_sel_pages) p.dbg.n_sel_pages[x.u] = 0;
          if (p.dbg.n_sel_keys) p.dbg.n_sel_keys[x.u] = 0;
          if (p.dbg.n_cand) p.dbg.n_cand[x.u] = 0;
        }
      }
      if (DENSE || x.L == 0) {
        cons_sync();
        if (tid == 0) {
          unit_ctrl(p, x.u)[CU_NKEYS] = DENSE ? (unsigned)x.L : 0u;
          __threadfence();
          st_release(unit_ctrl(p, x.u) + CU_SEL, 1u);
        }
      }
    } else if (ds.kind == IT_SCAN) {
      const unsigned nscan = (unsigned)((x.np + FZ_ROWS - 1) / FZ_ROWS);
      fz_finish(s, nfin, unit_ctrl(p, x.u) + CU_SCAN, 1u, nscan, TK_PSEL, x.u, 0, p.status);
    } else if (ds.kind == IT_SCORE) {
      fz_finish(s, nfin, unit_ctrl(p, x.u) + CU_SCORE, 1u, (unsigned)score_items(p, s, x), TK_KSEL, x.u, 0,
                p.status);
    } else if (ds.kind == IT_GATHER) {
      const int nch = nchunks_of((unsigned)ds.pad0);
      const int g = ds.chunk / FZ_GROUP;
      const int gsize = min(FZ_GROUP, nch - g * FZ_GROUP);
      fz_finish(s, nfin, group_ctrl(p, x.u, g), 1u, (unsigned)gsize, TK_GMERGE, x.u, g, p.status);
    }
  }
  if (tid == 0) {
    s.misc[1] = (int)nslot;
    __threadfence_block();
    misc[6] = 1;  // lets the finisher stop
  }
}

template <int G, int WORDS, bool DENSE>
__global__ void __launch_bounds__(FZ_THREADS, 1) hhr_fused_kernel(FzParams p) {
  extern __shared__ __align__(128) unsigned char fz_smem[];
  const FzShared s = fz_shared(fz_smem);
  const int tid = threadIdx.x;
  if (tid == 0) {
    for (int i = 0; i < FZ_NSLOT; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < FZ_NDESC; ++i) {
      mbar_init(&s.dfull[i], 1);
      mbar_init(&s.dempty[i], 1);
    }
    for (int i = 0; i < FZ_NFIN; ++i) {
      mbar_init(&s.ffull[i], 1);
      mbar_init(&s.fempty[i], 1);
    }
    for (int i = 0; i < 8; ++i) s.misc[i] = 0;
    fence_mbar_init();
  }
  for (int i = tid; i < FZ_UCACHE; i += blockDim.x) s.ucache[i] = 0u;
  for (int b = tid; b < min(p.dm.B, FZ_SEQ); b += blockDim.x) {
    s.seqp[b] = seq_len_of(p.dm, p.seq_lens, b);
    if constexpr (!DENSE) {  // full attention has no budgets
      s.seqp[FZ_SEQ + b] = __ldg(p.n_keep + b);
      s.seqp[2 * FZ_SEQ + b] = __ldg(p.top_k + b);
    }
  }
  __syncthreads();
  const int warp = tid >> 5;
  if (warp >= FZ_CWARPS) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(FZ_REGS_AUX));
    if (warp == FZ_PRODUCER_WARP) fz_producer<G, WORDS, DENSE>(p, s);
    else if (warp == FZ_FINISHER_WARP) fz_finisher(p, s);
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(FZ_REGS_CONS));
    fz_consumer<G, WORDS, DENSE>(p, s);
  }
  __syncthreads();
  // drain copies that were armed but never consumed (only after an abort)
  if (tid == 0) {
    const unsigned armed = (unsigned)s.misc[4], consumed = (unsigned)s.misc[1];
    for (unsigned gs = consumed; gs < armed; ++gs) {
      const long long t0 = clock64();
      while (!mbar_try_wait(&s.full[gs % FZ_NSLOT], (gs / FZ_NSLOT) & 1)) {
        if (clock64() - t0 > FZ_WAIT_CYCLES) break;
      }
    }
  }
  // the last CTA to leave resets the control words for the next call
  __shared__ int s_last;
  if (tid == 0) {
    __threadfence();
    const unsigned old = atomicAdd(p.wk.ctrl + 1, 1u);
    s_last = (old == gridDim.x - 1);
  }
  __syncthreads();
  if (s_last) {
    __threadfence();
    const int U = p.dm.B * p.dm.Hkv;
    for (int i = tid; i < U * (CU_STRIDE + p.wk.max_groups); i += blockDim.x) p.wk.ctrl[4 + i] = 0u;
    if (tid == 0) {
      p.wk.ctrl[0] = 0u;
      p.wk.ctrl[1] = 0u;
      p.wk.ctrl[2] = 0u;
      p.wk.ctrl[3] = 0u;
    }
  }
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
template <int G, int WORDS, bool DENSE>
static cudaError_t launch_fused_t(const FzParams& prm, int grid, cudaStream_t st) {
  static bool configured[64] = {false};  // the attribute is per function and device
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(hhr_fused_kernel<G, WORDS, DENSE>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)FZ_SMEM);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  hhr_fused_kernel<G, WORDS, DENSE><<<grid, FZ_THREADS, FZ_SMEM, st>>>(prm);
  return cudaGetLastError();
}

static FzParams make_params(const DecodeArgs& a, bool dense) {
  FzParams prm;
  prm.dm = a.dm;
  prm.wk = a.wk;
  prm.q = a.q;
  prm.R = a.R;
  prm.W = a.W;
  prm.Kr = a.Kr;
  prm.Vc = a.Vc;
  prm.pmin = a.pmin;
  prm.pmax = a.pmax;
  prm.codes = a.codes;
  prm.seq_lens = a.seq_lens;
  prm.table = a.table;
  prm.n_keep = a.n_keep;
  prm.top_k = a.top_k;
  prm.sm_scale = a.sm_scale;
  prm.out = a.out;
  prm.dbg = a.dbg;
  prm.status = a.status;
  const int U = a.dm.B * a.dm.Hkv;
  prm.items_per_unit_scan = dense ? 0 : a.wk.C1;
  prm.items_per_unit_score = dense ? 0 : a.wk.C2;
  prm.items_per_unit_gather = a.wk.C3;
  prm.total_items = U * (1 + prm.items_per_unit_scan + prm.items_per_unit_score + prm.items_per_unit_gather);
  return prm;
}

template <int G>
cudaError_t launch_dense(const DecodeArgs& a) {
  const FzParams prm = make_params(a, true);
  const int grid = std::min(a.num_sms, prm.total_items);
  return launch_fused_t<G, 1, true>(prm, grid, a.stream);
}

#define HHR_INSTANTIATE_DECODE(G)                           \
  template cudaError_t launch_decode<G>(const DecodeArgs&); \
  template cudaError_t launch_dense<G>(const DecodeArgs&);

}  // namespace hhr
