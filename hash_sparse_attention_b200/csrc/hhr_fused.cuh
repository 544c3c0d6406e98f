// HHR decode step as one persistent, warp-specialised kernel per layer (sm_100a).
//
// Work is a queue of items claimed in order by the CTAs (one CTA per SM).
// For units u = (sequence b, KV head h) the queue holds, in this order:
//   PREP(u)        for every unit: q' = R_h q, then the query codes
//   SCAN(u, c)     for every unit in turn: page bounds of pages
//                  [128c, 128c + 128)
//   GATHER(u, c)   for every unit in turn: softmax attention over kept rows
//                  [128c, 128c + 128), written as a partial per chunk
// Three more steps run as local tasks of the CTA that completes their
// inputs (it sees its own counter increment reach the target):
//   SELECT(u)      after the last scan chunk and the query codes of u: page
//                  top-N, Hamming scores of the kept pages' rows, key top-k
//   GMERGE(u, g)   after the 16 chunks of group g: their partials, merged
//   MERGE(u)       after the last group: the groups, merged into the output
// So no CTA ever waits for another CTA's consumers; only the producer waits,
// for q' (scan) or the selection (gather) of a unit claimed before.  The
// queue is unit-major, so late units are scanned while early units are
// selected and gathered.
//
// Warps 0-7 consume; warp 8 (producer) claims items and moves their bytes
// (R_h, W_h, q or q', page metadata rows, K'/V rows) into a ring of shared
// memory slots with cp.async.bulk, each slot completing on an mbarrier;
// warp 9 (finisher) publishes completions (a gpu-scope fence, then an
// acquire-release counter increment) and posts the tasks that become ready.
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
// 1-D bulk copy global -> shared (16-byte aligned, size a multiple of 16)
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void st_release(unsigned* p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
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
constexpr int FZ_CONS = 256;                 // consumer threads (warps 0-7)
constexpr int FZ_PRODUCER_WARP = 8;
constexpr int FZ_FINISHER_WARP = 9;
constexpr int FZ_THREADS = FZ_CONS + 64;
constexpr int FZ_NSLOT = 8;                  // ring slots
constexpr int FZ_SLOT = 16384;               // bytes per slot (64 rows of 256 B)
constexpr int FZ_NDESC = 4;                  // descriptor ring
constexpr int FZ_NFIN = 8;                   // finisher ring
constexpr int FZ_NTASK = 16;                 // local task ring
constexpr int FZ_QBUF = 4096;                // q (bf16) or q' (fp32) of one unit
constexpr int FZ_ROWS = FUSED_ROWS;          // pages per SCAN item, rows per GATHER item
constexpr int FZ_GROUP = FUSED_GROUP;        // gather chunks per group merge
constexpr int FZ_WORK = 57344;               // consumer scratch (select, softmax, merges)
constexpr long long FZ_WAIT_CYCLES = 4000000000ll;  // ~2 s at 1.9 GHz

constexpr size_t FZ_OFF_RING = 0;
constexpr size_t FZ_OFF_QBUF = FZ_OFF_RING + (size_t)FZ_NSLOT * FZ_SLOT;
constexpr size_t FZ_OFF_WORK = FZ_OFF_QBUF + (size_t)FZ_NDESC * FZ_QBUF;
constexpr size_t FZ_OFF_DESC = FZ_OFF_WORK + FZ_WORK;
constexpr size_t FZ_OFF_FINQ = FZ_OFF_DESC + FZ_NDESC * 32;
constexpr size_t FZ_OFF_TASK = FZ_OFF_FINQ + FZ_NFIN * 32;
constexpr size_t FZ_OFF_BAR = FZ_OFF_TASK + FZ_NTASK * 16;
constexpr size_t FZ_OFF_MISC = FZ_OFF_BAR + 8 * (2 * FZ_NSLOT + 2 * FZ_NDESC + 2 * FZ_NFIN);
constexpr size_t FZ_SMEM = FZ_OFF_MISC + 256;

enum : int { IT_PREP = 0, IT_SCAN = 1, IT_SELECT = 2, IT_GATHER = 3, IT_GMERGE = 4, IT_MERGE = 5, IT_END = 6 };
// (SELECT, GMERGE and MERGE are local tasks, never queue items)

struct __align__(16) FzDesc {
  int kind, unit, chunk, n;
  int nslots, pad0, pad1, pad2;
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
  CU_SEL = 2,     // kept rows published (sel_keys, n_keys)
  CU_SCAN = 3,    // scan chunks finished + query codes finished
  CU_MERGED = 4,  // groups merged
  CU_NKEYS = 5,   // kept rows
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
  int items_per_unit_gather;  // C3
  int total_items;
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
  int* misc;  // [0] abort, [1] consumed slots, [2] tasks posted, [3] tasks taken,
              // [4] armed slots, [5] finisher requests done, [6] consumers finished
};

__device__ __forceinline__ FzShared fz_shared(unsigned char* base) {
  FzShared s;
  s.ring = base + FZ_OFF_RING;
  s.qbuf = base + FZ_OFF_QBUF;
  s.work = base + FZ_OFF_WORK;
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

// barrier among the 256 consumer threads only
__device__ __forceinline__ void cons_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

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

// Acquires a phase another thread of the CTA has already seen complete (so the
// slot's bytes are visible to this thread too); bounded like every wait.
__device__ __forceinline__ void mbar_confirm(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > FZ_WAIT_CYCLES) break;
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
__device__ __forceinline__ Unit unit_of(const FzParams& p, int u) {
  Unit x;
  x.u = u;
  x.b = u / p.dm.Hkv;
  x.h = u - x.b * p.dm.Hkv;
  x.L = seq_len_of(p.dm, p.seq_lens, x.b);
  x.np = (x.L + p.dm.P - 1) / p.dm.P;
  return x;
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
  if (item < U * p.items_per_unit_scan) {
    kind = IT_SCAN;
    u = item / p.items_per_unit_scan;
    c = item - u * p.items_per_unit_scan;
    return;
  }
  item -= U * p.items_per_unit_scan;
  if (item < U * p.items_per_unit_gather) {
    kind = IT_GATHER;
    u = item / p.items_per_unit_gather;
    c = item - u * p.items_per_unit_gather;
    return;
  }
  kind = IT_END;
}

// ---------------------------------------------------------------------------
// producer (warp 8): claims items and fills slots
// ---------------------------------------------------------------------------
template <int G, int WORDS, bool DENSE>
__device__ void fz_producer(const FzParams& p, const FzShared& s) {
  const int lane = threadIdx.x & 31;
  const Dims& dm = p.dm;
  const int prep_slots = DENSE ? 4 : 4 + dm.nb / 64;  // R_h, then W_h (not needed without hashing)
  unsigned nslot = 0, ndesc = 0, armed = 0;
  while (true) {
    int item = 0;
    if (lane == 0) item = (int)atomicAdd(p.wk.ctrl + 0, 1u);
    item = __shfl_sync(0xffffffffu, item, 0);
    int kind, u, c;
    decode_item(p, item, kind, u, c);
    const Unit x = unit_of(p, u);
    int n = 0;
    unsigned nk = 0;
    if (kind == IT_SCAN) {
      n = min(FZ_ROWS, x.np - c * FZ_ROWS);
      if (n <= 0) continue;
    } else if (kind == IT_GATHER) {
      bool ok = true;
      if (lane == 0) ok = fz_wait_count(s, unit_ctrl(p, u) + CU_SEL, 1u, p.status);
      if (__shfl_sync(0xffffffffu, (int)ok, 0) == 0) break;
      (void)ld_acquire(unit_ctrl(p, u) + CU_SEL);  // every lane reads what the selecting CTA wrote
      nk = __ldcg(unit_ctrl(p, u) + CU_NKEYS);
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
    const int nslots = kind == IT_PREP ? prep_slots : ((kind == IT_SCAN || kind == IT_GATHER) ? 4 : 0);
    // the unit's q or q' goes to the descriptor's q buffer, completing on the first slot
    uint32_t qbytes = 0;
    const void* qsrc = nullptr;
    if (kind == IT_PREP) {
      qbytes = G * D * 2;
      qsrc = p.q + ((long long)x.b * dm.Hq + x.h * G) * D;
    } else if (kind == IT_SCAN || kind == IT_GATHER) {
      if (kind == IT_SCAN) {
        bool ok = true;
        if (lane == 0) ok = fz_wait_count(s, unit_ctrl(p, u) + CU_PREP, 1u, p.status);
        if (__shfl_sync(0xffffffffu, (int)ok, 0) == 0) break;
      }
      fence_proxy_async_global();  // q' was written by another CTA with ordinary stores
      qbytes = G * D * 4;
      qsrc = p.wk.qrot + ((long long)x.b * dm.Hq + x.h * G) * D;
    }
    unsigned char* qdst = s.qbuf + d * FZ_QBUF;
    // kept-row ids of a sparse gather chunk: lane holds rows lane + 32 i
    int rid[4] = {0, 0, 0, 0};
    if (!DENSE && kind == IT_GATHER) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int jj = lane + 32 * i;
        if (jj < n) rid[i] = __ldcg(p.wk.sel_keys + (long long)u * p.wk.Kmax + (long long)c * FZ_ROWS + jj);
      }
    }
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
      unsigned char* dst = s.ring + (size_t)slot * FZ_SLOT;
      // Each lane issues its own copies; lane 0 then arms the barrier with the
      // warp's byte total (the phase cannot complete before that arrival,
      // whichever order the copies land in).
      uint32_t mine = 0;
      if (kind == IT_PREP) {
        if (lane == 0) {
          const void* src = (k < 4) ? (const void*)(p.R + (long long)x.h * D * D + (long long)k * 32 * D)
                                    : (const void*)(p.W + ((long long)x.h * dm.nb + (long long)(k - 4) * 64) * D);
          bulk_g2s(dst, src, FZ_SLOT, &s.full[slot]);
          mine += FZ_SLOT;
        }
      } else if (kind == IT_SCAN) {
        const __nv_bfloat16* base = (k < 2) ? p.pmin : p.pmax;
        const int j0 = (k & 1) * 64;  // first page of this slot within the chunk
        const int rows = max(0, min(64, n - j0));
        if (!dm.paged) {
          if (lane == 0 && rows > 0) {
            bulk_g2s(dst, base + ((long long)(x.b * dm.Hkv + x.h) * dm.np_max + (long long)c * FZ_ROWS + j0) * D,
                     rows * 256, &s.full[slot]);
            mine += rows * 256;
          }
        } else {
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int j = lane + 32 * i;
            if (j < rows) {
              const int pg = c * FZ_ROWS + j0 + j;
              const int blk = __ldg(p.table + (long long)x.b * dm.max_blocks + pg);
              if ((unsigned)blk < (unsigned)dm.num_blocks) {
                bulk_g2s(dst + j * 256, base + ((long long)blk * dm.Hkv + x.h) * D, 256, &s.full[slot]);
                mine += 256;
              } else {
                set_status(p.status, HHR_ERR_BAD_BLOCK);
              }
            }
          }
        }
      } else {  // IT_GATHER
        const __nv_bfloat16* base = (k < 2) ? p.Kr : p.Vc;
        const int j0 = (k & 1) * 64;
        const int rows = max(0, min(64, n - j0));
        if (DENSE && !dm.paged) {
          if (lane == 0 && rows > 0) {
            bulk_g2s(dst, base + ((long long)(x.b * dm.Hkv + x.h) * dm.T + (long long)c * FZ_ROWS + j0) * D,
                     rows * 256, &s.full[slot]);
            mine += rows * 256;
          }
        } else {
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int j = lane + 32 * i;
            if (j < rows) {
              // row j0 + j = lane + 32 (2 (k & 1) + i): its id is rid[2 (k & 1) + i]
              const int t = DENSE ? c * FZ_ROWS + j0 + j : (((k & 1) == 0) ? rid[i] : rid[2 + i]);
              const long long off = kv_row(dm, p.table, x.b, x.h, t, p.status);
              if (off >= 0) {
                bulk_g2s(dst + j * 256, base + off, 256, &s.full[slot]);
                mine += 256;
              }
            }
          }
        }
      }
      if (k == 0 && lane == 0 && qbytes) {
        bulk_g2s(qdst, qsrc, qbytes, &s.full[slot]);
        mine += qbytes;
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) mine += __shfl_xor_sync(0xffffffffu, mine, o);
      if (lane == 0) mbar_arrive_expect_tx(&s.full[slot], mine);
      __syncwarp();
      armed = gs + 1;
    }
    if (aborted) break;
    if (lane == 0) {
      FzDesc& ds = s.desc[d];
      ds.kind = kind;
      ds.unit = u;
      ds.chunk = c;
      ds.n = n;
      ds.nslots = nslots;
      ds.pad0 = (int)nk;  // gather: the unit's kept rows
      mbar_arrive(&s.dfull[d]);
    }
    __syncwarp();
    nslot += nslots;
    ++ndesc;
    if (kind == IT_END) break;
  }
  if (lane == 0) s.misc[4] = (int)armed;  // slots armed with copies (drained at exit)
}

// ---------------------------------------------------------------------------
// finisher (warp 9): gpu-scope fence, the counter increment, task posting
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
    if (r.target != 0u && old + r.value == r.target) {
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

// One halving round of a transposed butterfly over WIDTH lanes: the lane
// keeps the half of its N values selected by bit `o` of its lane index and
// adds the partner's copy of that half.
template <int N, int WIDTH>
__device__ __forceinline__ void halving_round(float* v, int ln, int o) {
  const bool up = (ln & o) != 0;
#pragma unroll
  for (int i = 0; i < N / 2; ++i) {
    const float send = up ? v[i] : v[i + N / 2];
    const float keep = up ? v[i + N / 2] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o, WIDTH);
  }
}

// Sums NV per-lane values over the 16 lanes of a half-warp.  With NV >= 16
// lane l ends with the sums of values [ (NV/16) l, (NV/16)(l+1) ) in
// v[0 .. NV/16); with NV < 16 every lane ends with value index
// l >> (4 - log2 NV) in v[0] (the last rounds are plain butterflies).
template <int NV>
__device__ __forceinline__ void half_reduce(float* v, int ln) {
  if constexpr (NV >= 2) halving_round<NV, 16>(v, ln, 8); else v[0] += __shfl_xor_sync(0xffffffffu, v[0], 8, 16);
  if constexpr (NV >= 4) halving_round<NV / 2, 16>(v, ln, 4); else v[0] += __shfl_xor_sync(0xffffffffu, v[0], 4, 16);
  if constexpr (NV >= 8) halving_round<NV / 4, 16>(v, ln, 2); else v[0] += __shfl_xor_sync(0xffffffffu, v[0], 2, 16);
  if constexpr (NV >= 16) halving_round<NV / 8, 16>(v, ln, 1); else v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1, 16);
}

// Sums NV (>= 32) per-lane values over the 32 lanes of a warp; lane l ends
// with the sums of values [ (NV/32) l, (NV/32)(l+1) ) in v[0 .. NV/32).
template <int NV>
__device__ __forceinline__ void warp_reduce_t(float* v, int lane) {
  halving_round<NV, 32>(v, lane, 16);
  halving_round<NV / 2, 32>(v, lane, 8);
  halving_round<NV / 4, 32>(v, lane, 4);
  halving_round<NV / 8, 32>(v, lane, 2);
  halving_round<NV / 16, 32>(v, lane, 1);
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
    int t = lane < FZ_CONS / 32 ? red[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    red[lane] = t;
  }
  cons_sync();
  const int before = (warp > 0 ? red[warp - 1] : 0) + x - v;
  *total = red[FZ_CONS / 32 - 1];
  cons_sync();
  return before;
}

// ---- PREP: q' = R_h q, then the query codes --------------------------------
template <int G, bool DENSE>
__device__ void fz_prep(const FzParams& p, const FzShared& s, const Unit& x, int d, int s0, unsigned& nfin) {
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
  // q'_i = sum_j R_h[i][j] q_j: warp w takes rows 16w .. 16w+15 in blocks of
  // RB rows; the RB x GP partial sums are reduced together (transposed)
  constexpr int RB = GP == 4 ? 16 : 8;
  for (int rb = 0; rb < 16; rb += RB) {
    float v[RB * GP];
#pragma unroll
    for (int r = 0; r < RB; ++r) {
      const int i = warp * 16 + rb + r;
      const float4 rr = *reinterpret_cast<const float4*>(
          s.ring + (size_t)((s0 + i / 32) % FZ_NSLOT) * FZ_SLOT + (i % 32) * 512 + lane * 16);
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        float a = 0.f;
        if (g < G) {
          a = rr.x * qv[g][0];
          a = fmaf(rr.y, qv[g][1], a);
          a = fmaf(rr.z, qv[g][2], a);
          a = fmaf(rr.w, qv[g][3], a);
        }
        v[r * GP + g] = a;
      }
    }
    warp_reduce_t<RB * GP>(v, lane);
    // lane holds values [2 lane, 2 lane + 2): row (2 lane + e) / GP, head (2 lane + e) % GP
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int vi = 2 * lane + e;
      const int r = vi / GP, g = vi % GP;
      if (g < G) {
        const int i = warp * 16 + rb + r;
        const long long idx = ((long long)x.b * dm.Hq + x.h * G + g) * D + i;
        p.wk.qrot[idx] = v[e];
        if (p.dbg.q_rot) p.dbg.q_rot[idx] = v[e];
      }
    }
  }
  // publish q' now: the scans of this unit need only q'
  __threadfence();
  cons_sync();
  if (tid == 0) st_release(unit_ctrl(p, x.u) + CU_PREP, 1u);
  if constexpr (DENSE) return;  // full attention needs no codes (and has no W_h)
  // Query codes: bit j = [ (W_h q)_j > 0 ].  Products of bf16 values are exact
  // in fp32; the 128-term fp32 sum errs by at most 127 * 2^-24 * sum|w q|, so
  // below 2^-14 * sum|w q| the sign is taken from an fp64 recompute.  Warp w
  // takes bits [w nb/8, (w+1) nb/8) in blocks of NBB bits; after the
  // transposed reduction lane l holds (sum, magnitude) of bit l / GP of the
  // block and head l % GP.
  constexpr int NBB = 32 / GP;  // 8 (GP 4) or 4 (GP 8) bits per block
  const int bits_per_warp = dm.nb / (FZ_CONS / 32);
  for (int jb = 0; jb < bits_per_warp; jb += NBB) {
    float v[2 * NBB * GP];  // [bit][head][sum, magnitude]
#pragma unroll
    for (int bb = 0; bb < NBB; ++bb) {
      const int j = warp * bits_per_warp + jb + bb;
      const uint2 wv = *reinterpret_cast<const uint2*>(s.ring + (size_t)((s0 + 4 + j / 64) % FZ_NSLOT) * FZ_SLOT +
                                                       (j % 64) * 256 + lane * 8);
      const float w4[4] = {bf_lo(wv.x), bf_hi(wv.x), bf_lo(wv.y), bf_hi(wv.y)};
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
    const int j = warp * bits_per_warp + jb + bb;
    bool bit = v[0] > 0.f;
    if (g < G && fabsf(v[0]) <= ldexpf(v[1], -14)) {
      double ad = 0.0;
      const unsigned char* wrow = s.ring + (size_t)((s0 + 4 + j / 64) % FZ_NSLOT) * FZ_SLOT + (j % 64) * 256;
      for (int c = 0; c < D; c += 2) {
        const uint32_t w2 = *reinterpret_cast<const uint32_t*>(wrow + c * 2);
        ad += (double)bf_lo(w2) * (double)qf[g * D + c];
        ad += (double)bf_hi(w2) * (double)qf[g * D + c + 1];
      }
      bit = ad > 0.0;
    }
    if (g < G && bit) atomicOr(&qc[g * 8 + j / 32], 1u << (j % 32));
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
  // the query codes count like one more scan chunk toward the unit's select
  const unsigned nscan = (unsigned)((x.np + FZ_ROWS - 1) / FZ_ROWS);
  fz_finish(s, nfin, unit_ctrl(p, x.u) + CU_SCAN, 1u, x.np > 0 ? nscan + 1u : 0u, IT_SELECT, x.u, 0, p.status);
}

// ---- SCAN: page bounds of one chunk ------------------------------------------
template <int G>
__device__ void fz_scan(const FzParams& p, const FzShared& s, const Unit& x, int c, int n, int d, int s0) {
  constexpr int GP = G <= 4 ? 4 : 8;
  const Dims& dm = p.dm;
  const int tid = threadIdx.x, hw = tid >> 4, ln = tid & 15;
  const float* qs = reinterpret_cast<const float*>(s.qbuf + d * FZ_QBUF);
  // channels 8 ln .. 8 ln + 7 of each head, as channel pairs.  For G <= 4
  // the positive and negative parts of q' are kept apart so that the bound
  // is two packed FMAs per channel pair; for larger groups q' itself is kept
  // and each channel picks min or max by the sign of q'.
  constexpr int QS = G <= 4 ? 2 : 1;
  float2 qh[QS][G][4];
#pragma unroll
  for (int g = 0; g < G; ++g) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 v = *reinterpret_cast<const float2*>(qs + g * D + ln * 8 + 2 * k);
      if constexpr (QS == 2) {
        qh[0][g][k] = make_float2(fmaxf(v.x, 0.f), fmaxf(v.y, 0.f));
        qh[QS - 1][g][k] = make_float2(fminf(v.x, 0.f), fminf(v.y, 0.f));
      } else {
        qh[0][g][k] = v;
      }
    }
  }
  // Two pages per half-warp step: values [page][head].  After the reduction
  // lane ln holds value index ln >> HSH, i.e. page pl and head hidx below.
  constexpr int NV = 2 * GP;
  constexpr int HSH = GP == 4 ? 1 : 0;
  const int vi = ln >> HSH;
  const int pl = vi / GP, hidx = vi % GP;
#pragma unroll 1
  for (int r = 0; r < 4; ++r) {
    float a[NV];
#pragma unroll
    for (int pp = 0; pp < 2; ++pp) {
      const int j = hw + 16 * (2 * r + pp);  // page within the chunk
      const size_t off = (size_t)(j % 64) * 256 + ln * 16;
      const uint4 mnv = *reinterpret_cast<const uint4*>(s.ring + (size_t)((s0 + j / 64) % FZ_NSLOT) * FZ_SLOT + off);
      const uint4 mxv = *reinterpret_cast<const uint4*>(s.ring + (size_t)((s0 + 2 + j / 64) % FZ_NSLOT) * FZ_SLOT + off);
      const uint32_t mw[4] = {mnv.x, mnv.y, mnv.z, mnv.w};
      const uint32_t xw[4] = {mxv.x, mxv.y, mxv.z, mxv.w};
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        float sum = 0.f;
        if (g < G) {
          float2 acc = make_float2(0.f, 0.f);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 hi2 = make_float2(bf_lo(xw[k]), bf_hi(xw[k]));
            const float2 lo2 = make_float2(bf_lo(mw[k]), bf_hi(mw[k]));
            if constexpr (QS == 2) {
              acc = __ffma2_rn(qh[0][g][k], hi2, acc);
              acc = __ffma2_rn(qh[QS - 1][g][k], lo2, acc);
            } else {
              const float2 q2 = qh[0][g][k];
              acc = __ffma2_rn(q2, make_float2(q2.x >= 0.f ? hi2.x : lo2.x, q2.y >= 0.f ? hi2.y : lo2.y), acc);
            }
          }
          sum = acc.x + acc.y;
        }
        a[pp * GP + g] = sum;
      }
    }
    half_reduce<NV>(a, ln);
    // U = max over the real heads of the lane's page (the 8 lanes of that page)
    float U = hidx < G ? a[0] : -INFINITY;
#pragma unroll
    for (int o = 1 << HSH; o < 8; o <<= 1) U = fmaxf(U, __shfl_xor_sync(0xffffffffu, U, o, 16));
    const int j = hw + 16 * (2 * r + pl);
    if (j < n) {
      const int pg = c * FZ_ROWS + j;
      if ((ln & 7) == 0) {
        p.wk.U[(long long)x.u * dm.np_max + pg] = U;
        if (p.dbg.page_U) p.dbg.page_U[(long long)x.u * dm.np_max + pg] = U;
      }
      if (p.dbg.page_ub && hidx < G && (ln & ((1 << HSH) - 1)) == 0)
        p.dbg.page_ub[((long long)x.b * dm.Hq + x.h * G + hidx) * dm.np_max + pg] = a[0];
    }
  }
}

// ---- SELECT: page top-N, Hamming scores, key top-k --------------------------
// Shared scratch of the select (byte offsets into the work area).
constexpr int SEL_US = 0;                      // float [np + np/32] bounds, later uint16 scores (padded)
constexpr int SEL_HIST = 33792;                // int [2112]
constexpr int SEL_SPAGE = SEL_HIST + 8448;     // int [2048] kept pages
constexpr int SEL_CAND = SEL_SPAGE + 8192;     // int [512] members of the threshold bin
constexpr int SEL_FLAG = SEL_CAND + 2048;      // u32 [256] bitmap of kept threshold-bin members
constexpr int SEL_RED = SEL_FLAG + 1024;       // int [48] scan scratch and broadcasts
constexpr int SEL_CQ = SEL_RED + 192;          // u64 [G * WORDS]
constexpr int SEL_NBIN = 1024;                 // value bins of the page select
constexpr int SEL_MAX_CAND = 512;

// padded index: one spare word per 32 so that blocked per-thread ranges read
// shared memory without bank conflicts
__device__ __forceinline__ int pad32(int i) { return i + (i >> 5); }

// Bin of a bound: monotone non-decreasing in the value, so the N-th largest
// lies in one bin and every larger bin is kept whole.
__device__ __forceinline__ int value_bin(float v, float lo, float scale) {
  const float t = (v - lo) * scale;
  return min(SEL_NBIN - 1, max(0, (int)t));
}

// Block-wide min and max of one value per consumer thread (scratch: 16 floats).
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
  for (int w = 1; w < FZ_CONS / 32; ++w) {
    lo = fminf(lo, wr[w * 2 + 0]);
    hi = fmaxf(hi, wr[w * 2 + 1]);
  }
  cons_sync();
}

template <int G, int WORDS>
__device__ void fz_select(const FzParams& p, const FzShared& s, const Unit& x) {
  const Dims& dm = p.dm;
  const Work& wk = p.wk;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float* Us = reinterpret_cast<float*>(s.work + SEL_US);
  int* hist = reinterpret_cast<int*>(s.work + SEL_HIST);
  int* spage = reinterpret_cast<int*>(s.work + SEL_SPAGE);
  int* cand = reinterpret_cast<int*>(s.work + SEL_CAND);
  unsigned* flag = reinterpret_cast<unsigned*>(s.work + SEL_FLAG);
  int* red = reinterpret_cast<int*>(s.work + SEL_RED);
  int* bc = red + 36;  // broadcasts [0..11]
  uint64_t* cq = reinterpret_cast<uint64_t*>(s.work + SEL_CQ);
  float* wr = reinterpret_cast<float*>(hist + 2048);  // 16 floats of min / max scratch
  const int np = x.np;
  const int N = min(min(max(__ldg(p.n_keep + x.b), 1), wk.Nmax), np);
  int* gsel = wk.sel_pages + (long long)x.u * wk.Nmax;
  int* dsel = p.dbg.sel_pages ? p.dbg.sel_pages + (long long)x.u * wk.Nmax : nullptr;

  if (N >= np) {
    for (int i = tid; i < np; i += FZ_CONS) {
      spage[i] = i;
      gsel[i] = i;
      if (dsel) dsel[i] = i;
    }
    cons_sync();
  } else {
    // ---- bounds into shared memory (coalesced, 8 loads in flight per thread) ----
    const float* Ug = wk.U + (long long)x.u * dm.np_max;
    float lo = INFINITY, hi = -INFINITY;
    for (int base = 0; base < np; base += FZ_CONS * 8) {
      float v[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int i = base + r * FZ_CONS + tid;
        v[r] = i < np ? __ldcg(Ug + i) : 0.f;
      }
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int i = base + r * FZ_CONS + tid;
        if (i < np) {
          Us[pad32(i)] = v[r];
          lo = fminf(lo, v[r]);
          hi = fmaxf(hi, v[r]);
        }
      }
    }
    cons_minmax(lo, hi, wr);
    // ---- threshold by value bins.  Each thread owns a blocked range of at
    // most 32 pages; `member` marks pages still undecided, `keep` the kept.
    // A level bins the members over their value range (bins are monotone in
    // the value), keeps every bin above the one holding the need-th largest
    // member and descends into that bin; a small bin is then ranked exactly,
    // a bin of equal values is taken in index order. ----
    const int kpt = (np + FZ_CONS - 1) / FZ_CONS;
    const int i0 = min(np, tid * kpt), cnt = min(np, i0 + kpt) - i0;
    unsigned member = cnt >= 32 ? 0xffffffffu : ((1u << cnt) - 1u);
    unsigned keep = 0u;
    int need = N, nbin = 0;
    bool tie = false;
#pragma unroll 1
    for (int level = 0; level < 4; ++level) {
      tie = !(hi > lo);
      if (tie) break;
      const float scale = (float)SEL_NBIN / (hi - lo);
      for (int i = tid; i < SEL_NBIN; i += FZ_CONS) hist[i] = 0;
      cons_sync();
      for (int k = 0; k < cnt; ++k)
        if ((member >> k) & 1u) atomicAdd(&hist[value_bin(Us[pad32(i0 + k)], lo, scale)], 1);
      cons_sync();
      {
        constexpr int BPT = SEL_NBIN / FZ_CONS;  // 4 bins per thread, counted from the top
        int c4 = 0;
#pragma unroll
        for (int e = 0; e < BPT; ++e) c4 += hist[SEL_NBIN - 1 - (tid * BPT + e)];
        int tot;
        const int before = cons_excl_scan(c4, red, &tot);
        if (before < need && before + c4 >= need) {
          int run = before;
#pragma unroll
          for (int e = 0; e < BPT; ++e) {
            const int bi = SEL_NBIN - 1 - (tid * BPT + e);
            if (run + hist[bi] >= need) {
              bc[0] = bi;
              bc[1] = need - run;
              bc[2] = hist[bi];
              break;
            }
            run += hist[bi];
          }
        }
        cons_sync();
      }
      const int bstar = bc[0];
      need = bc[1];
      nbin = bc[2];
      float nlo = INFINITY, nhi = -INFINITY;
      for (int k = 0; k < cnt; ++k) {
        if (!((member >> k) & 1u)) continue;
        const float v = Us[pad32(i0 + k)];
        const int bn = value_bin(v, lo, scale);
        if (bn > bstar) {
          keep |= 1u << k;
          member &= ~(1u << k);
        } else if (bn < bstar) {
          member &= ~(1u << k);
        } else {
          nlo = fminf(nlo, v);
          nhi = fmaxf(nhi, v);
        }
      }
      if (nbin <= SEL_MAX_CAND) break;
      cons_minmax(nlo, nhi, wr);
      lo = nlo;
      hi = nhi;
    }
    if (tie || nbin > SEL_MAX_CAND) {
      // equal values (or still crowded): members in index order, the first `need`
      int m = __popc(member);
      int tot;
      const int mb = cons_excl_scan(m, red, &tot);
      int take = max(0, min(m, need - mb));
      for (int k = 0; k < cnt && take > 0; ++k) {
        if ((member >> k) & 1u) {
          keep |= 1u << k;
          --take;
        }
      }
    } else {
      // exact ranking of the (few) members: larger value first, then lower index
      if (tid == 0) bc[4] = 0;
      for (int i = tid; i < (np + 31) / 32; i += FZ_CONS) flag[i] = 0u;
      cons_sync();
      for (int k = 0; k < cnt; ++k)
        if ((member >> k) & 1u) cand[atomicAdd(&bc[4], 1)] = i0 + k;
      cons_sync();
      for (int a = tid; a < nbin; a += FZ_CONS) {
        const int ia = cand[a];
        const float va = Us[pad32(ia)];
        int rank = 0;
        for (int b2 = 0; b2 < nbin; ++b2) {
          const int ib = cand[b2];
          const float vb = Us[pad32(ib)];
          rank += (vb > va) || (vb == va && ib < ia);
        }
        if (rank < need) atomicOr(&flag[ia >> 5], 1u << (ia & 31));
      }
      cons_sync();
      for (int k = 0; k < cnt; ++k) {
        const int i = i0 + k;
        if (((member >> k) & 1u) && ((flag[i >> 5] >> (i & 31)) & 1u)) keep |= 1u << k;
      }
    }
    // ---- kept pages in index order ----
    int tot;
    int pos = cons_excl_scan(__popc(keep), red, &tot);
    for (int k = 0; k < cnt; ++k) {
      if ((keep >> k) & 1u) {
        const int i = i0 + k;
        spage[pos] = i;
        gsel[pos] = i;
        if (dsel) dsel[pos] = i;
        ++pos;
      }
    }
    cons_sync();
  }
  if (tid == 0 && p.dbg.n_sel_pages) p.dbg.n_sel_pages[x.u] = N;
  // ---- Hamming scores of the kept pages' rows (candidate ci = round * 256 + tid) ----
  const int nbins = G * dm.nb + 1;
  for (int i = tid; i < nbins; i += FZ_CONS) hist[i] = 0;
  if (tid < G * WORDS) cq[tid] = __ldcg(wk.qcodes + ((long long)x.b * dm.Hq + x.h * G) * WORDS + tid);
  cons_sync();
  unsigned short* sc = reinterpret_cast<unsigned short*>(s.work + SEL_US);
  const int ncs = N * dm.P;
  int* dsc = p.dbg.key_scores ? p.dbg.key_scores + (long long)x.u * wk.Nmax * dm.P : nullptr;
  constexpr int RB = WORDS >= 4 ? 4 : 8;  // rows per thread in flight
  for (int base = 0; base < ncs; base += FZ_CONS * RB) {
    uint64_t cw[RB][WORDS];
    bool valid[RB];
#pragma unroll
    for (int r = 0; r < RB; ++r) {
      const int ci = base + r * FZ_CONS + tid;
      valid[r] = false;
#pragma unroll
      for (int w2 = 0; w2 < WORDS; ++w2) cw[r][w2] = 0ull;
      if (ci < ncs) {
        const int slot = ci / dm.P;
        const int t = spage[slot] * dm.P + (ci - slot * dm.P);
        if (t < x.L) {
          const long long off = code_row(dm, p.table, x.b, x.h, t, p.status);
          if (off >= 0) {
            valid[r] = true;
            if constexpr (WORDS == 1) {
              cw[r][0] = __ldg(p.codes + off);
            } else {
#pragma unroll
              for (int w2 = 0; w2 < WORDS; w2 += 2) {
                const ulonglong2 v = __ldg(reinterpret_cast<const ulonglong2*>(p.codes + off + w2));
                cw[r][w2] = v.x;
                cw[r][w2 + 1] = v.y;
              }
            }
          }
        }
      }
    }
#pragma unroll
    for (int r = 0; r < RB; ++r) {
      const int ci = base + r * FZ_CONS + tid;
      if (ci < ncs) {
        int S = 0;
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
          for (int w2 = 0; w2 < WORDS; ++w2) S += __popcll(cq[g * WORDS + w2] ^ cw[r][w2]);
        sc[ci] = valid[r] ? (unsigned short)S : (unsigned short)0xFFFFu;
        if (dsc) dsc[ci] = valid[r] ? S : INT_MAX;
        if (valid[r]) atomicAdd(&hist[S], 1);
      }
    }
  }
  cons_sync();
  // ---- key top-k: counting select on the score histogram ----
  const int bpt = (nbins + FZ_CONS - 1) / FZ_CONS;
  int local = 0;
  for (int e = 0; e < bpt; ++e) {
    const int bi = tid * bpt + e;
    if (bi < nbins) local += hist[bi];
  }
  int n_cand;
  const int before = cons_excl_scan(local, red, &n_cand);
  const int keff = min(min(max(__ldg(p.top_k + x.b), 1), wk.Kmax), n_cand);
  if (keff > 0 && before < keff && before + local >= keff) {
    int run = before;
    for (int e = 0; e < bpt; ++e) {
      const int bi = tid * bpt + e;
      const int c2 = bi < nbins ? hist[bi] : 0;
      if (run + c2 >= keff) {
        bc[2] = bi;
        bc[3] = keff - run;
        break;
      }
      run += c2;
    }
  }
  cons_sync();
  if (keff > 0) {
    // Kept rows in candidate order, written coalesced: candidates go in
    // rounds of 256 (thread t takes candidate round * 256 + t); per round
    // and warp the counts of S < T and S == T are scanned once, then each
    // warp places its rows with ballots.
    const int T = bc[2], need_eq = bc[3];
    const int rounds = (ncs + FZ_CONS - 1) / FZ_CONS;  // <= 64
    int* wcnt = reinterpret_cast<int*>(s.work + SEL_CAND);  // [rounds][8] packed (lt << 16 | eq)
    const unsigned lanemask_lt = (1u << lane) - 1u;
    for (int r = 0; r < rounds; ++r) {
      const int ci = r * FZ_CONS + tid;
      const int v = ci < ncs ? sc[ci] : 0xFFFF;
      const unsigned blt = __ballot_sync(0xffffffffu, v < T);
      const unsigned beq = __ballot_sync(0xffffffffu, v == T);
      if (lane == 0) wcnt[r * 8 + warp] = (__popc(blt) << 16) | __popc(beq);
    }
    cons_sync();
    // exclusive scan over the rounds * 8 packed counts (2 per thread)
    {
      const int n2 = rounds * 8;
      const int a0 = 2 * tid, a1 = 2 * tid + 1;
      const int c0 = a0 < n2 ? wcnt[a0] : 0, c1 = a1 < n2 ? wcnt[a1] : 0;
      int tot;
      const int bsum = cons_excl_scan(c0 + c1, red, &tot);
      if (a0 < n2) wcnt[a0] = bsum;
      if (a1 < n2) wcnt[a1] = bsum + c0;
      cons_sync();
    }
    int* out = wk.sel_keys + (long long)x.u * wk.Kmax;
    int* dout = p.dbg.sel_keys ? p.dbg.sel_keys + (long long)x.u * wk.Kmax : nullptr;
    for (int r = 0; r < rounds; ++r) {
      const int ci = r * FZ_CONS + tid;
      const int v = ci < ncs ? sc[ci] : 0xFFFF;
      const bool lt = v < T, eq = v == T;
      const unsigned beq = __ballot_sync(0xffffffffu, eq);
      const int base2 = wcnt[r * 8 + warp];
      const int lt_before = base2 >> 16, eq_before = base2 & 0xffff;
      const int eq_rank = eq_before + __popc(beq & lanemask_lt);
      const bool take = lt || (eq && eq_rank < need_eq);
      const unsigned btake = __ballot_sync(0xffffffffu, take);
      const int pos = lt_before + min(eq_before, need_eq) + __popc(btake & lanemask_lt);
      if (take) {
        const int slot = ci / dm.P;
        const int t = spage[slot] * dm.P + (ci - slot * dm.P);
        out[pos] = t;
        if (dout) dout[pos] = t;
      }
    }
  }
  if (tid == 0) {
    unit_ctrl(p, x.u)[CU_NKEYS] = (unsigned)keff;
    if (p.dbg.n_sel_keys) p.dbg.n_sel_keys[x.u] = keff;
    if (p.dbg.n_cand) p.dbg.n_cand[x.u] = n_cand;
  }
}

// ---- GATHER: softmax attention over one chunk of kept rows ---------------------
// Writes the chunk's partial (unnormalised output, max and sum of weights per
// head, in log2 units) to its fixed slot part[u][c].
template <int G>
__device__ void fz_gather(const FzParams& p, const FzShared& s, const Unit& x, int c, int n, int d, int s0) {
  constexpr int GP = G <= 4 ? 4 : 8;  // heads padded to a power of two
  constexpr int CH = GP == 4 ? 8 : 4; // rows per half-warp per pass
  constexpr int NPASS = FZ_ROWS / (16 * CH);
  constexpr int NV = CH * GP;         // partial logits per lane
  constexpr int KPL = NV / 16;        // logits a lane keeps after the reduction
  constexpr int HS = GP / 2;          // heads per softmax thread (two head slots)
  constexpr int NKG = FZ_CONS / 64;   // key groups of the V accumulation
  const int tid = threadIdx.x, hw = tid >> 4, ln = tid & 15, lane = tid & 31, warp = tid >> 5;
  float* S = reinterpret_cast<float*>(s.work);                  // [128][GP] logits (log2 units)
  float2* PP = reinterpret_cast<float2*>(s.work + 4096);        // [128][GP] (p, p)
  float* red = reinterpret_cast<float*>(s.work + 4096 + 8192);  // [8 warps][HS]
  float2* OR = reinterpret_cast<float2*>(s.work + 16384);       // [NKG][G][64]
  const float* qs = reinterpret_cast<const float*>(s.qbuf + d * FZ_QBUF);
  const float qscale = p.sm_scale * 1.4426950408889634f;
  // ---- logits: pass r, half-warp hw takes rows 16 CH r + CH hw + kk; lane owns 8 channels ----
  {
    float2 qv[G][4];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 v = *reinterpret_cast<const float2*>(qs + g * D + ln * 8 + 2 * k);
        qv[g][k] = make_float2(v.x * qscale, v.y * qscale);
      }
#pragma unroll 1
    for (int pass = 0; pass < NPASS; ++pass) {
      const int row0 = pass * 16 * CH + CH * hw;
      float val[NV];
#pragma unroll
      for (int kk = 0; kk < CH; ++kk) {
        const int j = row0 + kk;
        const uint4 kv = *reinterpret_cast<const uint4*>(s.ring + (size_t)((s0 + j / 64) % FZ_NSLOT) * FZ_SLOT +
                                                         (j % 64) * 256 + ln * 16);
        const uint32_t kw[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
        for (int g = 0; g < GP; ++g) {
          float a = 0.f;
          if (g < G) {
            float2 acc = make_float2(0.f, 0.f);
#pragma unroll
            for (int k = 0; k < 4; ++k) acc = __ffma2_rn(qv[g][k], make_float2(bf_lo(kw[k]), bf_hi(kw[k])), acc);
            a = acc.x + acc.y;
          }
          val[g * CH + kk] = a;
        }
      }
      half_reduce<NV>(val, ln);
      // lane holds values [KPL ln, KPL ln + KPL): head (KPL ln) / CH, rows (KPL ln) % CH + i
#pragma unroll
      for (int i = 0; i < KPL; ++i) {
        const int vi = KPL * ln + i;
        const int g = vi / CH, kk = vi % CH;
        const int j = row0 + kk;
        S[j * GP + g] = (j < n) ? val[i] : -INFINITY;
      }
    }
  }
  cons_sync();
  // ---- chunk max per head, weights, sums ----
  // thread t: row j = t & 127, head slot gsl = t >> 7; heads gsl + 2e, e < HS
  const int j = tid & 127, gsl = tid >> 7;
  float sv[HS];
#pragma unroll
  for (int e = 0; e < HS; ++e) {
    sv[e] = S[j * GP + gsl + 2 * e];
    float m = sv[e];
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) red[warp * HS + e] = m;
  }
  cons_sync();
  float mh[GP];
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    const int sl = g & 1, e = g >> 1;
    float cm = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) cm = fmaxf(cm, red[(sl * 4 + w) * HS + e]);
    mh[g] = cm;
  }
  float ps[HS];
#pragma unroll
  for (int e = 0; e < HS; ++e) {
    const int g = gsl + 2 * e;
    float mg = mh[0];
#pragma unroll
    for (int gg = 1; gg < GP; ++gg)
      if (gg == g) mg = mh[gg];
    const float pv = (g < G && j < n) ? exp2f(sv[e] - mg) : 0.f;
    PP[j * GP + g] = make_float2(pv, pv);
    float t = pv;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    ps[e] = t;
  }
  cons_sync();  // every thread has read the maxima before red is reused for sums
  if (lane == 0) {
#pragma unroll
    for (int e = 0; e < HS; ++e) red[warp * HS + e] = ps[e];
  }
  cons_sync();  // weights and sums complete
  // ---- V accumulation: channel pair cp of every head, rows of key group kg ----
  const int cp = tid & 63, kg = tid >> 6;
  float2 o2[G];
#pragma unroll
  for (int g = 0; g < G; ++g) o2[g] = make_float2(0.f, 0.f);
  constexpr int RPG = FZ_ROWS / NKG;  // rows per key group
#pragma unroll 4
  for (int r = 0; r < RPG; ++r) {
    const int jr = kg * RPG + r;
    if (jr < n) {
      const uint32_t vw = *reinterpret_cast<const uint32_t*>(
          s.ring + (size_t)((s0 + 2 + jr / 64) % FZ_NSLOT) * FZ_SLOT + (jr % 64) * 256 + cp * 4);
      const float2 v2 = make_float2(bf_lo(vw), bf_hi(vw));
#pragma unroll
      for (int g = 0; g < G; ++g) o2[g] = __ffma2_rn(PP[jr * GP + g], v2, o2[g]);
    }
  }
#pragma unroll
  for (int g = 0; g < G; ++g) OR[(kg * G + g) * 64 + cp] = o2[g];
  cons_sync();
  // ---- the chunk's partial: key groups summed in order ----
  const int PS = G * D + 16;  // partial: o[G][D], m at G D, l at G D + 8 (16-byte rows)
  float* part = p.wk.part + ((long long)x.u * p.wk.C3 + c) * PS;
  for (int e = tid; e < G * 64; e += FZ_CONS) {
    const int g = e / 64, c2 = e % 64;
    float2 a = OR[(0 * G + g) * 64 + c2];
#pragma unroll
    for (int k = 1; k < NKG; ++k) {
      const float2 v = OR[(k * G + g) * 64 + c2];
      a.x += v.x;
      a.y += v.y;
    }
    *reinterpret_cast<float2*>(part + g * D + 2 * c2) = a;
  }
  if (tid < G) {
    const int sl = tid & 1, e = tid >> 1;
    float cs = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) cs += red[(sl * 4 + w) * HS + e];
    float mt = mh[0];
#pragma unroll
    for (int gg = 1; gg < GP; ++gg)
      if (gg == tid) mt = mh[gg];
    part[G * D + tid] = mt;
    part[G * D + 8 + tid] = cs;
  }
}

// Merges K partials src[0 .. K) (stride G D + 16 floats) in index order:
// M = max m_k, w_k = 2^(m_k - M), L = sum w_k l_k, O = sum w_k o_k.  With
// dst, the merged partial (O, M, L) is written there; otherwise out = O / L.
// K <= 256.  Loads are issued in batches so that a merge costs a few L2
// round trips, not one per partial.
template <int G>
__device__ void fz_merge(const FzShared& s, const float* src, int K, float* dst, float* out) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int PS = G * D + 16;
  float* wsm = reinterpret_cast<float*>(s.work + 32768);  // [256][G] weights, then M[8], L[8]
  float* MH = wsm + 256 * G;
  float* LH = MH + 8;
  cons_sync();  // the work area's previous readers are done
  if (warp < G) {
    const int g = warp;
    float mk[8], lk[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int k = lane + 32 * i;
      mk[i] = (k < K) ? __ldcg(src + (long long)k * PS + G * D + g) : -INFINITY;
      lk[i] = (k < K) ? __ldcg(src + (long long)k * PS + G * D + 8 + g) : 0.f;
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
      if (k < K) wsm[k * G + g] = w;
      L = fmaf(lk[i], w, L);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    if (lane == 0) {
      MH[g] = M;
      LH[g] = L;
    }
  }
  cons_sync();
  for (int f = tid; f < 32 * G; f += FZ_CONS) {
    const int g = f >> 5, c4 = f & 31;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int k0 = 0; k0 < K; k0 += 8) {
      float4 v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        v[i] = (k0 + i < K) ? __ldcg(reinterpret_cast<const float4*>(src + (long long)(k0 + i) * PS + g * D) + c4)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float w = (k0 + i < K) ? wsm[(k0 + i) * G + g] : 0.f;
        acc.x = fmaf(v[i].x, w, acc.x);
        acc.y = fmaf(v[i].y, w, acc.y);
        acc.z = fmaf(v[i].z, w, acc.z);
        acc.w = fmaf(v[i].w, w, acc.w);
      }
    }
    if (dst) {
      *reinterpret_cast<float4*>(dst + g * D + 4 * c4) = acc;
    } else {
      const float L = LH[g];
      const float r = L > 0.f ? 1.f / L : 0.f;
      *reinterpret_cast<float4*>(out + g * D + 4 * c4) = make_float4(acc.x * r, acc.y * r, acc.z * r, acc.w * r);
    }
  }
  if (dst && tid < G) {
    dst[G * D + tid] = MH[tid];
    dst[G * D + 8 + tid] = LH[tid];
  }
}

// ---------------------------------------------------------------------------
// consumer loop (warps 0-7)
// ---------------------------------------------------------------------------
template <int G, int WORDS, bool DENSE>
__device__ void fz_run_task(const FzParams& p, const FzShared& s, int kind, int u, int arg, unsigned& nfin) {
  const int tid = threadIdx.x;
  const int PS = G * D + 16;
  const Unit x = unit_of(p, u);
  // every thread acquires what the counted CTAs wrote before reading it
  if (kind == IT_SELECT) (void)ld_acquire(unit_ctrl(p, u) + CU_SCAN);
  else if (kind == IT_GMERGE) (void)ld_acquire(group_ctrl(p, u, arg));
  else (void)ld_acquire(unit_ctrl(p, u) + CU_MERGED);
  if (kind == IT_SELECT) {
    if constexpr (!DENSE) {
      fz_select<G, WORDS>(p, s, x);
      __threadfence();
      cons_sync();
      if (tid == 0) st_release(unit_ctrl(p, u) + CU_SEL, 1u);
    }
    return;
  }
  const unsigned nk = __ldcg(unit_ctrl(p, u) + CU_NKEYS);
  const int nch = nchunks_of(nk);
  const int ngroups = (nch + FZ_GROUP - 1) / FZ_GROUP;
  if (kind == IT_GMERGE) {
    const int gsize = min(FZ_GROUP, nch - arg * FZ_GROUP);
    const float* src = p.wk.part + ((long long)u * p.wk.C3 + (long long)arg * FZ_GROUP) * PS;
    float* gp = p.wk.gpart + ((long long)u * p.wk.max_groups + arg) * PS;
    fz_merge<G>(s, src, gsize, gp, nullptr);
    cons_sync();
    fz_finish(s, nfin, unit_ctrl(p, u) + CU_MERGED, 1u, (unsigned)ngroups, IT_MERGE, u, 0, p.status);
  } else if (kind == IT_MERGE) {
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
  int* dec = s.misc + 16;  // decisions broadcast by thread 0 (outside every scratch area)
  while (true) {
    const int d = (int)(ndesc % FZ_NDESC);
    const uint32_t dpar = (ndesc / FZ_NDESC) & 1;
    // Thread 0 alone waits (bounded) for the next thing to do and broadcasts
    // it, so all consumer threads act together: 1 = a local task, 2 = the
    // next descriptor, 0 = stop.  Tasks come first.
    if (tid == 0) {
      int res = 0;
      const long long t0 = clock64();
      while (true) {
        if (misc[3] != misc[2]) {
          __threadfence_block();
          const FzTask tk = s.tasks[misc[3] % FZ_NTASK];
          dec[4] = tk.kind;
          dec[5] = tk.unit;
          dec[6] = tk.arg;
          misc[3] = misc[3] + 1;
          res = 1;
          break;
        }
        if (!ended) {
          if (mbar_try_wait(&s.dfull[d], dpar)) {
            res = 2;
            break;
          }
        } else if (misc[5] == (int)nfin) {
          // every request handled; a task posted by the last one is visible
          // now (the finisher posts before it counts the request)
          __threadfence_block();
          if (misc[3] == misc[2]) break;  // none pending: done
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
    mbar_confirm(&s.dfull[d], dpar);
    const FzDesc ds = s.desc[d];
    cons_sync();  // everyone holds the descriptor before dec is written again
    if (ds.kind == IT_END) {
      ended = true;
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.dempty[d]);
      ++ndesc;
      continue;
    }
    const int nslots = ds.nslots;
    const int s0 = (int)(nslot % FZ_NSLOT);
    if (nslots > 0) {
      if (tid == 0) {
        bool ok = true;
        for (int k = 0; k < nslots && ok; ++k) {
          const unsigned gs = nslot + k;
          ok = fz_wait(s, &s.full[gs % FZ_NSLOT], (gs / FZ_NSLOT) & 1, p.status);
        }
        dec[2] = ok ? 1 : 0;
      }
      cons_sync();
      if (!dec[2]) break;
      for (int k = 0; k < nslots; ++k) {
        const unsigned gs = nslot + k;
        mbar_confirm(&s.full[gs % FZ_NSLOT], (gs / FZ_NSLOT) & 1);
      }
    }
    const Unit x = unit_of(p, ds.unit);
    if (ds.kind == IT_PREP) {
      fz_prep<G, DENSE>(p, s, x, d, s0, nfin);
    } else if (ds.kind == IT_SCAN) {
      if constexpr (!DENSE) fz_scan<G>(p, s, x, ds.chunk, ds.n, d, s0);
    } else if (ds.kind == IT_GATHER) {
      fz_gather<G>(p, s, x, ds.chunk, ds.n, d, s0);
    }
    // release the slots and the descriptor (one arrival per consumer warp)
    __syncwarp();
    if (lane == 0) {
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
        if (tid == 0) unit_ctrl(p, x.u)[CU_NKEYS] = DENSE ? (unsigned)x.L : 0u;
        __threadfence();
        cons_sync();
        if (tid == 0) st_release(unit_ctrl(p, x.u) + CU_SEL, 1u);
      }
    } else if (ds.kind == IT_SCAN) {
      cons_sync();
      const unsigned nscan = (unsigned)((x.np + FZ_ROWS - 1) / FZ_ROWS);
      fz_finish(s, nfin, unit_ctrl(p, x.u) + CU_SCAN, 1u, nscan + 1u, IT_SELECT, x.u, 0, p.status);
    } else if (ds.kind == IT_GATHER) {
      cons_sync();
      const int nch = nchunks_of((unsigned)ds.pad0);
      const int g = ds.chunk / FZ_GROUP;
      const int gsize = min(FZ_GROUP, nch - g * FZ_GROUP);
      fz_finish(s, nfin, group_ctrl(p, x.u, g), 1u, (unsigned)gsize, IT_GMERGE, x.u, g, p.status);
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
      mbar_init(&s.empty[i], FZ_CONS / 32);
    }
    for (int i = 0; i < FZ_NDESC; ++i) {
      mbar_init(&s.dfull[i], 1);
      mbar_init(&s.dempty[i], FZ_CONS / 32);
    }
    for (int i = 0; i < FZ_NFIN; ++i) {
      mbar_init(&s.ffull[i], 1);
      mbar_init(&s.fempty[i], 1);
    }
    for (int i = 0; i < 8; ++i) s.misc[i] = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const int warp = tid >> 5;
  if (warp == FZ_PRODUCER_WARP) {
    fz_producer<G, WORDS, DENSE>(p, s);
  } else if (warp == FZ_FINISHER_WARP) {
    fz_finisher(p, s);
  } else {
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
  prm.items_per_unit_gather = a.wk.C3;
  prm.total_items = U * (1 + prm.items_per_unit_scan + prm.items_per_unit_gather);
  return prm;
}

template <int G>
cudaError_t launch_decode(const DecodeArgs& a) {
  const FzParams prm = make_params(a, false);
  const int grid = std::min(a.num_sms, prm.total_items);
  switch (a.dm.words) {
    case 1: return launch_fused_t<G, 1, false>(prm, grid, a.stream);
    case 2: return launch_fused_t<G, 2, false>(prm, grid, a.stream);
    case 4: return launch_fused_t<G, 4, false>(prm, grid, a.stream);
  }
  return cudaErrorInvalidValue;
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
