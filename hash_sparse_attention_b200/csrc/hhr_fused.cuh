// HHR decode step as one persistent, warp-specialised kernel per layer (sm_100a).
//
// Work is a queue of items claimed in order by the CTAs (one CTA per SM):
//   PREP(u)       q' = R_h q and the query sign codes of unit u = (b, h)
//   SCAN(u, c)    page bounds of pages [128c, 128c + 128) of unit u; the CTA
//                 that finishes the last chunk of u runs SELECT(u): page
//                 top-N, Hamming scores of the kept pages' rows, key top-k
//   GATHER(u, c)  softmax attention over kept rows [128c, 128c + 128) of u;
//                 a CTA keeps a running (max, sum, output) over consecutive
//                 chunks of one unit and writes one partial when it moves
//                 on; the CTA that writes the last partial merges them
// The queue is unit-major, so while the last units are still being scanned
// and selected, the first units are already being gathered.
//
// Inside a CTA, warp 8 is the producer: it claims items and moves their
// bytes (R_h, W_h, q or q', page metadata rows, K'/V rows) into a ring of
// shared-memory slots with cp.async.bulk, each slot completing on an
// mbarrier.  Warps 0-7 consume the slots in order.
//
// Every wait (mbarrier or global flag) is bounded by a clock budget; on
// expiry the kernel records HHR_ERR_TIMEOUT in the status word, drains its
// own copies in flight and returns, so a fault elsewhere cannot hang it.
// A wait only ever targets an item claimed earlier (queue order), so waits
// end without any co-residency assumption.
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
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
// barrier among the 256 consumer threads only (the producer warp never joins)
__device__ __forceinline__ void cons_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// ---------------------------------------------------------------------------
// parameters of the fused kernel
// ---------------------------------------------------------------------------
constexpr int FZ_CONS = 256;                 // consumer threads (8 warps)
constexpr int FZ_THREADS = FZ_CONS + 32;     // + one producer warp
constexpr int FZ_NSLOT = 8;                  // ring slots
constexpr int FZ_SLOT = 16384;               // bytes per slot (64 rows of 256 B)
constexpr int FZ_NDESC = 4;                  // descriptor ring
constexpr int FZ_QBUF = 4096;                // q (bf16) or q' (fp32) of one unit
constexpr int FZ_ROWS = 128;                 // pages per SCAN item, rows per GATHER item
constexpr int FZ_WORK = 57344;               // consumer scratch (select, softmax, merges)
constexpr long long FZ_WAIT_CYCLES = 4000000000ll;  // ~2 s at 1.9 GHz

constexpr size_t FZ_OFF_RING = 0;
constexpr size_t FZ_OFF_QBUF = FZ_OFF_RING + (size_t)FZ_NSLOT * FZ_SLOT;
constexpr size_t FZ_OFF_WORK = FZ_OFF_QBUF + (size_t)FZ_NDESC * FZ_QBUF;
constexpr size_t FZ_OFF_DESC = FZ_OFF_WORK + FZ_WORK;
constexpr size_t FZ_OFF_BAR = FZ_OFF_DESC + FZ_NDESC * 32;
constexpr size_t FZ_OFF_MISC = FZ_OFF_BAR + 8 * (2 * FZ_NSLOT + 2 * FZ_NDESC);
constexpr size_t FZ_SMEM = FZ_OFF_MISC + 256;

enum : int { IT_PREP = 0, IT_SCAN = 1, IT_GATHER = 2, IT_END = 3 };

struct __align__(16) FzDesc {
  int kind, unit, chunk, n;
  int nslots, pad0, pad1, pad2;
};

// per-unit control words (kept at zero between calls; the last CTA resets them)
enum : int { CU_PREP = 0, CU_SEL = 1, CU_SCAN = 2, CU_GATHER = 3, CU_NPART = 4, CU_NKEYS = 5, CU_STRIDE = 8 };

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
  int total_items;
};

struct FzShared {
  unsigned char* ring;
  unsigned char* qbuf;
  unsigned char* work;
  FzDesc* desc;
  uint64_t* full;
  uint64_t* empty;
  uint64_t* dfull;
  uint64_t* dempty;
  int* misc;  // [0] abort, [1] consumed slots, [2..] broadcast
};

__device__ __forceinline__ FzShared fz_shared(unsigned char* base) {
  FzShared s;
  s.ring = base + FZ_OFF_RING;
  s.qbuf = base + FZ_OFF_QBUF;
  s.work = base + FZ_OFF_WORK;
  s.desc = reinterpret_cast<FzDesc*>(base + FZ_OFF_DESC);
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + FZ_OFF_BAR);
  s.full = bars;
  s.empty = bars + FZ_NSLOT;
  s.dfull = bars + 2 * FZ_NSLOT;
  s.dempty = bars + 2 * FZ_NSLOT + FZ_NDESC;
  s.misc = reinterpret_cast<int*>(base + FZ_OFF_MISC);
  return s;
}

__device__ __forceinline__ volatile int* abort_flag(const FzShared& s) { return s.misc; }

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

// Bounded wait for a global flag set by another CTA (acquire).
__device__ __forceinline__ bool fz_wait_flag(const FzShared& s, const unsigned* flag, int* status) {
  if (ld_acquire(flag)) return true;
  const long long t0 = clock64();
  while (true) {
    __nanosleep(128);
    if (ld_acquire(flag)) return true;
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

// unit geometry
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

// ---------------------------------------------------------------------------
// producer: claims items and fills slots
// ---------------------------------------------------------------------------
template <int G, int WORDS, bool DENSE>
__device__ void fz_producer(const FzParams& p, const FzShared& s) {
  const int lane = threadIdx.x & 31;
  const Dims& dm = p.dm;
  const int U = dm.B * dm.Hkv;
  const int C1 = p.wk.C1, C3 = p.wk.C3;
  const int prep_slots = DENSE ? 4 : 4 + dm.nb / 64;  // R_h, then W_h (not needed without hashing)
  unsigned nslot = 0, ndesc = 0, armed = 0;
  while (true) {
    int item = 0;
    if (lane == 0) item = (int)atomicAdd(p.wk.ctrl + 0, 1u);
    item = __shfl_sync(0xffffffffu, item, 0);
    int kind, u = 0, c = 0;
    if (item < U) {
      kind = IT_PREP;
      u = item;
    } else if (!DENSE && item < U + U * C1) {
      kind = IT_SCAN;
      u = (item - U) / C1;
      c = (item - U) - u * C1;
    } else if (item < p.total_items) {
      const int g = item - U - (DENSE ? 0 : U * C1);
      kind = IT_GATHER;
      u = g / C3;
      c = g - u * C3;
    } else {
      kind = IT_END;
    }
    const Unit x = unit_of(p, u);
    int n = 0;
    if (kind == IT_SCAN) {
      n = min(FZ_ROWS, x.np - c * FZ_ROWS);
      if (n <= 0) continue;
    } else if (kind == IT_GATHER) {
      bool ok = true;
      if (lane == 0) ok = fz_wait_flag(s, unit_ctrl(p, u) + CU_SEL, p.status);
      ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
      if (!ok) break;
      (void)ld_acquire(unit_ctrl(p, u) + CU_SEL);  // every lane reads what the selecting CTA wrote
      const int nk = (int)__ldcg(unit_ctrl(p, u) + CU_NKEYS);
      n = min(FZ_ROWS, nk - c * FZ_ROWS);
      if (n <= 0) continue;
    } else if (kind == IT_PREP) {
      n = x.L;
    }
    // descriptor slot
    const int d = (int)(ndesc % FZ_NDESC);
    if (ndesc >= FZ_NDESC) {
      bool ok = true;
      if (lane == 0) ok = fz_wait(s, &s.dempty[d], ((ndesc / FZ_NDESC) - 1) & 1, p.status);
      if (__shfl_sync(0xffffffffu, (int)ok, 0) == 0) break;
    }
    const int nslots = kind == IT_PREP ? prep_slots : (kind == IT_END ? 0 : 4);
    // the unit's q or q' goes to the descriptor's q buffer, completing on the first slot
    uint32_t qbytes = 0;
    const void* qsrc = nullptr;
    if (kind == IT_PREP) {
      qbytes = G * D * 2;
      qsrc = p.q + ((long long)x.b * dm.Hq + x.h * G) * D;
    } else if (kind != IT_END) {
      if (kind == IT_SCAN) {
        bool ok = true;
        if (lane == 0) ok = fz_wait_flag(s, unit_ctrl(p, u) + CU_PREP, p.status);
        if (__shfl_sync(0xffffffffu, (int)ok, 0) == 0) break;
      }
      fence_proxy_async_global();  // q' was written by other CTAs with ordinary stores
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
        if (__shfl_sync(0xffffffffu, (int)ok, 0) == 0) { aborted = true; break; }
      }
      unsigned char* dst = s.ring + (size_t)slot * FZ_SLOT;
      // ---- this slot's copies: each lane issues its own; lane 0 then arms the
      // barrier with the warp's byte total (the phase cannot complete before
      // that arrival, whichever order the copies land in) ----
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
      } else if (kind == IT_GATHER) {
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
// consumers
// ---------------------------------------------------------------------------

// One halving round of a transposed butterfly over the 16 lanes of a
// half-warp: the lane keeps the half of its N values selected by bit `o` of
// its lane index and adds the partner's copy of that half.
template <int N>
__device__ __forceinline__ void halving_round(float* v, int ln, int o) {
  const bool up = (ln & o) != 0;
#pragma unroll
  for (int i = 0; i < N / 2; ++i) {
    const float send = up ? v[i] : v[i + N / 2];
    const float keep = up ? v[i + N / 2] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o, 16);
  }
}

// Sums NV per-lane values over the 16 lanes of a half-warp.  With NV >= 16
// lane l ends with the sums of values [ (NV/16) l, (NV/16)(l+1) ) in
// v[0 .. NV/16); with NV < 16 every lane ends with value index
// l >> (4 - log2 NV) in v[0] (the last rounds are plain butterflies).
template <int NV>
__device__ __forceinline__ void half_reduce(float* v, int ln) {
  if constexpr (NV >= 2) halving_round<NV>(v, ln, 8); else v[0] += __shfl_xor_sync(0xffffffffu, v[0], 8, 16);
  if constexpr (NV >= 4) halving_round<NV / 2>(v, ln, 4); else v[0] += __shfl_xor_sync(0xffffffffu, v[0], 4, 16);
  if constexpr (NV >= 8) halving_round<NV / 4>(v, ln, 2); else v[0] += __shfl_xor_sync(0xffffffffu, v[0], 2, 16);
  if constexpr (NV >= 16) halving_round<NV / 8>(v, ln, 1); else v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1, 16);
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

// ---- PREP ------------------------------------------------------------------
template <int G, bool DENSE>
__device__ void fz_prep(const FzParams& p, const FzShared& s, const Unit& x, int d, int s0) {
  const Dims& dm = p.dm;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float* qf = reinterpret_cast<float*>(s.work);               // [G][128]
  unsigned* qc = reinterpret_cast<unsigned*>(s.work + 4096);  // [G][8] 32-bit code words
  const __nv_bfloat16* qb = reinterpret_cast<const __nv_bfloat16*>(s.qbuf + d * FZ_QBUF);
  for (int i = tid; i < G * D; i += FZ_CONS) qf[i] = __bfloat162float(qb[i]);
  if (tid < G * 8) qc[tid] = 0u;
  cons_sync();
  // lane owns channels 4l .. 4l+3
  float qv[G][4];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float4 t = *reinterpret_cast<const float4*>(qf + g * D + 4 * lane);
    qv[g][0] = t.x; qv[g][1] = t.y; qv[g][2] = t.z; qv[g][3] = t.w;
  }
  // q'_i = sum_j R_h[i][j] q_j: warp w takes rows 16w .. 16w+15
  for (int r = 0; r < 16; ++r) {
    const int i = warp * 16 + r;
    const float4 rr = *reinterpret_cast<const float4*>(
        s.ring + (size_t)((s0 + i / 32) % FZ_NSLOT) * FZ_SLOT + (i % 32) * 512 + lane * 16);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float a = rr.x * qv[g][0];
      a = fmaf(rr.y, qv[g][1], a);
      a = fmaf(rr.z, qv[g][2], a);
      a = fmaf(rr.w, qv[g][3], a);
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
      if (lane == g) {
        const long long idx = ((long long)x.b * dm.Hq + x.h * G + g) * D + i;
        p.wk.qrot[idx] = a;
        if (p.dbg.q_rot) p.dbg.q_rot[idx] = a;
      }
    }
  }
  if constexpr (DENSE) return;  // full attention needs no codes (and has no W_h)
  // query codes: bit j = [ (W_h q)_j > 0 ]; products of bf16 values are exact
  // in fp32; the 128-term fp32 sum errs by at most 127 * 2^-24 * sum|w q|, so
  // below 2^-14 * sum|w q| the sign is taken from an fp64 recompute
  const int bits_per_warp = dm.nb / (FZ_CONS / 32);
  for (int r = 0; r < bits_per_warp; ++r) {
    const int j = warp * bits_per_warp + r;
    const int ws = 4 + j / 64;
    const uint2 wv = *reinterpret_cast<const uint2*>(s.ring + (size_t)((s0 + ws) % FZ_NSLOT) * FZ_SLOT +
                                                     (j % 64) * 256 + lane * 8);
    const float w4[4] = {bf_lo(wv.x), bf_hi(wv.x), bf_lo(wv.y), bf_hi(wv.y)};
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float a = 0.f, m = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float pe = w4[e] * qv[g][e];
        a += pe;
        m += fabsf(pe);
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) {
        a += __shfl_xor_sync(0xffffffffu, a, o);
        m += __shfl_xor_sync(0xffffffffu, m, o);
      }
      bool bit = a > 0.f;
      if (fabsf(a) <= ldexpf(m, -14)) {
        double ad = 0.0;
#pragma unroll
        for (int e = 0; e < 4; ++e) ad += (double)w4[e] * (double)qv[g][e];
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) ad += __shfl_xor_sync(0xffffffffu, ad, o);
        bit = ad > 0.0;
      }
      if (lane == 0 && bit) atomicOr(&qc[g * 8 + j / 32], 1u << (j % 32));
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
}

// ---- SCAN ------------------------------------------------------------------
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
  constexpr int HSH = GP == 4 ? 2 : 1;  // lane -> head index shift after the reduction
  const int hidx = ln >> HSH;
  for (int r = 0; r < 8; ++r) {
    const int j = hw + 16 * r;  // page within the chunk
    const size_t off = (size_t)(j % 64) * 256 + ln * 16;
    const uint4 mnv = *reinterpret_cast<const uint4*>(s.ring + (size_t)((s0 + j / 64) % FZ_NSLOT) * FZ_SLOT + off);
    const uint4 mxv = *reinterpret_cast<const uint4*>(s.ring + (size_t)((s0 + 2 + j / 64) % FZ_NSLOT) * FZ_SLOT + off);
    const uint32_t mw[4] = {mnv.x, mnv.y, mnv.z, mnv.w};
    const uint32_t xw[4] = {mxv.x, mxv.y, mxv.z, mxv.w};
    float a[GP];
#pragma unroll
    for (int g = 0; g < G; ++g) {
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
      a[g] = acc.x + acc.y;
    }
#pragma unroll
    for (int g = G; g < GP; ++g) a[g] = 0.f;
    half_reduce<GP>(a, ln);
    // lane holds the bound of head hidx; U = max over the real heads
    float U = hidx < G ? a[0] : -INFINITY;
#pragma unroll
    for (int o = 16 >> (4 - HSH); o <= 8; o <<= 1) U = fmaxf(U, __shfl_xor_sync(0xffffffffu, U, o, 16));
    if (j < n) {
      const int pg = c * FZ_ROWS + j;
      if (ln == 0) {
        p.wk.U[(long long)x.u * dm.np_max + pg] = U;
        if (p.dbg.page_U) p.dbg.page_U[(long long)x.u * dm.np_max + pg] = U;
      }
      if (p.dbg.page_ub && hidx < G && (ln & ((1 << HSH) - 1)) == 0)
        p.dbg.page_ub[((long long)x.b * dm.Hq + x.h * G + hidx) * dm.np_max + pg] = a[0];
    }
  }
}

// ---- SELECT: page top-N, Hamming scores, key top-k -------------------------
template <int G, int WORDS>
__device__ void fz_select(const FzParams& p, const FzShared& s, const Unit& x) {
  const Dims& dm = p.dm;
  const Work& wk = p.wk;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int* spage = reinterpret_cast<int*>(s.work);                          // [<= 2048]
  unsigned short* sc = reinterpret_cast<unsigned short*>(s.work + 8192);  // [<= 16384]
  int* hist = reinterpret_cast<int*>(s.work + 8192 + 32768);             // [<= 2049 + pad]
  int* red = reinterpret_cast<int*>(s.work + 8192 + 32768 + 8448);       // [40]
  int* bc = red + 36;
  const int np = x.np;
  const int N = min(min(max(__ldg(p.n_keep + x.b), 1), wk.Nmax), np);
  int* gsel = wk.sel_pages + (long long)x.u * wk.Nmax;
  int* dsel = p.dbg.sel_pages ? p.dbg.sel_pages + (long long)x.u * wk.Nmax : nullptr;

  // ---- page top-N: exact radix select on order-preserving keys (11, 11, 10 bits) ----
  if (N >= np) {
    for (int i = tid; i < np; i += FZ_CONS) {
      spage[i] = i;
      gsel[i] = i;
      if (dsel) dsel[i] = i;
    }
  } else {
    constexpr int KPT = MAX_SELECT_PAGES / FZ_CONS;  // 64
    const int kpt = (np + FZ_CONS - 1) / FZ_CONS;
    const float* U = wk.U + (long long)x.u * dm.np_max;
    uint32_t key[KPT];
#pragma unroll
    for (int i = 0; i < KPT; ++i) {
      const int idx = tid * kpt + i;
      key[i] = (i < kpt && idx < np) ? order_key(__ldcg(U + idx)) : 0u;
    }
    uint32_t prefix = 0u, pmask = 0u;
    int need = N;
    const int shifts[3] = {21, 10, 0};
    const int widths[3] = {11, 11, 10};
#pragma unroll 1
    for (int ps = 0; ps < 3; ++ps) {
      const int shift = shifts[ps];
      const int nbins = 1 << widths[ps];
      const uint32_t dmask = (uint32_t)nbins - 1u;
      for (int i = tid; i < nbins; i += FZ_CONS) hist[i] = 0;
      cons_sync();
#pragma unroll
      for (int i = 0; i < KPT; ++i) {
        if (i < kpt) {
          const int idx = tid * kpt + i;
          const bool m = idx < np && (key[i] & pmask) == prefix;
          if (__any_sync(0xffffffffu, m)) {
            const unsigned dg = (key[i] >> shift) & dmask;
            const unsigned bin = m ? dg : (0x10000u | lane);
            const unsigned peers = __match_any_sync(0xffffffffu, bin);
            if (m && lane == __ffs(peers) - 1) atomicAdd(&hist[dg], __popc(peers));
          }
        }
      }
      cons_sync();
      // find the digit holding the need-th largest: thread t owns bins from the top
      const int bpt = nbins / FZ_CONS;  // 8 or 4
      int cnt = 0;
      for (int e = 0; e < bpt; ++e) cnt += hist[nbins - 1 - (tid * bpt + e)];
      int tot;
      const int before = cons_excl_scan(cnt, red, &tot);
      if (before < need && before + cnt >= need) {
        int run = before;
        for (int e = 0; e < bpt; ++e) {
          const int bi = nbins - 1 - (tid * bpt + e);
          if (run + hist[bi] >= need) {
            bc[0] = bi;
            bc[1] = need - run;
            break;
          }
          run += hist[bi];
        }
      }
      cons_sync();
      prefix |= (uint32_t)bc[0] << shift;
      pmask |= dmask << shift;
      need = bc[1];
      cons_sync();
    }
    int gt = 0, eq = 0;
#pragma unroll
    for (int i = 0; i < KPT; ++i) {
      const int idx = tid * kpt + i;
      if (i < kpt && idx < np) {
        gt += key[i] > prefix;
        eq += key[i] == prefix;
      }
    }
    int tot;
    const int eq_before = cons_excl_scan(eq, red, &tot);
    const int take_eq = max(0, min(eq, need - eq_before));
    int pos = cons_excl_scan(gt + take_eq, red, &tot);
    int taken = 0;
#pragma unroll
    for (int i = 0; i < KPT; ++i) {
      const int idx = tid * kpt + i;
      if (i < kpt && idx < np) {
        const bool is_eq = key[i] == prefix;
        if (key[i] > prefix || (is_eq && taken < take_eq)) {
          spage[pos] = idx;
          gsel[pos] = idx;
          if (dsel) dsel[pos] = idx;
          ++pos;
          taken += is_eq;
        }
      }
    }
  }
  if (tid == 0 && p.dbg.n_sel_pages) p.dbg.n_sel_pages[x.u] = N;
  // ---- Hamming scores of the kept pages' rows ----
  const int nbins = G * dm.nb + 1;
  for (int i = tid; i < nbins; i += FZ_CONS) hist[i] = 0;
  cons_sync();
  uint64_t* cq = reinterpret_cast<uint64_t*>(s.work + 8192 + 32768 + 8448 + 256);  // [G * WORDS]
  if (tid < G * WORDS) cq[tid] = __ldcg(wk.qcodes + ((long long)x.b * dm.Hq + x.h * G) * WORDS + tid);
  cons_sync();
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
      int S = 0;
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int w2 = 0; w2 < WORDS; ++w2) S += __popcll(cq[g * WORDS + w2] ^ cw[r][w2]);
      if (ci < ncs) {
        sc[ci] = valid[r] ? (unsigned short)S : (unsigned short)0xFFFFu;
        if (dsc) dsc[ci] = valid[r] ? S : INT_MAX;
      }
      const bool v = ci < ncs && valid[r];
      if (__any_sync(0xffffffffu, v)) {
        const unsigned bin = v ? (unsigned)S : (0x10000u | lane);
        const unsigned peers = __match_any_sync(0xffffffffu, bin);
        if (v && lane == __ffs(peers) - 1) atomicAdd(&hist[S], __popc(peers));
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
      const int cnt = bi < nbins ? hist[bi] : 0;
      if (run + cnt >= keff) {
        bc[2] = bi;
        bc[3] = keff - run;
        break;
      }
      run += cnt;
    }
  }
  cons_sync();
  if (keff > 0) {
    const int T = bc[2], need_eq = bc[3];
    const int cpt = (ncs + FZ_CONS - 1) / FZ_CONS;
    int lt = 0, eq = 0;
    for (int i = 0; i < cpt; ++i) {
      const int ci = tid * cpt + i;
      if (ci < ncs) {
        const int v = sc[ci];
        lt += v < T;
        eq += v == T;
      }
    }
    int tot;
    const int eq_before = cons_excl_scan(eq, red, &tot);
    const int take_eq = max(0, min(eq, need_eq - eq_before));
    int pos = cons_excl_scan(lt + take_eq, red, &tot);
    int taken = 0;
    int* out = wk.sel_keys + (long long)x.u * wk.Kmax;
    int* dout = p.dbg.sel_keys ? p.dbg.sel_keys + (long long)x.u * wk.Kmax : nullptr;
    for (int i = 0; i < cpt; ++i) {
      const int ci = tid * cpt + i;
      if (ci < ncs) {
        const int v = sc[ci];
        const bool is_eq = v == T;
        if (v < T || (is_eq && taken < take_eq)) {
          const int slot = ci / dm.P;
          const int t = spage[slot] * dm.P + (ci - slot * dm.P);
          out[pos] = t;
          if (dout) dout[pos] = t;
          ++pos;
          taken += is_eq;
        }
      }
    }
  }
  if (tid == 0) {
    unit_ctrl(p, x.u)[CU_NKEYS] = (unsigned)keff;
    if (p.dbg.n_sel_keys) p.dbg.n_sel_keys[x.u] = keff;
    if (p.dbg.n_cand) p.dbg.n_cand[x.u] = n_cand;
  }
  (void)warp;
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
  const int PS = G * (D + 2);
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
    part[G * D + tid] = mh[0];
#pragma unroll
    for (int gg = 1; gg < G; ++gg)
      if (gg == tid) part[G * D + tid] = mh[gg];
    part[G * D + G + tid] = cs;
  }
}

// Merges K partials src[0 .. K) (stride G (D + 2) floats) in index order:
// M = max m_k, w_k = 2^(m_k - M), L = sum w_k l_k, O = sum w_k o_k.  With
// dst, the merged partial (O, M, L) is written there; otherwise out = O / L.
// K <= 256.  Loads are issued in batches so that a merge costs a few L2
// round trips, not one per partial.
template <int G>
__device__ void fz_merge(const FzShared& s, const float* src, int K, float* dst, float* out) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int PS = G * (D + 2);
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
      lk[i] = (k < K) ? __ldcg(src + (long long)k * PS + G * D + G + g) : 0.f;
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
    dst[G * D + G + tid] = LH[tid];
  }
}

// After a chunk's partial is written: the last chunk of its group of
// FZ_GROUP chunks merges the group (in chunk order) into gpart[u][group];
// the last group of the unit merges the groups (in order) into the output.
constexpr int FZ_GROUP = FUSED_GROUP;

template <int G>
__device__ void fz_gather_done(const FzParams& p, const FzShared& s, const Unit& x, int c) {
  const int tid = threadIdx.x;
  const int PS = G * (D + 2);
  int* bc = reinterpret_cast<int*>(s.work + FZ_WORK - 64);
  const unsigned nk = __ldcg(unit_ctrl(p, x.u) + CU_NKEYS);
  const int nchunks = (int)((nk + FZ_ROWS - 1) / FZ_ROWS);
  const int ngroups = (nchunks + FZ_GROUP - 1) / FZ_GROUP;
  const int grp = c / FZ_GROUP;
  const int gsize = min(FZ_GROUP, nchunks - grp * FZ_GROUP);
  __threadfence();
  cons_sync();
  if (tid == 0) {
    unsigned* gc = p.wk.ctrl + 4 + (p.dm.B * p.dm.Hkv) * CU_STRIDE + x.u * p.wk.max_groups + grp;
    bc[0] = (atomicAdd(gc, 1u) + 1u == (unsigned)gsize) ? 1 : 0;
  }
  cons_sync();
  if (!bc[0]) return;
  __threadfence();
  const float* chunk_parts = p.wk.part + ((long long)x.u * p.wk.C3 + grp * FZ_GROUP) * PS;
  float* gp = p.wk.gpart + ((long long)x.u * p.wk.max_groups + grp) * PS;
  fz_merge<G>(s, chunk_parts, gsize, gp, nullptr);
  __threadfence();
  cons_sync();
  if (tid == 0) bc[1] = (atomicAdd(unit_ctrl(p, x.u) + CU_GATHER, 1u) + 1u == (unsigned)ngroups) ? 1 : 0;
  cons_sync();
  if (!bc[1]) return;
  __threadfence();
  fz_merge<G>(s, p.wk.gpart + (long long)x.u * p.wk.max_groups * PS, ngroups, nullptr,
              p.out + ((long long)x.b * p.dm.Hq + x.h * G) * D);
}

template <int G, int WORDS, bool DENSE>
__device__ void fz_consumer(const FzParams& p, const FzShared& s) {
  const Dims& dm = p.dm;
  const int tid = threadIdx.x, lane = tid & 31;
  const int prep_slots = DENSE ? 4 : 4 + dm.nb / 64;  // R_h, then W_h (not needed without hashing)
  unsigned nslot = 0, ndesc = 0;
  int* dec = reinterpret_cast<int*>(s.work + FZ_WORK - 32);  // wait decisions of thread 0
  while (true) {
    const int d = (int)(ndesc % FZ_NDESC);
    // Thread 0 alone runs the bounded waits and broadcasts the outcome, so all
    // consumer threads leave or continue together (a barrier never strands one).
    if (tid == 0) dec[0] = fz_wait(s, &s.dfull[d], (ndesc / FZ_NDESC) & 1, p.status) ? 1 : 0;
    cons_sync();
    if (!dec[0]) break;
    mbar_confirm(&s.dfull[d], (ndesc / FZ_NDESC) & 1);
    const FzDesc ds = s.desc[d];
    cons_sync();  // everyone holds the descriptor before dec is written again
    if (ds.kind == IT_END) break;
    const int nslots = ds.kind == IT_PREP ? prep_slots : 4;
    const int s0 = (int)(nslot % FZ_NSLOT);
    if (tid == 0) {
      bool ok = true;
      for (int k = 0; k < nslots && ok; ++k) {
        const unsigned gs = nslot + k;
        ok = fz_wait(s, &s.full[gs % FZ_NSLOT], (gs / FZ_NSLOT) & 1, p.status);
      }
      dec[1] = ok ? 1 : 0;
    }
    cons_sync();
    if (!dec[1]) break;
    for (int k = 0; k < nslots; ++k) {
      const unsigned gs = nslot + k;
      mbar_confirm(&s.full[gs % FZ_NSLOT], (gs / FZ_NSLOT) & 1);
    }
    const Unit x = unit_of(p, ds.unit);
    if (ds.kind == IT_PREP) {
      fz_prep<G, DENSE>(p, s, x, d, s0);
    } else if (ds.kind == IT_SCAN) {
      if constexpr (!DENSE) fz_scan<G>(p, s, x, ds.chunk, ds.n, d, s0);
    } else {
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
    // ---- completion of the item ----
    if (ds.kind == IT_PREP) {
      if (x.L == 0) {
        for (int e = tid; e < G * D; e += FZ_CONS)
          p.out[((long long)x.b * dm.Hq + x.h * G) * D + e] = 0.f;
        if (tid == 0) {
          if (p.dbg.n_sel_pages) p.dbg.n_sel_pages[x.u] = 0;
          if (p.dbg.n_sel_keys) p.dbg.n_sel_keys[x.u] = 0;
          if (p.dbg.n_cand) p.dbg.n_cand[x.u] = 0;
        }
      }
      if (tid == 0) unit_ctrl(p, x.u)[CU_NKEYS] = DENSE ? (unsigned)x.L : 0u;
      __threadfence();
      cons_sync();
      if (tid == 0) {
        st_release(unit_ctrl(p, x.u) + CU_PREP, 1u);
        if (DENSE || x.L == 0) st_release(unit_ctrl(p, x.u) + CU_SEL, 1u);
      }
    } else if (ds.kind == IT_GATHER) {
      fz_gather_done<G>(p, s, x, ds.chunk);
    } else if (ds.kind == IT_SCAN) {
      __threadfence();
      cons_sync();
      int* bc = reinterpret_cast<int*>(s.work + FZ_WORK - 64);
      if (tid == 0) {
        const unsigned done = atomicAdd(unit_ctrl(p, x.u) + CU_SCAN, 1u) + 1u;
        const unsigned need = (unsigned)((x.np + FZ_ROWS - 1) / FZ_ROWS);
        bc[0] = done == need;
      }
      cons_sync();
      if (bc[0]) {
        __threadfence();
        if constexpr (!DENSE) fz_select<G, WORDS>(p, s, x);
        __threadfence();
        cons_sync();
        if (tid == 0) st_release(unit_ctrl(p, x.u) + CU_SEL, 1u);
      }
    }
  }
  if (tid == 0) s.misc[1] = (int)nslot;
  (void)DENSE;
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
    for (int i = 0; i < 8; ++i) s.misc[i] = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (tid >= FZ_CONS) {
    fz_producer<G, WORDS, DENSE>(p, s);
  } else {
    fz_consumer<G, WORDS, DENSE>(p, s);
  }
  __syncthreads();
  // drain copies that were issued but never consumed (only after an abort)
  if (tid == 0) {
    const unsigned issued = (unsigned)s.misc[4], consumed = (unsigned)s.misc[1];
    for (unsigned gs = consumed; gs < issued; ++gs) {
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

static FzParams make_params(const DecodeArgs& a) {
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
  return prm;
}

template <int G>
cudaError_t launch_decode(const DecodeArgs& a) {
  FzParams prm = make_params(a);
  const int U = a.dm.B * a.dm.Hkv;
  prm.total_items = U * (1 + a.wk.C1 + a.wk.C3);
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
  FzParams prm = make_params(a);
  const int U = a.dm.B * a.dm.Hkv;
  prm.total_items = U * (1 + a.wk.C3);
  const int grid = std::min(a.num_sms, prm.total_items);
  return launch_fused_t<G, 1, true>(prm, grid, a.stream);
}

#define HHR_INSTANTIATE_DECODE(G)                           \
  template cudaError_t launch_decode<G>(const DecodeArgs&); \
  template cudaError_t launch_dense<G>(const DecodeArgs&);

}  // namespace hhr
