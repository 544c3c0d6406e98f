"""Runs the CUDA path through the C ABI and compares every stage with the oracle.

Stage-wise parity: each stage's oracle consumes the GPU's output of the
previous stage (exported through hhr_debug), so integer and index stages are
compared bit for bit on identical inputs.  Float stages are compared with the
fp64 oracle within the tolerances below.  End-to-end: the oracle runs its own
pipeline from the raw inputs; index differences are counted, outputs compared
within tolerance where the selections agree.

Tolerances and exemptions:
  * attention output: per query head max|o - o^| / max|o^| <= 2e-3
  * page bounds: |ub - ub^| <= 2e-3 * sum_i |q'_i| max(|mn_i|, |mx_i|)
  * K': equal, bit for bit, to the oracle's bf16_rne(R_h k)
  * a hash bit is exempt when |fp64 projection| < 1e-5 |x|; a page is exempt
    when |U_p - thr| <= 1e-4 |thr| (thr = the N-th largest fp64 bound)
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

from hash_sparse_attention_b200 import hhr
from hash_sparse_attention_b200.synth import LayerInputs, Workload, from_pool
from oracle import hhr_oracle as O

OUT_RTOL = 2e-3
BOUND_RTOL = 2e-3
HASH_EXEMPT = 1e-5
PAGE_EXEMPT = 1e-4
INT32_MAX = 2**31 - 1


def config_for(w: Workload, li: LayerInputs) -> hhr.HHRConfig:
    if w.paged:
        return hhr.make_config(w.batch, w.num_q_heads, w.num_kv_heads, w.page_size, w.hash_bits, w.context,
                               paged=True, num_blocks=li.K.shape[0], max_blocks_per_seq=li.block_table.shape[1],
                               page_agg=w.page_agg, key_agg=w.key_agg)
    return hhr.make_config(w.batch, w.num_q_heads, w.num_kv_heads, w.page_size, w.hash_bits, w.context,
                           page_agg=w.page_agg, key_agg=w.key_agg)


@dataclass
class GpuRun:
    cfg: object
    lens: list
    Krot: np.ndarray       # logical [B, Hkv, T, d] float64
    V: np.ndarray
    pmin: np.ndarray       # logical [B, Hkv, np_max, d]
    pmax: np.ndarray
    codes: np.ndarray      # logical uint64 [B, Hkv, T, w]
    out: np.ndarray
    dbg: dict
    status: int
    Nmax: int
    Kmax: int
    extra: dict = field(default_factory=dict)


def _logical_meta(pool_meta: torch.Tensor, table: torch.Tensor, lens, P, np_max):
    B = table.shape[0]
    out = torch.zeros(B, pool_meta.shape[1], np_max, pool_meta.shape[2], dtype=pool_meta.dtype,
                      device=pool_meta.device)
    for b, L in enumerate(lens):
        n = -(-L // P)
        if n:
            out[b, :, :n] = pool_meta[table[b, :n].long()].permute(1, 0, 2)
    return out


def run_gpu(w: Workload, li: LayerInputs, max_keep: int | None = None, max_topk: int | None = None,
            n_keep: torch.Tensor | None = None, top_k: torch.Tensor | None = None, with_dbg: bool = True,
            dense: bool = False, to_host: bool = True) -> GpuRun:
    dev = torch.device("cuda")
    mv = lambda t: None if t is None else t.to(dev)  # noqa: E731
    K, V, q, R, W = mv(li.K), mv(li.V), mv(li.q), mv(li.R), mv(li.W)
    seq = mv(li.seq_lens)
    table = mv(li.block_table)
    n_keep = mv(n_keep if n_keep is not None else li.n_keep)
    top_k = mv(top_k if top_k is not None else li.top_k)
    lens = [int(x) for x in li.seq_lens.cpu()]
    cfg = config_for(w, li)
    P = w.page_size
    np_max = -(-w.context // P)
    Nmax = max_keep if max_keep is not None else int(n_keep.max())
    Kmax = max_topk if max_topk is not None else int(top_k.max())
    cache = hhr.alloc_cache(cfg, dev)
    hhr.build_cache(cfg, K, V, R, W, seq, table, cache)
    out = torch.full((w.batch, w.num_q_heads, w.head_dim), float("nan"), device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    dbg = hhr.alloc_debug(cfg, Nmax, Kmax, dev) if with_dbg else None
    if dense:
        ws = hhr.dense_workspace(cfg, dev)
        hhr.dense_decode(cfg, q, R, cache, seq, table, out, ws, status=status)
    else:
        ws = hhr.decode_workspace(cfg, Nmax, Kmax, dev)
        hhr.decode_step(cfg, q, R, W, cache, seq, table, n_keep, top_k, Nmax, Kmax, out, ws, dbg=dbg,
                        status=status)
    torch.cuda.synchronize()
    if not to_host:
        return GpuRun(cfg, lens, None, None, None, None, None, out, {}, int(status.item()), Nmax, Kmax,
                      extra=dict(cache=cache, ws=ws, dbg=dbg))
    if w.paged:
        Kr = from_pool(cache.Krot, table, lens, w.context)
        Vl = from_pool(cache.V, table, lens, w.context)
        cd = from_pool(cache.codes, table, lens, w.context)
        pmn = _logical_meta(cache.page_min, table, lens, P, np_max)
        pmx = _logical_meta(cache.page_max, table, lens, P, np_max)
    else:
        Kr, Vl, cd, pmn, pmx = cache.Krot, cache.V, cache.codes, cache.page_min, cache.page_max
    d = {}
    if dbg is not None:
        for name in ("q_rot", "page_ub", "page_U", "sel_pages", "n_sel_pages", "q_codes", "key_scores",
                     "n_cand", "sel_keys", "n_sel_keys"):
            t = getattr(dbg, name).cpu()
            d[name] = t.numpy().view(np.uint64) if name == "q_codes" else t.numpy()
    return GpuRun(cfg, lens, Kr.double().cpu().numpy(), Vl.double().cpu().numpy(), pmn.double().cpu().numpy(),
                  pmx.double().cpu().numpy(), cd.cpu().numpy().view(np.uint64), out.cpu().numpy().astype(np.float64),
                  d, int(status.item()), Nmax, Kmax)


def rel_err(a: np.ndarray, ref: np.ndarray) -> float:
    den = np.abs(ref).max()
    return float(np.abs(a - ref).max() / den) if den > 0 else float(np.abs(a).max())


@dataclass
class Report:
    kprime_flips: int = 0
    kprime_elems: int = 0
    code_exempt_bits: int = 0
    code_exempt_mismatch: int = 0
    qcode_exempt_bits: int = 0
    qcode_exempt_mismatch: int = 0
    page_exempt_diff: int = 0
    e2e_page_diff: int = 0
    e2e_key_diff: int = 0
    max_out_err: float = 0.0
    max_e2e_err: float = 0.0
    max_bound_err: float = 0.0
    max_qrot_err: float = 0.0
    heads: int = 0


def check_build(w: Workload, li: LayerInputs, g: GpuRun, rep: Report, heads=None) -> None:
    Klog = (li.K_logical if w.paged else li.K).double().cpu().numpy()
    Wn = li.W.double().cpu().numpy()
    R32 = li.R.double().cpu().numpy()
    P = w.page_size
    for b, L in enumerate(g.lens):
        for h in (heads if heads is not None else range(w.num_kv_heads)):
            if L == 0:
                continue
            Kx = Klog[b, h, :L]
            Kp_ref = O.rotate_keys_stored(R32[h], Kx)
            Kp = g.Krot[b, h, :L]
            diff = Kp != Kp_ref
            rep.kprime_flips += int(diff.sum())
            rep.kprime_elems += diff.size
            # the build rounds the exact product once (elements near a rounding
            # midpoint are recomputed in fp64), so K' equals the oracle's bit for bit
            assert np.array_equal(Kp, Kp_ref), f"K' differs from bf16_rne(R_h k) in {int(diff.sum())} elements"
            # page metadata: stage-wise on the GPU's stored K'
            mn, mx = O.page_minmax(Kp, L, P)
            n = mn.shape[0]
            assert np.array_equal(g.pmin[b, h, :n], mn), f"page_min b{b} h{h}"
            assert np.array_equal(g.pmax[b, h, :n], mx), f"page_max b{b} h{h}"
            # key codes: bit-exact outside the exempt band
            proj = O.hash_projection(Wn[h], Kx)
            ref = O.hash_codes(Wn[h], Kx)
            got = g.codes[b, h, :L]
            mism = _bits(np.bitwise_xor(got, ref), w.hash_bits)
            exempt = np.abs(proj) < HASH_EXEMPT * np.linalg.norm(Kx, axis=1)[:, None]
            assert not np.any(mism & ~exempt), f"key code mismatch outside the exempt band b{b} h{h}"
            rep.code_exempt_bits += int(exempt.sum())
            rep.code_exempt_mismatch += int((mism & exempt).sum())


def _bits(words: np.ndarray, nb: int) -> np.ndarray:
    n = words.shape[0]
    out = np.zeros((n, nb), dtype=bool)
    for j in range(nb):
        out[:, j] = ((words[:, j // 64] >> np.uint64(j % 64)) & np.uint64(1)).astype(bool)
    return out


def check_decode(w: Workload, li: LayerInputs, g: GpuRun, rep: Report, heads=None, e2e: bool = True,
                 scale: float | None = None) -> None:
    G, P, d = w.group, w.page_size, w.head_dim
    scale = scale if scale is not None else 1.0 / math.sqrt(d)
    R32 = li.R.double().cpu().numpy()
    Wn = li.W.double().cpu().numpy()
    qn = li.q.double().cpu().numpy()
    Klog = (li.K_logical if w.paged else li.K).double().cpu().numpy() if e2e else None
    Vlog = (li.V_logical if w.paged else li.V).double().cpu().numpy() if e2e else None
    nk = li.n_keep.cpu().numpy()
    tk = li.top_k.cpu().numpy()
    dg = g.dbg
    for b, L in enumerate(g.lens):
        N = min(max(int(nk[b]), 1), g.Nmax)
        k = min(max(int(tk[b]), 1), g.Kmax)
        for h in (heads if heads is not None else range(w.num_kv_heads)):
            rep.heads += 1
            hq = slice(h * G, (h + 1) * G)
            Q = qn[b, hq]
            Qr = O.rotate_query(R32[h], Q)
            rep.max_qrot_err = max(rep.max_qrot_err, rel_err(dg["q_rot"][b, hq], Qr))
            assert rep.max_qrot_err <= OUT_RTOL
            # query codes
            projq = O.hash_projection(Wn[h], Q)
            cq_ref = O.hash_codes(Wn[h], Q)
            cq = dg["q_codes"][b, hq]
            mism = _bits(np.bitwise_xor(cq, cq_ref), w.hash_bits)
            ex = np.abs(projq) < HASH_EXEMPT * np.linalg.norm(Q, axis=1)[:, None]
            assert not np.any(mism & ~ex), "query code mismatch outside the exempt band"
            rep.qcode_exempt_bits += int(ex.sum())
            rep.qcode_exempt_mismatch += int((mism & ex).sum())
            bh_out = g.out[b, hq]
            if L == 0:
                assert dg["n_sel_pages"][b, h] == 0 and dg["n_sel_keys"][b, h] == 0
                assert np.all(bh_out == 0)
                continue
            np_b = -(-L // P)
            mn, mx = g.pmin[b, h, :np_b], g.pmax[b, h, :np_b]
            ub_ref = O.page_bounds(Qr, mn, mx)
            ub = dg["page_ub"][b, hq, :np_b]
            tol = BOUND_RTOL * (np.abs(Qr)[:, None, :] * np.maximum(np.abs(mn), np.abs(mx))[None]).sum(-1)
            err = np.abs(ub - ub_ref)
            assert np.all(err <= tol), "page bound outside tolerance"
            rep.max_bound_err = max(rep.max_bound_err, float((err / np.maximum(tol / BOUND_RTOL, 1e-300)).max()))
            U = dg["page_U"][b, h, :np_b]
            if w.page_agg == "max":
                assert np.array_equal(U, ub.max(axis=0)), "U is not the group max of ub"
            else:  # fp32 sum of G terms in the kernel's order
                Us = ub.astype(np.float64).sum(axis=0)
                assert np.all(np.abs(U - Us) <= 2.0 ** -21 * G * np.abs(ub).sum(axis=0)), "U is not the group sum of ub"
            # page top-N: bit exact on the GPU's bounds
            Neff = min(N, np_b)
            assert dg["n_sel_pages"][b, h] == Neff
            sel_p = dg["sel_pages"][b, h, :Neff]
            assert np.array_equal(sel_p, O.select_pages(U.astype(np.float64), Neff)), "page select differs"
            # against the fp64 bounds, outside the exempt band
            U64 = O.group_bound(ub_ref, w.page_agg)
            ref_p = O.select_pages(U64, Neff)
            if Neff < np_b:
                thr = np.sort(U64)[::-1][Neff - 1]
                band = PAGE_EXEMPT * abs(thr) if thr > 0 else BOUND_RTOL * float(tol.max())
                sym = np.setxor1d(sel_p, ref_p)
                assert np.all(np.abs(U64[sym] - thr) <= band), "page select differs outside the exempt band"
                rep.page_exempt_diff += len(sym)
            # Hamming on the GPU's codes of the GPU's candidates
            cand = O.candidates(sel_p, L, P)
            S_ref = O.hamming(cq, g.codes[b, h][cand], w.key_agg)
            assert dg["n_cand"][b, h] == len(cand)
            sc = dg["key_scores"][b, h, :Neff * P]
            slot_tok = (sel_p[:, None] * P + np.arange(P)[None]).reshape(-1)
            valid = slot_tok < L
            assert np.array_equal(sc[valid], S_ref), "Hamming scores differ"
            assert np.all(sc[~valid] == INT32_MAX)
            keff = min(k, len(cand))
            assert dg["n_sel_keys"][b, h] == keff
            sel_k = dg["sel_keys"][b, h, :keff]
            assert np.array_equal(sel_k, O.select_keys(S_ref, cand, keff)), "key select differs"
            # attention on the GPU's kept rows of the GPU's cache
            o_ref = O.attention(Qr, g.Krot[b, h], g.V[b, h], sel_k, scale)
            for gg in range(G):
                e = rel_err(bh_out[gg], o_ref[gg])
                rep.max_out_err = max(rep.max_out_err, e)
                assert e <= OUT_RTOL, f"attention output rel err {e:.3g} b{b} h{h} g{gg}"
            if e2e:
                Kp, mn_o, mx_o, codes_o = O.build_head(Klog[b, h], R32[h], Wn[h], L, P)
                r = O.decode_head(Q, R32[h], Wn[h], Kp, Vlog[b, h, :L], mn_o, mx_o, codes_o, L, P, N, k, scale,
                                  page_agg=w.page_agg, key_agg=w.key_agg)
                dp = len(np.setxor1d(r["sel_pages"], sel_p))
                dk = len(np.setxor1d(r["sel_keys"], sel_k))
                rep.e2e_page_diff += dp
                rep.e2e_key_diff += dk
                if dp == 0 and dk == 0:
                    for gg in range(G):
                        e = rel_err(bh_out[gg], r["out"][gg])
                        rep.max_e2e_err = max(rep.max_e2e_err, e)
                        assert e <= OUT_RTOL, f"end-to-end rel err {e:.3g}"


def check_dense(w: Workload, li: LayerInputs, g: GpuRun, scale: float | None = None) -> float:
    G, d = w.group, w.head_dim
    scale = scale if scale is not None else 1.0 / math.sqrt(d)
    R32 = li.R.double().cpu().numpy()
    qn = li.q.double().cpu().numpy()
    worst = 0.0
    for b, L in enumerate(g.lens):
        for h in range(w.num_kv_heads):
            hq = slice(h * G, (h + 1) * G)
            o_ref = O.dense_head(qn[b, hq], R32[h], g.Krot[b, h, :L], g.V[b, h, :L], L, scale)
            for gg in range(G):
                e = rel_err(g.out[b, hq][gg], o_ref[gg]) if L else float(np.abs(g.out[b, hq][gg]).max())
                worst = max(worst, e)
    return worst
