"""Exact ties of page bounds across the top-N threshold, on the GPU.

The page select keeps the N largest bounds U_p and gives equal bounds to the
lower page index (rit.work explainer, section "Два уровня маршрутизации
решают разные ошибки": whole pages are dropped by their bound; the tie rule is
this library's reading).  Random bf16 data never produces two bitwise-equal
bounds, so these tests build caches whose pages repeat:

  dup    whole pages repeated: page j holds the rows of page j mod 8, so U
         takes 8 values, each on many pages;
  zero   every other page is all zeros: their bounds are +0 or -0, which must
         tie with each other (and key codes of zero keys are all 0);
  const  every row of page j is the same vector, one of 5 repeated vectors, so
         min == max on every page and bounds repeat.

N is chosen so that the N-th largest bound sits inside a group of equal
bounds (the test checks that it does), so the kernel must choose among equal
bounds by page index.  Duplicated rows also make equal Hamming scores at the
key threshold.  Every stage is compared with the oracle bit for bit on the
GPU's previous-stage outputs (tests/parity.py).
"""
import numpy as np
import pytest
import torch

from hash_sparse_attention_b200.synth import WORKLOADS, make_layer, scaled, to_pool

pytestmark = pytest.mark.gpu

import parity  # noqa: E402


def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _tie_pattern(K: torch.Tensor, lens, P: int, mode: str, gen: torch.Generator) -> torch.Tensor:
    """Rewrites the logical K [B, Hkv, T, d] so that page bounds tie exactly."""
    K = K.clone()
    B, H, T, d = K.shape
    for b, L in enumerate(lens):
        npg = -(-L // P)
        for j in range(npg):
            t0, t1 = j * P, min((j + 1) * P, L)
            if mode == "dup":
                src = (j % 8) * P
                if j >= 8 and src + (t1 - t0) <= L:
                    K[b, :, t0:t1] = K[b, :, src:src + (t1 - t0)]
            elif mode == "zero":
                if j % 2 == 1:
                    K[b, :, t0:t1] = 0
            elif mode == "const":
                v = K[b, :, (j % 5) * P]  # [H, d]: row 0 of page j mod 5 (taken before it is rewritten)
                K[b, :, t0:t1] = v[:, None, :]
            else:
                raise ValueError(mode)
        if L < T:
            K[b, :, L:] = 0
    return K


def _layer(G: int, P: int, mode: str, paged: bool, seed: int):
    w = scaled(WORKLOADS["tiny_4k"], num_q_heads=2 * G, num_kv_heads=2, hash_bits=128, page_size=P,
               context=2048, batch=2, keep_pages=None, keep_den=8, top_k=None, topk_den=10, seed=seed,
               paged=paged, ragged_min=1500 if paged else None)
    li = make_layer(w)
    gen = torch.Generator().manual_seed(seed)
    if paged:
        lens = [int(x) for x in li.seq_lens]
        Klog = _tie_pattern(li.K_logical, lens, P, mode, gen)
        li.K_logical = Klog
        li.K = to_pool(Klog, li.block_table, lens, P, li.K.shape[0])
    else:
        li.K = _tie_pattern(li.K, [int(x) for x in li.seq_lens], P, mode, gen)
    return w, li


def _budgets_across_ties(w, li, rng):
    """Runs once with debug outputs to read U, then picks per sequence an N
    whose N-th largest bound lies strictly inside a group of equal bounds, and
    a k that cuts through equal Hamming scores where the candidates allow it."""
    g = parity.run_gpu(w, li, n_keep=torch.full((w.batch,), 10**6, dtype=torch.int32),
                       top_k=torch.full((w.batch,), 10**6, dtype=torch.int32),
                       max_keep=-(-w.context // w.page_size), max_topk=w.context)
    assert g.status == 0
    n_keep, top_k = [], []
    for b, L in enumerate(g.lens):
        npg = -(-L // w.page_size)
        U = g.dbg["page_U"][b, 0, :npg].astype(np.float64)
        vals, counts = np.unique(U, return_counts=True)  # -0 and +0 count as one value
        order = np.argsort(-vals)
        vals, counts = vals[order], counts[order]
        above = np.concatenate([[0], np.cumsum(counts)[:-1]])
        tied = [i for i in range(len(vals)) if counts[i] >= 3 and above[i] >= 1]
        assert tied, "no group of equal bounds below the top: the pattern did not make ties"
        i = tied[int(rng.integers(len(tied)))]
        N = int(above[i] + 1 + rng.integers(counts[i] - 1))  # strictly inside the group
        n_keep.append(N)
        top_k.append(max(1, (N * w.page_size) // 2 + 1))
    return (torch.tensor(n_keep, dtype=torch.int32), torch.tensor(top_k, dtype=torch.int32))


def _check_cut_inside_ties(g, w, n_keep):
    for b, L in enumerate(g.lens):
        npg = -(-L // w.page_size)
        N = int(n_keep[b])
        for h in range(w.num_kv_heads):
            U = g.dbg["page_U"][b, h, :npg].astype(np.float64)
            thr = np.sort(U)[::-1][N - 1]
            n_gt, n_ge = int((U > thr).sum()), int((U >= thr).sum())
            if h == 0:  # budgets were chosen on head 0
                assert n_gt < N < n_ge, "the N-th bound is not inside a tie group"


@pytest.mark.parametrize("G,P,mode,paged", [
    (1, 16, "dup", False), (4, 16, "dup", False), (7, 32, "dup", False),
    (1, 32, "zero", False), (4, 16, "zero", False), (7, 16, "zero", False),
    (4, 32, "const", False), (7, 16, "const", False), (1, 16, "const", False),
    (4, 16, "dup", True), (4, 32, "zero", True),
])
def test_page_bound_ties_select_lower_pages(G, P, mode, paged):
    _cuda()
    w, li = _layer(G, P, mode, paged, seed=100 + 7 * G + P)
    rng = np.random.default_rng(G * 1000 + P)
    n_keep, top_k = _budgets_across_ties(w, li, rng)
    li.n_keep, li.top_k = n_keep, top_k
    g = parity.run_gpu(w, li, n_keep=n_keep, top_k=top_k)
    assert g.status == 0
    _check_cut_inside_ties(g, w, n_keep)
    rep = parity.Report()
    parity.check_build(w, li, g, rep)
    # stage-wise: sel_pages == oracle select on the GPU's bounds (ties -> lower page),
    # sel_keys == oracle select on the GPU's scores (ties -> lower token)
    parity.check_decode(w, li, g, rep, e2e=True)
    print(rep)
