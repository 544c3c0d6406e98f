"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Sizes: the tiny 4K workload and the 32K Llama layer run in full; the GQA-7,
paged and 128K workloads run at full size on sampled heads, in the same
launch configuration as the benchmark; smaller variants span several tiles
and ragged tails; edge cases cover empty, one-row and partial pages,
budgets at and above the candidate count, and every group size 1..8.
"""
import math

import numpy as np
import pytest
import torch

from hash_sparse_attention_b200 import hhr
from hash_sparse_attention_b200.synth import WORKLOADS, make_layer, scaled

pytestmark = pytest.mark.gpu

import parity  # noqa: E402  (tests/ is on sys.path under pytest)


def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _run_and_check(w, li, heads=None, e2e=True, **kw):
    g = parity.run_gpu(w, li, **kw)
    assert g.status == 0
    rep = parity.Report()
    parity.check_build(w, li, g, rep, heads=heads)
    parity.check_decode(w, li, g, rep, heads=heads, e2e=e2e)
    return g, rep


def test_tiny_4k_full():
    _cuda()
    w = WORKLOADS["tiny_4k"]
    li = make_layer(w)
    g, rep = _run_and_check(w, li)
    print(rep)
    assert rep.e2e_key_diff == 0 and rep.e2e_page_diff == 0
    assert rep.max_out_err < 1e-4


def test_llama_layer_32k_full():
    _cuda()
    w = WORKLOADS["llama_layer_32k"]
    li = make_layer(w)
    g, rep = _run_and_check(w, li)
    print(rep)
    assert rep.max_out_err < 1e-4


@pytest.mark.parametrize("ctx", [5000, 20011])
def test_qwen_gqa7_small(ctx):
    _cuda()
    w = scaled(WORKLOADS["qwen_gqa7_128k"], context=ctx, batch=2)
    li = make_layer(w)
    _run_and_check(w, li)


def test_qwen_gqa7_full_sampled():
    _cuda()
    w = WORKLOADS["qwen_gqa7_128k"]
    li = make_layer(w, device="cuda")
    _run_and_check(w, li, heads=[0, 3])


def test_paged_ragged_small():
    _cuda()
    w = scaled(WORKLOADS["paged_b16_ragged"], batch=5, context=4096, ragged_min=1000)
    li = make_layer(w)
    _run_and_check(w, li)


def test_paged_ragged_full_sampled():
    _cuda()
    w = WORKLOADS["paged_b16_ragged"]
    li = make_layer(w, device="cuda")
    _run_and_check(w, li, heads=[2, 7])


@pytest.mark.parametrize("layer", [0, 31])
def test_llama_128k_layer_sampled(layer):
    """The headline workload's per-layer call, full size, two KV heads checked."""
    _cuda()
    w = WORKLOADS["llama_32l_128k"]
    li = make_layer(w, layer=layer, device="cuda")
    _run_and_check(w, li, heads=[1, 6])


def test_llama_128k_keep8_sampled():
    _cuda()
    w = WORKLOADS["llama_32l_128k_keep8"]
    li = make_layer(w, layer=3, device="cuda")
    _run_and_check(w, li, heads=[4])


@pytest.mark.parametrize("G,bits,P", [(1, 64, 16), (2, 128, 32), (3, 256, 16), (4, 64, 32),
                                      (5, 128, 16), (6, 256, 32), (7, 128, 16), (8, 64, 16)])
def test_group_sizes_bits_pages(G, bits, P):
    _cuda()
    w = scaled(WORKLOADS["tiny_4k"], num_q_heads=2 * G, num_kv_heads=2, hash_bits=bits, page_size=P,
               context=3001, keep_pages=None, keep_den=8, top_k=None, topk_den=10, batch=2, seed=G)
    li = make_layer(w)
    _run_and_check(w, li)


def test_edge_lengths_and_budgets():
    """seq_len 0, 1, 15, 16, 17, 33; N above the page count; k above the candidates."""
    _cuda()
    w = scaled(WORKLOADS["tiny_4k"], batch=6, context=64, keep_pages=3, top_k=40, seed=11)
    li = make_layer(w, seq_lens=[0, 1, 15, 16, 17, 33])
    _run_and_check(w, li)
    # budgets above everything: every page and every row is kept
    big = torch.tensor([1000] * 6, dtype=torch.int32)
    _run_and_check(w, li, n_keep=big, top_k=big, max_keep=1000, max_topk=1000)


def test_keep_everything_equals_dense():
    _cuda()
    w = scaled(WORKLOADS["llama_layer_32k"], context=5003, batch=2)
    li = make_layer(w)
    allp = torch.full((2,), 10**6, dtype=torch.int32)
    g = parity.run_gpu(w, li, n_keep=allp, top_k=allp, max_keep=-(-5003 // 16), max_topk=5003)
    gd = parity.run_gpu(w, li, dense=True)
    assert np.allclose(g.out, gd.out, rtol=0, atol=2e-5 * np.abs(gd.out).max())
    assert parity.check_dense(w, li, gd) <= parity.OUT_RTOL


def test_dense_parity_paged():
    _cuda()
    w = scaled(WORKLOADS["paged_b16_ragged"], batch=3, context=3000, ragged_min=500)
    li = make_layer(w)
    gd = parity.run_gpu(w, li, dense=True)
    assert parity.check_dense(w, li, gd) <= parity.OUT_RTOL


def test_paged_equals_contiguous_bitwise():
    _cuda()
    wp = scaled(WORKLOADS["paged_b16_ragged"], batch=3, context=6000, ragged_min=2000, seed=5)
    lp = make_layer(wp)
    wc = scaled(wp, paged=False)
    lc = make_layer(wc, seq_lens=[int(x) for x in lp.seq_lens])
    assert torch.equal(lc.K, lp.K_logical) and torch.equal(lc.V, lp.V_logical)
    gp = parity.run_gpu(wp, lp)
    gc = parity.run_gpu(wc, lc)
    assert np.array_equal(gp.out, gc.out)
    for name in ("sel_pages", "sel_keys", "key_scores", "page_U"):
        assert np.array_equal(gp.dbg[name], gc.dbg[name]), name


def test_batch_independence_and_determinism():
    _cuda()
    w = scaled(WORKLOADS["llama_layer_32k"], context=7000, batch=3)
    li = make_layer(w)
    g1 = parity.run_gpu(w, li)
    g2 = parity.run_gpu(w, li)
    assert np.array_equal(g1.out, g2.out)
    for name in g1.dbg:
        assert np.array_equal(g1.dbg[name], g2.dbg[name]), name
    # sequence 1 alone gives bit-identical results
    w1 = scaled(w, batch=1)
    solo = make_layer(w1)
    for f in ("K", "V", "q"):
        setattr(solo, f, getattr(li, f)[1:2].clone())
    gs = parity.run_gpu(w1, solo)
    # the selections are identical; the attention sum is split over a different
    # number of CTAs per KV head alone than in the batch, so the output agrees
    # to rounding (it is bit-identical for a given batch shape, as above)
    for name in ("sel_pages", "sel_keys", "key_scores", "q_codes"):
        assert np.array_equal(gs.dbg[name][0], g1.dbg[name][1]), name
    assert np.allclose(gs.out[0], g1.out[1], rtol=0, atol=1e-6 * np.abs(g1.out[1]).max())


def test_bad_block_id_sets_status_without_fault():
    _cuda()
    w = scaled(WORKLOADS["paged_b16_ragged"], batch=2, context=512, ragged_min=300, seed=9)
    li = make_layer(w)
    cfg = parity.config_for(w, li)
    dev = torch.device("cuda")
    table = li.block_table.clone()
    table[1, 2] = cfg.num_blocks + 5  # outside the pool: the kernels must skip it and report
    K, V, q, R, W = (t.to(dev) for t in (li.K, li.V, li.q, li.R, li.W))
    seq, tb = li.seq_lens.to(dev), table.to(dev)
    cache = hhr.alloc_cache(cfg, dev)
    hhr.build_cache(cfg, K, V, R, W, seq, tb, cache)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    ws = hhr.decode_workspace(cfg, 64, 64, dev)
    out = torch.zeros(2, w.num_q_heads, 128, device=dev)
    hhr.decode_step(cfg, q, R, W, cache, seq, tb, li.n_keep.to(dev), li.top_k.to(dev), 64, 64, out, ws,
                    status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 6  # HHR_ERR_BAD_BLOCK
    assert torch.isfinite(out).all()


def test_more_units_than_sms():
    """160 (sequence, KV head) units on a grid of at most one CTA per SM: some
    CTA groups decode several units one after another (the shared-memory ring,
    the slot counts and the per-unit counters carry over).  Three calls on one
    workspace (its counters reset by the kernel) give identical results."""
    _cuda()
    w = scaled(WORKLOADS["llama_layer_32k"], context=3000, batch=20, seed=21)
    li = make_layer(w)
    g, rep = _run_and_check(w, li, e2e=False)
    r = parity.run_gpu(w, li, to_host=False)
    assert r.status == 0
    cache, ws = r.extra["cache"], r.extra["ws"]
    dev = torch.device("cuda")
    q, R, W = li.q.to(dev), li.R.to(dev), li.W.to(dev)
    seq, nk, tk = li.seq_lens.to(dev), li.n_keep.to(dev), li.top_k.to(dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    for _ in range(2):
        out = torch.full_like(r.out, float("nan"))
        hhr.decode_step(r.cfg, q, R, W, cache, seq, None, nk, tk, r.Nmax, r.Kmax, out, ws, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.equal(out, r.out)
    assert np.array_equal(g.out, r.out.cpu().numpy().astype(np.float64))


def test_bounded_wait_runs_out_and_reports_timeout():
    """A device-side wait that runs out ends the launch with HHR_ERR_TIMEOUT in
    the status word (no trap, no hang); after the workspace is zeroed again the
    next call is bit-identical to a clean run.  The wait limit is cut to a few
    hundred SM cycles, far below the skew between the CTAs of a group, so the
    group barriers of this 8-unit layer (18 CTAs per KV head) run out."""
    _cuda()
    from hash_sparse_attention_b200 import _lib
    w = scaled(WORKLOADS["llama_layer_32k"], context=8192, batch=1, seed=33)
    li = make_layer(w)
    clean = parity.run_gpu(w, li, to_host=False)
    assert clean.status == 0
    cache, ws = clean.extra["cache"], clean.extra["ws"]
    dev = torch.device("cuda")
    q, R, W = li.q.to(dev), li.R.to(dev), li.W.to(dev)
    seq, nk, tk = li.seq_lens.to(dev), li.n_keep.to(dev), li.top_k.to(dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    out = torch.zeros_like(clean.out)
    L = _lib.lib()
    try:
        L.hhr_set_wait_limit(300)
        hhr.decode_step(clean.cfg, q, R, W, cache, seq, None, nk, tk, clean.Nmax, clean.Kmax, out, ws, status=status)
        torch.cuda.synchronize()
    finally:
        L.hhr_set_wait_limit(0)
    assert int(status.item()) == _lib.HHR_ERR_TIMEOUT
    # the context is usable; zero the workspace again, then a clean call
    ws.zero_()
    status.zero_()
    out2 = torch.full_like(clean.out, float("nan"))
    hhr.decode_step(clean.cfg, q, R, W, cache, seq, None, nk, tk, clean.Nmax, clean.Kmax, out2, ws, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(out2, clean.out)


@pytest.mark.parametrize("bits", [64, 128, 256])
def test_orthogonal_hash_projection(bits):
    """The random-orthogonal-projection hash (paper page, Figure 2 caption) at
    each code width (Figure 10's bit sweep): the same kernels, another W."""
    _cuda()
    w = scaled(WORKLOADS["llama_layer_32k"], context=6000, batch=2, hash_bits=bits, hash_law="orthogonal",
               seed=90 + bits)
    li = make_layer(w)
    _run_and_check(w, li)


@pytest.mark.parametrize("G,page_agg,key_agg", [(4, "sum", "sum"), (4, "max", "min"), (7, "sum", "min"),
                                                (1, "sum", "min"), (8, "sum", "sum")])
def test_group_aggregation_modes(G, page_agg, key_agg):
    """The alternatives to the library's readings for grouped query heads: the
    page bound summed over the group, the Hamming distance of the closest head."""
    _cuda()
    w = scaled(WORKLOADS["llama_layer_32k"], num_q_heads=2 * G, num_kv_heads=2, context=5000, batch=2,
               page_agg=page_agg, key_agg=key_agg, seed=100 + G)
    li = make_layer(w)
    _run_and_check(w, li)


def test_build_exact_when_the_rotation_split_is_inexact():
    """K' stays the correctly rounded product when some entries of R_h are
    fp32 subnormals, whose three bf16 terms do not add back to them: the
    build's exact recompute then reads R_h from global memory instead of its
    staged terms.  Other heads keep the staged path."""
    _cuda()
    w = scaled(WORKLOADS["llama_layer_32k"], context=3000, batch=1, seed=77)
    li = make_layer(w)
    R = li.R.clone()
    R[0, 3, 7] = 1.0e-39   # subnormal: its bf16 split is inexact
    R[0, 90, 11] = -3.3e-40
    li.R = R
    _run_and_check(w, li, e2e=False)
