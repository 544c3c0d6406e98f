"""hhr_append_cache: growing the cache token by token gives, bit for bit, the
cache a full build produces (rit.work explainer, section "Когда HHR меняет
планы запуска модели": the page bounds are stored with the cache, so every
generated key must update its page).

Each case builds the cache over initial lengths, then appends rows (one at a
time, or several per call) across page boundaries, and compares K', V, the
page min/max and the codes with hhr_build_cache over the final lengths, then
checks the appended cache against the fp64 oracle (tests/parity.py).
"""
import numpy as np
import pytest
import torch

from hash_sparse_attention_b200 import hhr
from hash_sparse_attention_b200.synth import WORKLOADS, from_pool, make_layer, scaled

pytestmark = pytest.mark.gpu

import parity  # noqa: E402


def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _logical(w, tb, cache, lens):
    if not w.paged:
        return cache.Krot, cache.V, cache.codes, cache.page_min, cache.page_max
    np_max = -(-w.context // w.page_size)
    return (from_pool(cache.Krot, tb, lens, w.context), from_pool(cache.V, tb, lens, w.context),
            from_pool(cache.codes, tb, lens, w.context),
            parity._logical_meta(cache.page_min, tb, lens, w.page_size, np_max),
            parity._logical_meta(cache.page_max, tb, lens, w.page_size, np_max))


@pytest.mark.parametrize("P,paged,step", [(16, False, 1), (32, False, 1), (16, True, 1), (16, False, 5),
                                          (32, True, 3)])
def test_append_equals_full_build(P, paged, step):
    _cuda()
    dev = torch.device("cuda")
    final = [1040, 777, 64]
    grow = 40
    w = scaled(WORKLOADS["llama_layer_32k"], batch=3, context=1100, page_size=P, num_q_heads=8, num_kv_heads=2,
               paged=paged, ragged_min=None, seed=61 + P)
    li = make_layer(w, seq_lens=final)
    cfg = parity.config_for(w, li)
    K, V, R, W = (t.to(dev) for t in (li.K, li.V, li.R, li.W))
    tb = None if li.block_table is None else li.block_table.to(dev)
    # reference: one build over the final lengths
    ref = hhr.alloc_cache(cfg, dev)
    hhr.build_cache(cfg, K, V, R, W, torch.tensor(final, dtype=torch.int32, device=dev), tb, ref)
    # build over the initial lengths, then append `step` rows per call
    start = [max(0, L - grow) for L in final]
    cache = hhr.alloc_cache(cfg, dev)
    hhr.build_cache(cfg, K, V, R, W, torch.tensor(start, dtype=torch.int32, device=dev), tb, cache)
    cur = list(start)
    while cur != final:
        nxt = [min(L, c + step) for c, L in zip(cur, final)]
        hhr.append_cache(cfg, K, V, R, W, torch.tensor(cur, dtype=torch.int32, device=dev),
                         torch.tensor(nxt, dtype=torch.int32, device=dev), step, tb, cache)
        cur = nxt
    torch.cuda.synchronize()
    got = _logical(w, tb, cache, final)
    exp = _logical(w, tb, ref, final)
    for b, L in enumerate(final):
        npg = -(-L // P)
        for name, g, e in zip(("K'", "V", "codes", "page_min", "page_max"), got, exp):
            n = npg if name.startswith("page") else L
            assert torch.equal(g[b, :, :n].cpu(), e[b, :, :n].cpu()), f"{name} differs, sequence {b}"
    # and the appended cache against the oracle's build
    gr = parity.GpuRun(cfg, final, *[t.double().cpu().numpy() for t in got[:2]],
                       got[3].double().cpu().numpy(), got[4].double().cpu().numpy(),
                       got[2].cpu().numpy().view(np.uint64), None, {}, 0, 1, 1)
    rep = parity.Report()
    parity.check_build(w, li, gr, rep)
    assert rep.kprime_elems > 0


def test_append_in_place_key_rows():
    """K may alias Krot: the raw key of the new token is written into the
    cache's own row, then appended (only rows >= old_lens are read)."""
    _cuda()
    dev = torch.device("cuda")
    w = scaled(WORKLOADS["tiny_4k"], context=300, batch=1, seed=71)
    final = [300]
    li = make_layer(w, seq_lens=final)
    cfg = parity.config_for(w, li)
    K, V, R, W = (t.to(dev) for t in (li.K, li.V, li.R, li.W))
    ref = hhr.alloc_cache(cfg, dev)
    hhr.build_cache(cfg, K, V, R, W, torch.tensor(final, dtype=torch.int32, device=dev), None, ref)
    Kc, Vc = K.clone(), V.clone()
    cache = hhr.alloc_cache(cfg, dev, Krot=Kc, V=Vc)
    hhr.build_cache(cfg, Kc, Vc, R, W, torch.tensor([290], dtype=torch.int32, device=dev), None, cache)
    for t in range(290, 300):
        Kc[:, :, t] = K[:, :, t]  # the new token's raw key lands in its cache row
        hhr.append_cache(cfg, Kc, Vc, R, W, torch.tensor([t], dtype=torch.int32, device=dev),
                         torch.tensor([t + 1], dtype=torch.int32, device=dev), 1, None, cache)
    torch.cuda.synchronize()
    assert torch.equal(cache.Krot[:, :, :300], ref.Krot[:, :, :300])
    assert torch.equal(cache.codes[:, :, :300], ref.codes[:, :, :300])
    assert torch.equal(cache.page_min[:, :, :19], ref.page_min[:, :, :19])
    assert torch.equal(cache.page_max[:, :, :19], ref.page_max[:, :, :19])
