"""Exact top-k keys and the recall of HHR's selection against them, on the GPU
("Top-10% key recall", thelatestinai.com page, Figure 4 caption).

Stage-wise, as the decode parity: the scores are compared with the fp64
oracle within tolerance, the top-k bit for bit with the oracle's select on the
GPU's scores (ties to the lower token), and against the fp64 scores outside an
exemption band around the threshold; the recall equals the oracle's recall of
the GPU's own selections.
"""
import math

import numpy as np
import pytest
import torch

from hash_sparse_attention_b200 import hhr
from hash_sparse_attention_b200.synth import WORKLOADS, make_layer, scaled
from oracle import hhr_oracle as O

pytestmark = pytest.mark.gpu

import parity  # noqa: E402

SCORE_RTOL = 2e-3
EXEMPT = 1e-4


def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("name,kw", [
    ("llama_layer_32k", dict(context=5000, batch=2, seed=81)),
    ("qwen_gqa7_128k", dict(context=3000, batch=2, seed=82)),
    ("paged_b16_ragged", dict(batch=3, context=3000, ragged_min=800, seed=83)),
    ("tiny_4k", dict(seed=84)),
])
def test_exact_topk_and_recall(name, kw):
    _cuda()
    w = scaled(WORKLOADS[name], **kw)
    li = make_layer(w)
    g = parity.run_gpu(w, li, to_host=False)
    assert g.status == 0
    dev = torch.device("cuda")
    cache, dbg = g.extra["cache"], g.extra["dbg"]
    q, R = li.q.to(dev), li.R.to(dev)
    seq, tk = li.seq_lens.to(dev), li.top_k.to(dev)
    tb = None if li.block_table is None else li.block_table.to(dev)
    Kmax = int(li.top_k.max())
    logits, sel, n_sel = hhr.exact_topk(g.cfg, q, R, cache, seq, tb, tk, Kmax)
    rec = hhr.recall(g.cfg, dbg.sel_keys, dbg.n_sel_keys, sel, n_sel)
    torch.cuda.synchronize()
    full = parity.run_gpu(w, li)  # host copies of the same cache (deterministic build)
    z_gpu = logits.cpu().numpy().astype(np.float64)
    sel_g, n_g, rec_g = sel.cpu().numpy(), n_sel.cpu().numpy(), rec.cpu().numpy()
    hsel, hn = dbg.sel_keys.cpu().numpy(), dbg.n_sel_keys.cpu().numpy()
    R64 = li.R.double().cpu().numpy()
    qn = li.q.double().cpu().numpy()
    G = w.group
    for b, L in enumerate(full.lens):
        k = min(max(int(li.top_k[b]), 1), Kmax, L)
        for h in range(w.num_kv_heads):
            Qr = O.rotate_query(R64[h], qn[b, h * G:(h + 1) * G])
            Kp = full.Krot[b, h, :L]
            z64 = O.key_scores_exact(Qr, Kp)
            tol = SCORE_RTOL * (np.abs(Kp) @ np.abs(Qr).T).max(axis=1)
            assert np.all(np.abs(z_gpu[b, h, :L] - z64) <= tol), "scores outside tolerance"
            assert np.all(np.isneginf(z_gpu[b, h, L:])), "scores past the sequence end must be -inf"
            assert n_g[b, h] == k
            got = sel_g[b, h, :k]
            # bit-exact on the GPU's scores
            assert np.array_equal(got, O.exact_topk(z_gpu[b, h, :L], k)), "top-k differs on the GPU's scores"
            # against the fp64 scores, outside the band around the threshold
            ref = O.exact_topk(z64, k)
            if k < L:
                thr = np.sort(z64)[::-1][k - 1]
                sym = np.setxor1d(got, ref)
                assert np.all(np.abs(z64[sym] - thr) <= EXEMPT * max(abs(thr), float(tol.max()))), \
                    "top-k differs outside the exemption band"
            r_ref = O.recall(hsel[b, h, :hn[b, h]], got)
            assert math.isclose(float(rec_g[b, h]), r_ref, rel_tol=0, abs_tol=1e-6)
            print(f"{name} b{b} h{h}: recall {r_ref:.3f} (k={k}, HHR kept {hn[b, h]})")
