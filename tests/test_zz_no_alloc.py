"""hhr_decode_step_noalloc: the decode step for callers that cannot allocate.

Callers such as code running under another framework's CUDA graph capture,
or inference-runtime plugins restricted to the host runtime's memory pool,
cannot call cudaMalloc for a workspace.  The no-alloc entry point runs the
same decode step in the library's built-in device scratch.  These tests call
it through the C ABI twice in a row and compare with hhr_decode_step on a
caller-provided workspace.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from hash_sparse_attention_b200 import _lib, hhr
from hash_sparse_attention_b200.synth import WORKLOADS, make_layer, scaled

pytestmark = pytest.mark.gpu

OUT_RTOL = 2e-3  # the attention-output tolerance of the parity tests


def _rel(a, b):
    return float((a - b).abs().max() / b.abs().max())


def test_noalloc_matches_workspace_path_twice():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda")
    w = scaled(WORKLOADS["llama_layer_32k"], context=9001, batch=2)
    li = make_layer(w)
    cfg = hhr.make_config(w.batch, w.num_q_heads, w.num_kv_heads, w.page_size, w.hash_bits, w.context)
    K, V, q, R, W = (t.to(dev) for t in (li.K, li.V, li.q, li.R, li.W))
    seq, nk, tk = li.seq_lens.to(dev), li.n_keep.to(dev), li.top_k.to(dev)
    Nmax, Kmax = int(li.n_keep.max()), int(li.top_k.max())
    cache = hhr.alloc_cache(cfg, dev)
    hhr.build_cache(cfg, K, V, R, W, seq, None, cache)
    ws = hhr.decode_workspace(cfg, Nmax, Kmax, dev)
    ref = torch.empty(w.batch, w.num_q_heads, 128, device=dev)
    hhr.decode_step(cfg, q, R, W, cache, seq, None, nk, tk, Nmax, Kmax, ref, ws)
    L = _lib.lib()
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream().cuda_stream
    outs = []
    for _ in range(2):
        out = torch.full_like(ref, float("nan"))
        st = L.hhr_decode_step_noalloc(
            ctypes.byref(cfg), q.data_ptr(), R.data_ptr(), W.data_ptr(), cache.Krot.data_ptr(), cache.V.data_ptr(),
            cache.page_min.data_ptr(), cache.page_max.data_ptr(), cache.codes.data_ptr(), seq.data_ptr(), None,
            nk.data_ptr(), tk.data_ptr(), Nmax, Kmax, 1.0 / np.sqrt(128.0), out.data_ptr(), None,
            status.data_ptr(), stream)
        assert st == _lib.HHR_OK, L.hhr_last_error()
        outs.append(out)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for out in outs:
        assert torch.isfinite(out).all()
        assert _rel(out, ref) <= OUT_RTOL
    # same kernels, same order of arithmetic: the results are in fact identical
    assert torch.equal(outs[0], ref) and torch.equal(outs[1], ref)


def test_noalloc_rejects_sizes_beyond_the_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    cfg = hhr.make_config(64, 32, 8, 16, 256, 131072)
    need = _lib.lib().hhr_decode_workspace_size(ctypes.byref(cfg), 1024, 13108)
    assert need > _lib.NOALLOC_SCRATCH_BYTES
    fake = [0x10000 + 256 * i for i in range(12)]
    st = _lib.lib().hhr_decode_step_noalloc(ctypes.byref(cfg), *fake, 1024, 13108, 0.1, 0x90000, None, None, None)
    assert st == _lib.HHR_ERR_WORKSPACE
    assert b"scratch" in _lib.lib().hhr_last_error()
