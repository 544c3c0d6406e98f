"""hhr_decode_step_noalloc: the decode step for callers that cannot allocate.

Callers such as inference-runtime plugins that must take every byte of device
memory from the host runtime's pool, or serving loops where an allocation is
not allowed, cannot call cudaMalloc for a workspace.  The no-alloc entry point
runs the same decode step in the library's built-in device scratch.  These
tests call it through the C ABI twice in a row, then with a different shape
after a larger one (the scratch keeps the previous call's contents), and
compare with hhr_decode_step on a caller-provided workspace.  This file is
collected last on purpose.
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


def _noalloc(cfg, q, R, W, cache, seq, nk, tk, Nmax, Kmax, out, status):
    return _lib.lib().hhr_decode_step_noalloc(
        ctypes.byref(cfg), q.data_ptr(), R.data_ptr(), W.data_ptr(), cache.Krot.data_ptr(), cache.V.data_ptr(),
        cache.page_min.data_ptr(), cache.page_max.data_ptr(), cache.codes.data_ptr(), seq.data_ptr(), None,
        nk.data_ptr(), tk.data_ptr(), Nmax, Kmax, 1.0 / np.sqrt(128.0), out.data_ptr(), None,
        status.data_ptr(), torch.cuda.current_stream().cuda_stream)


def test_noalloc_after_a_larger_call_of_another_shape():
    """A larger call leaves data all over the scratch; a following call of a
    smaller shape with another group size and code width must clear what it
    uses and match hhr_decode_step bit for bit."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda")
    runs = []
    for w in (scaled(WORKLOADS["llama_layer_32k"], batch=3, context=20000, seed=4),
              scaled(WORKLOADS["qwen_gqa7_128k"], batch=1, context=5000, seed=5)):
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
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        out = torch.full_like(ref, float("nan"))
        assert _noalloc(cfg, q, R, W, cache, seq, nk, tk, Nmax, Kmax, out, status) == _lib.HHR_OK
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        runs.append((out, ref))
    for out, ref in runs:
        assert torch.equal(out, ref)


def test_noalloc_rejects_bad_arguments_like_the_workspace_path():
    """Same status and message as hhr_decode_step for rejected arguments,
    returned before anything is enqueued (no device pointer is touched: the
    pointers below are never dereferenced)."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L = _lib.lib()
    cfg = hhr.make_config(1, 32, 8, 16, 128, 32768)
    fake = [0x10000 + 256 * i for i in range(12)]
    # max_keep_pages above the kernel's kept-page capacity
    st_ws = L.hhr_decode_step(ctypes.byref(cfg), *fake, 4096, 100, 0.1, 0x90000, None, 0xA0000, 1 << 30, None, None)
    msg_ws = L.hhr_last_error().replace(b"hhr_decode_step", b"")
    st_na = L.hhr_decode_step_noalloc(ctypes.byref(cfg), *fake, 4096, 100, 0.1, 0x90000, None, None, None)
    msg_na = L.hhr_last_error().replace(b"hhr_decode_step_noalloc", b"")
    assert st_ws == st_na == _lib.HHR_ERR_UNSUPPORTED
    assert msg_ws == msg_na
    # a NULL q: rejected before the scratch is cleared
    st = L.hhr_decode_step_noalloc(ctypes.byref(cfg), None, *fake[1:], 64, 100, 0.1, 0x90000, None, None, None)
    assert st == _lib.HHR_ERR_INVALID_ARG

