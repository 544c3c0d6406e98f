"""The C ABI library loads on the CPU and exports what include/hhr.h declares.

No compute call is made here (there is no GPU): only host-side functions and
argument validation paths, which return before any CUDA call.
"""
import ctypes
import os
import re
import subprocess

import pytest

from hash_sparse_attention_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hhr.h")


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"HHR_API\s+[\w\s\*]+?\b(hhr_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(_lib.LIB_PATH):
        import __graft_entry__
        __graft_entry__.build()
    return _lib.lib()


def test_header_declares_the_boundary():
    fns = declared_functions()
    assert fns == sorted(["hhr_status_string", "hhr_last_error", "hhr_set_wait_limit", "hhr_build_cache",
                          "hhr_append_cache", "hhr_exact_topk", "hhr_recall",
                          "hhr_decode_workspace_size",
                          "hhr_workspace_init", "hhr_decode_step", "hhr_decode_step_noalloc",
                          "hhr_dense_workspace_size", "hhr_dense_decode"])
    # the binding declares exactly the same functions
    assert sorted(_lib.SIGNATURES) == fns


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True).stdout
    exported = sorted(set(re.findall(r"\bT\s+(hhr_\w+)", out)))
    assert exported == declared_functions()
    for name in declared_functions():
        assert getattr(L, name) is not None


def test_status_strings(L):
    assert L.hhr_status_string(0) == b"HHR_OK"
    assert L.hhr_status_string(3) == b"HHR_ERR_WORKSPACE"
    assert L.hhr_status_string(6) == b"HHR_ERR_BAD_BLOCK"
    assert L.hhr_status_string(99) == b"HHR_ERR_UNKNOWN"


def _cfg(**kw):
    base = dict(batch=1, num_q_heads=32, num_kv_heads=8, head_dim=128, page_size=16, hash_bits=128,
                max_seq_len=32768, paged=0, num_blocks=0, max_blocks_per_seq=0)
    base.update(kw)
    return _lib.HHRConfig(**base)


def test_workspace_size_is_host_arithmetic(L):
    c = _cfg()
    n = L.hhr_decode_workspace_size(ctypes.byref(c), 256, 3277)
    assert n > 0 and n % 256 == 0
    # larger budgets never need less
    assert L.hhr_decode_workspace_size(ctypes.byref(c), 512, 8192) >= n
    assert L.hhr_dense_workspace_size(ctypes.byref(c)) > 0
    # invalid configurations report zero
    assert L.hhr_decode_workspace_size(ctypes.byref(_cfg(head_dim=64)), 256, 3277) == 0
    assert L.hhr_decode_workspace_size(ctypes.byref(c), 0, 3277) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(head_dim=64), _lib.HHR_ERR_UNSUPPORTED),
    (dict(num_q_heads=36), _lib.HHR_ERR_UNSUPPORTED),    # group size 9... 36/8 not integral
    (dict(num_q_heads=30), _lib.HHR_ERR_INVALID_ARG),    # not a multiple
    (dict(page_size=8), _lib.HHR_ERR_UNSUPPORTED),
    (dict(hash_bits=96), _lib.HHR_ERR_UNSUPPORTED),
    (dict(max_seq_len=1 << 20), _lib.HHR_ERR_UNSUPPORTED),  # more pages than supported
    (dict(max_seq_len=1 << 18), _lib.HHR_ERR_UNSUPPORTED),  # more pages than the page select holds
    (dict(paged=1, num_blocks=0), _lib.HHR_ERR_INVALID_ARG),
    (dict(paged=1, num_blocks=10, max_blocks_per_seq=3), _lib.HHR_ERR_INVALID_ARG),
])
def test_validation_rejects_bad_configs(L, kw, code):
    c = _cfg(**kw)
    if kw.get("num_q_heads") == 36:
        c.num_kv_heads = 4  # group size 9
    st = L.hhr_decode_step(ctypes.byref(c), *([None] * 12), 1, 1, 0.1, None, None, None, 0, None, None)
    assert st == code, L.hhr_last_error()
    assert L.hhr_last_error() != b""


def test_null_pointers_and_alignment(L):
    c = _cfg()
    st = L.hhr_decode_step(ctypes.byref(c), *([None] * 12), 1, 1, 0.1, None, None, None, 0, None, None)
    assert st == _lib.HHR_ERR_INVALID_ARG
    st = L.hhr_build_cache(ctypes.byref(c), *([None] * 11), None)
    assert st == _lib.HHR_ERR_INVALID_ARG
    # misaligned (fake, never dereferenced) pointers are rejected before any launch
    fake = [0x1000 + 16 * i for i in range(12)]
    fake[2] += 2  # W
    st = L.hhr_decode_step(ctypes.byref(c), *fake, 256, 3277, 0.1, 0x9000, None, 0xA000, 1 << 30, None, None)
    assert st == _lib.HHR_ERR_INVALID_ARG and b"aligned" in L.hhr_last_error()
    # workspace too small
    fake[2] -= 2
    st = L.hhr_decode_step(ctypes.byref(c), *fake, 256, 3277, 0.1, 0x9000, None, 0xA000, 100, None, None)
    assert st == _lib.HHR_ERR_WORKSPACE
    # workspace not 256-byte aligned
    st = L.hhr_decode_step(ctypes.byref(c), *fake, 256, 3277, 0.1, 0x9000, None, 0xA010, 1 << 30, None, None)
    assert st == _lib.HHR_ERR_INVALID_ARG
    # non-positive softmax scale
    st = L.hhr_decode_step(ctypes.byref(c), *fake, 256, 3277, 0.0, 0x9000, None, 0xA000, 1 << 30, None, None)
    assert st == _lib.HHR_ERR_INVALID_ARG
