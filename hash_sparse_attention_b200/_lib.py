"""ctypes declarations of libhhr.so (the C ABI in include/hhr.h).

Argument marshalling only: every step of the decode path runs in the CUDA
kernels behind these entry points.  Loading fails loudly when the library has
not been built; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhhr.so")

HHR_OK = 0
HHR_ERR_INVALID_ARG = 1
HHR_ERR_UNSUPPORTED = 2
HHR_ERR_WORKSPACE = 3
HHR_ERR_CUDA = 4
HHR_ERR_TIMEOUT = 5
HHR_ERR_BAD_BLOCK = 6
NOALLOC_SCRATCH_BYTES = 16 << 20  # HHR_NOALLOC_SCRATCH_BYTES in include/hhr.h


class HHRConfig(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "batch", "num_q_heads", "num_kv_heads", "head_dim", "page_size", "hash_bits",
        "max_seq_len", "paged", "num_blocks", "max_blocks_per_seq", "page_group_agg", "key_group_agg")]

    def as_dict(self) -> dict:
        return {n: getattr(self, n) for n, _ in self._fields_}


class HHRDebug(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "q_rot", "page_ub", "page_U", "sel_pages", "n_sel_pages", "q_codes",
        "key_scores", "n_cand", "sel_keys", "n_sel_keys")]


_vp = ctypes.c_void_p
_i32 = ctypes.c_int32
_sz = ctypes.c_size_t
_cfgp = ctypes.POINTER(HHRConfig)

# name -> (restype, argtypes); the same set of functions include/hhr.h declares
SIGNATURES = {
    "hhr_status_string": (ctypes.c_char_p, [_i32]),
    "hhr_last_error": (ctypes.c_char_p, []),
    "hhr_set_wait_limit": (None, [ctypes.c_int64]),
    "hhr_build_cache": (_i32, [_cfgp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "hhr_append_cache": (_i32, [_cfgp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "hhr_decode_workspace_size": (_sz, [_cfgp, _i32, _i32]),
    "hhr_workspace_init": (_i32, [_vp, _sz, _vp]),
    "hhr_decode_step": (_i32, [_cfgp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                               _i32, _i32, ctypes.c_float, _vp, ctypes.POINTER(HHRDebug), _vp, _sz,
                               _vp, _vp]),
    "hhr_decode_step_noalloc": (_i32, [_cfgp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                       _i32, _i32, ctypes.c_float, _vp, ctypes.POINTER(HHRDebug), _vp, _vp]),
    "hhr_dense_workspace_size": (_sz, [_cfgp]),
    "hhr_exact_topk": (_i32, [_cfgp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _vp, _vp]),
    "hhr_recall": (_i32, [_cfgp, _vp, _vp, _i32, _vp, _vp, _i32, _vp, _vp]),
    "hhr_dense_decode": (_i32, [_cfgp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_float, _vp, _vp, _sz,
                                _vp, _vp]),
}

_LIB = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -c 'import __graft_entry__ as g; g.build()'` "
                "or `python -m hash_sparse_attention_b200.build_lib` (there is no CPU fallback)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


class HHRError(RuntimeError):
    def __init__(self, status: int, where: str):
        L = lib()
        msg = L.hhr_last_error().decode() or L.hhr_status_string(status).decode()
        super().__init__(f"{where}: {L.hhr_status_string(status).decode()}: {msg}")
        self.status = status


def check(status: int, where: str) -> None:
    if status != HHR_OK:
        raise HHRError(status, where)
