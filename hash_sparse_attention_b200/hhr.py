"""Python binding of the HHR decode path (argument marshalling only).

Every function here checks tensor placement, dtype and shape, turns tensors
into device pointers and calls the C ABI of libhhr.so on the current CUDA
stream.  The computation happens entirely in the library's kernels.
"""
from __future__ import annotations

import ctypes
import math
from dataclasses import dataclass

import torch

from ._lib import HHRConfig, HHRDebug, check, lib

__all__ = ["HHRConfig", "HHRDebug", "make_config", "Cache", "alloc_cache", "build_cache", "append_cache",
           "exact_topk", "recall",
           "decode_workspace", "dense_workspace", "decode_step", "decode_step_noalloc", "dense_decode", "DebugOutputs",
           "alloc_debug"]


AGG = {"max": 0, "sum": 1, "min": 1}


def make_config(batch: int, num_q_heads: int, num_kv_heads: int, page_size: int, hash_bits: int,
                max_seq_len: int, paged: bool = False, num_blocks: int = 0,
                max_blocks_per_seq: int = 0, head_dim: int = 128, page_agg: str = "max",
                key_agg: str = "sum") -> HHRConfig:
    """page_agg: "max" (default) or "sum" of the group's page bounds;
    key_agg: "sum" (default) or "min" of the group's Hamming distances."""
    if page_agg not in ("max", "sum") or key_agg not in ("sum", "min"):
        raise ValueError("page_agg is 'max' or 'sum'; key_agg is 'sum' or 'min'")
    return HHRConfig(batch, num_q_heads, num_kv_heads, head_dim, page_size, hash_bits, max_seq_len,
                     1 if paged else 0, num_blocks, max_blocks_per_seq, 1 if page_agg == "sum" else 0,
                     1 if key_agg == "min" else 0)


def _ptr(t: torch.Tensor | None) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _stream(stream: torch.cuda.Stream | None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _expect(t: torch.Tensor, dtype: torch.dtype, shape: tuple, name: str) -> None:
    if t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")


@dataclass
class Cache:
    """Device tensors of one layer's HHR cache (see include/hhr.h for layouts)."""
    Krot: torch.Tensor
    V: torch.Tensor
    page_min: torch.Tensor
    page_max: torch.Tensor
    codes: torch.Tensor  # int64 storage of the uint64 code words


def cache_shapes(cfg: HHRConfig) -> dict:
    d, P, Hkv = cfg.head_dim, cfg.page_size, cfg.num_kv_heads
    w = cfg.hash_bits // 64
    if cfg.paged:
        nb = cfg.num_blocks
        return dict(kv=(nb, Hkv, P, d), meta=(nb, Hkv, d), codes=(nb, Hkv, P, w))
    np_max = -(-cfg.max_seq_len // P)
    T, B = cfg.max_seq_len, cfg.batch
    return dict(kv=(B, Hkv, T, d), meta=(B, Hkv, np_max, d), codes=(B, Hkv, T, w))


def alloc_cache(cfg: HHRConfig, device="cuda", Krot: torch.Tensor | None = None,
                V: torch.Tensor | None = None) -> Cache:
    """Allocates cache tensors; Krot / V may be given to build in place."""
    sh = cache_shapes(cfg)
    Krot = Krot if Krot is not None else torch.empty(sh["kv"], dtype=torch.bfloat16, device=device)
    V = V if V is not None else torch.empty(sh["kv"], dtype=torch.bfloat16, device=device)
    return Cache(Krot=Krot, V=V,
                 page_min=torch.empty(sh["meta"], dtype=torch.bfloat16, device=device),
                 page_max=torch.empty(sh["meta"], dtype=torch.bfloat16, device=device),
                 codes=torch.empty(sh["codes"], dtype=torch.int64, device=device))


def build_cache(cfg: HHRConfig, K: torch.Tensor, V: torch.Tensor, R: torch.Tensor, W: torch.Tensor,
                seq_lens: torch.Tensor, block_table: torch.Tensor | None, cache: Cache,
                stream: torch.cuda.Stream | None = None) -> Cache:
    sh = cache_shapes(cfg)
    _expect(K, torch.bfloat16, sh["kv"], "K")
    _expect(V, torch.bfloat16, sh["kv"], "V")
    _expect(R, torch.float32, (cfg.num_kv_heads, cfg.head_dim, cfg.head_dim), "R")
    _expect(W, torch.bfloat16, (cfg.num_kv_heads, cfg.hash_bits, cfg.head_dim), "W")
    _expect(seq_lens, torch.int32, (cfg.batch,), "seq_lens")
    st = lib().hhr_build_cache(ctypes.byref(cfg), _ptr(K), _ptr(V), _ptr(R), _ptr(W), _ptr(seq_lens),
                               _ptr(block_table), _ptr(cache.Krot), _ptr(cache.V), _ptr(cache.page_min),
                               _ptr(cache.page_max), _ptr(cache.codes), _stream(stream))
    check(st, "hhr_build_cache")
    return cache


def append_cache(cfg: HHRConfig, K: torch.Tensor, V: torch.Tensor, R: torch.Tensor, W: torch.Tensor,
                 old_lens: torch.Tensor, new_lens: torch.Tensor, max_new: int, block_table: torch.Tensor | None,
                 cache: Cache, stream: torch.cuda.Stream | None = None) -> Cache:
    """Builds rows [old_lens[b], new_lens[b]) of every sequence into `cache`
    (rotation, codes, V, page min/max merged with the page's earlier rows)."""
    sh = cache_shapes(cfg)
    _expect(K, torch.bfloat16, sh["kv"], "K")
    _expect(V, torch.bfloat16, sh["kv"], "V")
    _expect(old_lens, torch.int32, (cfg.batch,), "old_lens")
    _expect(new_lens, torch.int32, (cfg.batch,), "new_lens")
    st = lib().hhr_append_cache(ctypes.byref(cfg), _ptr(K), _ptr(V), _ptr(R), _ptr(W), _ptr(old_lens),
                                _ptr(new_lens), max_new, _ptr(block_table), _ptr(cache.Krot), _ptr(cache.V),
                                _ptr(cache.page_min), _ptr(cache.page_max), _ptr(cache.codes), _stream(stream))
    check(st, "hhr_append_cache")
    return cache


def decode_workspace(cfg: HHRConfig, max_keep_pages: int, max_top_k: int, device="cuda") -> torch.Tensor:
    n = lib().hhr_decode_workspace_size(ctypes.byref(cfg), max_keep_pages, max_top_k)
    if n == 0:
        raise ValueError("invalid configuration for the decode workspace")
    ws = torch.zeros(n, dtype=torch.uint8, device=device)
    return ws


def dense_workspace(cfg: HHRConfig, device="cuda") -> torch.Tensor:
    n = lib().hhr_dense_workspace_size(ctypes.byref(cfg))
    if n == 0:
        raise ValueError("invalid configuration for the dense workspace")
    return torch.zeros(n, dtype=torch.uint8, device=device)


@dataclass
class DebugOutputs:
    q_rot: torch.Tensor
    page_ub: torch.Tensor
    page_U: torch.Tensor
    sel_pages: torch.Tensor
    n_sel_pages: torch.Tensor
    q_codes: torch.Tensor
    key_scores: torch.Tensor
    n_cand: torch.Tensor
    sel_keys: torch.Tensor
    n_sel_keys: torch.Tensor

    def struct(self) -> HHRDebug:
        return HHRDebug(*[getattr(self, n).data_ptr() for n, _ in HHRDebug._fields_])


def alloc_debug(cfg: HHRConfig, max_keep_pages: int, max_top_k: int, device="cuda") -> DebugOutputs:
    B, Hq, Hkv, d, P = cfg.batch, cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim, cfg.page_size
    np_max = -(-cfg.max_seq_len // P)
    Nmax = min(max_keep_pages, np_max)
    w = cfg.hash_bits // 64
    z = lambda *s, dt=torch.int32: torch.full(s, -7, dtype=dt, device=device)  # noqa: E731
    return DebugOutputs(
        q_rot=torch.zeros(B, Hq, d, device=device), page_ub=torch.zeros(B, Hq, np_max, device=device),
        page_U=torch.zeros(B, Hkv, np_max, device=device), sel_pages=z(B, Hkv, Nmax), n_sel_pages=z(B, Hkv),
        q_codes=torch.zeros(B, Hq, w, dtype=torch.int64, device=device), key_scores=z(B, Hkv, Nmax * P),
        n_cand=z(B, Hkv), sel_keys=z(B, Hkv, max_top_k), n_sel_keys=z(B, Hkv))


def decode_step(cfg: HHRConfig, q: torch.Tensor, R: torch.Tensor, W: torch.Tensor, cache: Cache,
                seq_lens: torch.Tensor, block_table: torch.Tensor | None, n_keep: torch.Tensor,
                top_k: torch.Tensor, max_keep_pages: int, max_top_k: int, out: torch.Tensor,
                workspace: torch.Tensor, sm_scale: float | None = None, dbg: DebugOutputs | None = None,
                status: torch.Tensor | None = None, stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    _expect(q, torch.bfloat16, (cfg.batch, cfg.num_q_heads, cfg.head_dim), "q")
    _expect(out, torch.float32, (cfg.batch, cfg.num_q_heads, cfg.head_dim), "out")
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(cfg.head_dim)
    d = dbg.struct() if dbg is not None else None
    st = lib().hhr_decode_step(
        ctypes.byref(cfg), _ptr(q), _ptr(R), _ptr(W), _ptr(cache.Krot), _ptr(cache.V), _ptr(cache.page_min),
        _ptr(cache.page_max), _ptr(cache.codes), _ptr(seq_lens), _ptr(block_table), _ptr(n_keep), _ptr(top_k),
        max_keep_pages, max_top_k, sm_scale, _ptr(out), ctypes.byref(d) if d is not None else None,
        _ptr(workspace), workspace.numel(), _ptr(status), _stream(stream))
    check(st, "hhr_decode_step")
    return out


def decode_step_noalloc(cfg: HHRConfig, q: torch.Tensor, R: torch.Tensor, W: torch.Tensor, cache: Cache,
                        seq_lens: torch.Tensor, block_table: torch.Tensor | None, n_keep: torch.Tensor,
                        top_k: torch.Tensor, max_keep_pages: int, max_top_k: int, out: torch.Tensor,
                        sm_scale: float | None = None, dbg: DebugOutputs | None = None,
                        status: torch.Tensor | None = None,
                        stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """decode_step without a workspace tensor: the library's built-in device
    scratch is used instead (see hhr_decode_step_noalloc in include/hhr.h)."""
    _expect(q, torch.bfloat16, (cfg.batch, cfg.num_q_heads, cfg.head_dim), "q")
    _expect(out, torch.float32, (cfg.batch, cfg.num_q_heads, cfg.head_dim), "out")
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(cfg.head_dim)
    d = dbg.struct() if dbg is not None else None
    st = lib().hhr_decode_step_noalloc(
        ctypes.byref(cfg), _ptr(q), _ptr(R), _ptr(W), _ptr(cache.Krot), _ptr(cache.V), _ptr(cache.page_min),
        _ptr(cache.page_max), _ptr(cache.codes), _ptr(seq_lens), _ptr(block_table), _ptr(n_keep), _ptr(top_k),
        max_keep_pages, max_top_k, sm_scale, _ptr(out), ctypes.byref(d) if d is not None else None,
        _ptr(status), _stream(stream))
    check(st, "hhr_decode_step_noalloc")
    return out


def dense_decode(cfg: HHRConfig, q: torch.Tensor, R: torch.Tensor, cache: Cache, seq_lens: torch.Tensor,
                 block_table: torch.Tensor | None, out: torch.Tensor, workspace: torch.Tensor,
                 sm_scale: float | None = None, status: torch.Tensor | None = None,
                 stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    _expect(q, torch.bfloat16, (cfg.batch, cfg.num_q_heads, cfg.head_dim), "q")
    _expect(out, torch.float32, (cfg.batch, cfg.num_q_heads, cfg.head_dim), "out")
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(cfg.head_dim)
    st = lib().hhr_dense_decode(ctypes.byref(cfg), _ptr(q), _ptr(R), _ptr(cache.Krot), _ptr(cache.V),
                                _ptr(seq_lens), _ptr(block_table), sm_scale, _ptr(out), _ptr(workspace),
                                workspace.numel(), _ptr(status), _stream(stream))
    check(st, "hhr_dense_decode")
    return out


def exact_topk(cfg: HHRConfig, q: torch.Tensor, R: torch.Tensor, cache: Cache, seq_lens: torch.Tensor,
               block_table: torch.Tensor | None, top_k: torch.Tensor, max_top_k: int,
               stream: torch.cuda.Stream | None = None):
    """The k keys with the largest max-over-the-group logit per (sequence, KV
    head): returns (logits [B, Hkv, T] fp32, sel [B, Hkv, max_top_k], n_sel [B, Hkv])."""
    _expect(q, torch.bfloat16, (cfg.batch, cfg.num_q_heads, cfg.head_dim), "q")
    dev = q.device
    logits = torch.empty(cfg.batch, cfg.num_kv_heads, cfg.max_seq_len, dtype=torch.float32, device=dev)
    sel = torch.full((cfg.batch, cfg.num_kv_heads, max_top_k), -1, dtype=torch.int32, device=dev)
    n_sel = torch.zeros(cfg.batch, cfg.num_kv_heads, dtype=torch.int32, device=dev)
    st = lib().hhr_exact_topk(ctypes.byref(cfg), _ptr(q), _ptr(R), _ptr(cache.Krot), _ptr(seq_lens),
                              _ptr(block_table), _ptr(top_k), max_top_k, _ptr(logits), _ptr(sel), _ptr(n_sel),
                              None, _stream(stream))
    check(st, "hhr_exact_topk")
    return logits, sel, n_sel


def recall(cfg: HHRConfig, sel_a: torch.Tensor, n_a: torch.Tensor, sel_b: torch.Tensor, n_b: torch.Tensor,
           stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """|A n B| / |B| per (sequence, KV head) for index lists [B, Hkv, *]."""
    out = torch.empty(cfg.batch, cfg.num_kv_heads, dtype=torch.float32, device=sel_a.device)
    st = lib().hhr_recall(ctypes.byref(cfg), _ptr(sel_a.contiguous()), _ptr(n_a.contiguous()), sel_a.shape[-1],
                          _ptr(sel_b.contiguous()), _ptr(n_b.contiguous()), sel_b.shape[-1], _ptr(out),
                          _stream(stream))
    check(st, "hhr_recall")
    return out

