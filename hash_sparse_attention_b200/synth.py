"""Seeded synthetic inputs for the HHR decode path.

This module holds no arithmetic of the method: it only draws random tensors
and lays them out.  It is shared by the tests, the benchmark and the oracle
harness so that the CUDA path and the oracle see the same bytes.

Workloads follow the shapes of the HHR paper (Hierarchical Hash Retrieval for
Efficient LLM Generation): the Llama-3.1-8B attention shape of its Table 3
(32 layers, 32 query heads, 8 KV heads, hidden 4096 so head_dim 128, 131072
context), 128-bit codes (Table 4), and a "top-10%" key budget (Figure 4).
The learned per-head transforms R_h (GKR) and W_h (LHP) are replaced by
seeded stand-ins: R_h is a QR-orthogonalised Gaussian and W_h a Gaussian
projection rounded to bf16.

Draw recipe, per (workload, layer):
  * a CPU generator seeded with ``seed`` draws, for each KV head in order:
    R_h (fp64 Gaussian d x d, QR, column signs fixed so diag(R_qr) > 0,
    stored as fp32), W_h (N(0,1), nb x d, rounded RNE to bf16); then the
    data law's per-head channel structure for K and then for V;
    for ragged workloads the sequence lengths come first, then the block
    table permutation.
  * a generator on the target device seeded with ``seed + 7919`` draws K,
    V and q (fp32 N(0,1), shaped [B, Hkv, T, d] / [B, Hq, d]), which are then
    scaled by the channel structure and rounded RNE to bf16.
W_h law: "gaussian" (default) or "orthogonal" (rows of QR-orthogonalised
Gaussian d x d matrices, the random-orthogonal-projection hash of the paper's
Figure 2, one d x d block per d bits).
Data laws: "outlier" = 4 channels per (layer, KV head) drawn without
replacement, independently for K and V, multiplied by 10; "student_t3" =
per (KV head, channel) scale |t_3| (t_3 = z / sqrt(chi2_3 / 3)), separately
for K and V.  q is always N(0,1).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    page_size: int
    hash_bits: int
    context: int                  # fixed context, or the upper end of the ragged range
    layers: int = 1
    keep_den: int = 8             # keep ceil(np / keep_den) pages ...
    keep_pages: int | None = None  # ... unless a fixed page count is given
    topk_den: int = 10            # top-k = ceil(L / topk_den) keys ...
    top_k: int | None = None      # ... unless a fixed k is given
    law: str = "outlier"          # "outlier" or "student_t3"
    hash_law: str = "gaussian"    # W_h: "gaussian" (N(0,1)) or "orthogonal" (rows of random orthogonal matrices)
    page_agg: str = "max"         # page bound over the group's query heads: "max" or "sum"
    key_agg: str = "sum"          # Hamming score over the group's query heads: "sum" or "min"
    paged: bool = False
    ragged_min: int | None = None  # ragged contexts drawn uniform in [ragged_min, context]
    seed: int = 0
    layer_seed_base: int | None = None  # per-layer seed = base + layer (else seed)

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def words(self) -> int:
        return self.hash_bits // 64

    def layer_seed(self, layer: int) -> int:
        if self.layer_seed_base is not None:
            return self.layer_seed_base + layer
        return self.seed

    def keep_for(self, seq_len: int) -> int:
        np_pages = -(-seq_len // self.page_size)
        if self.keep_pages is not None:
            return self.keep_pages
        return -(-np_pages // self.keep_den)

    def topk_for(self, seq_len: int) -> int:
        if self.top_k is not None:
            return self.top_k
        return -(-seq_len // self.topk_den)


# The five workloads of the HHR decode benchmark (shapes from the paper's
# Table 3 model configuration; budgets and data laws as stated beside each).
WORKLOADS: dict[str, Workload] = {
    # tiny single step: B1, GQA 4 (4 q heads / 1 KV head), T 4096, P 16, 64-bit codes
    "tiny_4k": Workload("tiny_4k", 1, 4, 1, 128, 16, 64, 4096,
                        keep_pages=32, top_k=256, seed=0),
    # one Llama-3.1-8B-shaped layer at 32K, keep 1/8 of pages, top 10% keys
    "llama_layer_32k": Workload("llama_layer_32k", 1, 32, 8, 128, 16, 128, 32768,
                                keep_den=8, topk_den=10, seed=1),
    # all 32 layers at 128K, keep 1/16 of pages, top 10% keys (clamped to the candidates)
    "llama_32l_128k": Workload("llama_32l_128k", 1, 32, 8, 128, 16, 128, 131072,
                               layers=32, keep_den=16, topk_den=10, seed=1000,
                               layer_seed_base=1000),
    # same, keep 1/8 of pages so that the key top-k really prunes
    "llama_32l_128k_keep8": Workload("llama_32l_128k_keep8", 1, 32, 8, 128, 16, 128, 131072,
                                     layers=32, keep_den=8, topk_den=10, seed=1000,
                                     layer_seed_base=1000),
    # batch 16 paged, ragged contexts in [8192, 32768], 16-token blocks
    "paged_b16_ragged": Workload("paged_b16_ragged", 16, 32, 8, 128, 16, 128, 32768,
                                 keep_den=8, topk_den=10, paged=True, ragged_min=8192, seed=2),
    # Qwen-like GQA 7 stress: B4, 28/4 heads, 128K, P 32, 256-bit codes
    "qwen_gqa7_128k": Workload("qwen_gqa7_128k", 4, 28, 4, 128, 32, 256, 131072,
                               keep_den=32, top_k=2048, law="student_t3", seed=3),
}


def scaled(w: Workload, **changes) -> Workload:
    """A copy of a workload with some fields changed (smaller test cases)."""
    d = dict(w.__dict__)
    d.update(changes)
    return Workload(**d)


def orthogonal_from_gaussian(g: torch.Generator, d: int) -> np.ndarray:
    """QR-orthogonalised Gaussian, made unique by positive diag of the R factor (fp64)."""
    a = torch.randn(d, d, generator=g, dtype=torch.float64).numpy()
    qm, rm = np.linalg.qr(a)
    s = np.sign(np.diag(rm))
    s[s == 0] = 1.0
    return qm * s[None, :]


def hash_projection(w: Workload, g: torch.Generator) -> torch.Tensor:
    """W_h before rounding to bf16 (fp32, nb x d).

    "gaussian": N(0,1) entries, the stand-in for the learned projection.
    "orthogonal": the random-orthogonal-projection hash of the paper's
    Figure 2 caption (random orthogonal projection, then sign): rows of
    QR-orthogonalised Gaussian d x d matrices, as many blocks of d rows as nb
    needs (256 bits at d = 128: two independent blocks)."""
    nb, d = w.hash_bits, w.head_dim
    if w.hash_law == "gaussian":
        return torch.randn(nb, d, generator=g, dtype=torch.float32)
    if w.hash_law == "orthogonal":
        blocks = [torch.from_numpy(orthogonal_from_gaussian(g, d).T.copy()) for _ in range(-(-nb // d))]
        return torch.cat(blocks, 0)[:nb].to(torch.float32)
    raise ValueError(f"unknown hash law {w.hash_law!r}")


def _channel_scales(w: Workload, g: torch.Generator) -> torch.Tensor:
    """Per-channel multipliers for one KV head of one tensor (K or V)."""
    d = w.head_dim
    if w.law == "outlier":
        sc = torch.ones(d, dtype=torch.float32)
        idx = torch.randperm(d, generator=g)[:4]
        sc[idx] = 10.0
        return sc
    if w.law == "student_t3":
        z = torch.randn(d, generator=g, dtype=torch.float64)
        chi2 = (torch.randn(3, d, generator=g, dtype=torch.float64) ** 2).sum(0)
        t3 = z / torch.sqrt(chi2 / 3.0)
        return t3.abs().to(torch.float32)
    raise ValueError(f"unknown data law {w.law!r}")


@dataclass
class LayerInputs:
    """One layer's inputs.  Tensors live on the requested device.

    K, V: bf16, contiguous [B, Hkv, T, d] (T = max context), or, when paged,
          the block pool [nblocks, Hkv, P, d] addressed by ``block_table``.
    q:    bf16 [B, Hq, d].
    R:    fp32 [Hkv, d, d] (k' = R_h k);  R64 the fp64 matrices it came from.
    W:    bf16 [Hkv, nb, d].
    seq_lens: int32 [B];  block_table: int32 [B, max_blocks] (-1 = unused) or None.
    n_keep, top_k: int32 [B] per-sequence budgets.
    K_logical/V_logical: for paged inputs, the per-sequence view [B, Hkv, T, d]
          that the pool was scattered from (zeros beyond each length).
    """
    K: torch.Tensor
    V: torch.Tensor
    q: torch.Tensor
    R: torch.Tensor
    R64: np.ndarray
    W: torch.Tensor
    seq_lens: torch.Tensor
    block_table: torch.Tensor | None
    n_keep: torch.Tensor
    top_k: torch.Tensor
    K_logical: torch.Tensor | None = None
    V_logical: torch.Tensor | None = None
    extra: dict = field(default_factory=dict)


def draw_seq_lens(w: Workload, g: torch.Generator) -> list[int]:
    if w.ragged_min is None:
        return [w.context] * w.batch
    lens = torch.randint(w.ragged_min, w.context + 1, (w.batch,), generator=g)
    return [int(x) for x in lens]


def make_layer(w: Workload, layer: int = 0, device: str | torch.device = "cpu",
               seq_lens: list[int] | None = None) -> LayerInputs:
    """Draw one layer's inputs following the recipe in the module docstring.

    ``seq_lens`` overrides the drawn lengths (edge-case tests); the random
    stream is unchanged otherwise.
    """
    device = torch.device(device)
    seed = w.layer_seed(layer)
    g = torch.Generator().manual_seed(seed)
    B, Hq, Hkv, d, P, nb = w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.page_size, w.hash_bits
    T = w.context

    drawn = draw_seq_lens(w, g)
    lens = list(seq_lens) if seq_lens is not None else drawn
    assert len(lens) == B and all(0 <= L <= T for L in lens)

    R64 = np.empty((Hkv, d, d), dtype=np.float64)
    Wb = torch.empty(Hkv, nb, d, dtype=torch.bfloat16)
    ksc = torch.empty(Hkv, d, dtype=torch.float32)
    vsc = torch.empty(Hkv, d, dtype=torch.float32)
    for h in range(Hkv):
        R64[h] = orthogonal_from_gaussian(g, d)
        Wb[h] = hash_projection(w, g).to(torch.bfloat16)
        ksc[h] = _channel_scales(w, g)
        vsc[h] = _channel_scales(w, g)

    gd = torch.Generator(device=device).manual_seed(seed + 7919)
    K = torch.randn(B, Hkv, T, d, generator=gd, device=device, dtype=torch.float32)
    K.mul_(ksc.to(device)[None, :, None, :])
    K = K.to(torch.bfloat16)
    V = torch.randn(B, Hkv, T, d, generator=gd, device=device, dtype=torch.float32)
    V.mul_(vsc.to(device)[None, :, None, :])
    V = V.to(torch.bfloat16)
    q = torch.randn(B, Hq, d, generator=gd, device=device, dtype=torch.float32).to(torch.bfloat16)
    # zero the rows beyond each sequence's length (they are never part of the cache)
    for b, L in enumerate(lens):
        if L < T:
            K[b, :, L:] = 0
            V[b, :, L:] = 0

    n_keep = torch.tensor([w.keep_for(L) for L in lens], dtype=torch.int32)
    top_k = torch.tensor([w.topk_for(L) for L in lens], dtype=torch.int32)
    R = torch.from_numpy(R64.astype(np.float32))

    block_table = None
    K_logical = V_logical = None
    if w.paged:
        nblk = [-(-L // P) for L in lens]
        max_blocks = -(-T // P)
        pool = sum(nblk)
        perm = torch.randperm(max(pool, 1), generator=g)
        table = torch.full((B, max_blocks), -1, dtype=torch.int32)
        pos = 0
        for b in range(B):
            table[b, :nblk[b]] = perm[pos:pos + nblk[b]].to(torch.int32)
            pos += nblk[b]
        block_table = table
        K_logical, V_logical = K, V
        K = to_pool(K, table, lens, P, max(pool, 1))
        V = to_pool(V, table, lens, P, max(pool, 1))

    return LayerInputs(
        K=K, V=V, q=q.to(device), R=R.to(device), R64=R64, W=Wb.to(device),
        seq_lens=torch.tensor(lens, dtype=torch.int32, device=device),
        block_table=None if block_table is None else block_table.to(device),
        n_keep=n_keep.to(device), top_k=top_k.to(device),
        K_logical=K_logical, V_logical=V_logical)


def to_pool(X: torch.Tensor, table: torch.Tensor, lens: list[int], P: int, nblocks: int) -> torch.Tensor:
    """Scatter per-sequence rows [B, H, T, d] into a block pool [nblocks, H, P, d]."""
    B, H, T, d = X.shape
    pool = torch.zeros(nblocks, H, P, d, dtype=X.dtype, device=X.device)
    for b, L in enumerate(lens):
        nb_ = -(-L // P)
        if nb_ == 0:
            continue
        pad = nb_ * P
        rows = X[b, :, :pad] if pad <= T else torch.nn.functional.pad(X[b], (0, 0, 0, pad - T))
        rows = rows.reshape(H, nb_, P, d).permute(1, 0, 2, 3)
        pool[table[b, :nb_].long().to(X.device)] = rows
    return pool


def from_pool(pool: torch.Tensor, table: torch.Tensor, lens: list[int], T: int) -> torch.Tensor:
    """Gather a block pool [nblocks, H, P, ...] back into per-sequence rows [B, H, T, ...]
    (zeros past each length)."""
    nblocks, H, P = pool.shape[:3]
    rest = tuple(pool.shape[3:])
    B = table.shape[0]
    out = torch.zeros((B, H, T) + rest, dtype=pool.dtype, device=pool.device)
    for b, L in enumerate(lens):
        nb_ = -(-L // P)
        if nb_ == 0:
            continue
        rows = pool[table[b, :nb_].long().to(pool.device)].transpose(0, 1).reshape((H, nb_ * P) + rest)
        out[b, :, :L] = rows[:, :L]
    return out


def num_pages(seq_len: int, page_size: int) -> int:
    return -(-seq_len // page_size)


def l2_flush_bytes() -> int:
    """Size of a buffer that evicts the whole L2 of the current device (2x L2)."""
    props = torch.cuda.get_device_properties(torch.cuda.current_device())
    return 2 * int(getattr(props, "L2_cache_size", 128 << 20))


__all__ = ["Workload", "WORKLOADS", "LayerInputs", "make_layer", "scaled", "to_pool",
           "from_pool", "num_pages", "orthogonal_from_gaussian", "hash_projection", "l2_flush_bytes"]
