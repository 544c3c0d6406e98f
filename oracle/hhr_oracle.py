"""HHR decode-path oracle: plain, slow, fp64 CPU reference.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
baseline leg of the benchmark may import this module.  The CUDA library never
calls it and shares no code with it; the two meet only through the seeded
inputs of ``hash_sparse_attention_b200.synth``.

What it computes follows "HHR: Hierarchical Hash Retrieval for Efficient LLM
Generation" (paper card, Abstract) and the rit.work explainer of the same
paper (section "Два уровня маршрутизации решают разные ошибки", the two
routing levels):

  cache build   K' = R_h k (stored bf16), per-page channel min/max of K',
                per-key sign codes of W_h k                 (build_head)
  GKR           q' = R_h q, page logit upper bounds, keep the top-N pages
                                                            (rotate_query,
                                                             page_bounds,
                                                             select_pages)
  LHP           query codes, Hamming distance over the keys of surviving
                pages, keep the top-k keys                  (hash_codes,
                                                             hamming,
                                                             select_keys)
  attention     exact softmax attention over the kept keys  (attention)

Everything is float64 (np.float64) or exact integers.  Inputs that are bf16
on the GPU side arrive here as float64 arrays holding the same values.
Readings where the pages are silent are marked "READING" below.

Parity status: every function here is pinned by tests/test_oracle.py
(closed forms, brute force, a library routine, or invariants) -- see the
header of that file for which pin covers which function.
"""
from __future__ import annotations

import math

import numpy as np

# ---------------------------------------------------------------------------
# bf16 rounding (storage format of K' and of the page metadata)
# ---------------------------------------------------------------------------

_BF16_MIN_NORMAL = 2.0 ** -126
_BF16_SUB_QUANTUM = 2.0 ** -133


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bf16 value, ties to even (RNE).

    bf16 keeps 8 significant bits.  For a normal number x = m * 2^e with
    m in [0.5, 1), the nearest bf16 value is rint(m * 256) / 256 * 2^e, where
    rint rounds half to even; every step is exact in float64.  Below the
    smallest normal the grid is uniform with spacing 2^-133.
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    normal = np.ldexp(np.rint(m * 256.0) / 256.0, e)
    sub = np.rint(x / _BF16_SUB_QUANTUM) * _BF16_SUB_QUANTUM
    return np.where(np.abs(x) < _BF16_MIN_NORMAL, sub, normal)


# ---------------------------------------------------------------------------
# GKR: orthogonal transform R_h
# ---------------------------------------------------------------------------

def rotate(R: np.ndarray, X: np.ndarray) -> np.ndarray:
    """x' = R_h x for every row x of X ([n, d] -> [n, d]).

    GKR's head-wise orthogonal transform (paper card, Abstract; rit.work,
    two-level routing section: it redistributes values across coordinates
    while keeping every query-key product exact).  READING: the stored key is
    k' = R_h k and the query is q' = R_h q, so q'.k' = q.k for orthogonal R_h.
    """
    return np.asarray(X, dtype=np.float64) @ np.asarray(R, dtype=np.float64).T


def rotate_keys_stored(R: np.ndarray, K: np.ndarray) -> np.ndarray:
    """K' as the cache stores it: R_h k computed in fp64, then rounded RNE to bf16."""
    return round_bf16(rotate(R, K))


def rotate_query(R: np.ndarray, Q: np.ndarray) -> np.ndarray:
    """q' = R_h q for the G query heads of one KV head ([G, d]); kept in fp64."""
    return rotate(R, Q)


# ---------------------------------------------------------------------------
# Pages and their metadata
# ---------------------------------------------------------------------------

def num_pages(L: int, P: int) -> int:
    return -(-L // P)


def page_minmax(Kp: np.ndarray, L: int, P: int) -> tuple[np.ndarray, np.ndarray]:
    """Per-page, per-channel min and max of the stored keys.

    Neighbouring keys are grouped into pages (rit.work, two-level routing
    section); each page keeps what its bound needs.  READING: the metadata is
    the channel-wise minimum and maximum over the page's valid keys (rows
    < L); a partial last page uses only its valid rows.
    """
    n = num_pages(L, P)
    d = Kp.shape[1]
    mn = np.empty((n, d), dtype=np.float64)
    mx = np.empty((n, d), dtype=np.float64)
    for p in range(n):
        rows = Kp[p * P:min((p + 1) * P, L)]
        mn[p] = rows.min(axis=0)
        mx[p] = rows.max(axis=0)
    return mn, mx


def page_bounds(Qr: np.ndarray, mn: np.ndarray, mx: np.ndarray) -> np.ndarray:
    """Page-level logit upper bound ub[g, p] for each query head g of the group.

    The paper card's Abstract names "page-level logit bounds" derived after
    the transform; rit.work (two-level routing section) describes the bound as
    the highest score any key of the page can reach.  The pages do not print
    the formula.  READING: the bound of a channel box,
        ub[g, p] = sum_i max(q'_gi * mn_pi, q'_gi * mx_pi),
    which is >= q'_g . k' for every key k' of page p, and equal to it when the
    page holds one key.  Unscaled (no 1/sqrt(d)); rankings do not change.
    """
    Qr = np.asarray(Qr, dtype=np.float64)
    G, d = Qr.shape
    ub = np.empty((G, mn.shape[0]), dtype=np.float64)
    for g in range(G):
        a = Qr[g][None, :] * mn
        b = Qr[g][None, :] * mx
        ub[g] = np.maximum(a, b).sum(axis=1)
    return ub


def group_bound(ub: np.ndarray, mode: str = "max") -> np.ndarray:
    """U_p = max over the query heads of the group of ub[g, p].

    READING (pages silent on GQA): the max keeps U_p an upper bound for every
    query head that shares the KV head, so one page selection serves them all.
    mode "sum" is the alternative aggregation: U_p = sum over the heads (a bound
    of the group's summed logits).
    """
    if mode == "max":
        return ub.max(axis=0)
    if mode == "sum":
        return ub.sum(axis=0)
    raise ValueError(mode)


def select_pages(U: np.ndarray, N: int) -> np.ndarray:
    """Coarse pruning: keep the N pages with the largest U_p (ascending ids).

    Low-bound pages are dropped whole (rit.work, two-level routing section;
    paper card Abstract: "pruning of low-logit keys").  READING: equal bounds
    go to the lower page index; N larger than the page count keeps all pages.
    """
    U = np.asarray(U, dtype=np.float64)
    N = min(int(N), U.shape[0])
    order = np.argsort(-U, kind="stable")  # stable: equal values keep index order
    return np.sort(order[:N]).astype(np.int64)


def candidates(sel_pages: np.ndarray, L: int, P: int) -> np.ndarray:
    """Token ids of the valid keys inside the kept pages, ascending.

    LHP ranks only the keys of surviving pages (rit.work, two-level routing
    section).  Positions >= L are not keys.
    """
    out = []
    for p in np.sort(sel_pages):
        out.extend(range(int(p) * P, min((int(p) + 1) * P, L)))
    return np.asarray(out, dtype=np.int64)


# ---------------------------------------------------------------------------
# LHP: sign hash codes and Hamming distance
# ---------------------------------------------------------------------------

def hash_projection(W: np.ndarray, X: np.ndarray) -> np.ndarray:
    """The projection W_h x for every row x ([n, d] -> [n, nb]) in fp64."""
    return np.asarray(X, dtype=np.float64) @ np.asarray(W, dtype=np.float64).T


def hash_codes(W: np.ndarray, X: np.ndarray) -> np.ndarray:
    """Binary codes of the rows of X packed into uint64 words ([n, nb/64]).

    Queries and keys become binary codes by sign(.) of a learned head-wise
    projection (paper card Abstract; Figure 2 caption on the paper page:
    projection followed by sign(.)).  READINGS: the hash uses the unrotated
    vector (W_h k, W_h q); bit b is 1 iff (W_h x)_b > 0 (zero gives 0); bit b
    sits in word b // 64 at position b % 64 (least significant first).
    """
    proj = hash_projection(W, X)
    n, nb = proj.shape
    words = nb // 64
    bits = (proj > 0.0)
    out = np.zeros((n, words), dtype=np.uint64)
    for b in range(nb):
        out[:, b // 64] |= bits[:, b].astype(np.uint64) << np.uint64(b % 64)
    return out


def hamming(cq: np.ndarray, codes: np.ndarray, mode: str = "sum") -> np.ndarray:
    """S_j = sum over the group's query codes of the number of differing bits.

    Hamming distance counts mismatching bits (paper card Abstract; rit.work,
    first section).  READING (pages silent on GQA): the group score is the sum
    over its query heads, i.e. the distance between concatenated codes.
    mode "min" is the alternative: the distance to the closest query head.
    cq: uint64 [G, w]; codes: uint64 [n, w] -> int64 [n].
    """
    x = np.bitwise_xor(codes[None, :, :], cq[:, None, :])  # [G, n, w]
    per_head = np.bitwise_count(x).astype(np.int64).sum(axis=2)  # [G, n]
    if mode == "sum":
        return per_head.sum(axis=0)
    if mode == "min":
        return per_head.min(axis=0)
    raise ValueError(mode)


def select_keys(S: np.ndarray, cand: np.ndarray, k: int) -> np.ndarray:
    """Fine retrieval: keep the k candidates with the smallest S (ascending ids).

    READING: equal distances go to the lower token index; k is clamped to the
    number of candidates ("top-10% key recall", Figure 4 caption, fixes the
    budget style but not the clamp).
    """
    k = min(int(k), S.shape[0])
    order = np.argsort(S, kind="stable")  # cand is ascending, so ties -> lower token id
    return np.sort(cand[order[:k]]).astype(np.int64)


# ---------------------------------------------------------------------------
# Attention over the kept keys
# ---------------------------------------------------------------------------

def attention(Qr: np.ndarray, Kp: np.ndarray, V: np.ndarray, sel: np.ndarray,
              scale: float) -> np.ndarray:
    """Exact softmax attention restricted to the selected keys, per query head.

    Attention is computed exactly on the retrieved keys only (rit.work, first
    section).  s_j = scale * q'_g . k'_j over j in sel, o_g = sum_j softmax(s)_j v_j.
    READINGS: V is stored unrotated; the softmax is renormalised over the
    selected set; an empty set gives a zero output.  Returns float64 [G, d].
    """
    G, d = Qr.shape
    if len(sel) == 0:
        return np.zeros((G, d), dtype=np.float64)
    Ks = Kp[sel]
    Vs = V[sel]
    out = np.empty((G, d), dtype=np.float64)
    for g in range(G):
        s = scale * (Ks @ Qr[g])
        e = np.exp(s - s.max())
        out[g] = (e @ Vs) / e.sum()
    return out


# ---------------------------------------------------------------------------
# Whole head: build, then one decode step
# ---------------------------------------------------------------------------

def build_head(K: np.ndarray, R: np.ndarray, W: np.ndarray, L: int, P: int):
    """Cache build for one (sequence, KV head): stored K', page min/max, key codes.

    K: [>=L, d] bf16 values as float64; only rows < L are keys.
    Returns (Kp [L, d], mn [np, d], mx [np, d], codes uint64 [L, w]).
    """
    Kv = np.asarray(K[:L], dtype=np.float64)
    Kp = rotate_keys_stored(R, Kv)
    mn, mx = page_minmax(Kp, L, P)
    codes = hash_codes(W, Kv)
    return Kp, mn, mx, codes


def decode_head(Q: np.ndarray, R: np.ndarray, W: np.ndarray, Kp: np.ndarray, V: np.ndarray,
                mn: np.ndarray, mx: np.ndarray, codes: np.ndarray, L: int, P: int,
                N: int, k: int, scale: float | None = None, page_agg: str = "max",
                key_agg: str = "sum") -> dict:
    """One decode step of HHR for the G query heads of one KV head, all stages.

    Q: [G, d] query rows; the other arrays as returned by build_head.
    Returns every intermediate so that stages can be compared one by one.
    """
    d = Q.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    Qr = rotate_query(R, Q)
    if L == 0:
        G = Q.shape[0]
        return dict(q_rot=Qr, ub=np.zeros((G, 0)), U=np.zeros(0), sel_pages=np.zeros(0, np.int64),
                    q_codes=hash_codes(W, Q), cand=np.zeros(0, np.int64), scores=np.zeros(0, np.int64),
                    sel_keys=np.zeros(0, np.int64), out=np.zeros((G, d)))
    ub = page_bounds(Qr, mn, mx)
    U = group_bound(ub, page_agg)
    sel_p = select_pages(U, N)
    cq = hash_codes(W, Q)
    cand = candidates(sel_p, L, P)
    S = hamming(cq, codes[cand], key_agg)
    sel_k = select_keys(S, cand, k)
    out = attention(Qr, Kp, V, sel_k, scale)
    return dict(q_rot=Qr, ub=ub, U=U, sel_pages=sel_p, q_codes=cq, cand=cand, scores=S,
                sel_keys=sel_k, out=out)


def dense_head(Q: np.ndarray, R: np.ndarray, Kp: np.ndarray, V: np.ndarray, L: int,
               scale: float | None = None) -> np.ndarray:
    """Full attention over all L stored keys (the comparison row of the paper's tables)."""
    d = Q.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    return attention(rotate_query(R, Q), Kp, V, np.arange(L), scale)


# ---------------------------------------------------------------------------
# Exact top-k and recall (the fidelity measure of the paper's Figure 4)
# ---------------------------------------------------------------------------

def key_scores_exact(Qr: np.ndarray, Kp: np.ndarray) -> np.ndarray:
    """z_t = max over the group's query heads of q'_g . k'_t (fp64).

    "Top-10% key recall" (thelatestinai.com page, Figure 4 caption) measures
    retrieval against the truly highest-scoring keys.  READING: with grouped
    query heads sharing one KV head, a key's score is the largest logit of the
    group (a key matters if any head of the group attends to it; the same
    aggregation as the page bound's U_p)."""
    return (np.asarray(Kp, dtype=np.float64) @ np.asarray(Qr, dtype=np.float64).T).max(axis=1)


def exact_topk(z: np.ndarray, k: int) -> np.ndarray:
    """The k keys with the largest score, ascending ids; READING: equal scores
    go to the lower token, k is clamped to the number of keys."""
    z = np.asarray(z, dtype=np.float64)
    k = min(int(k), z.shape[0])
    order = np.argsort(-z, kind="stable")
    return np.sort(order[:k]).astype(np.int64)


def recall(sel: np.ndarray, exact: np.ndarray) -> float:
    """|sel n exact| / |exact| (0 for an empty reference)."""
    exact = np.asarray(exact)
    if exact.size == 0:
        return 0.0
    return float(np.intersect1d(np.asarray(sel), exact).size) / float(exact.size)

