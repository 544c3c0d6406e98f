"""Pins for the fp64 oracle (CPU only).

Each oracle function is checked against something other than itself:

  round_bf16      torch's fp32->bf16 conversion (a library routine, RNE) on
                  fp32-exact inputs, including constructed ties
  rotate          orientation on a cyclic shift (closed form); invariance
                  |q.k - q'.k'| <= 1e-9 |q||k| for QR-orthogonal R (the
                  passage: the transform keeps query-key products exact)
  page_minmax     brute force over rows, partial last page
  page_bounds     brute force over the 2^d corners of the channel box (the
                  maximum of a linear function on a box); P=1 gives the exact
                  logit; ub >= every logit of the page
  select_pages    brute-force rank definition (count of strictly better pages)
  candidates      hand example
  hash_codes      bit-by-bit construction with Python integers; the SimHash
                  law E[Hamming]/bits = angle/pi for Gaussian projections
  hamming         bit-by-bit count with Python integers; H(x,x)=0, H(x,~x)=bits
  select_keys     brute-force rank definition
  attention       torch scaled_dot_product_attention in fp64 when every key
                  is kept; one key gives v; q=0 gives the mean of V
  decode_head     the hand-derived fixture tests/golden/hhr_hand_example.json
  key_scores_exact  rotation invariance (scores of rotated vectors equal the
                  max over heads of the unrotated q.k, computed without the
                  oracle) and a hand example where max and sum differ
  exact_topk      brute-force rank definition (largest first, ties to the
                  lower index)
  recall          hand examples (the denominator is the reference set)
  group_bound / hamming aggregation modes (sum of bounds, min distance):
                  hand examples where the modes differ

The last test plants plausible mistakes in copies of oracle functions and
checks that some pin rejects each of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import hhr_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hhr_hand_example.json")


def _rng(seed=0):
    return np.random.default_rng(seed)


def _bf16_values(rng, shape, scale=1.0):
    x = torch.from_numpy(rng.standard_normal(shape).astype(np.float32) * scale)
    return x.to(torch.bfloat16).to(torch.float64).numpy()


def _orth(rng, d):
    q, r = np.linalg.qr(rng.standard_normal((d, d)))
    return q * np.sign(np.diag(r))[None, :]


# ---------------------------------------------------------------------------
# pin functions (take the functions under test as arguments so that planted
# mistakes can be run through them)
# ---------------------------------------------------------------------------

def pin_round_bf16(round_bf16):
    rng = _rng(1)
    x32 = (rng.standard_normal(20000) * np.exp(rng.uniform(-30, 30, 20000))).astype(np.float32)
    # constructed ties: low 16 bits exactly 0x8000, both parities of the kept bit
    u = rng.integers(0x3F000000, 0x47000000, 4000, dtype=np.uint32)
    ties = ((u & np.uint32(0xFFFF0000)) | np.uint32(0x8000)).view(np.float32)
    x32 = np.concatenate([x32, ties, -ties, np.float32([0.0, 1.0, -1.0, 3.0e-39, -7.1e-40])])
    ref = torch.from_numpy(x32).to(torch.bfloat16).to(torch.float64).numpy()
    got = round_bf16(x32.astype(np.float64))
    assert np.array_equal(got, ref)


def pin_rotate_orientation(rotate):
    d = 8
    R = np.zeros((d, d))
    for i in range(d):
        R[i, (i + 1) % d] = 1.0          # (R x)_i = x_{i+1}
    x = np.arange(1.0, d + 1.0)[None, :]
    assert np.array_equal(rotate(R, x)[0], np.roll(x[0], -1))


def pin_rotate_invariance(rotate):
    rng = _rng(2)
    for d in (4, 64, 128):
        R = _orth(rng, d)
        assert np.abs(R.T @ R - np.eye(d)).max() <= 1e-12
        q = rng.standard_normal((5, d)) * 3
        k = rng.standard_normal((7, d)) * 3
        k[:, :4] *= 10
        lhs = q @ k.T
        rhs = rotate(R, q) @ rotate(R, k).T
        scale = np.linalg.norm(q, axis=1)[:, None] * np.linalg.norm(k, axis=1)[None, :]
        assert np.all(np.abs(lhs - rhs) <= 1e-9 * scale)


def pin_page_minmax(page_minmax):
    rng = _rng(3)
    for L, P in ((37, 16), (32, 16), (1, 16), (17, 16), (65, 32), (5, 2)):
        Kp = _bf16_values(rng, (L, 6))
        mn, mx = page_minmax(Kp, L, P)
        n = -(-L // P)
        assert mn.shape == (n, 6) and mx.shape == (n, 6)
        for p in range(n):
            for c in range(6):
                lo = hi = None
                for j in range(p * P, min(p * P + P, L)):
                    v = Kp[j, c]
                    lo = v if lo is None or v < lo else lo
                    hi = v if hi is None or v > hi else hi
                assert mn[p, c] == lo and mx[p, c] == hi


def pin_page_bounds_corners(page_bounds):
    rng = _rng(4)
    d = 6
    for _ in range(20):
        Qr = rng.standard_normal((3, d))
        a = rng.standard_normal((4, d))
        b = rng.standard_normal((4, d))
        mn, mx = np.minimum(a, b), np.maximum(a, b)
        ub = page_bounds(Qr, mn, mx)
        for g in range(3):
            for p in range(4):
                best = -np.inf
                for mask in range(1 << d):
                    corner = np.array([mx[p, i] if (mask >> i) & 1 else mn[p, i] for i in range(d)])
                    best = max(best, float(Qr[g] @ corner))
                assert abs(ub[g, p] - best) <= 1e-12 * (1 + np.abs(Qr[g]).sum() * np.abs(np.r_[mn[p], mx[p]]).max())


def pin_page_bounds_safe(page_bounds, page_minmax):
    rng = _rng(5)
    d, L, P = 128, 100, 16
    Kp = _bf16_values(rng, (L, d))
    Kp[:, :4] *= 10
    Qr = rng.standard_normal((4, d))
    mn, mx = page_minmax(Kp, L, P)
    ub = page_bounds(Qr, mn, mx)
    logits = Qr @ Kp.T
    for p in range(mn.shape[0]):
        rows = slice(p * P, min(p * P + P, L))
        terms = np.abs(Qr).sum(axis=1) * np.abs(Kp[rows]).max()
        assert np.all(ub[:, p] >= logits[:, rows].max(axis=1) - 1e-12 * terms)
    # one key per page: the bound is the logit itself
    mn1, mx1 = page_minmax(Kp, L, 1)
    ub1 = page_bounds(Qr, mn1, mx1)
    assert np.allclose(ub1, logits, rtol=0, atol=1e-11)


def _rank_select_largest(U, N):
    out = []
    for p in range(len(U)):
        better = sum(1 for r in range(len(U)) if U[r] > U[p] or (U[r] == U[p] and r < p))
        if better < N:
            out.append(p)
    return out


def pin_select_pages(select_pages):
    rng = _rng(6)
    for n, N in ((50, 7), (64, 64), (10, 20), (33, 1)):
        U = np.round(rng.standard_normal(n) * 2) / 2  # many ties
        assert list(select_pages(U, N)) == _rank_select_largest(list(U), N)
    assert list(select_pages(np.array([3.0, 5.0, 5.0, 1.0, 5.0]), 2)) == [1, 2]
    assert list(select_pages(np.array([-0.0, 0.0]), 1)) == [0]


def pin_candidates(candidates):
    assert list(candidates(np.array([2, 0]), 5, 2)) == [0, 1, 4]
    assert list(candidates(np.array([1]), 40, 16)) == list(range(16, 32))
    assert list(candidates(np.array([2]), 40, 16)) == list(range(32, 40))


def _py_codes(W, X):
    proj = X @ W.T
    out = []
    for row in proj:
        words = [0] * (len(row) // 64)
        for b, v in enumerate(row):
            if v > 0:
                words[b // 64] += 1 << (b % 64)
        out.append(words)
    return out


def pin_hash_codes(hash_codes):
    rng = _rng(7)
    W = _bf16_values(rng, (128, 16))
    X = _bf16_values(rng, (9, 16))
    X[0] = 0.0  # all projections zero -> all bits 0
    got = hash_codes(W, X)
    ref = _py_codes(W, X)
    assert [[int(w) for w in r] for r in got] == ref
    # unit rows: bit b = sign of coordinate b
    Wi = np.zeros((64, 4))
    Wi[:4] = np.eye(4)
    assert [int(w) for w in hash_codes(Wi, np.array([[2.0, -1.0, 0.0, 1.0]]))[0]] == [9]


def pin_simhash_angle(hash_codes, hamming):
    rng = _rng(8)
    d, nb = 64, 4096
    W = rng.standard_normal((nb, d))
    for theta in (0.3, math.pi / 4, 1.2, 2.5):
        u = rng.standard_normal(d)
        u /= np.linalg.norm(u)
        v = rng.standard_normal(d)
        v -= (v @ u) * u
        v /= np.linalg.norm(v)
        q = u
        k = math.cos(theta) * u + math.sin(theta) * v
        h = hamming(hash_codes(W, q[None, :]), hash_codes(W, k[None, :]))[0]
        p = theta / math.pi
        assert abs(h / nb - p) <= 5 * math.sqrt(p * (1 - p) / nb)


def pin_hamming(hamming):
    rng = _rng(9)
    G, n, w = 3, 20, 2
    cq = rng.integers(0, 2**63, (G, w), dtype=np.uint64) * np.uint64(2) + rng.integers(0, 2, (G, w), dtype=np.uint64)
    codes = rng.integers(0, 2**63, (n, w), dtype=np.uint64) * np.uint64(2) + rng.integers(0, 2, (n, w), dtype=np.uint64)
    S = hamming(cq, codes)
    for j in range(n):
        cnt = 0
        for g in range(G):
            for t in range(w):
                a, c = int(cq[g, t]), int(codes[j, t])
                cnt += sum(1 for b in range(64) if ((a >> b) & 1) != ((c >> b) & 1))
        assert S[j] == cnt
    assert np.all(hamming(cq[:1], cq[:1]) == 0)
    assert np.all(hamming(cq[:1], ~cq[:1]) == 64 * w)


def _rank_select_smallest(S, ids, k):
    out = []
    for a in range(len(S)):
        better = sum(1 for b in range(len(S)) if S[b] < S[a] or (S[b] == S[a] and ids[b] < ids[a]))
        if better < k:
            out.append(int(ids[a]))
    return sorted(out)


def pin_select_keys(select_keys):
    rng = _rng(10)
    for n, k in ((40, 9), (16, 16), (5, 50), (31, 1)):
        ids = np.sort(rng.choice(1000, n, replace=False))
        S = rng.integers(0, 6, n)
        assert list(select_keys(S, ids, k)) == _rank_select_smallest(list(S), list(ids), k)


def pin_attention(attention):
    rng = _rng(11)
    G, d, L = 4, 128, 77
    Q = rng.standard_normal((G, d))
    K = rng.standard_normal((L, d))
    V = rng.standard_normal((L, d))
    scale = 1 / math.sqrt(d)
    got = attention(Q, K, V, np.arange(L), scale)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q)[None, :, None, :], torch.from_numpy(K)[None, None].expand(1, G, L, d),
        torch.from_numpy(V)[None, None].expand(1, G, L, d), scale=scale)[0, :, 0].numpy()
    assert np.allclose(got, ref, rtol=0, atol=1e-12)
    assert np.array_equal(attention(Q, K, V, np.array([13]), scale), np.repeat(V[13][None], G, 0))
    sel = np.array([1, 5, 9, 40])
    assert np.allclose(attention(np.zeros((G, d)), K, V, sel, scale), V[sel].mean(0)[None].repeat(G, 0),
                       rtol=0, atol=1e-14)


def pin_hand_example(O_):
    ex = json.load(open(GOLDEN))
    e = ex["expected"]
    R = np.array(ex["R"], float)
    K = np.array(ex["K"], float)
    V = np.array(ex["V"], float)
    Q = np.array(ex["Q"], float)
    L, P = ex["seq_len"], ex["page_size"]
    W = np.zeros((ex["hash_bits"], ex["d"]))
    W[:ex["W_unit_rows"]] = np.eye(ex["d"])
    Kp, mn, mx, codes = O_.build_head(K, R, W, L, P)
    assert np.array_equal(Kp, np.array(e["K_rot"], float))
    assert np.array_equal(mn, np.array(e["page_min"], float))
    assert np.array_equal(mx, np.array(e["page_max"], float))
    assert [int(c) for c in codes[:, 0]] == e["key_codes"]
    r = O_.decode_head(Q, R, W, Kp, V, mn, mx, codes, L, P, N=2, k=3, scale=math.log(2.0))
    assert np.array_equal(r["q_rot"], np.array(e["q_rot"], float))
    assert np.array_equal(r["ub"], np.array(e["ub"], float))
    assert np.array_equal(r["U"], np.array(e["U"], float))
    assert list(r["sel_pages"]) == e["sel_pages_N2"]
    assert [int(c) for c in r["q_codes"][:, 0]] == e["q_codes"]
    assert list(r["cand"]) == e["candidates_N2"]
    assert list(r["scores"]) == e["scores_N2"]
    assert list(r["sel_keys"]) == e["sel_keys_k3"]
    exact = np.array([[a / b for a, b in row] for row in e["out_k3_exact"]])
    assert np.allclose(r["out"], exact, rtol=0, atol=1e-15)
    assert np.allclose(r["out"], np.array(e["out_k3"]), rtol=0, atol=1e-15)
    r1 = O_.decode_head(Q, R, W, Kp, V, mn, mx, codes, L, P, N=1, k=2, scale=math.log(2.0))
    assert list(r1["sel_pages"]) == e["sel_pages_N1"]
    r2 = O_.decode_head(Q, R, W, Kp, V, mn, mx, codes, L, P, N=2, k=2, scale=math.log(2.0))
    assert list(r2["sel_keys"]) == e["sel_keys_k2"]


# ---------------------------------------------------------------------------
# the tests
# ---------------------------------------------------------------------------

def test_round_bf16():
    pin_round_bf16(O.round_bf16)


def test_rotate_orientation():
    pin_rotate_orientation(O.rotate)


def test_rotate_invariance():
    pin_rotate_invariance(O.rotate)


def test_synth_rotation_is_orthogonal():
    from hash_sparse_attention_b200.synth import orthogonal_from_gaussian
    R = orthogonal_from_gaussian(torch.Generator().manual_seed(5), 128)
    assert np.abs(R.T @ R - np.eye(128)).max() <= 1e-12
    assert np.all(np.diag(np.linalg.qr(R)[1]) != 0)


def test_page_minmax():
    pin_page_minmax(O.page_minmax)


def test_page_bounds_corners():
    pin_page_bounds_corners(O.page_bounds)


def test_page_bounds_safe():
    pin_page_bounds_safe(O.page_bounds, O.page_minmax)


def test_select_pages():
    pin_select_pages(O.select_pages)


def test_candidates():
    pin_candidates(O.candidates)


def test_hash_codes():
    pin_hash_codes(O.hash_codes)


def test_simhash_angle():
    pin_simhash_angle(O.hash_codes, O.hamming)


def test_hamming():
    pin_hamming(O.hamming)


def test_select_keys():
    pin_select_keys(O.select_keys)


def test_attention():
    pin_attention(O.attention)


def test_hand_example():
    pin_hand_example(O)


def test_keep_everything_is_dense_attention():
    """Keeping every page and every key reproduces full attention on (q', K')."""
    rng = _rng(12)
    d, L, P, G = 128, 203, 16, 4
    K = _bf16_values(rng, (L, d))
    V = _bf16_values(rng, (L, d))
    Q = _bf16_values(rng, (G, d))
    R = _orth(rng, d).astype(np.float32).astype(np.float64)
    W = _bf16_values(rng, (128, d))
    Kp, mn, mx, codes = O.build_head(K, R, W, L, P)
    r = O.decode_head(Q, R, W, Kp, V, mn, mx, codes, L, P, N=10**6, k=10**6)
    assert list(r["sel_keys"]) == list(range(L))
    dense = O.dense_head(Q, R, Kp, V, L)
    assert np.array_equal(r["out"], dense)
    Qr = O.rotate(R, Q)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Qr)[None, :, None, :], torch.from_numpy(Kp)[None, None].expand(1, G, L, d),
        torch.from_numpy(V)[None, None].expand(1, G, L, d), scale=1 / math.sqrt(d))[0, :, 0].numpy()
    assert np.allclose(r["out"], ref, rtol=0, atol=1e-12)


def test_rotation_spreads_outlier_channels():
    """Fig. 3 analogue: after a random orthogonal R, the largest channel magnitude drops."""
    from hash_sparse_attention_b200.synth import WORKLOADS, make_layer, scaled
    w = scaled(WORKLOADS["tiny_4k"], context=512)
    li = make_layer(w)
    K = li.K[0, 0].double().numpy()
    Kp = O.rotate(li.R64[0], K)
    assert np.abs(Kp).max(axis=0).max() < 0.6 * np.abs(K).max(axis=0).max()


# ---------------------------------------------------------------------------
# planted mistakes: each mutant must be rejected by some pin
def pin_key_scores(key_scores_exact):
    rng = _rng(41)
    d, G = 16, 3
    R = _orth(rng, d)
    Q = rng.standard_normal((G, d))
    K = rng.standard_normal((50, d)) * 2
    z = key_scores_exact(Q @ R.T, K @ R.T)  # rotated query and keys (R applied by matmul)
    ref = np.array([max(float(np.dot(Q[g], K[t])) for g in range(G)) for t in range(50)])
    assert np.all(np.abs(z - ref) <= 1e-9 * np.linalg.norm(K, axis=1) * np.linalg.norm(Q, axis=1).max())
    # hand example: two heads, max over heads (a sum would give [-1, 3, 0])
    z = key_scores_exact(np.array([[1.0, 0.0], [0.0, 1.0]]), np.array([[2.0, -3.0], [-1.0, 4.0], [0.0, 0.0]]))
    assert np.array_equal(z, [2.0, 4.0, 0.0])


def pin_exact_topk(exact_topk):
    rng = _rng(42)
    for n, k in ((30, 7), (30, 30), (10, 40), (25, 1)):
        z = rng.integers(0, 6, n).astype(np.float64)  # many ties
        got = exact_topk(z, k)
        keep = [t for t in range(n)
                if sum(1 for u in range(n) if z[u] > z[t] or (z[u] == z[t] and u < t)) < min(k, n)]
        assert np.array_equal(got, keep)


def pin_recall(recall):
    assert recall(np.array([1, 2, 3]), np.array([2, 3, 4, 5])) == 0.5
    assert recall(np.array([7]), np.array([7])) == 1.0
    assert recall(np.array([], dtype=np.int64), np.array([1])) == 0.0
    assert recall(np.array([1, 2]), np.array([], dtype=np.int64)) == 0.0
    assert recall(np.array([1, 2, 3, 4]), np.array([4])) == 1.0


def pin_aggregation_modes(group_bound, hamming):
    ub = np.array([[3.0, 1.0, -2.0], [2.0, 2.0, 1.0]])
    assert np.array_equal(group_bound(ub, "max"), [3.0, 2.0, 1.0])
    assert np.array_equal(group_bound(ub, "sum"), [5.0, 3.0, -1.0])
    cq = np.array([[0b1011], [0b0000]], dtype=np.uint64)      # two heads, one word
    codes = np.array([[0b1010], [0b1111], [0b0000]], dtype=np.uint64)
    assert np.array_equal(hamming(cq, codes, "sum"), [1 + 2, 1 + 4, 3 + 0])
    assert np.array_equal(hamming(cq, codes, "min"), [1, 1, 0])


def test_aggregation_modes():
    pin_aggregation_modes(O.group_bound, O.hamming)


def test_key_scores_exact():
    pin_key_scores(O.key_scores_exact)


def test_exact_topk():
    pin_exact_topk(O.exact_topk)


def test_recall():
    pin_recall(O.recall)


# ---------------------------------------------------------------------------

def _fails(fn, *args):
    try:
        fn(*args)
    except AssertionError:
        return True
    return False


def test_planted_mistakes_are_caught():
    # rounding through fp32 first (double rounding) / truncation instead of RNE
    assert _fails(pin_round_bf16, lambda x: np.floor(np.frexp(x)[0] * 256) / 256 * 2.0 ** np.frexp(x)[1])
    # transposed rotation
    assert _fails(pin_rotate_orientation, lambda R, X: np.asarray(X) @ np.asarray(R))
    # off-by-one page range
    def minmax_off(Kp, L, P):
        n = -(-L // P)
        mn = np.stack([Kp[p * P:min(p * P + P + 1, L)].min(0) for p in range(n)])
        mx = np.stack([Kp[p * P:min(p * P + P + 1, L)].max(0) for p in range(n)])
        return mn, mx
    assert _fails(pin_page_minmax, minmax_off)
    # bound that ignores the min side, or uses |q'| on max only
    assert _fails(pin_page_bounds_corners, lambda Qr, mn, mx: Qr @ mx.T)
    assert _fails(pin_page_bounds_corners, lambda Qr, mn, mx: np.abs(Qr) @ mx.T)
    # a dropped term: mid-point instead of the box corner
    assert _fails(pin_page_bounds_safe, lambda Qr, mn, mx: Qr @ ((mn + mx) / 2).T, O.page_minmax)
    # ties going to the higher page index / selecting the smallest
    def sel_ties_high(U, N):
        n = len(U)
        order = np.argsort(-U[::-1], kind="stable")  # reversed: ties go to the higher index
        return np.sort(n - 1 - order[:min(N, n)])
    assert _fails(pin_select_pages, sel_ties_high)
    assert _fails(pin_select_pages, lambda U, N: np.sort(np.argsort(U, kind="stable")[:min(N, len(U))]))
    # candidates ignoring the sequence end
    assert _fails(pin_candidates, lambda s, L, P: np.concatenate([np.arange(p * P, p * P + P) for p in np.sort(s)]))
    # MSB-first packing / sign flipped / >= 0 at zero
    def codes_msb(W, X):
        proj = np.asarray(X) @ np.asarray(W).T
        out = np.zeros((proj.shape[0], proj.shape[1] // 64), np.uint64)
        for b in range(proj.shape[1]):
            out[:, b // 64] |= (proj[:, b] > 0).astype(np.uint64) << np.uint64(63 - b % 64)
        return out
    assert _fails(pin_hash_codes, codes_msb)
    assert _fails(pin_hash_codes, lambda W, X: O.hash_codes(-np.asarray(W), X))
    def codes_ge(W, X):
        proj = np.asarray(X) @ np.asarray(W).T
        out = np.zeros((proj.shape[0], proj.shape[1] // 64), np.uint64)
        for b in range(proj.shape[1]):
            out[:, b // 64] |= (proj[:, b] >= 0).astype(np.uint64) << np.uint64(b % 64)
        return out
    assert _fails(pin_hash_codes, codes_ge)
    # one side's code complemented -> the SimHash law breaks
    assert _fails(pin_simhash_angle, O.hash_codes, lambda a, b: O.hamming(a, ~b))
    # Hamming with AND instead of XOR / counting only the first word
    assert _fails(pin_hamming, lambda cq, c: np.bitwise_count(c[None] & cq[:, None]).astype(np.int64).sum((0, 2)))
    assert _fails(pin_hamming, lambda cq, c: np.bitwise_count(c[None, :, :1] ^ cq[:, None, :1]).astype(np.int64).sum((0, 2)))
    # key top-k keeping the largest distances / ties to the higher token
    assert _fails(pin_select_keys, lambda S, c, k: np.sort(c[np.argsort(-S, kind="stable")[:min(k, len(S))]]))
    assert _fails(pin_select_keys, lambda S, c, k: np.sort(c[::-1][np.argsort(S[::-1], kind="stable")[:min(k, len(S))]]))
    # attention without the max shift is fine numerically; without normalisation / scale it is not
    assert _fails(pin_attention, lambda Q, K, V, s, sc: np.stack([np.exp(sc * (K[s] @ q)) @ V[s] for q in Q]))
    assert _fails(pin_attention, lambda Q, K, V, s, sc: O.attention(Q, K, V, s, 1.0))
    # key scores summed over the group instead of the max; top-k ties to the higher
    # index; recall over the selection's size
    assert _fails(pin_key_scores, lambda Qr, Kp: (np.asarray(Kp) @ np.asarray(Qr).T).sum(axis=1))
    def topk_ties_high(z, k):
        n = len(z)
        order = np.argsort(-z[::-1], kind="stable")
        return np.sort(n - 1 - order[:min(k, n)])
    assert _fails(pin_exact_topk, topk_ties_high)
    assert _fails(pin_recall, lambda a, b: float(np.intersect1d(a, b).size) / max(1, np.asarray(a).size))
    # the modes swapped
    assert _fails(pin_aggregation_modes, lambda ub, m="max": O.group_bound(ub, "sum" if m == "max" else "max"),
                  O.hamming)
    assert _fails(pin_aggregation_modes, O.group_bound,
                  lambda cq, c, m="sum": O.hamming(cq, c, "min" if m == "sum" else "sum"))

