"""The seeded input generator (CPU): the random-orthogonal hash projection
(the paper page's Figure 2 caption: random orthogonal projection, then sign)
has orthonormal rows within each d x d block; the default law is unchanged."""
import numpy as np
import torch

from hash_sparse_attention_b200.synth import WORKLOADS, hash_projection, make_layer, scaled


def test_orthogonal_hash_projection_rows():
    for bits in (64, 128, 256):
        w = scaled(WORKLOADS["tiny_4k"], hash_bits=bits, hash_law="orthogonal")
        W = hash_projection(w, torch.Generator().manual_seed(bits)).double().numpy()
        assert W.shape == (bits, 128)
        for b0 in range(0, bits, 128):
            blk = W[b0:b0 + 128]
            gram = blk @ blk.T
            assert np.abs(gram - np.eye(blk.shape[0])).max() < 1e-6
        if bits == 256:  # two independent blocks, not copies
            assert np.abs(W[:128] @ W[128:].T).max() > 0.05


def test_gaussian_law_is_the_default_and_deterministic():
    w = scaled(WORKLOADS["tiny_4k"], context=256)
    a, b = make_layer(w), make_layer(w)
    assert w.hash_law == "gaussian"
    assert torch.equal(a.W, b.W) and torch.equal(a.K, b.K)
    wo = scaled(w, hash_law="orthogonal")
    c = make_layer(wo)
    assert not torch.equal(a.W, c.W)
    assert torch.equal(a.R, c.R)  # R_h is drawn before W_h
