"""Pins for the fp64 layer oracle (oracle/layer.py): it must reduce to the pinned
forward oracle with identity projections, its projections must equal explicit
per-element loops, and grouped key/value heads must equal repeating each key/value
head's projection columns for its query heads."""
import numpy as np
import pytest

import oracle
import oracle.layer as ol
from oracle import DELTA, LINEAR

RNG = np.random.default_rng(321)


@pytest.mark.parametrize("mode", [LINEAR, DELTA])
def test_identity_projections_give_the_forward(mode):
    B, L, H, d, N = 2, 12, 2, 4, 5
    x = RNG.standard_normal((B, L, H * d))
    beta = RNG.standard_normal(H)
    eye = np.eye(H * d)
    y, M, z = ol.layer_forward(x, eye, eye, eye, eye, beta, N, mode, H, H, d)
    heads = x.reshape(B, L, H, d).transpose(0, 2, 1, 3)
    out, M_ref, z_ref = oracle.forward(heads, heads, heads, beta, N, mode)
    assert np.allclose(y, out.transpose(0, 2, 1, 3).reshape(B, L, H * d), rtol=0, atol=1e-13)
    assert np.allclose(M, M_ref, rtol=0, atol=1e-12) and np.allclose(z, z_ref, rtol=0, atol=1e-12)


def test_projection_is_the_matrix_product():
    x = RNG.standard_normal((1, 3, 5))
    W = RNG.standard_normal((5, 4))
    got = ol.project(x, W)
    for l in range(3):
        for j in range(4):
            ref = sum(x[0, l, i] * W[i, j] for i in range(5))
            assert abs(got[0, l, j] - ref) <= 1e-13


@pytest.mark.parametrize("mode", [LINEAR, DELTA])
def test_grouped_heads_equal_repeated_projections(mode):
    """H = 4 query heads on H_kv = 2 key/value heads equals H_kv = H with each key/value
    head's columns of W_K, W_V repeated for the two query heads that read it."""
    B, L, D, H, Hkv, d, N = 1, 10, 6, 4, 2, 3, 4
    x = RNG.standard_normal((B, L, D))
    Wq = RNG.standard_normal((D, H * d))
    Wk = RNG.standard_normal((D, Hkv * d))
    Wv = RNG.standard_normal((D, Hkv * d))
    Wo = RNG.standard_normal((H * d, D))
    beta = RNG.standard_normal(H)
    y, M, z = ol.layer_forward(x, Wq, Wk, Wv, Wo, beta, N, mode, H, Hkv, d)
    rep = lambda W: np.concatenate([W[:, (h // 2) * d:(h // 2) * d + d] for h in range(H)], axis=1)
    y2, M2, z2 = ol.layer_forward(x, Wq, rep(Wk), rep(Wv), Wo, beta, N, mode, H, H, d)
    assert np.allclose(y, y2, rtol=0, atol=1e-12)
    assert np.allclose(M, M2[:, ::2], rtol=0, atol=1e-12)
    assert np.allclose(z, z2[:, ::2], rtol=0, atol=1e-12)


def test_planted_wrong_head_split_fails():
    """Splitting the projection's columns head-minor instead of head-major must break
    the identity reduction (checks the pin can see a transposed head layout)."""
    B, L, H, d, N = 1, 6, 2, 3, 3
    x = RNG.standard_normal((B, L, H * d))
    beta = RNG.standard_normal(H)
    eye = np.eye(H * d)
    heads_bad = x.reshape(B, L, d, H).transpose(0, 3, 1, 2)
    out_bad, _, _ = oracle.forward(heads_bad, heads_bad, heads_bad, beta, N, LINEAR)
    y, _, _ = ol.layer_forward(x, eye, eye, eye, eye, beta, N, LINEAR, H, H, d)
    assert not np.allclose(y, out_bad.transpose(0, 2, 1, 3).reshape(B, L, H * d), atol=1e-6)
