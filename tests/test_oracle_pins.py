"""Pins for the fp64 oracle: each test ties the oracle to something other than itself.

P1 brute-force attention, P2 segment-length invariance of the Linear state,
P3 gate limits, P4 delta fixed point, P5 hand-computed worked example (golden file),
P6 stream equivalence, P7 causal kernel linear attention as a special case.
Plus planted-mistake checks: a wrong variant of the oracle must fail a pin.
"""
import math
import os

import numpy as np
import pytest

import oracle
from oracle import DELTA, LINEAR

RNG = np.random.default_rng(12345)


def rand(*shape):
    return RNG.standard_normal(shape)


# ----------------------------------------------------------------------------
# P1: brute-force masked softmax attention (explicit N x N matrix, pure loops)
# ----------------------------------------------------------------------------
def brute_attention(q, k, v):
    """Explicit lower-triangular softmax(QK^T/sqrt(d))V with plain Python loops and
    no max subtraction: weights exp(c_ij) / sum_j exp(c_ij) over j <= i."""
    n, d = q.shape
    out = np.zeros((n, v.shape[1]))
    for i in range(n):
        ws = []
        for j in range(n):
            if j <= i:
                c = sum(q[i, t] * k[j, t] for t in range(d)) / math.sqrt(d)
                ws.append(math.exp(c))
            else:
                ws.append(0.0)
        tot = sum(ws)
        for c in range(v.shape[1]):
            out[i, c] = sum(ws[j] * v[j, c] for j in range(n)) / tot
    return out


@pytest.mark.parametrize("d,n", [(2, 1), (2, 2), (4, 3), (4, 8), (64, 8), (8, 64)])
def test_p1_bruteforce_attention(d, n):
    q, k, v = rand(n, d), rand(n, d), rand(n, d)
    ref = brute_attention(q, k, v)
    got = oracle.local_attention(q, k, v)
    assert np.max(np.abs(got - ref)) <= 1e-13 * max(1.0, np.max(np.abs(ref)))
    # the same through the full forward with g = 0 (beta = -inf), one segment
    out, _, _ = oracle.forward(q[None, None], k[None, None], v[None, None],
                               [-np.inf], n, LINEAR)
    assert np.max(np.abs(out[0, 0] - ref)) <= 1e-13 * max(1.0, np.max(np.abs(ref)))


def test_p1_single_token_returns_value():
    q, k, v = rand(1, 5), rand(1, 5), rand(1, 5)
    assert np.array_equal(oracle.local_attention(q, k, v), v)


# ----------------------------------------------------------------------------
# P2: Linear final state does not depend on the segment length
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("N", [1, 2, 4, 8, 16, 32, 5, 7])
def test_p2_linear_state_segment_invariance(N):
    L, d = 32, 6
    q, k, v = rand(1, 2, L, d), rand(1, 2, L, d), rand(1, 2, L, d)
    _, M, z = oracle.forward(q, k, v, [0.3, -0.7], N, LINEAR)
    for h in range(2):
        phik = np.where(k[0, h] > 0, k[0, h] + 1.0, np.exp(np.minimum(k[0, h], 0)))
        M_ref = np.einsum("tk,tc->kc", phik, v[0, h])   # whole-sequence sum of bindings
        z_ref = phik.sum(axis=0)
        assert np.linalg.norm(M[0, h] - M_ref) <= 1e-12 * np.linalg.norm(M_ref)
        assert np.linalg.norm(z[0, h] - z_ref) <= 1e-12 * np.linalg.norm(z_ref)


def test_p2_with_initial_state():
    L, d, N = 24, 4, 8
    q, k, v = rand(1, 1, L, d), rand(1, 1, L, d), rand(1, 1, L, d)
    M0, z0 = rand(1, 1, d, d), np.abs(rand(1, 1, d)) + 1
    _, M, z = oracle.forward(q, k, v, [0.0], N, LINEAR, M0, z0)
    phik = np.where(k[0, 0] > 0, k[0, 0] + 1.0, np.exp(np.minimum(k[0, 0], 0)))
    assert np.allclose(M[0, 0], M0[0, 0] + phik.T @ v[0, 0], rtol=1e-12, atol=1e-12)
    assert np.allclose(z[0, 0], z0[0, 0] + phik.sum(0), rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------
# sigma = ELU + 1 against its textbook definition and a library ELU
# ----------------------------------------------------------------------------
def test_sigma_matches_elu_plus_one():
    import torch
    x = np.concatenate([rand(1000) * 5, [0.0, -0.0, 1e-300, -1e-300, -50.0, 50.0]])
    ref = torch.nn.functional.elu(torch.from_numpy(x), alpha=1.0).numpy() + 1.0
    assert np.max(np.abs(oracle.sigma(x) - ref)) <= 1e-15 * np.max(np.abs(ref))
    assert oracle.sigma(np.array([0.0]))[0] == 1.0
    assert np.all(oracle.sigma(x) > 0)


def test_gate_value_limits():
    assert oracle.gate_value(0.0) == 0.5
    assert oracle.gate_value(np.inf) == 1.0
    assert oracle.gate_value(-np.inf) == 0.0
    assert abs(oracle.gate_value(2.0) - 1 / (1 + math.exp(-2.0))) < 1e-16
    assert abs(oracle.gate_value(-2.0) - 1 / (1 + math.exp(2.0))) < 1e-16


# ----------------------------------------------------------------------------
# P3: gate limits
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("mode", [LINEAR, DELTA])
def test_p3_gate_limits(mode):
    B, H, L, d, N = 1, 2, 12, 4, 4
    q, k, v = rand(B, H, L, d), rand(B, H, L, d), rand(B, H, L, d)
    # beta -> -inf: pure local causal attention, segment by segment
    out, _, _ = oracle.forward(q, k, v, [-np.inf, -40.0], N, mode)
    for h in range(H):
        for s0 in range(0, L, N):
            ref = brute_attention(q[0, h, s0:s0 + N], k[0, h, s0:s0 + N], v[0, h, s0:s0 + N])
            assert np.max(np.abs(out[0, h, s0:s0 + N] - ref)) <= 1e-12
    # beta -> +inf: pure memory retrieval, exactly 0 in the first segment
    out, _, _ = oracle.forward(q, k, v, [np.inf, 40.0], N, mode)
    assert np.all(out[0, 0, :N] == 0.0)
    assert np.max(np.abs(out[0, 1, :N])) < 1e-15
    # retrieval against an independent per-row loop with the running state
    for h in range(H):
        M = np.zeros((d, d))
        z = np.zeros(d)
        for s0 in range(0, L, N):
            for i in range(s0, s0 + N):
                fq = [oracle.sigma(np.array([x]))[0] for x in q[0, h, i]]
                den = sum(fq[a] * z[a] for a in range(d))
                for c in range(d):
                    num = sum(fq[a] * M[a, c] for a in range(d))
                    ref = num / den if den != 0 else 0.0
                    assert abs(out[0, h, i, c] - ref) <= 1e-12 * max(1, abs(ref)) + 1e-15
            fk = oracle.sigma(k[0, h, s0:s0 + N])
            if mode == LINEAR:
                M = M + fk.T @ v[0, h, s0:s0 + N]
            else:
                dk = fk @ z
                R = np.zeros((N, d))
                for t in range(N):
                    if dk[t] != 0:
                        R[t] = (fk[t] @ M) / dk[t]
                M = M + fk.T @ (v[0, h, s0:s0 + N] - R)
            z = z + fk.sum(0)


# ----------------------------------------------------------------------------
# P4: delta fixed point
# ----------------------------------------------------------------------------
def test_p4_delta_fixed_point():
    d, N = 5, 6
    q1, k1, v1 = rand(N, d), rand(N, d), rand(N, d)
    _, M1, z1 = oracle.head_forward(q1, k1, v1, 0.5, N, DELTA)
    assert np.all(z1 > 0)
    k2 = rand(N, d)
    fk2 = oracle.sigma(k2)
    v2 = (fk2 @ M1) / (fk2 @ z1)[:, None]         # bindings already in the memory
    q2 = rand(N, d)
    _, M2, z2 = oracle.head_forward(q2, k2, v2, 0.5, N, DELTA, M1, z1)
    assert np.linalg.norm(M2 - M1) <= 1e-12 * np.linalg.norm(M1)
    assert np.allclose(z2, z1 + fk2.sum(0), rtol=1e-14, atol=0)
    # the Linear rule does change M on the same data
    _, M2l, _ = oracle.head_forward(q2, k2, v2, 0.5, N, LINEAR, M1, z1)
    assert np.linalg.norm(M2l - M1) > 1e-3 * np.linalg.norm(M1)


def test_p4_delta_first_segment_equals_linear():
    L, d = 16, 4
    q, k, v = rand(1, 1, L, d), rand(1, 1, L, d), rand(1, 1, L, d)
    o_l, M_l, z_l = oracle.forward(q, k, v, [0.2], L, LINEAR)
    o_d, M_d, z_d = oracle.forward(q, k, v, [0.2], L, DELTA)
    assert np.array_equal(o_l, o_d)
    assert np.array_equal(M_l, M_d) and np.array_equal(z_l, z_d)


# ----------------------------------------------------------------------------
# P5: hand-computed worked example (tests/golden/worked_example_d2.txt)
# ----------------------------------------------------------------------------
def load_golden(path):
    vals = {}
    w = 1.0 / (1.0 + math.exp(-1.0 / math.sqrt(2.0)))
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, rhs = [s.strip() for s in line.split("=", 1)]
            vals[key] = np.array([eval(t, {"w": w}) for t in rhs.split(",")], dtype=np.float64)
    return vals


def test_p5_worked_example(golden_dir):
    g = load_golden(os.path.join(golden_dir, "worked_example_d2.txt"))
    d = int(g["d"][0])
    q = g["q"].reshape(1, 1, 2, d)
    k = g["k"].reshape(1, 1, 2, d)
    v = g["v"].reshape(1, 1, 2, d)
    beta = [g["beta"][0]]
    for mode, tag in ((LINEAR, "linear"), (DELTA, "delta")):
        out, M, z = oracle.forward(q, k, v, beta, 1, mode)
        assert np.allclose(out.ravel(), g["N1.out"], rtol=0, atol=1e-14)
        assert np.allclose(M.ravel(), g[f"N1.{tag}.M"], rtol=0, atol=1e-14)
        assert np.allclose(z.ravel(), g[f"N1.{tag}.z"], rtol=0, atol=1e-14)
        out, M, z = oracle.forward(q, k, v, beta, 2, mode)
        assert np.allclose(out.ravel(), g["N2.out"], rtol=0, atol=1e-14)
        assert np.allclose(M.ravel(), g["N2.M"], rtol=0, atol=1e-14)
        assert np.allclose(z.ravel(), g["N2.z"], rtol=0, atol=1e-14)


# ----------------------------------------------------------------------------
# P6: stream equivalence (step with carried state == forward; split + resume)
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("mode", [LINEAR, DELTA])
def test_p6_stream_equivalence(mode):
    B, H, L, d, N = 2, 2, 24, 4, 6
    q, k, v = rand(B, H, L, d), rand(B, H, L, d), rand(B, H, L, d)
    beta = [0.4, -1.1]
    out, M, z = oracle.forward(q, k, v, beta, N, mode)
    Ms, zs = None, None
    outs = []
    for s0 in range(0, L, N):
        o, Ms, zs = oracle.step(q[:, :, s0:s0 + N], k[:, :, s0:s0 + N], v[:, :, s0:s0 + N],
                                beta, mode, Ms, zs)
        outs.append(o)
    assert np.array_equal(np.concatenate(outs, axis=2), out)
    assert np.array_equal(Ms, M) and np.array_equal(zs, z)
    o1, M1, z1 = oracle.forward(q[:, :, :12], k[:, :, :12], v[:, :, :12], beta, N, mode)
    o2, M2, z2 = oracle.forward(q[:, :, 12:], k[:, :, 12:], v[:, :, 12:], beta, N, mode, M1, z1)
    assert np.array_equal(np.concatenate([o1, o2], axis=2), out)
    assert np.array_equal(M2, M) and np.array_equal(z2, z)


def test_ragged_tail_is_a_short_segment():
    L, d, N = 10, 3, 4
    q, k, v = rand(1, 1, L, d), rand(1, 1, L, d), rand(1, 1, L, d)
    for mode in (LINEAR, DELTA):
        out, M, z = oracle.forward(q, k, v, [0.1], N, mode)
        o1, M1, z1 = oracle.forward(q[:, :, :8], k[:, :, :8], v[:, :, :8], [0.1], N, mode)
        o2, M2, z2 = oracle.forward(q[:, :, 8:], k[:, :, 8:], v[:, :, 8:], [0.1], 2, mode, M1, z1)
        assert np.array_equal(out, np.concatenate([o1, o2], axis=2))
        assert np.array_equal(M, M2) and np.array_equal(z, z2)


def test_empty_sequence_passes_state_through():
    M0, z0 = rand(1, 1, 3, 3), np.abs(rand(1, 1, 3))
    e = np.zeros((1, 1, 0, 3))
    out, M, z = oracle.forward(e, e, e, [0.0], 4, DELTA, M0, z0)
    assert out.shape == (1, 1, 0, 3)
    assert np.array_equal(M, M0) and np.array_equal(z, z0)


# ----------------------------------------------------------------------------
# P7: N = 1, Linear, g = 1 is causal kernel linear attention with exclusive prefix
# ----------------------------------------------------------------------------
def test_p7_causal_linear_attention():
    L, d = 20, 5
    q, k, v = rand(L, d), rand(L, d), rand(L, d)
    out, _, _ = oracle.head_forward(q, k, v, 1.0, 1, LINEAR)
    S = np.zeros((d, d))
    Z = np.zeros(d)
    for t in range(L):
        fq = np.array([x + 1 if x > 0 else math.exp(x) for x in q[t]])
        den = float(fq @ Z)
        ref = np.zeros(d) if den == 0 else (fq @ S) / den
        assert np.max(np.abs(out[t] - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))
        fk = np.array([x + 1 if x > 0 else math.exp(x) for x in k[t]])
        S += np.outer(fk, v[t])
        Z += fk


# ----------------------------------------------------------------------------
# Planted mistakes: each plausible bug in the oracle must fail at least one pin.
# ----------------------------------------------------------------------------
def _worked_example_ok(fwd):
    g = load_golden(os.path.join(os.path.dirname(__file__), "golden", "worked_example_d2.txt"))
    q = g["q"].reshape(1, 1, 2, 2)
    k = g["k"].reshape(1, 1, 2, 2)
    v = g["v"].reshape(1, 1, 2, 2)
    ok = True
    for mode, tag in ((LINEAR, "linear"), (DELTA, "delta")):
        out, M, z = fwd(q, k, v, [0.0], 1, mode)
        ok &= np.allclose(out.ravel(), g["N1.out"], atol=1e-12)
        ok &= np.allclose(M.ravel(), g[f"N1.{tag}.M"], atol=1e-12)
        out, M, z = fwd(q, k, v, [0.0], 2, mode)
        ok &= np.allclose(out.ravel(), g["N2.out"], atol=1e-12)
    return bool(ok)


@pytest.mark.parametrize("bug", ["transpose_M", "update_before_read", "delta_sign",
                                 "scale_d", "mask_excl_diag", "gate_swapped",
                                 "den_from_M_sum", "elu_no_plus_one"])
def test_planted_mistakes_are_caught(monkeypatch, bug):
    import oracle as o
    assert _worked_example_ok(o.forward)
    if bug == "transpose_M":
        orig = o.retrieve
        monkeypatch.setattr(o, "retrieve", lambda p, M, z: orig(p, M.T, z))
    elif bug == "update_before_read":
        def seg(q, k, v, M, z, g, mode):
            pk = o.sigma(k)
            M2, z2 = (o.update_linear if mode == LINEAR else o.update_delta)(pk, v, M, z)
            out = g * o.retrieve(o.sigma(q), M2, z2) + (1 - g) * o.local_attention(q, k, v)
            return out, M2, z2
        monkeypatch.setattr(o, "segment", seg)
    elif bug == "delta_sign":
        monkeypatch.setattr(o, "update_delta", lambda pk, v, M, z: (
            M + pk.T @ (v + o.retrieve(pk, M, z)), z + pk.sum(0)))
    elif bug == "scale_d":
        def att(q, k, v):
            n, d = q.shape
            s = np.where(np.triu(np.ones((n, n), bool), 1), -np.inf, (q @ k.T) / d)
            w = np.exp(s - s.max(1, keepdims=True))
            return (w @ v) / w.sum(1, keepdims=True)
        monkeypatch.setattr(o, "local_attention", att)
    elif bug == "mask_excl_diag":
        def att(q, k, v):
            n, d = q.shape
            s = np.where(np.triu(np.ones((n, n), bool), 0), -1e300, (q @ k.T) / np.sqrt(d))
            w = np.exp(s - s.max(1, keepdims=True))
            return (w @ v) / w.sum(1, keepdims=True)
        monkeypatch.setattr(o, "local_attention", att)
    elif bug == "gate_swapped":
        monkeypatch.setattr(o, "gate_value", lambda b: 1.0 / (1.0 + np.exp(b)))
    elif bug == "den_from_M_sum":
        monkeypatch.setattr(o, "retrieve", lambda p, M, z: np.nan_to_num(
            (p @ M) / (p @ M.sum(1))[:, None]))
    elif bug == "elu_no_plus_one":
        monkeypatch.setattr(o, "sigma", lambda x: np.where(np.asarray(x) > 0, x, np.exp(np.minimum(x, 0)) - 1))
    assert not (_worked_example_ok(o.forward) and _gate_limit_ok(o.forward))


def _gate_limit_ok(fwd):
    """P3 in miniature: beta = +inf retrieves exactly 0 in the first segment and
    beta = -inf gives plain causal attention."""
    q, k, v = rand(1, 1, 4, 3), rand(1, 1, 4, 3), rand(1, 1, 4, 3)
    out, _, _ = fwd(q, k, v, [np.inf], 2, LINEAR)
    ok = bool(np.all(out[0, 0, :2] == 0.0))
    out, _, _ = fwd(q, k, v, [-np.inf], 4, LINEAR)
    return ok and np.allclose(out[0, 0], brute_attention(q[0, 0], k[0, 0], v[0, 0]), atol=1e-12)
