"""Pins for the fp64 backward oracle: every gradient it returns must equal a central
finite difference of the forward oracle (itself pinned in test_oracle_pins.py) for
the loss sum(dout * out) + sum(dM_out * M_S) + sum(dz_out * z_S). Small shapes with
several segments and a ragged last one, both update rules, a carried state, and the
zero state (whose first segment retrieves the constant 0). Planted mistakes in the
backward (a dropped term, a wrong sign) must fail the same check."""
import numpy as np
import pytest

import oracle
import oracle.backward as ob
from oracle import DELTA, LINEAR

H_FD = 1e-6


def make_case(seed, B=1, H=2, L=7, d=4, state=True):
    rng = np.random.default_rng(seed)
    q, k, v = (rng.standard_normal((B, H, L, d)) for _ in range(3))
    beta = rng.standard_normal(H)
    dout = rng.standard_normal((B, H, L, d))
    dM_out = rng.standard_normal((B, H, d, d))
    dz_out = rng.standard_normal((B, H, d))
    M_in = rng.standard_normal((B, H, d, d)) if state else None
    z_in = (np.abs(rng.standard_normal((B, H, d))) + 0.5) if state else None
    return dict(q=q, k=k, v=v, beta=beta, dout=dout, dM_out=dM_out, dz_out=dz_out,
                M_in=M_in, z_in=z_in)


def loss(c, N, mode):
    out, M, z = oracle.forward(c["q"], c["k"], c["v"], c["beta"], N, mode, c["M_in"], c["z_in"])
    return float((c["dout"] * out).sum() + (c["dM_out"] * M).sum() + (c["dz_out"] * z).sum())


def fd_grad(c, name, N, mode):
    """Central differences of the loss with respect to every element of c[name]."""
    x = c[name]
    g = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        idx = it.multi_index
        x0 = x[idx]
        x[idx] = x0 + H_FD
        lp = loss(c, N, mode)
        x[idx] = x0 - H_FD
        lm = loss(c, N, mode)
        x[idx] = x0
        g[idx] = (lp - lm) / (2 * H_FD)
    return g


def analytic(c, N, mode, fn=ob.backward):
    return fn(c["q"], c["k"], c["v"], c["beta"], N, mode, c["dout"], c["M_in"], c["z_in"],
              c["dM_out"], c["dz_out"])


def close(a, b):
    scale = max(1.0, float(np.max(np.abs(b))))
    return float(np.max(np.abs(a - b))) <= 1e-6 * scale


@pytest.mark.parametrize("mode", [LINEAR, DELTA])
@pytest.mark.parametrize("N", [3, 7])
def test_gradients_match_finite_differences(mode, N):
    """N = 3: segments 3, 3, 1 (a ragged last one); N = 7: one segment."""
    c = make_case(seed=100 + N + 10 * mode)
    dq, dk, dv, dbeta, dM, dz = analytic(c, N, mode)
    for name, got in (("q", dq), ("k", dk), ("v", dv), ("beta", dbeta), ("M_in", dM),
                      ("z_in", dz)):
        ref = fd_grad(c, name, N, mode)
        assert close(got, ref), f"d{name} mode={mode} N={N}"


@pytest.mark.parametrize("mode", [LINEAR, DELTA])
def test_gradients_zero_state(mode):
    """M_0 = z_0 = 0: the first segment retrieves the constant 0 and its Delta term is
    dropped. The state input is given as explicit zeros so that dM_in can be checked
    too (z_in is not: the zero-denominator rule makes the loss jump when z leaves 0)."""
    c = make_case(seed=7 + mode, H=1, L=8, state=False)
    d = c["q"].shape[-1]
    c["M_in"] = np.zeros((1, 1, d, d))
    c["z_in"] = np.zeros((1, 1, d))
    dq, dk, dv, dbeta, dM, _ = analytic(c, 4, mode)
    for name, got in (("q", dq), ("k", dk), ("v", dv), ("beta", dbeta), ("M_in", dM)):
        assert close(got, fd_grad(c, name, 4, mode)), f"d{name} mode={mode}"
    # the same call with the state omitted (None) gives the same gradients
    c2 = dict(c, M_in=None, z_in=None)
    r2 = analytic(c2, 4, mode)
    for a, b in zip((dq, dk, dv, dbeta, dM), r2[:5]):
        assert np.array_equal(a, b)


def test_gate_limit_gives_attention_gradient():
    """g = 0 (beta = -inf) and no state gradient: dq, dk, dv are those of plain causal
    softmax attention per segment, dM_in = 0."""
    c = make_case(seed=3, H=1, L=6)
    c["beta"] = np.array([-np.inf])
    c["dM_out"][:] = 0.0
    c["dz_out"][:] = 0.0
    dq, dk, dv, _, dM, dz = analytic(c, 3, LINEAR)
    for s0 in (0, 3):
        sl = slice(s0, s0 + 3)
        r = ob.local_attention_backward(c["q"][0, 0, sl], c["k"][0, 0, sl], c["v"][0, 0, sl],
                                        c["dout"][0, 0, sl])
        assert np.allclose(dq[0, 0, sl], r[0], rtol=0, atol=1e-13)
        assert np.allclose(dk[0, 0, sl], r[1], rtol=0, atol=1e-13)
        assert np.allclose(dv[0, 0, sl], r[2], rtol=0, atol=1e-13)
    assert np.count_nonzero(dM) == 0 and np.count_nonzero(dz) == 0


# ----------------------------------------------------------------------------
# planted mistakes: each variant must fail the finite-difference check
# ----------------------------------------------------------------------------
def _with_patch(monkeypatch, name, fn):
    monkeypatch.setattr(ob, name, fn)


def test_planted_dropped_denominator_term(monkeypatch):
    orig = ob.retrieve_backward

    def bad(phi, M, z, da):
        dphi, dM, dz = orig(phi, M, z, da)
        num = phi @ M
        den = phi @ z
        return (da / den[:, None]) @ M.T, dM, dz  # drops the d(den) term
    _with_patch(monkeypatch, "retrieve_backward", bad)
    c = make_case(seed=11)
    dq = analytic(c, 3, LINEAR)[0]
    assert not close(dq, fd_grad(c, "q", 3, LINEAR))


def test_planted_wrong_delta_sign(monkeypatch):
    orig = ob.update_backward

    def bad(phi_k, v, M, z, dM_new, dz_new, mode):
        r = oracle.retrieve(phi_k, M, z)
        du = phi_k @ dM_new
        dphi = (v + r) @ dM_new.T + dz_new[None, :]  # sign of R flipped
        dphi_r, dM_r, dz_r = ob.retrieve_backward(phi_k, M, z, -du)
        return dphi + dphi_r, du, dM_new + dM_r, dz_new + dz_r
    _with_patch(monkeypatch, "update_backward", bad)
    c = make_case(seed=12)
    dk = analytic(c, 3, DELTA)[1]
    assert not close(dk, fd_grad(c, "k", 3, DELTA))


def test_planted_missing_softmax_centering(monkeypatch):
    def bad(q, k, v, da):
        n, d = q.shape
        s = (q @ k.T) / np.sqrt(d)
        s = np.where(np.triu(np.ones((n, n), dtype=bool), k=1), -np.inf, s)
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        dp = da @ v.T
        ds = p * dp  # the row term of the softmax Jacobian is missing
        return ds @ k / np.sqrt(d), ds.T @ q / np.sqrt(d), p.T @ da
    _with_patch(monkeypatch, "local_attention_backward", bad)
    c = make_case(seed=13)
    dq = analytic(c, 3, LINEAR)[0]
    assert not close(dq, fd_grad(c, "q", 3, LINEAR))
