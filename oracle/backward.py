"""fp64 CPU oracle for the gradient of the Infini-attention forward.

TEST INFRASTRUCTURE ONLY, like the rest of this package: only the test suite, the
smoke check in ``__graft_entry__`` and the CPU legs of ``bench.py`` may use it; the
CUDA library shares no code with it.

The forward it differentiates is the one in ``oracle/__init__.py`` ("Leave No
Context Behind", arXiv 2404.07143, as quoted on llm-papers-study.pages.dev:
sections 3.1, 3.3, 3.4, 3.5, 3.8). The pages give no backward pass; this is the
chain rule applied to each forward step in reverse order, one function per step,
each the exact derivative of the step it names (no approximation). Conventions:

  * the loss is L = sum(dout * out) + sum(dM_out * M_S) + sum(dz_out * z_S), so the
    upstream gradients are dout [B,H,L,d], dM_out [B,H,d,d] and dz_out [B,H,d]
    (None: zero);
  * a row whose retrieval denominator is exactly 0 retrieves the constant 0 (the
    forward's zero-state rule), so no gradient flows through that row's retrieval
    (nor through the Delta term of a key row with a zero denominator);
  * sigma'(x) = 1 for x > 0 and exp(x) otherwise (ELU + 1 is continuously
    differentiable, both sides give 1 at 0);
  * beta's gradient is summed over the batch (beta has one value per head).

Pinned in ``tests/test_oracle_backward_pins.py`` by central finite differences of
the (separately pinned) forward oracle on small inputs.
"""
from __future__ import annotations

import numpy as np

from . import DELTA, LINEAR, gate_value, local_attention, retrieve, sigma


def dsigma(x: np.ndarray) -> np.ndarray:
    """Derivative of sigma = ELU + 1 (section 3.3): 1 for x > 0, exp(x) otherwise."""
    x = np.asarray(x, dtype=np.float64)
    return np.where(x > 0.0, 1.0, np.exp(np.minimum(x, 0.0)))


def local_attention_backward(q, k, v, da):
    """Gradient of A_dot = softmax(Q K^T / sqrt(d) + causal mask) V (section 3.1) for
    one head and one segment, given dA_dot. Returns (dq, dk, dv)."""
    n, d = q.shape
    c = 1.0 / np.sqrt(d)
    scores = (q @ k.T) * c
    future = np.triu(np.ones((n, n), dtype=bool), k=1)
    scores = np.where(future, -np.inf, scores)
    scores = scores - scores.max(axis=1, keepdims=True)
    w = np.exp(scores)
    p = w / w.sum(axis=1, keepdims=True)          # softmax rows
    dp = da @ v.T                                 # dL/dP
    dv = p.T @ da
    ds = p * (dp - (dp * p).sum(axis=1, keepdims=True))  # softmax Jacobian, row by row
    dq = (ds @ k) * c
    dk = (ds.T @ q) * c
    return dq, dk, dv


def retrieve_backward(phi, M, z, da):
    """Gradient of A = phi M / (phi z) row by row (section 3.3; rows with a zero
    denominator are the constant 0), given dA. Returns (dphi, dM, dz)."""
    num = phi @ M
    den = phi @ z
    nz = den != 0.0
    inv = np.zeros_like(den)
    inv[nz] = 1.0 / den[nz]
    a = num * inv[:, None]
    dnum = da * inv[:, None]                      # dL/d(num)
    dden = -(da * a).sum(axis=1) * inv            # dL/d(den)
    dphi = dnum @ M.T + dden[:, None] * z[None, :]
    return dphi, phi.T @ dnum, phi.T @ dden


def update_backward(phi_k, v, M, z, dM_new, dz_new, mode):
    """Gradient of one memory update (section 3.4) given the gradients of the new
    state. Returns (dphi_k, dv, dM_old, dz_old)."""
    if mode == LINEAR:
        # M_s = M_{s-1} + phi^T V ; z_s = z_{s-1} + sum_t phi_t
        dphi = v @ dM_new.T + dz_new[None, :]
        return dphi, phi_k @ dM_new, dM_new.copy(), dz_new.copy()
    if mode == DELTA:
        # M_s = M_{s-1} + phi^T (V - R), R = phi M_{s-1} / (phi z_{s-1})
        r = retrieve(phi_k, M, z)
        du = phi_k @ dM_new                       # dL/d(V - R)
        dphi = (v - r) @ dM_new.T + dz_new[None, :]
        dphi_r, dM_r, dz_r = retrieve_backward(phi_k, M, z, -du)
        return dphi + dphi_r, du, dM_new + dM_r, dz_new + dz_r
    raise ValueError(f"unknown mode {mode}")


def head_backward(q, k, v, beta_h, N, mode, dout, M0=None, z0=None, dM_end=None, dz_end=None):
    """One head's gradient over its [L, d] sequence in segments of N (the last one
    may be shorter). Returns (dq, dk, dv, dbeta_h, dM0, dz0)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    L, d = q.shape
    g = gate_value(beta_h)
    M = np.zeros((d, d)) if M0 is None else np.array(M0, dtype=np.float64)
    z = np.zeros(d) if z0 is None else np.array(z0, dtype=np.float64)
    # forward over the segments, keeping the state each segment reads
    bounds = [(s0, min(s0 + N, L)) for s0 in range(0, L, N)]
    states = []
    for s0, s1 in bounds:
        states.append((M, z))
        phi_k = sigma(k[s0:s1])
        if mode == LINEAR:
            M, z = M + phi_k.T @ v[s0:s1], z + phi_k.sum(axis=0)
        else:
            M, z = M + phi_k.T @ (v[s0:s1] - retrieve(phi_k, M, z)), z + phi_k.sum(axis=0)
    dM = np.zeros((d, d)) if dM_end is None else np.array(dM_end, dtype=np.float64)
    dz = np.zeros(d) if dz_end is None else np.array(dz_end, dtype=np.float64)
    dq = np.zeros((L, d))
    dk = np.zeros((L, d))
    dv = np.zeros((L, d))
    dg = 0.0
    for (s0, s1), (Ms, zs) in reversed(list(zip(bounds, states))):
        qs, ks, vs, do = q[s0:s1], k[s0:s1], v[s0:s1], dout[s0:s1]
        phi_q, phi_k = sigma(qs), sigma(ks)
        a_dot = local_attention(qs, ks, vs)
        a_mem = retrieve(phi_q, Ms, zs)
        # gate (section 3.5): out = g A_mem + (1 - g) A_dot
        dg += float((do * (a_mem - a_dot)).sum())
        dq_a, dk_a, dv_a = local_attention_backward(qs, ks, vs, (1.0 - g) * do)
        dphi_q, dM_q, dz_q = retrieve_backward(phi_q, Ms, zs, g * do)
        dphi_k, dv_u, dM_prev, dz_prev = update_backward(phi_k, vs, Ms, zs, dM, dz, mode)
        dq[s0:s1] = dq_a + dphi_q * dsigma(qs)
        dk[s0:s1] = dk_a + dphi_k * dsigma(ks)
        dv[s0:s1] = dv_a + dv_u
        dM = dM_prev + dM_q
        dz = dz_prev + dz_q
    return dq, dk, dv, dg * g * (1.0 - g), dM, dz


def backward(q, k, v, beta, N, mode, dout, M_in=None, z_in=None, dM_out=None, dz_out=None,
             heads=None):
    """Gradient of the whole-sequence forward for [B, H, L, d] inputs (heads are
    independent, section 3.6). Returns (dq, dk, dv [B,H,L,d], dbeta [H], dM_in
    [B,H,d,d], dz_in [B,H,d]) in float64; dbeta sums over the batch rows evaluated.
    heads: optional list of (b, h) to evaluate; the others are left as zeros."""
    q = np.asarray(q, dtype=np.float64)
    B, H, L, d = q.shape
    dq = np.zeros((B, H, L, d))
    dk = np.zeros((B, H, L, d))
    dv = np.zeros((B, H, L, d))
    dbeta = np.zeros(H)
    dM = np.zeros((B, H, d, d))
    dz = np.zeros((B, H, d))
    todo = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    for b, h in todo:
        r = head_backward(q[b, h], k[b, h], v[b, h], beta[h], N, mode, dout[b, h],
                          None if M_in is None else M_in[b, h],
                          None if z_in is None else z_in[b, h],
                          None if dM_out is None else dM_out[b, h],
                          None if dz_out is None else dz_out[b, h])
        dq[b, h], dk[b, h], dv[b, h] = r[0], r[1], r[2]
        dbeta[h] += r[3]
        dM[b, h], dz[b, h] = r[4], r[5]
    return dq, dk, dv, dbeta, dM, dz
