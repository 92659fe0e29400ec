"""fp64 CPU oracle for the Infini-attention forward pass.

TEST INFRASTRUCTURE ONLY. This package is the slow, plain, obviously correct
statement of what the layer computes. Only the test suite, the smoke check in
``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may import it. The
product path (the CUDA library and its Python binding) never imports or calls
anything here, and this package shares no code with it.

Source: "Leave No Context Behind: Efficient Infinite Context Transformers with
Infini-attention" (Munkhdalai, Faruqui, Golovnev; arXiv 2404.07143), as quoted on
the close-reading note llm-papers-study.pages.dev ("精读笔记：Infini-attention"),
sections 3.1 (scaled dot-product attention), 3.3 (memory retrieval), 3.4 (Linear
and Linear+Delta memory update), 3.5 (long-term context injection / gate), 3.6
(multi-head memories) and 3.8 (per-segment forward summary); and the book chapter
waylandz.com "第24章 Sparse与Infinite Attention", section 24.5 (read-then-write
order inside one segment).

Every step is evaluated in float64 with numpy. Matrix products use ``@`` (a
library matmul) as a single step; nothing is blocked, fused or reordered beyond
what the equations state.

Readings of points the pages leave open:
  * softmax scale is 1/sqrt(d_key) of the head (section 3.1 prints sqrt(d_model);
    the section 3.8 summary and the book's SDPA call use the head width);
  * the causal mask is inside the segment and includes the diagonal;
  * sigma = ELU + 1 with ELU's alpha = 1;
  * retrieval divides each row of sigma(Q) M by the scalar sigma(Q) z of that row;
  * a row whose denominator is exactly 0 (the zero state, e.g. the first segment
    with M_0 = 0, z_0 = 0) retrieves 0; the gate is still applied;
  * the Delta term uses the pre-update M_{s-1}, z_{s-1} for the whole segment and
    is dropped (R = 0) on rows whose denominator is exactly 0;
  * z is updated the same way in both modes;
  * beta has one value per head, shared across the batch;
  * a final segment shorter than N (L not a multiple of N) is processed as a
    segment of its own length.

Every function here is pinned by tests under ``tests/test_oracle_pins.py``
(brute force, closed forms, invariants, gate limits, delta fixed point and a
hand-computed worked example); no function is "parity unpinned".
"""
from __future__ import annotations

import numpy as np

LINEAR = 0
DELTA = 1


def sigma(x: np.ndarray) -> np.ndarray:
    """ELU(x) + 1 with alpha = 1: x + 1 for x > 0, exp(x) otherwise (section 3.3)."""
    x = np.asarray(x, dtype=np.float64)
    return np.where(x > 0.0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def gate_value(beta: float) -> float:
    """sigmoid(beta) in float64, stable for beta = +-inf (section 3.5)."""
    b = float(beta)
    if b >= 0.0:
        return 1.0 / (1.0 + np.exp(-b))
    e = np.exp(b)
    return e / (1.0 + e)


def local_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """A_dot = softmax(Q K^T / sqrt(d) + causal mask) V for one head and one segment.

    Section 3.1 equation for A_dot, with the causal mask of the section 3.8 summary
    (token i attends to tokens j <= i of its own segment).
    """
    n, d = q.shape
    scores = (q @ k.T) / np.sqrt(d)
    future = np.triu(np.ones((n, n), dtype=bool), k=1)
    scores = np.where(future, -np.inf, scores)
    scores = scores - scores.max(axis=1, keepdims=True)
    w = np.exp(scores)
    return (w @ v) / w.sum(axis=1, keepdims=True)


def retrieve(phi_x: np.ndarray, M: np.ndarray, z: np.ndarray) -> np.ndarray:
    """sigma(X) M / (sigma(X) z), row by row; rows with a zero denominator give 0.

    Section 3.3 (A_mem) when phi_x = sigma(Q); the same expression with sigma(K) is
    the retrieved value inside the Linear+Delta update of section 3.4.
    """
    num = phi_x @ M
    den = phi_x @ z
    out = np.zeros_like(num)
    nz = den != 0.0
    out[nz] = num[nz] / den[nz][:, None]
    return out


def update_linear(phi_k, v, M, z):
    """M_s = M_{s-1} + sigma(K)^T V ; z_s = z_{s-1} + sum_t sigma(K_t) (section 3.4)."""
    return M + phi_k.T @ v, z + phi_k.sum(axis=0)


def update_delta(phi_k, v, M, z):
    """M_s = M_{s-1} + sigma(K)^T (V - sigma(K) M_{s-1} / sigma(K) z_{s-1}) (section 3.4).

    z follows the Linear rule ("still tracking the same normalization term").
    """
    r = retrieve(phi_k, M, z)
    return M + phi_k.T @ (v - r), z + phi_k.sum(axis=0)


def segment(q, k, v, M, z, g, mode):
    """One head, one segment: read the old state, write the output, then update.

    Order as in the section 3.8 summary and the book's section 24.5: retrieval uses
    M_{s-1}, z_{s-1}; the update happens after the output is formed.
    Returns (out, M_s, z_s).
    """
    phi_q = sigma(q)
    a_dot = local_attention(q, k, v)
    a_mem = retrieve(phi_q, M, z)
    out = g * a_mem + (1.0 - g) * a_dot
    phi_k = sigma(k)
    if mode == LINEAR:
        M, z = update_linear(phi_k, v, M, z)
    elif mode == DELTA:
        M, z = update_delta(phi_k, v, M, z)
    else:
        raise ValueError(f"unknown mode {mode}")
    return out, M, z


def head_forward(q, k, v, g, N, mode, M0=None, z0=None):
    """Stream one head's [L, d] sequence through segments of N tokens (section 3.4:
    the new state is passed on to the next segment). Returns (out, M, z)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    L, d = q.shape
    M = np.zeros((d, d)) if M0 is None else np.array(M0, dtype=np.float64)
    z = np.zeros(d) if z0 is None else np.array(z0, dtype=np.float64)
    out = np.zeros((L, d))
    for s0 in range(0, L, N):
        s1 = min(s0 + N, L)
        out[s0:s1], M, z = segment(q[s0:s1], k[s0:s1], v[s0:s1], M, z, g, mode)
    return out, M, z


def forward(q, k, v, beta, N, mode, M_in=None, z_in=None, heads=None):
    """Whole-sequence forward for [B, H, L, d] inputs, heads independent (section 3.6).

    beta: [H]. M_in: [B, H, d, d] or None (zero state). z_in: [B, H, d] or None.
    heads: optional list of (b, h) to evaluate; the others are left as zeros.
    Returns (out [B,H,L,d], M_out [B,H,d,d], z_out [B,H,d]) in float64.
    """
    q = np.asarray(q, dtype=np.float64)
    B, H, L, d = q.shape
    out = np.zeros((B, H, L, d))
    M_out = np.zeros((B, H, d, d))
    z_out = np.zeros((B, H, d))
    todo = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    for b, h in todo:
        g = gate_value(beta[h])
        out[b, h], M_out[b, h], z_out[b, h] = head_forward(
            q[b, h], k[b, h], v[b, h], g, N, mode,
            None if M_in is None else M_in[b, h],
            None if z_in is None else z_in[b, h])
    return out, M_out, z_out


def step(q, k, v, beta, mode, M_in=None, z_in=None, heads=None):
    """One segment with carried state: the forward over a sequence of length N == L."""
    L = np.asarray(q).shape[2]
    return forward(q, k, v, beta, max(L, 1), mode, M_in, z_in, heads)
