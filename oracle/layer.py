"""fp64 CPU oracle for one Infini-attention layer with its projections.

TEST INFRASTRUCTURE ONLY, like the rest of this package.

The layer ("Leave No Context Behind", arXiv 2404.07143, as quoted on
llm-papers-study.pages.dev, sections 3.1 and 3.6): the input rows x [B, L, D_model]
are projected to per-head queries, keys and values (Q = x W_Q, K = x W_K, V = x W_V;
H query heads and H_kv key/value heads of width d, heads laid side by side in the
projection's columns), the heads run the Infini-attention forward of
``oracle/__init__.py`` (grouped: query head h reads key/value head h // (H / H_kv)),
and the concatenated head outputs are projected back, y = [A_1 ... A_H] W_O. Every
matrix product is one library ``@`` step in float64.

Pinned in ``tests/test_oracle_layer_pins.py``: identity projections reduce the layer
to the (pinned) forward; the projections against explicit per-element loops on a
tiny case; grouped heads against repeating each key/value head's projection columns
for its query heads.
"""
from __future__ import annotations

import numpy as np

from . import forward


def project(x, W):
    """x [B, L, D_in] @ W [D_in, D_out] in float64."""
    return np.asarray(x, dtype=np.float64) @ np.asarray(W, dtype=np.float64)


def split_heads(t, heads, d):
    """[B, L, heads * d] -> [B, heads, L, d] (head h = columns [h d, h d + d))."""
    B, L, _ = t.shape
    return t.reshape(B, L, heads, d).transpose(0, 2, 1, 3)


def merge_heads(t):
    """[B, heads, L, d] -> [B, L, heads * d]."""
    B, heads, L, d = t.shape
    return t.transpose(0, 2, 1, 3).reshape(B, L, heads * d)


def layer_forward(x, Wq, Wk, Wv, Wo, beta, N, mode, H, H_kv, d, M_in=None, z_in=None):
    """y [B, L, D_model] and the final state (M, z) [B, H_kv, d, d] / [B, H_kv, d]."""
    q = split_heads(project(x, Wq), H, d)
    k = split_heads(project(x, Wk), H_kv, d)
    v = split_heads(project(x, Wv), H_kv, d)
    G = H // H_kv
    k_rep = np.repeat(k, G, axis=1)  # query head h reads key/value head h // G
    v_rep = np.repeat(v, G, axis=1)
    M_rep = None if M_in is None else np.repeat(np.asarray(M_in, dtype=np.float64), G, axis=1)
    z_rep = None if z_in is None else np.repeat(np.asarray(z_in, dtype=np.float64), G, axis=1)
    out, M, z = forward(q, k_rep, v_rep, beta, N, mode, M_rep, z_rep)
    y = project(merge_heads(out), Wo)
    # the state of a key/value head is the same at every query head of its group
    return y, M[:, ::G], z[:, ::G]
