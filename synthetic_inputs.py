"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module only draws random numbers; it holds none of the layer's arithmetic.
Both the CUDA path and the fp64 oracle consume what it produces.

Recipe (the same for every workload):
  * Q, K, V are i.i.d. N(0, 1), drawn in float32 by a torch.Generator seeded with
    ``seed * 16 + tensor_id`` (q = 0, k = 1, v = 2, beta = 3), then rounded to the
    working dtype (bf16 by round-to-nearest-even, or kept in fp32);
  * beta is one value per head: an explicit list when given, otherwise N(0, 1);
  * small cases are drawn on the CPU generator and copied to the device; the full
    benchmark sizes are drawn on the device generator, and the oracle reads the
    sampled heads back to the host. Either way the oracle sees exactly the values
    the kernels see (bf16 -> float64 is exact).
"""
from __future__ import annotations

import torch

TENSOR_Q, TENSOR_K, TENSOR_V, TENSOR_BETA = 0, 1, 2, 3


def _gen(device, seed, tensor_id):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 16 + tensor_id)
    return g


def normal(shape, dtype, seed, tensor_id, device="cpu"):
    """i.i.d. N(0,1) float32 draws rounded to ``dtype``."""
    x = torch.randn(shape, generator=_gen(device, seed, tensor_id), device=device,
                    dtype=torch.float32)
    return x.to(dtype)


def make_inputs(B, H, L, d, dtype=torch.bfloat16, seed=0, device="cpu", beta=None,
                gen_device=None):
    """Return dict(q, k, v, beta) with q/k/v [B, H, L, d] and beta [H] float32.

    gen_device: where the generator runs (default: ``device``). Drawing on the CPU
    and moving to ``device`` gives the same values on every machine.
    """
    gd = device if gen_device is None else gen_device
    shape = (B, H, L, d)
    q = normal(shape, dtype, seed, TENSOR_Q, gd).to(device)
    k = normal(shape, dtype, seed, TENSOR_K, gd).to(device)
    v = normal(shape, dtype, seed, TENSOR_V, gd).to(device)
    if beta is None:
        b = normal((H,), torch.float32, seed, TENSOR_BETA, gd).to(device)
    else:
        b = torch.as_tensor(beta, dtype=torch.float32).to(device)
    return {"q": q.contiguous(), "k": k.contiguous(), "v": v.contiguous(), "beta": b}


def normal_state(B, H, d, seed, scale_M=1.0, scale_z=1.0, device="cpu"):
    """A non-zero carried state (M, z) for resume/step tests: M ~ N(0, scale_M),
    z ~ scale_z * (1 + |N(0,1)|) so that every denominator is positive."""
    M = normal((B, H, d, d), torch.float32, seed, 5, "cpu") * scale_M
    z = (1.0 + normal((B, H, d), torch.float32, seed, 6, "cpu").abs()) * scale_z
    return M.to(device).contiguous(), z.to(device).contiguous()
