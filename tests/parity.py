"""Shared helpers for the GPU-vs-oracle parity tests.

Tolerances (written here once, used by every parity test):
  bf16 inputs, fp32 accumulation:
    out: max-abs error <= 2e-2 and relative Frobenius error <= 5e-3
    M, z: relative Frobenius error <= 1e-3
  fp32 inputs: relative error <= 1e-4 (Frobenius, and max-abs relative to the
    largest reference magnitude) on out, M and z.
"""
import numpy as np
import torch

import oracle

BF16_OUT_MAXABS = 2e-2
BF16_OUT_RELF = 5e-3
BF16_STATE_RELF = 1e-3
F32_REL = 1e-4


def f64(t):
    return None if t is None else t.detach().to("cpu", torch.float64).numpy()


def relf(got, ref):
    den = np.linalg.norm(ref)
    num = np.linalg.norm(got - ref)
    return num / den if den > 0 else num


def run_oracle(inp, N, mode, M_in=None, z_in=None, heads=None):
    return oracle.forward(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["beta"]), N, mode,
                          f64(M_in), f64(z_in), heads=heads)


def check_bf16(out, M, z, ref, heads=None, what=""):
    r_out, r_M, r_z = ref
    o = f64(out)
    Mg, zg = f64(M), f64(z)
    if heads is not None:
        idx = tuple(np.array(heads).T)
        o, r_out = o[idx], r_out[idx]
        Mg, r_M, zg, r_z = Mg[idx], r_M[idx], zg[idx], r_z[idx]
    assert np.all(np.isfinite(o)), f"{what}: non-finite output"
    maxabs = float(np.max(np.abs(o - r_out))) if o.size else 0.0
    rf = relf(o, r_out)
    assert maxabs <= BF16_OUT_MAXABS, f"{what}: out max-abs {maxabs:.3e}"
    assert rf <= BF16_OUT_RELF, f"{what}: out rel-F {rf:.3e}"
    if M is not None:
        rM, rz = relf(Mg, r_M), relf(zg, r_z)
        assert rM <= BF16_STATE_RELF, f"{what}: M rel-F {rM:.3e}"
        assert rz <= BF16_STATE_RELF, f"{what}: z rel-F {rz:.3e}"
    return maxabs, rf


def check_f32(out, M, z, ref, what=""):
    for name, g, r in (("out", f64(out), ref[0]), ("M", f64(M), ref[1]), ("z", f64(z), ref[2])):
        if g is None:
            continue
        assert np.all(np.isfinite(g)), f"{what}: non-finite {name}"
        scale = max(1.0, float(np.max(np.abs(r)))) if r.size else 1.0
        err = float(np.max(np.abs(g - r))) if r.size else 0.0
        assert err <= F32_REL * scale, f"{what}: {name} max-abs {err:.3e} (scale {scale:.3e})"
        assert relf(g, r) <= F32_REL, f"{what}: {name} rel-F {relf(g, r):.3e}"
