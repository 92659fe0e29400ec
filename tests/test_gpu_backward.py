"""GPU parity of infini_attn_backward against the fp64 backward oracle
(oracle/backward.py, pinned by finite differences) on the same bf16 inputs.

Tolerances: dq, dk, dv are bf16 results of bf16 tensor-core products of rounded
operands (P, dS, sigma(Q), dnum, dM_s, U rounded to bf16: 2^-9 relative each) with
fp32 accumulation, then rounded to bf16 themselves; the flash-attention backward's
usual error at this precision is a few 1e-3 relative, so the bound is rel-F
<= 1e-2 and max-abs <= 3e-2 of the largest reference magnitude. dbeta is one sum
of ~1e5 such terms per head (relative 2e-2); the state gradients dM_in, dz_in are
fp32 sums over every segment of bf16 products (rel-F <= 1e-2)."""
import numpy as np
import pytest
import torch

import oracle.backward as ob
from parity import f64, relf
from synthetic_inputs import make_inputs, normal, normal_state

pytestmark = pytest.mark.gpu

LIN, DEL = 0, 1
GRAD_RELF = 1e-2
GRAD_MAXABS = 3e-2
DBETA_REL = 2e-2
STATE_GRAD_RELF = 1e-2


@pytest.fixture(scope="module")
def ia():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import compressive_memory_transformer_b200 as m
    assert m.device_status() == 0
    return m


def sync_ok(ia):
    torch.cuda.synchronize()
    assert ia.device_status() == 0, "a bounded device wait ran out"


def run(ia, B, H, L, N, mode, seed, beta=None, state=False, state_grad=False):
    inp = make_inputs(B, H, L, 128, torch.bfloat16, seed=seed, device="cuda", gen_device="cpu",
                      beta=beta)
    dout = normal((B, H, L, 128), torch.bfloat16, seed, 7).cuda()
    M0 = z0 = dM = dz = None
    if state:
        M0, z0 = normal_state(B, H, 128, seed=seed + 1, scale_M=3.0, scale_z=50.0, device="cuda")
    if state_grad:
        dM = (normal((B, H, 128, 128), torch.float32, seed, 8) * 0.05).cuda()
        dz = (normal((B, H, 128), torch.float32, seed, 9) * 0.05).cuda()
    got = ia.infini_attn_backward(inp["q"], inp["k"], inp["v"], inp["beta"], N, mode, dout,
                                  M0, z0, dM, dz)
    sync_ok(ia)
    c = lambda t: None if t is None else f64(t)
    ref = ob.backward(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["beta"]), N, mode,
                      f64(dout), c(M0), c(z0), c(dM), c(dz))
    return got, ref


def check(got, ref, what):
    for name, g, r in zip(("dq", "dk", "dv"), got[:3], ref[:3]):
        g = f64(g)
        rf = relf(g, r)
        ma = float(np.max(np.abs(g - r)))
        assert rf <= GRAD_RELF, f"{what}: {name} rel-F {rf:.3e}"
        assert ma <= GRAD_MAXABS * float(np.max(np.abs(r))), f"{what}: {name} max-abs {ma:.3e}"
    db = f64(got[3])
    assert np.all(np.abs(db - ref[3]) <= DBETA_REL * np.maximum(np.abs(ref[3]), 1e-3)), (
        f"{what}: dbeta {db} vs {ref[3]}")
    assert relf(f64(got[4]), ref[4]) <= STATE_GRAD_RELF, f"{what}: dM_in"
    assert relf(f64(got[5]), ref[5]) <= STATE_GRAD_RELF, f"{what}: dz_in"


@pytest.mark.parametrize("mode", [LIN, DEL])
def test_backward_matches_oracle(ia, mode):
    """Three segments of two tiles each, zero state, loss through the output only."""
    got, ref = run(ia, 1, 2, 768, 256, mode, seed=91)
    check(got, ref, f"mode={mode}")


@pytest.mark.parametrize("mode", [LIN, DEL])
def test_backward_carried_state_and_state_gradients(ia, mode):
    """A non-zero incoming state, gradients of the final state, and a gate that leans
    on the memory (beta = 2): every path of the memory's backward carries weight."""
    got, ref = run(ia, 2, 1, 512, 256, mode, seed=93, beta=[2.0], state=True, state_grad=True)
    check(got, ref, f"state mode={mode}")


def test_backward_one_tile_segments(ia):
    """N = 128 (one tile per segment, five segments), Delta, memory-dominated gate."""
    got, ref = run(ia, 1, 2, 640, 128, DEL, seed=95, beta=[3.0, -1.0], state_grad=True)
    check(got, ref, "N=128")


def test_backward_deterministic(ia):
    """Two calls give bitwise equal gradients (fixed reduction orders, no atomics)."""
    inp = make_inputs(1, 2, 512, 128, torch.bfloat16, seed=97, device="cuda", gen_device="cpu")
    dout = normal((1, 2, 512, 128), torch.bfloat16, 97, 7).cuda()
    a = ia.infini_attn_backward(inp["q"], inp["k"], inp["v"], inp["beta"], 256, DEL, dout)
    b = ia.infini_attn_backward(inp["q"], inp["k"], inp["v"], inp["beta"], 256, DEL, dout)
    sync_ok(ia)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_backward_zero_length(ia):
    """L = 0: dbeta = 0 and the state gradient passes through."""
    q = torch.empty((1, 2, 0, 128), device="cuda", dtype=torch.bfloat16)
    beta = torch.tensor([0.5, -0.5], device="cuda")
    dM = torch.randn((1, 2, 128, 128), device="cuda")
    dz = torch.randn((1, 2, 128), device="cuda")
    r = ia.infini_attn_backward(q, q.clone(), q.clone(), beta, 256, LIN, q.clone(), None, None,
                                dM, dz)
    sync_ok(ia)
    assert torch.count_nonzero(r[3]) == 0
    assert torch.equal(r[4], dM) and torch.equal(r[5], dz)


@pytest.mark.parametrize("mode", [LIN, DEL])
@pytest.mark.parametrize("state", [False, True])
def test_backward_single_segment(ia, mode, state):
    """L = N (one segment, S = 1): from the zero state every row retrieves the constant 0
    and no gradient reaches the state through the retrieval or the Delta term; with a
    carried state both paths carry weight. Final-state gradients included."""
    got, ref = run(ia, 1, 2, 256, 256, mode, seed=99 + mode, state=state, state_grad=True)
    check(got, ref, f"single segment mode={mode} state={state}")


@pytest.mark.parametrize("mode", [LIN, DEL])
def test_backward_at_the_benchmarked_segment_length(ia, mode):
    """N = 2048 (16 query tiles per segment, the heaviest-first tile order and the longest
    reverse chains of the benchmarked shape) over two segments, with a carried state and
    final-state gradients; B * H = 2 heads, so the state rebuild splits every segment
    into the most token chunks (8)."""
    got, ref = run(ia, 1, 2, 4096, 2048, mode, seed=105, state=True, state_grad=True)
    check(got, ref, f"N=2048 mode={mode}")
