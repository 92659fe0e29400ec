"""GPU parity: the CUDA library (through its C ABI) against the fp64 oracle, on
seeded inputs at sizes the oracle finishes in seconds (several tiles, ragged
segments and tails), plus the pages' degenerate cases."""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from parity import (check_bf16, check_f32, f64, relf, run_oracle)
from synthetic_inputs import make_inputs, normal_state

pytestmark = pytest.mark.gpu

LIN, DEL = 0, 1


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


# ---------------------------------------------------------------------------
# fp32 path
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("mode", [LIN, DEL])
def test_f32_tiny_config(ia, mode):
    """B=1, H=2, d=64, N=64, L=256, N(0,1) from seed 0, beta = [0, 1]."""
    inp = make_inputs(1, 2, 256, 64, torch.float32, seed=0, device="cuda", beta=[0.0, 1.0],
                      gen_device="cpu")
    out, M, z = ia.infini_attn_forward(inp["q"], inp["k"], inp["v"], inp["beta"], 64, mode)
    sync_ok(ia)
    check_f32(out, M, z, run_oracle(inp, 64, mode), f"f32 tiny mode={mode}")


@pytest.mark.parametrize("B,H,L,N,d", [(2, 3, 100, 32, 24), (1, 1, 1, 1, 5), (1, 2, 77, 77, 128),
                                       (1, 1, 130, 7, 33)])
@pytest.mark.parametrize("mode", [LIN, DEL])
def test_f32_ragged_shapes(ia, B, H, L, N, d, mode):
    inp = make_inputs(B, H, L, d, torch.float32, seed=3, device="cuda", gen_device="cpu")
    Mi, zi = normal_state(B, H, d, seed=4, device="cuda")
    out, M, z = ia.infini_attn_forward(inp["q"], inp["k"], inp["v"], inp["beta"], N, mode, Mi, zi)
    sync_ok(ia)
    check_f32(out, M, z, run_oracle(inp, N, mode, Mi, zi), f"f32 {B,H,L,N,d} mode={mode}")


def test_f32_worked_example(ia, golden_dir):
    from test_oracle_pins import load_golden
    g = load_golden(os.path.join(golden_dir, "worked_example_d2.txt"))
    mk = lambda a: torch.tensor(a, dtype=torch.float32, device="cuda").reshape(1, 1, 2, 2)
    q, k, v = mk(g["q"]), mk(g["k"]), mk(g["v"])
    beta = torch.tensor([g["beta"][0]], dtype=torch.float32, device="cuda")
    for mode, tag in ((LIN, "linear"), (DEL, "delta")):
        out, M, z = ia.infini_attn_forward(q, k, v, beta, 1, mode)
        sync_ok(ia)
        assert np.allclose(f64(out).ravel(), g["N1.out"], atol=1e-6)
        assert np.allclose(f64(M).ravel(), g[f"N1.{tag}.M"], atol=1e-5)
        assert np.allclose(f64(z).ravel(), g[f"N1.{tag}.z"], atol=1e-5)
        out, M, z = ia.infini_attn_forward(q, k, v, beta, 2, mode)
        sync_ok(ia)
        assert np.allclose(f64(out).ravel(), g["N2.out"], atol=1e-6)
        assert np.allclose(f64(M).ravel(), g["N2.M"], atol=1e-5)


def test_f32_delta_fixed_point(ia):
    """Bindings already in the memory leave M unchanged (Linear+Delta)."""
    d, N = 16, 8
    inp = make_inputs(1, 1, N, d, torch.float32, seed=7, device="cuda", gen_device="cpu")
    _, M1, z1 = ia.infini_attn_forward(inp["q"], inp["k"], inp["v"], inp["beta"], N, DEL)
    k2 = make_inputs(1, 1, N, d, torch.float32, seed=8, device="cuda", gen_device="cpu")["k"]
    fk = torch.nn.functional.elu(k2.double()) + 1
    v2 = (fk @ M1.double()) / (fk @ z1.double().unsqueeze(-1))
    _, M2, z2 = ia.infini_attn_forward(inp["q"], k2, v2.float().contiguous(), inp["beta"], N, DEL,
                                       M1, z1)
    sync_ok(ia)
    assert relf(f64(M2), f64(M1)) <= 1e-5
    assert relf(f64(z2), f64(z1) + f64(fk.sum(2))) <= 1e-6


# ---------------------------------------------------------------------------
# bf16 tensor-core path (d = 128)
# ---------------------------------------------------------------------------
BF16_SHAPES = [
    (1, 2, 512, 256),     # two full segments, two tiles each
    (2, 1, 640, 256),     # ragged final segment (128 tokens)
    (1, 2, 448, 192),     # N not a multiple of the tile: ragged tiles inside the sequence
    (1, 1, 128, 128),     # one tile
    (1, 1, 1000, 300),    # everything ragged
    (1, 3, 96, 2048),     # a single short segment
    (1, 1, 1, 64),        # one token
]


@pytest.mark.parametrize("B,H,L,N", BF16_SHAPES)
@pytest.mark.parametrize("mode", [LIN, DEL])
def test_bf16_small_shapes(ia, B, H, L, N, mode):
    inp = make_inputs(B, H, L, 128, torch.bfloat16, seed=11, device="cuda", gen_device="cpu")
    out, M, z = ia.infini_attn_forward(inp["q"], inp["k"], inp["v"], inp["beta"], N, mode)
    sync_ok(ia)
    check_bf16(out, M, z, run_oracle(inp, N, mode), what=f"bf16 {B,H,L,N} mode={mode}")


@pytest.mark.parametrize("mode", [LIN, DEL])
def test_bf16_memory_path_isolated(ia, mode):
    """beta = +30: out is A_mem (to fp32 rounding), so the retrieval is compared
    on its own instead of being hidden behind A_dot."""
    B, H, L, N = 1, 2, 2048, 512
    inp = make_inputs(B, H, L, 128, torch.bfloat16, seed=5, device="cuda", beta=[30.0, 30.0],
                      gen_device="cpu")
    out, M, z = ia.infini_attn_forward(inp["q"], inp["k"], inp["v"], inp["beta"], N, mode)
    sync_ok(ia)
    ref = run_oracle(inp, N, mode)
    check_bf16(out, M, z, ref, what=f"beta=+30 mode={mode}")
    # the first segment retrieves exactly nothing
    assert float(out[:, :, :N].abs().max()) < 1e-6


@pytest.mark.parametrize("mode", [LIN, DEL])
def test_bf16_gate_minus_inf_is_local_attention(ia, mode):
    B, H, L, N = 1, 1, 512, 256
    inp = make_inputs(B, H, L, 128, torch.bfloat16, seed=9, device="cuda", beta=[-math.inf],
                      gen_device="cpu")
    out, _, _ = ia.infini_attn_forward(inp["q"], inp["k"], inp["v"], inp["beta"], N, mode)
    sync_ok(ia)
    q, k, v = (f64(inp[x])[0, 0] for x in "qkv")
    ref = np.concatenate([oracle.local_attention(q[s:s + N], k[s:s + N], v[s:s + N])
                          for s in range(0, L, N)])
    got = f64(out)[0, 0]
    assert np.max(np.abs(got - ref)) <= 2e-2 and relf(got, ref) <= 5e-3


@pytest.mark.parametrize("mode", [LIN, DEL])
def test_bf16_carried_state_and_step(ia, mode):
    """forward with a given state == segment-by-segment steps with the state
    carried in place (the streaming loop of the pages)."""
    B, H, L, N = 2, 2, 768, 256
    inp = make_inputs(B, H, L, 128, torch.bfloat16, seed=21, device="cuda", gen_device="cpu")
    Mi, zi = normal_state(B, H, 128, seed=22, scale_M=3.0, scale_z=50.0, device="cuda")
    out, M, z = ia.infini_attn_forward(inp["q"], inp["k"], inp["v"], inp["beta"], N, mode, Mi, zi)
    sync_ok(ia)
    ref = run_oracle(inp, N, mode, Mi, zi)
    check_bf16(out, M, z, ref, what=f"carried mode={mode}")
    Ms, zs = Mi.clone(), zi.clone()
    outs = []
    for s0 in range(0, L, N):
        sl = slice(s0, s0 + N)
        o, _, _ = ia.infini_attn_step(inp["q"][:, :, sl].contiguous(), inp["k"][:, :, sl].contiguous(),
                                      inp["v"][:, :, sl].contiguous(), inp["beta"], mode, Ms, zs,
                                      M_out=Ms, z_out=zs)
        outs.append(o)
    sync_ok(ia)
    check_bf16(torch.cat(outs, dim=2), Ms, zs, ref, what=f"steps mode={mode}")


@pytest.mark.parametrize("mode", [LIN, DEL])
@pytest.mark.parametrize("growth", [0.0045, 0.008, 0.015, 0.05])
def test_bf16_rescale_every_key_tile(ia, mode, growth):
    """Scores that grow along the segment (keys k_t ~ growth t + N(0,1), queries
    ~ 1 + 0.1 N(0,1)): each key tile raises each row's running max by about
    2089 growth in exp2 units (128 features x 128 keys x log2(e)/sqrt(128)), i.e.
    about 9, 17, 31 and 104 for the four rates: past the 2^8 rescale threshold at
    every key tile, below and above the 2^24 bound under which a step keeps the P it
    computed against the previous step's maximum."""
    B, H, L, N = 1, 2, 1024, 512
    g = torch.Generator().manual_seed(41)
    t = torch.arange(L, dtype=torch.float32).view(1, 1, L, 1)
    q = (1.0 + 0.1 * torch.randn((B, H, L, 128), generator=g)).to(torch.bfloat16)
    k = (growth * (t % N) + torch.randn((B, H, L, 128), generator=g)).to(torch.bfloat16)
    v = torch.randn((B, H, L, 128), generator=g).to(torch.bfloat16)
    beta = torch.tensor([0.3, -0.7])
    inp = {"q": q.cuda(), "k": k.cuda(), "v": v.cuda(), "beta": beta.cuda()}
    out, M, z = ia.infini_attn_forward(inp["q"], inp["k"], inp["v"], inp["beta"], N, mode)
    sync_ok(ia)
    ref = run_oracle(inp, N, mode)
    check_bf16(out, M, z, ref, what=f"rescale mode={mode} growth={growth}")


@pytest.mark.parametrize("mode", [LIN, DEL])
def test_bf16_steps_under_graph_capture(ia, mode):
    """A one-segment call runs the state update on a second stream beside the
    attention (forked and joined inside the call). Captured into a CUDA graph and
    replayed, three carried steps give bitwise the results of plain calls, and
    both match the oracle."""
    B, H, N, S = 2, 2, 512, 3
    inp = make_inputs(B, H, N * S, 128, torch.bfloat16, seed=31, device="cuda", gen_device="cpu")
    segs = [tuple(inp[x][:, :, s * N:(s + 1) * N].contiguous() for x in ("q", "k", "v"))
            for s in range(S)]
    Mi, zi = normal_state(B, H, 128, seed=32, scale_M=3.0, scale_z=50.0, device="cuda")

    def run(M, z, outs):
        for s, (q, k, v) in enumerate(segs):
            ia.infini_attn_step(q, k, v, inp["beta"], mode, M, z, out=outs[s], M_out=M, z_out=z)

    M1, z1 = Mi.clone(), zi.clone()
    o1 = [torch.empty_like(segs[0][0]) for _ in range(S)]
    run(M1, z1, o1)
    sync_ok(ia)
    M2, z2 = Mi.clone(), zi.clone()
    o2 = [torch.empty_like(segs[0][0]) for _ in range(S)]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run(M2, z2, o2)
    M2.copy_(Mi)
    z2.copy_(zi)
    g.replay()
    sync_ok(ia)
    del g
    for a, b in zip(o1, o2):
        assert torch.equal(a, b)
    assert torch.equal(M1, M2) and torch.equal(z1, z2)
    ref = run_oracle(inp, N, mode, Mi, zi)
    check_bf16(torch.cat(o1, dim=2), M1, z1, ref, what=f"graph steps mode={mode}")


def test_bf16_output_only_16_byte_aligned(ia):
    """The attention kernel stores rows as 32-byte sectors when `out` allows it;
    an `out` aligned to 16 bytes only takes the 16-byte stores, same result."""
    B, H, L, N = 1, 2, 512, 256
    inp = make_inputs(B, H, L, 128, torch.bfloat16, seed=51, device="cuda", gen_device="cpu")
    n = B * H * L * 128
    buf = torch.empty(n + 8, dtype=torch.bfloat16, device="cuda")
    out16 = buf[8:].view(B, H, L, 128)
    assert out16.data_ptr() % 32 == 16
    for mode in (LIN, DEL):
        ref_out, _, _ = ia.infini_attn_forward(inp["q"], inp["k"], inp["v"], inp["beta"], N, mode)
        ia.infini_attn_forward(inp["q"], inp["k"], inp["v"], inp["beta"], N, mode, out=out16)
        sync_ok(ia)
        assert torch.equal(out16, ref_out)


def test_bf16_empty_sequence_passes_state(ia):
    B, H = 1, 2
    e = torch.empty((B, H, 0, 128), dtype=torch.bfloat16, device="cuda")
    beta = torch.zeros(H, device="cuda")
    Mi, zi = normal_state(B, H, 128, seed=1, device="cuda")
    out, M, z = ia.infini_attn_forward(e, e.clone(), e.clone(), beta, 64, DEL, Mi, zi)
    sync_ok(ia)
    assert out.shape == e.shape
    assert torch.equal(M, Mi) and torch.equal(z, zi)
    _, M0, z0 = ia.infini_attn_forward(e, e.clone(), e.clone(), beta, 64, LIN)
    sync_ok(ia)
    assert float(M0.abs().max()) == 0.0 and float(z0.abs().max()) == 0.0


def test_bf16_linear_state_is_deterministic(ia):
    B, H, L, N = 1, 2, 1024, 256
    inp = make_inputs(B, H, L, 128, torch.bfloat16, seed=2, device="cuda", gen_device="cpu")
    r1 = ia.infini_attn_forward(inp["q"], inp["k"], inp["v"], inp["beta"], N, LIN)
    r2 = ia.infini_attn_forward(inp["q"], inp["k"], inp["v"], inp["beta"], N, LIN)
    sync_ok(ia)
    for a, b in zip(r1, r2):
        assert torch.equal(a, b)


def test_timeout_is_reported_not_hung(ia):
    ia.selftest_timeout(2_000_000)   # a 2 ms wait on a barrier nothing arrives at
    assert ia.device_status() == -7
    assert ia.device_status() == 0   # the flag is cleared once read
