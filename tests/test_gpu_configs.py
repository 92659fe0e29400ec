"""Parity at the full sizes of the benchmark workloads, in the launch configuration
bench.py times: the GPU runs the whole workload; the fp64 oracle recomputes sampled
(batch, head) pairs over their full length. Heads are independent (one memory per
head), so a sampled head is compared exactly, output rows and final state.

Workloads (bf16 q/k/v i.i.d. N(0,1), beta ~ N(0,1) per head, zero initial state):
  1B-LM layer:      B=4, H=8,  d=128, N=2048, L=32768, Linear and Linear+Delta
                    (also with beta = +30 on every head: the retrieval on its own)
  8B 500K length:   B=1, H=1,  d=128, N=2048, L=524288, beta = +30, Linear+Delta
  1M-token stream:  B=1, H=8,  d=128, N=2048, 512 infini_attn_step calls, Linear+Delta
  8B 500K stream:   B=1, H=32, d=128, N=2048, L=524288, Linear+Delta, one forward
  segment sweep:    B=8, H=16, d=128, L=65536, N in {512, 1024, 2048, 4096}, both modes
"""
import numpy as np
import pytest
import torch

import oracle
from parity import BF16_OUT_MAXABS, BF16_OUT_RELF, BF16_STATE_RELF, relf
from synthetic_inputs import make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ia():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import compressive_memory_transformer_b200 as m
    return m


def head64(t, b, h):
    return t[b, h].detach().to("cpu", torch.float64).numpy()


def check_head(out, M, z, q, k, v, beta, b, h, N, mode, what):
    g = oracle.gate_value(float(beta[h]))
    r_out, r_M, r_z = oracle.head_forward(head64(q, b, h), head64(k, b, h), head64(v, b, h), g,
                                          N, mode)
    o = head64(out, b, h)
    assert np.all(np.isfinite(o)), what
    maxabs = float(np.max(np.abs(o - r_out)))
    rf = relf(o, r_out)
    rM = relf(M[b, h].double().cpu().numpy(), r_M)
    rz = relf(z[b, h].double().cpu().numpy(), r_z)
    assert maxabs <= BF16_OUT_MAXABS, f"{what} (b={b}, h={h}): out max-abs {maxabs:.3e}"
    assert rf <= BF16_OUT_RELF, f"{what} (b={b}, h={h}): out rel-F {rf:.3e}"
    assert rM <= BF16_STATE_RELF, f"{what} (b={b}, h={h}): M rel-F {rM:.3e}"
    assert rz <= BF16_STATE_RELF, f"{what} (b={b}, h={h}): z rel-F {rz:.3e}"


@pytest.mark.parametrize("mode", [0, 1])
def test_1b_layer_shape(ia, mode):
    B, H, L, N = 4, 8, 32768, 2048
    inp = make_inputs(B, H, L, 128, torch.bfloat16, seed=0, device="cuda", gen_device="cuda")
    out, M, z = ia.infini_attn_forward(inp["q"], inp["k"], inp["v"], inp["beta"], N, mode)
    torch.cuda.synchronize()
    assert ia.device_status() == 0
    beta = inp["beta"].cpu()
    for b, h in ((0, 0), (B - 1, H - 1)):
        check_head(out, M, z, inp["q"], inp["k"], inp["v"], beta, b, h, N, mode,
                   f"1B layer mode={mode}")


@pytest.mark.parametrize("mode", [0, 1])
def test_1b_layer_shape_memory_path_isolated(ia, mode):
    """beta = +30 on every head of the 1B-layer shape (16 segments of 2048): the output
    is the memory retrieval (the local attention's weight is 1e-13), so the retrieval
    with M rounded to bf16 is compared on its own at the full segment count, where z
    has grown over 15 segments."""
    B, H, L, N = 4, 8, 32768, 2048
    inp = make_inputs(B, H, L, 128, torch.bfloat16, seed=0, device="cuda", gen_device="cuda",
                      beta=[30.0] * H)
    out, M, z = ia.infini_attn_forward(inp["q"], inp["k"], inp["v"], inp["beta"], N, mode)
    torch.cuda.synchronize()
    assert ia.device_status() == 0
    beta = inp["beta"].cpu()
    for b, h in ((0, 0), (B - 1, H - 1)):
        check_head(out, M, z, inp["q"], inp["k"], inp["v"], beta, b, h, N, mode,
                   f"1B layer beta=+30 mode={mode}")
    # the first segment retrieves exactly nothing: only the 1e-13 local-attention share
    assert float(out[:, :, :N].abs().max()) < 1e-6


def test_8b_length_memory_path_isolated(ia):
    """beta = +30 over the 8B 500K stream's length (256 segments of 2048, Linear+Delta),
    one head: the retrieval after z has grown for half a million tokens."""
    B, H, L, N, mode = 1, 1, 524288, 2048, 1
    inp = make_inputs(B, H, L, 128, torch.bfloat16, seed=2, device="cuda", gen_device="cuda",
                      beta=[30.0])
    out, M, z = ia.infini_attn_forward(inp["q"], inp["k"], inp["v"], inp["beta"], N, mode)
    torch.cuda.synchronize()
    assert ia.device_status() == 0
    check_head(out, M, z, inp["q"], inp["k"], inp["v"], inp["beta"].cpu(), 0, 0, N, mode,
               "8B length beta=+30")
    del inp, out
    torch.cuda.empty_cache()


def test_1m_token_stream_steps(ia):
    B, H, N, S, mode = 1, 8, 2048, 512, 1
    seg = [make_inputs(B, H, N, 128, torch.bfloat16, seed=1000 + i, device="cuda",
                       gen_device="cuda") for i in range(S)]
    beta = seg[0]["beta"]
    M = torch.zeros((B, H, 128, 128), device="cuda")
    z = torch.zeros((B, H, 128), device="cuda")
    outs = []
    for i in range(S):
        o, _, _ = ia.infini_attn_step(seg[i]["q"], seg[i]["k"], seg[i]["v"], beta, mode, M, z,
                                      M_out=M, z_out=z)
        outs.append(o)
    torch.cuda.synchronize()
    assert ia.device_status() == 0
    h = 3
    cat = lambda key: torch.cat([s[key][:, h:h + 1] for s in seg], dim=2)
    q, k, v = cat("q"), cat("k"), cat("v")
    out = torch.cat([o[:, h:h + 1] for o in outs], dim=2)
    check_head(out, M[:, h:h + 1], z[:, h:h + 1], q, k, v, beta.cpu()[h:h + 1], 0, 0, N, mode,
               "1M stream")


def test_8b_500k_stream(ia):
    B, H, L, N, mode = 1, 32, 524288, 2048, 1
    inp = make_inputs(B, H, L, 128, torch.bfloat16, seed=0, device="cuda", gen_device="cuda")
    out, M, z = ia.infini_attn_forward(inp["q"], inp["k"], inp["v"], inp["beta"], N, mode)
    torch.cuda.synchronize()
    assert ia.device_status() == 0
    check_head(out, M, z, inp["q"], inp["k"], inp["v"], inp["beta"].cpu(), 0, 17, N, mode,
               "8B 500K")
    del inp, out
    torch.cuda.empty_cache()


@pytest.mark.parametrize("N", [512, 1024, 2048, 4096])
def test_segment_sweep(ia, N):
    B, H, L = 8, 16, 65536
    inp = make_inputs(B, H, L, 128, torch.bfloat16, seed=0, device="cuda", gen_device="cuda")
    beta = inp["beta"].cpu()
    for mode in (0, 1):
        out, M, z = ia.infini_attn_forward(inp["q"], inp["k"], inp["v"], inp["beta"], N, mode)
        torch.cuda.synchronize()
        assert ia.device_status() == 0
        b, h = (N // 512) % B, (N // 256) % H
        check_head(out, M, z, inp["q"], inp["k"], inp["v"], beta, b, h, N, mode,
                   f"sweep N={N} mode={mode}")
    del inp
    torch.cuda.empty_cache()
