"""GPU parity of the token-level streaming decode (infini_attn_decode) against the
fp64 oracle's whole-sequence forward: feeding a sequence through decode, one or a
few tokens at a time, must give every token the output the forward gives it (its
segment's causal attention up to itself, retrieval from the state of the segments
before), and the state after each completed segment must be the forward's state
after that many segments."""
import numpy as np
import pytest
import torch

from parity import check_bf16, f64, relf, run_oracle, BF16_STATE_RELF
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


def stream_decode(ia, inp, N, mode, chunks, M0=None, z0=None):
    """Feeds q/k/v [B, H, L, d] through decode in the given chunk sizes (a chunk
    never crosses a segment end). Returns the outputs and the states seen after
    each completed segment."""
    q, k, v, beta = inp["q"], inp["k"], inp["v"], inp["beta"]
    B, H, L, d = q.shape
    kc = torch.zeros((B, H, N, d), device="cuda", dtype=torch.bfloat16)
    vc = torch.zeros_like(kc)
    M = torch.zeros((B, H, d, d), device="cuda") if M0 is None else M0.clone()
    z = torch.zeros((B, H, d), device="cuda") if z0 is None else z0.clone()
    out = torch.empty_like(q)
    states = []
    t, pos, ci = 0, 0, 0
    while t < L:
        n = min(chunks[ci % len(chunks)], N - pos, L - t)
        ci += 1
        sl = slice(t, t + n)
        o = ia.infini_attn_decode(q[:, :, sl].contiguous(), k[:, :, sl].contiguous(),
                                  v[:, :, sl].contiguous(), beta, kc, vc, M, z, pos, mode)
        out[:, :, sl] = o
        t += n
        pos += n
        if pos == N:
            states.append((M.clone(), z.clone()))
            pos = 0
    sync_ok(ia)
    return out, states


@pytest.mark.parametrize("mode", [LIN, DEL])
def test_decode_token_by_token(ia, mode):
    """n = 1 for every token of 2.5 segments (N = 256, L = 640): the last segment is
    left half full, as in a stream that stops mid-segment."""
    B, H, L, N = 1, 2, 640, 256
    inp = make_inputs(B, H, L, 128, torch.bfloat16, seed=51, device="cuda", gen_device="cpu")
    out, states = stream_decode(ia, inp, N, mode, [1])
    ref = run_oracle(inp, N, mode)
    check_bf16(out, None, None, ref, what=f"decode n=1 mode={mode}")
    assert len(states) == 2
    for s, (M, z) in enumerate(states):
        sub = {x: inp[x][:, :, : (s + 1) * N] for x in ("q", "k", "v")}
        sub["beta"] = inp["beta"]
        _, r_M, r_z = run_oracle(sub, N, mode)
        assert relf(f64(M), r_M) <= BF16_STATE_RELF, f"M after segment {s}"
        assert relf(f64(z), r_z) <= BF16_STATE_RELF, f"z after segment {s}"


@pytest.mark.parametrize("mode", [LIN, DEL])
def test_decode_mixed_chunks_carried_state(ia, mode):
    """Chunks of 1, 3, 17, 40 (three query groups of up to 16) and 64 tokens, several
    heads and batch rows, a non-zero incoming state, N = 320 (a segment that is not a
    multiple of the 64-row cache chunk)."""
    B, H, L, N = 2, 3, 960, 320
    inp = make_inputs(B, H, L, 128, torch.bfloat16, seed=52, device="cuda", gen_device="cpu")
    M0, z0 = normal_state(B, H, 128, seed=53, scale_M=3.0, scale_z=50.0, device="cuda")
    out, states = stream_decode(ia, inp, N, mode, [1, 3, 17, 40, 64], M0, z0)
    ref = run_oracle(inp, N, mode, M0, z0)
    check_bf16(out, states[-1][0], states[-1][1], ref, what=f"decode mixed mode={mode}")


def test_decode_long_cache_many_splits(ia):
    """One token at the end of a 2048-token segment: the cache is split over many
    CTAs whose partial softmaxes are merged; 32 heads as in the 1B-layer workload."""
    B, H, N = 4, 8, 2048
    inp = make_inputs(B, H, N, 128, torch.bfloat16, seed=54, device="cuda", gen_device="cuda")
    kc = inp["k"].clone()
    vc = inp["v"].clone()
    M0, z0 = normal_state(B, H, 128, seed=55, scale_M=3.0, scale_z=50.0, device="cuda")
    M, z = M0.clone(), z0.clone()
    last = slice(N - 1, N)
    o = ia.infini_attn_decode(inp["q"][:, :, last].contiguous(), inp["k"][:, :, last].contiguous(),
                              inp["v"][:, :, last].contiguous(), inp["beta"], kc, vc, M, z, N - 1,
                              LIN)
    sync_ok(ia)
    heads = [(0, 0), (3, 7), (1, 4)]
    ref = run_oracle({x: inp[x] for x in ("q", "k", "v", "beta")}, N, LIN, M0, z0, heads=heads)
    for (b, h) in heads:
        r_out = ref[0][b, h, N - 1]
        g = f64(o)[b, h, 0]
        assert np.max(np.abs(g - r_out)) <= 2e-2 and relf(g, r_out) <= 5e-3, f"head {(b, h)}"
        assert relf(f64(M)[b, h], ref[1][b, h]) <= BF16_STATE_RELF
        assert relf(f64(z)[b, h], ref[2][b, h]) <= BF16_STATE_RELF


def test_decode_state_untouched_mid_segment(ia):
    """Before the segment is complete the state is only read."""
    B, H, N = 1, 2, 256
    inp = make_inputs(B, H, 100, 128, torch.bfloat16, seed=56, device="cuda", gen_device="cpu")
    kc = torch.zeros((B, H, N, 128), device="cuda", dtype=torch.bfloat16)
    vc = torch.zeros_like(kc)
    M0, z0 = normal_state(B, H, 128, seed=57, scale_M=3.0, scale_z=50.0, device="cuda")
    M, z = M0.clone(), z0.clone()
    ia.infini_attn_decode(inp["q"], inp["k"], inp["v"], inp["beta"], kc, vc, M, z, 0, DEL)
    sync_ok(ia)
    assert torch.equal(M, M0) and torch.equal(z, z0)
    assert torch.equal(kc[:, :, :100], inp["k"]) and torch.equal(vc[:, :, :100], inp["v"])
    assert torch.count_nonzero(kc[:, :, 100:]) == 0
