"""GPU parity of the state-only entry points (infini_attn_state_update,
infini_attn_state_sum) and of the Linear-mode sequence sharding they make possible,
emulated on one GPU: the sequence is cut into consecutive ranges, each range's
state sum is taken from the zero state, and each range's forward starts from the
sum of the ranges before it, as sequence_sharded_linear_forward does across ranks."""
import numpy as np
import pytest
import torch

from parity import BF16_STATE_RELF, check_bf16, f64, relf, run_oracle
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


@pytest.mark.parametrize("mode", [LIN, DEL])
@pytest.mark.parametrize("inplace", [False, True])
def test_state_update_matches_oracle(ia, mode, inplace):
    """Several segments and a ragged last one, a non-zero incoming state."""
    B, H, L, N = 2, 2, 1000, 256
    inp = make_inputs(B, H, L, 128, torch.bfloat16, seed=71, device="cuda", gen_device="cpu")
    M0, z0 = normal_state(B, H, 128, seed=72, scale_M=3.0, scale_z=50.0, device="cuda")
    M_in, z_in = M0.clone(), z0.clone()
    if inplace:
        M, z = ia.infini_attn_state_update(inp["k"], inp["v"], N, mode, M_in, z_in, M_in, z_in)
    else:
        M, z = ia.infini_attn_state_update(inp["k"], inp["v"], N, mode, M_in, z_in)
        assert torch.equal(M_in, M0) and torch.equal(z_in, z0)
    sync_ok(ia)
    _, r_M, r_z = run_oracle(inp, N, mode, M0, z0)
    assert relf(f64(M), r_M) <= BF16_STATE_RELF and relf(f64(z), r_z) <= BF16_STATE_RELF


def test_state_sum(ia):
    """Blocks added to the incoming state in block order; zero blocks pass it through."""
    B, H, d, count = 2, 3, 128, 4
    g = torch.Generator().manual_seed(73)
    dM = torch.randn((count, B, H, d, d), generator=g).cuda()
    dz = torch.rand((count, B, H, d), generator=g).cuda()
    M0 = torch.randn((B, H, d, d), generator=g).cuda()
    z0 = torch.rand((B, H, d), generator=g).cuda()
    M, z = ia.infini_attn_state_sum(dM, dz, M0, z0)
    sync_ok(ia)
    refM = f64(M0) + f64(dM).sum(0)
    refz = f64(z0) + f64(dz).sum(0)
    assert np.max(np.abs(f64(M) - refM)) <= 1e-5 * np.max(np.abs(refM))
    assert np.max(np.abs(f64(z) - refz)) <= 1e-5 * np.max(np.abs(refz))
    M1, z1 = ia.infini_attn_state_sum(dM[:0], dz[:0], M0, z0)
    M2, z2 = ia.infini_attn_state_sum(dM[:0], dz[:0])
    sync_ok(ia)
    assert torch.equal(M1, M0) and torch.equal(z1, z0)
    assert torch.count_nonzero(M2) == 0 and torch.count_nonzero(z2) == 0


def test_linear_sequence_sharding_emulated(ia):
    """Three ranges (3, 1 and 2 segments, the last one ragged) of a Linear-mode
    sequence with a non-zero incoming state: outputs and final state equal the
    oracle's single forward over the whole sequence."""
    B, H, N = 1, 4, 256
    ranges = [3 * N, 1 * N, 2 * N - 100]
    L = sum(ranges)
    inp = make_inputs(B, H, L, 128, torch.bfloat16, seed=74, device="cuda", gen_device="cpu")
    M0, z0 = normal_state(B, H, 128, seed=75, scale_M=3.0, scale_z=50.0, device="cuda")
    bounds = np.cumsum([0] + ranges)
    parts = [{x: inp[x][:, :, bounds[r]:bounds[r + 1]].contiguous() for x in ("q", "k", "v")}
             for r in range(len(ranges))]
    sums = [ia.infini_attn_state_update(p["k"], p["v"], N, LIN) for p in parts]
    dM_all = torch.stack([s[0] for s in sums])
    dz_all = torch.stack([s[1] for s in sums])
    out = torch.empty_like(inp["q"])
    for r, p in enumerate(parts):
        M_pre, z_pre = ia.infini_attn_state_sum(dM_all[:r], dz_all[:r], M0, z0)
        o, _, _ = ia.infini_attn_forward(p["q"], p["k"], p["v"], inp["beta"], N, LIN, M_pre, z_pre,
                                         state_out=False)
        out[:, :, bounds[r]:bounds[r + 1]] = o
    M_end, z_end = ia.infini_attn_state_sum(dM_all, dz_all, M0, z0)
    sync_ok(ia)
    ref = run_oracle(inp, N, LIN, M0, z0)
    check_bf16(out, M_end, z_end, ref, what="sharded Linear forward")
