"""GPU parity of infini_attn_forward_gqa: grouped key/value heads (H query heads
sharing H_kv key/value heads) and the [B, L, H, d] layout, against the fp64 oracle
run on the same tokens expanded to one key/value head per query head and moved to
[B, H, L, d]. The memory is built from K and V alone, so every query head of a
group sees the same state: the library keeps it once per key/value head."""
import numpy as np
import pytest
import torch

from parity import check_bf16, f64, run_oracle
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


def case(ia, B, H, H_kv, L, N, mode, layout, seed, state=False):
    G = H // H_kv
    qi = make_inputs(B, H, L, 128, torch.bfloat16, seed=seed, device="cuda", gen_device="cpu")
    kv = make_inputs(B, H_kv, L, 128, torch.bfloat16, seed=seed + 1, device="cuda",
                     gen_device="cpu")
    q, k, v, beta = qi["q"], kv["k"], kv["v"], qi["beta"]  # [B, heads, L, d]
    M0 = z0 = None
    if state:
        M0, z0 = normal_state(B, H_kv, 128, seed=seed + 2, scale_M=3.0, scale_z=50.0,
                              device="cuda")
    if layout == ia.LAYOUT_BLHD:
        args = [t.transpose(1, 2).contiguous() for t in (q, k, v)]
    else:
        args = [q, k, v]
    out, M, z = ia.infini_attn_forward_gqa(*args, beta, N, mode, layout, M0, z0)
    sync_ok(ia)
    if layout == ia.LAYOUT_BLHD:
        out = out.transpose(1, 2)
    # the oracle on one key/value head per query head
    ref_inp = {"q": q, "k": k.repeat_interleave(G, dim=1), "v": v.repeat_interleave(G, dim=1),
               "beta": beta}
    Mr = None if M0 is None else M0.repeat_interleave(G, dim=1)
    zr = None if z0 is None else z0.repeat_interleave(G, dim=1)
    r_out, r_M, r_z = run_oracle(ref_inp, N, mode, Mr, zr)
    # one state per key/value head: the oracle's copy at the group's first query head
    ref = (r_out, r_M[:, ::G], r_z[:, ::G])
    check_bf16(out, M, z, ref, what=f"gqa H={H} H_kv={H_kv} layout={layout} mode={mode}")
    return out, M, z


@pytest.mark.parametrize("mode", [LIN, DEL])
def test_gqa_bhld(ia, mode):
    """4 query heads on 2 key/value heads, several segments and a ragged last one."""
    case(ia, 2, 4, 2, 640, 256, mode, ia.LAYOUT_BHLD, seed=81)


@pytest.mark.parametrize("mode", [LIN, DEL])
def test_blhd_layout(ia, mode):
    """[B, L, H, d] with one key/value head per query head, a non-zero state."""
    case(ia, 2, 3, 3, 512, 256, mode, ia.LAYOUT_BLHD, seed=83, state=True)


@pytest.mark.parametrize("mode", [LIN, DEL])
def test_gqa_blhd_one_segment(ia, mode):
    """8 query heads on 1 key/value head in [B, L, H, d], one segment (the path that
    runs the state update beside the attention), N not a multiple of 128."""
    case(ia, 1, 8, 1, 320, 320, mode, ia.LAYOUT_BLHD, seed=85, state=True)


def test_gqa_with_one_group_is_forward(ia):
    """H_kv == H and [B, H, L, d]: bitwise the output and state of infini_attn_forward."""
    inp = make_inputs(2, 2, 768, 128, torch.bfloat16, seed=87, device="cuda", gen_device="cpu")
    a = ia.infini_attn_forward(inp["q"], inp["k"], inp["v"], inp["beta"], 256, DEL)
    b = ia.infini_attn_forward_gqa(inp["q"], inp["k"], inp["v"], inp["beta"], 256, DEL,
                                   ia.LAYOUT_BHLD)
    sync_ok(ia)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
