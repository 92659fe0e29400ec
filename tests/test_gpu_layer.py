"""GPU parity of the projection GEMM (infini_attn_gemm_bf16) and of the whole layer
(infini_attn_layer_forward) against the fp64 layer oracle (oracle/layer.py) on the
same bf16 inputs.

Tolerances: the GEMM multiplies exact bf16 values with fp32 accumulation and rounds
the result to bf16 (2^-9 relative), so rel-F <= 4e-3 and max-abs <= 8e-3 of the
largest reference magnitude. The layer rounds the projections q, k, v and the heads'
outputs to bf16 before the next step (each 2^-9) and runs the bf16 forward (rel-F
<= 5e-3 against its own oracle): rel-F <= 1e-2 for y, and 5e-3 for the state, whose
per-token rounding errors average over the sequence."""
import numpy as np
import pytest
import torch

import oracle.layer as ol
from parity import f64, relf
from synthetic_inputs import normal

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


@pytest.mark.parametrize("M,N,K", [(256, 384, 640), (128, 128, 128), (2048, 1024, 1024),
                                   (640, 512, 256), (8320, 1024, 256), (4224, 768, 1152)])
def test_gemm_matches_fp64(ia, M, N, K):
    """Several tiles in each direction, several k-steps, more tiles than SMs in the
    largest cases (each CTA takes several tiles and reuses its two accumulators). N a
    multiple of 256 takes the CTA-pair kernel (256 x 256 tiles); an odd number of
    128-row blocks (640, 8320, 4224 rows) leaves the last tile's second half past the
    end, and K = 256 gives fewer k-steps than ring stages."""
    A = normal((M, K), torch.bfloat16, 61, 0).cuda()
    B = (normal((K, N), torch.float32, 61, 1) / np.sqrt(K)).to(torch.bfloat16).cuda()
    C = ia.infini_attn_gemm_bf16(A, B)
    sync_ok(ia)
    ref = ol.project(f64(A)[None], f64(B))[0]
    got = f64(C)
    assert relf(got, ref) <= 4e-3
    assert np.max(np.abs(got - ref)) <= 8e-3 * np.max(np.abs(ref))


def layer_case(ia, B, L, D, H, Hkv, N, mode, seed, state=False):
    d = 128
    x = normal((B, L, D), torch.bfloat16, seed, 0).cuda()
    W = lambda tid, r, c: (normal((r, c), torch.float32, seed, tid) / np.sqrt(r)).to(
        torch.bfloat16).cuda()
    Wq, Wk, Wv, Wo = W(1, D, H * d), W(2, D, Hkv * d), W(3, D, Hkv * d), W(4, H * d, D)
    beta = normal((H,), torch.float32, seed, 5).cuda()
    M0 = z0 = None
    if state:
        M0 = (normal((B, Hkv, d, d), torch.float32, seed, 6) * 3.0).cuda()
        z0 = ((1.0 + normal((B, Hkv, d), torch.float32, seed, 7).abs()) * 50.0).cuda()
    y, M, z = ia.infini_attn_layer_forward(x, Wq, Wk, Wv, Wo, beta, N, mode, H, Hkv, M0, z0)
    sync_ok(ia)
    c = lambda t: None if t is None else f64(t)
    r_y, r_M, r_z = ol.layer_forward(f64(x), f64(Wq), f64(Wk), f64(Wv), f64(Wo), f64(beta), N,
                                     mode, H, Hkv, d, c(M0), c(z0))
    got = f64(y)
    assert relf(got, r_y) <= 1e-2, f"y rel-F {relf(got, r_y):.3e}"
    assert np.max(np.abs(got - r_y)) <= 3e-2 * np.max(np.abs(r_y))
    assert relf(f64(M), r_M) <= 5e-3 and relf(f64(z), r_z) <= 5e-3


@pytest.mark.parametrize("mode", [LIN, DEL])
def test_layer_matches_oracle(ia, mode):
    """Two heads, D_model = 256, three segments with a ragged last one."""
    layer_case(ia, 1, 640, 256, 2, 2, 256, mode, seed=71)


@pytest.mark.parametrize("mode", [LIN, DEL])
def test_layer_grouped_heads_with_state(ia, mode):
    """4 query heads on 2 key/value heads, two batch rows, a carried state."""
    layer_case(ia, 2, 384, 384, 4, 2, 128, mode, seed=73, state=True)


@pytest.mark.parametrize("mode", [LIN, DEL])
def test_layer_projection_widths_off_the_wide_tile(ia, mode):
    """3 query heads on 1 key/value head: the projection widths (384, 128) are not
    multiples of 256, so the three products take three launches of the 128-wide GEMM
    instead of the one grouped launch."""
    layer_case(ia, 1, 384, 256, 3, 1, 128, mode, seed=77)


def test_layer_grouped_projection_many_row_blocks(ia):
    """6 query heads on 2 key/value heads over 2 x 1024 rows: the grouped projection
    launch spans 16 row blocks and 3 + 1 + 1 wide column tiles (more tiles than SMs)."""
    layer_case(ia, 2, 1024, 512, 6, 2, 512, DEL, seed=79, state=True)


def test_layer_workspace_and_events_give_the_same_result(ia):
    """A caller workspace (infini_attn_layer_forward_ex) gives bitwise the same outputs
    as the library's own scratch, and the three stage events are recorded in order."""
    B, L, D, H, N = 1, 256, 256, 2, 128
    x = normal((B, L, D), torch.bfloat16, 75, 0).cuda()
    Ws = [(normal(shape, torch.float32, 75, 1 + i) / np.sqrt(shape[0])).to(torch.bfloat16).cuda()
          for i, shape in enumerate([(D, H * 128)] * 3 + [(H * 128, D)])]
    beta = normal((H,), torch.float32, 75, 5).cuda()
    a = ia.infini_attn_layer_forward(x, *Ws, beta, N, DEL, H)
    ws = torch.empty(ia.layer_workspace_size(B, L, D, H, H, N), dtype=torch.uint8, device="cuda")
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    for e in evs:
        e.record()
    b = ia.infini_attn_layer_forward(x, *Ws, beta, N, DEL, H, workspace=ws, stage_events=evs)
    sync_ok(ia)
    for u, w in zip(a, b):
        assert torch.equal(u, w)
    assert evs[0].elapsed_time(evs[1]) >= 0 and evs[1].elapsed_time(evs[2]) >= 0
