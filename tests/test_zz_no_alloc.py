"""infini_attn_step_static: the streaming step for callers that must not allocate.

Some callers cannot let a library allocate device memory while they run: a
serving loop that reserved its whole memory budget at start-up, or a framework
whose allocator owns all device memory. infini_attn_step_static keeps its scratch
in a fixed array reserved when the library loads. This test calls it through the
C ABI twice in a row (the second call carries the state of the first, in place,
so a stale scratch would show) and checks both against infini_attn_step, the
allocating call, within the bf16 tolerances the parity tests use. It also checks
that sizes beyond the fixed array are refused before anything runs.

Kept in a file that pytest collects last.
"""
import numpy as np
import pytest
import torch

from parity import BF16_OUT_MAXABS, BF16_OUT_RELF, BF16_STATE_RELF, f64, relf
from synthetic_inputs import make_inputs

pytestmark = pytest.mark.gpu


def _static_step(ia, q, k, v, beta, M_in, z_in, out, M_out, z_out, mode):
    B, H, N, d = q.shape
    p = lambda t: None if t is None else t.data_ptr()
    return ia.raw_call("infini_attn_step_static", p(q), p(k), p(v), p(beta), p(M_in), p(z_in),
                       p(out), p(M_out), p(z_out), B, H, N, d, mode,
                       torch.cuda.current_stream().cuda_stream)


def _close(a_out, a_M, a_z, b_out, b_M, b_z):
    o1, o2 = f64(a_out), f64(b_out)
    assert np.all(np.isfinite(o1))
    assert float(np.max(np.abs(o1 - o2))) <= BF16_OUT_MAXABS
    assert relf(o1, o2) <= BF16_OUT_RELF
    assert relf(f64(a_M), f64(b_M)) <= BF16_STATE_RELF
    assert relf(f64(a_z), f64(b_z)) <= BF16_STATE_RELF


@pytest.mark.parametrize("mode", [1, 0])
def test_static_step_matches_allocating_step_twice(mode):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import compressive_memory_transformer_b200 as ia
    B, H, N, d = 1, 8, 2048, 128
    seg1 = make_inputs(B, H, N, d, torch.bfloat16, seed=31, device="cuda")
    seg2 = make_inputs(B, H, N, d, torch.bfloat16, seed=32, device="cuda")
    beta = seg1["beta"]

    # reference: the allocating step, segment 1 then segment 2 with the state carried
    r1 = ia.infini_attn_step(seg1["q"], seg1["k"], seg1["v"], beta, mode)
    r2 = ia.infini_attn_step(seg2["q"], seg2["k"], seg2["v"], beta, mode, r1[1], r1[2])

    # allocation-free step, twice in a row, the state advanced in place
    out1 = torch.empty_like(seg1["q"])
    out2 = torch.empty_like(seg2["q"])
    M = torch.empty((B, H, d, d), device="cuda")
    z = torch.empty((B, H, d), device="cuda")
    st = _static_step(ia, seg1["q"], seg1["k"], seg1["v"], beta, None, None, out1, M, z, mode)
    assert st == 0, ia.strerror(st)
    torch.cuda.synchronize()
    M1, z1 = M.clone(), z.clone()
    st = _static_step(ia, seg2["q"], seg2["k"], seg2["v"], beta, M, z, out2, M, z, mode)
    assert st == 0, ia.strerror(st)
    torch.cuda.synchronize()
    assert ia.device_status() == 0

    _close(out1, M1, z1, *r1)
    _close(out2, M, z, *r2)


def test_static_step_refuses_sizes_beyond_its_array():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import compressive_memory_transformer_b200 as ia
    # never dereferenced: the size check comes before any launch (addresses 8 GiB
    # apart so that no two of the 2 GiB operands overlap)
    gap = 1 << 33
    q, k, v, beta, out = ((1 << 20) + i * gap for i in range(5))
    st = ia.raw_call("infini_attn_step_static", q, k, v, beta, None, None, out, None, None,
                     1, 4096, 2048, 128, 1, None)
    assert st == -9
    assert "scratch" in ia.strerror(st)
