"""infini_attn_step_static: the streaming step for callers that must not allocate.

Some callers cannot let a library allocate device memory while they run: a
serving loop that reserved its whole memory budget at start-up, or a framework
whose allocator owns all device memory. infini_attn_step_static keeps its scratch
in a fixed array reserved when the library loads. These tests call it through the
C ABI twice in a row (the second call carries the state of the first, in place,
so a stale scratch would show) and check both against infini_attn_step, the
allocating call, within the bf16 tolerances the parity tests use; they check that
the call takes nothing from the device's stream-ordered memory pool (the pool the
allocating call draws its scratch from), that the largest size the array holds
still matches the allocating call, and that the first size beyond it is refused
before anything runs.

Kept in a file that pytest collects last.
"""
import numpy as np
import pytest
import torch

from parity import BF16_OUT_MAXABS, BF16_OUT_RELF, BF16_STATE_RELF, f64, relf
from synthetic_inputs import make_inputs

pytestmark = pytest.mark.gpu

# With d = 128 and one segment, one head's scratch without token chunking is
# 197632 bytes, so the fixed 8 MiB array holds 42 heads and refuses 43.
MAX_HEADS = 42


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


class PoolWatermark:
    """High watermark of the device's default stream-ordered memory pool (the pool
    that cudaMallocAsync draws from when no other pool is set)."""

    def __init__(self):
        from cuda.bindings import driver as dr
        from cuda.bindings import runtime as rt
        self.rt, self.dr = rt, dr
        err, self.pool = rt.cudaDeviceGetDefaultMemPool(torch.cuda.current_device())
        assert err == rt.cudaError_t.cudaSuccess

    def reset(self):
        torch.cuda.synchronize()
        (err,) = self.rt.cudaMemPoolSetAttribute(
            self.pool, self.rt.cudaMemPoolAttr.cudaMemPoolAttrUsedMemHigh, self.dr.cuuint64_t(0))
        assert err == self.rt.cudaError_t.cudaSuccess

    def high(self):
        torch.cuda.synchronize()
        err, val = self.rt.cudaMemPoolGetAttribute(
            self.pool, self.rt.cudaMemPoolAttr.cudaMemPoolAttrUsedMemHigh)
        assert err == self.rt.cudaError_t.cudaSuccess
        return int(val)


@pytest.fixture(scope="module")
def ia():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import compressive_memory_transformer_b200 as m
    return m


@pytest.mark.parametrize("mode", [1, 0])
def test_static_step_matches_allocating_step_twice(ia, mode):
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


def test_static_step_takes_nothing_from_the_memory_pool(ia):
    """The allocating step raises the pool's high watermark (so the probe sees its
    scratch); the static step, on the same arguments, leaves it at zero."""
    B, H, N, d = 1, 8, 2048, 128
    seg = make_inputs(B, H, N, d, torch.bfloat16, seed=33, device="cuda")
    out = torch.empty_like(seg["q"])
    M = torch.empty((B, H, d, d), device="cuda")
    z = torch.empty((B, H, d), device="cuda")
    pool = PoolWatermark()
    pool.reset()
    ia.infini_attn_step(seg["q"], seg["k"], seg["v"], seg["beta"], 1, out=out, M_out=M, z_out=z)
    assert pool.high() > 0
    # first call on the device (address look-up), then a measured pair of calls
    assert _static_step(ia, seg["q"], seg["k"], seg["v"], seg["beta"], None, None, out, M, z,
                        1) == 0
    pool.reset()
    free_before = torch.cuda.mem_get_info()[0]
    for _ in range(2):
        st = _static_step(ia, seg["q"], seg["k"], seg["v"], seg["beta"], M, z, out, M, z, 1)
        assert st == 0, ia.strerror(st)
    assert pool.high() == 0
    assert torch.cuda.mem_get_info()[0] == free_before
    assert ia.device_status() == 0


def test_static_step_at_the_largest_size_it_holds(ia):
    """42 heads of one 2048-token segment (no token chunking left) against the
    allocating step, twice with the state carried in place."""
    B, H, N, d, mode = 1, MAX_HEADS, 2048, 128, 1
    seg1 = make_inputs(B, H, N, d, torch.bfloat16, seed=35, device="cuda")
    seg2 = make_inputs(B, H, N, d, torch.bfloat16, seed=36, device="cuda")
    beta = seg1["beta"]
    r1 = ia.infini_attn_step(seg1["q"], seg1["k"], seg1["v"], beta, mode)
    r2 = ia.infini_attn_step(seg2["q"], seg2["k"], seg2["v"], beta, mode, r1[1], r1[2])
    out1, out2 = torch.empty_like(seg1["q"]), torch.empty_like(seg2["q"])
    M = torch.empty((B, H, d, d), device="cuda")
    z = torch.empty((B, H, d), device="cuda")
    assert _static_step(ia, seg1["q"], seg1["k"], seg1["v"], beta, None, None, out1, M, z,
                        mode) == 0
    torch.cuda.synchronize()
    M1, z1 = M.clone(), z.clone()
    assert _static_step(ia, seg2["q"], seg2["k"], seg2["v"], beta, M, z, out2, M, z, mode) == 0
    torch.cuda.synchronize()
    assert ia.device_status() == 0
    _close(out1, M1, z1, *r1)
    _close(out2, M, z, *r2)


@pytest.mark.parametrize("B,H", [(1, MAX_HEADS + 1), (1, 4096)])
def test_static_step_refuses_sizes_beyond_its_array(ia, B, H):
    # never dereferenced: the size check comes before any launch (addresses 8 GiB
    # apart so that no two of the operands overlap)
    gap = 1 << 33
    q, k, v, beta, out = ((1 << 20) + i * gap for i in range(5))
    st = ia.raw_call("infini_attn_step_static", q, k, v, beta, None, None, out, None, None,
                     B, H, 2048, 128, 1, None)
    assert st == -9
    assert "scratch" in ia.strerror(st)
