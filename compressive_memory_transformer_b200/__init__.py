"""Python binding of libinfini_attn.so (the B200 Infini-attention forward).

Argument marshalling only: every step of the computation runs in the CUDA
library. torch supplies device memory and the stream. There is no CPU fallback:
importing this package fails when the library is missing or cannot be loaded.

Entry points (same names as the C ABI in include/infini_attn.h):
    infini_attn_forward(q, k, v, beta, N, mode, M_in=None, z_in=None, ...)
    infini_attn_step(q, k, v, beta, mode, M_in=None, z_in=None, ...)
    infini_attn_decode(q, k, v, beta, k_cache, v_cache, M, z, pos, mode, ...)
    infini_attn_forward_gqa(q, k, v, beta, N, mode, layout, ...)
    infini_attn_state_update(k, v, N, mode, M_in=None, z_in=None, ...)
    infini_attn_state_sum(dM, dz, M_in=None, z_in=None, ...)
    infini_attn_backward(q, k, v, beta, N, mode, dout, M_in=None, z_in=None, ...)
    infini_attn_layer_forward(x, Wq, Wk, Wv, Wo, beta, N, mode, H, H_kv, ...)
    infini_attn_gemm_bf16(A, B)
q, k, v: [B, H, L, d] CUDA tensors, bf16 (d = 128) or fp32 (d <= 128);
beta: [H] fp32; M: [B, H, d, d] fp32; z: [B, H, d] fp32.
"""
from __future__ import annotations

import ctypes
import os

import torch

LINEAR = 0
DELTA = 1
LAYOUT_BHLD = 0  # [B, H, L, d]
LAYOUT_BLHD = 1  # [B, L, H, d]
DTYPE_BF16 = 0
DTYPE_F32 = 1

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libinfini_attn.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing; build it with "
        "`python -m compressive_memory_transformer_b200.build` (nvcc, sm_100a)")

_lib = ctypes.CDLL(LIB_PATH)

_vp = ctypes.c_void_p
_i = ctypes.c_int
_ll = ctypes.c_longlong


class Opts(ctypes.Structure):
    _fields_ = [("workspace", _vp), ("workspace_bytes", ctypes.c_size_t),
                ("stage_events", _vp * 3)]


_SIGS = {
    "infini_attn_forward": [_vp] * 9 + [_i, _i, _ll, _i, _i, _i, _vp],
    "infini_attn_step": [_vp] * 9 + [_i, _i, _i, _i, _i, _vp],
    "infini_attn_step_static": [_vp] * 9 + [_i, _i, _i, _i, _i, _vp],
    "infini_attn_forward_f32": [_vp] * 9 + [_i, _i, _ll, _i, _i, _i, _vp],
    "infini_attn_step_f32": [_vp] * 9 + [_i, _i, _i, _i, _i, _vp],
    "infini_attn_forward_ex": [_vp] * 9 + [_i, _i, _ll, _i, _i, _i, _i, ctypes.POINTER(Opts), _vp],
    "infini_attn_decode": [_vp] * 9 + [_i] * 7 + [_vp],
    "infini_attn_state_update": [_vp] * 6 + [_i, _i, _ll, _i, _i, _i, _vp],
    "infini_attn_forward_gqa": [_vp] * 9 + [_i, _i, _i, _ll, _i, _i, _i, _i, _vp],
    "infini_attn_state_sum": [_vp, _vp, _i] + [_vp] * 4 + [_i, _i, _i, _vp],
    "infini_attn_backward": [_vp] * 15 + [_i, _i, _ll, _i, _i, _i, _vp],
    "infini_attn_backward_ex": [_vp] * 15 + [_i, _i, _ll, _i, _i, _i, ctypes.POINTER(Opts), _vp],
    "infini_attn_backward_workspace_size": [_i, _i, _ll, _i, _i, _i],
    "infini_attn_layer_forward": [_vp] * 11 + [_i, _ll, _i, _i, _i, _i, _i, _i, _vp],
    "infini_attn_gemm_bf16": [_vp, _vp, _vp, _ll, _i, _i, _vp],
    "infini_attn_layer_forward_ex": [_vp] * 11 + [_i, _ll, _i, _i, _i, _i, _i, _i,
                                                  ctypes.POINTER(Opts), _vp],
    "infini_attn_layer_workspace_size": [_i, _ll, _i, _i, _i, _i, _i, _i],
    "infini_attn_workspace_size": [_i, _i, _ll, _i, _i, _i, _i],
    "infini_attn_device_status": [],
    "infini_attn_selftest_timeout": [_ll, _vp],
    "infini_attn_strerror": [_i],
    "infini_attn_version": [],
}
for _name, _args in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = _i
_lib.infini_attn_strerror.restype = ctypes.c_char_p
_lib.infini_attn_workspace_size.restype = ctypes.c_size_t
_lib.infini_attn_backward_workspace_size.restype = ctypes.c_size_t
_lib.infini_attn_layer_workspace_size.restype = ctypes.c_size_t

# every symbol the header declares (checked by the CPU tests)
EXPORTED = tuple(_SIGS)


class InfiniError(RuntimeError):
    def __init__(self, status: int):
        self.status = status
        super().__init__(f"infini_attn status {status}: {strerror(status)}")


def strerror(status: int) -> str:
    return _lib.infini_attn_strerror(int(status)).decode()


def version() -> int:
    return _lib.infini_attn_version()


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream_handle(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _check(st):
    if st != 0:
        raise InfiniError(st)


def _prepare(q, k, v, beta, M_in, z_in, out, M_out, z_out, state_out):
    if q.dim() != 4:
        raise ValueError("q, k, v must be [B, H, L, d]")
    B, H, L, d = q.shape
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.shape != q.shape or t.dtype != q.dtype or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor shaped and typed like q")
    if beta.dtype != torch.float32 or beta.numel() != H or not beta.is_cuda:
        raise ValueError("beta must be a CUDA fp32 tensor with H elements")
    if out is None:
        out = torch.empty_like(q)
    if state_out and M_out is None:
        M_out = torch.empty((B, H, d, d), device=q.device, dtype=torch.float32)
        z_out = torch.empty((B, H, d), device=q.device, dtype=torch.float32)
    for t in (M_in, z_in, M_out, z_out):
        if t is not None and (t.dtype != torch.float32 or not t.is_contiguous() or not t.is_cuda):
            raise ValueError("M and z must be contiguous CUDA fp32 tensors")
    return B, H, L, d, out, M_out, z_out


def infini_attn_forward(q, k, v, beta, N, mode=LINEAR, M_in=None, z_in=None, out=None,
                        M_out=None, z_out=None, state_out=True, stream=None):
    """Whole-sequence forward; returns (out, M_out, z_out)."""
    B, H, L, d, out, M_out, z_out = _prepare(q, k, v, beta, M_in, z_in, out, M_out, z_out,
                                             state_out)
    fn = _lib.infini_attn_forward if q.dtype == torch.bfloat16 else _lib.infini_attn_forward_f32
    if q.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("q/k/v must be bf16 or fp32")
    _check(fn(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(M_in), _ptr(z_in), _ptr(out),
              _ptr(M_out), _ptr(z_out), B, H, L, int(N), d, int(mode), _stream_handle(stream)))
    return out, M_out, z_out


def infini_attn_step(q, k, v, beta, mode=LINEAR, M_in=None, z_in=None, out=None, M_out=None,
                     z_out=None, state_out=True, stream=None):
    """One segment (L == N) with carried state; returns (out, M_out, z_out).
    Pass M_out=M_in, z_out=z_in to advance the state in place."""
    B, H, L, d, out, M_out, z_out = _prepare(q, k, v, beta, M_in, z_in, out, M_out, z_out,
                                             state_out)
    fn = _lib.infini_attn_step if q.dtype == torch.bfloat16 else _lib.infini_attn_step_f32
    if q.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("q/k/v must be bf16 or fp32")
    _check(fn(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(M_in), _ptr(z_in), _ptr(out),
              _ptr(M_out), _ptr(z_out), B, H, L, d, int(mode), _stream_handle(stream)))
    return out, M_out, z_out


def infini_attn_forward_ex(q, k, v, beta, N, mode=LINEAR, M_in=None, z_in=None, out=None,
                           M_out=None, z_out=None, workspace=None, stage_events=None,
                           state_out=True, stream=None):
    """Forward with options: a caller-owned workspace tensor (uint8, CUDA) and up to
    three torch.cuda.Event objects recorded around the state kernels and the
    fused attention kernel."""
    B, H, L, d, out, M_out, z_out = _prepare(q, k, v, beta, M_in, z_in, out, M_out, z_out,
                                             state_out)
    dtype = DTYPE_BF16 if q.dtype == torch.bfloat16 else DTYPE_F32
    o = Opts()
    if workspace is not None:
        o.workspace = workspace.data_ptr()
        o.workspace_bytes = workspace.numel() * workspace.element_size()
    if stage_events is not None:
        for i_, ev in enumerate(stage_events):
            o.stage_events[i_] = None if ev is None else ev.cuda_event
    _check(_lib.infini_attn_forward_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(M_in),
                                       _ptr(z_in), _ptr(out), _ptr(M_out), _ptr(z_out), B, H, L,
                                       int(N), d, int(mode), dtype, ctypes.byref(o),
                                       _stream_handle(stream)))
    return out, M_out, z_out


def infini_attn_forward_gqa(q, k, v, beta, N, mode=LINEAR, layout=LAYOUT_BHLD, M_in=None,
                            z_in=None, out=None, M_out=None, z_out=None, state_out=True,
                            stream=None):
    """Forward with grouped key/value heads and a choice of layout (bf16, d = 128).
    LAYOUT_BHLD: q [B, H, L, d], k/v [B, H_kv, L, d]; LAYOUT_BLHD: q [B, L, H, d], k/v
    [B, L, H_kv, d]; out is laid out as q. M/z are per key/value head: [B, H_kv, d, d]
    and [B, H_kv, d]. Returns (out, M_out, z_out)."""
    if q.dim() != 4 or q.dtype != torch.bfloat16:
        raise ValueError("q, k, v must be 4-d bf16 tensors")
    if layout == LAYOUT_BHLD:
        B, H, L, d = q.shape
        H_kv = k.shape[1]
        kv_shape = (B, H_kv, L, d)
    elif layout == LAYOUT_BLHD:
        B, L, H, d = q.shape
        H_kv = k.shape[2]
        kv_shape = (B, L, H_kv, d)
    else:
        raise ValueError("layout must be LAYOUT_BHLD or LAYOUT_BLHD")
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA bf16 tensor")
    if tuple(k.shape) != kv_shape or tuple(v.shape) != kv_shape:
        raise ValueError(f"k and v must be {kv_shape}")
    if beta.dtype != torch.float32 or beta.numel() != H or not beta.is_cuda:
        raise ValueError("beta must be a CUDA fp32 tensor with H elements")
    if out is None:
        out = torch.empty_like(q)
    if state_out and M_out is None:
        M_out = torch.empty((B, H_kv, d, d), device=q.device, dtype=torch.float32)
        z_out = torch.empty((B, H_kv, d), device=q.device, dtype=torch.float32)
    for t in (M_in, z_in, M_out, z_out):
        if t is not None and (t.dtype != torch.float32 or not t.is_contiguous() or not t.is_cuda):
            raise ValueError("M and z must be contiguous CUDA fp32 tensors")
    _check(_lib.infini_attn_forward_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(M_in),
                                        _ptr(z_in), _ptr(out), _ptr(M_out), _ptr(z_out), B, H,
                                        H_kv, L, int(N), d, int(mode), int(layout),
                                        _stream_handle(stream)))
    return out, M_out, z_out


def infini_attn_state_update(k, v, N, mode=LINEAR, M_in=None, z_in=None, M_out=None, z_out=None,
                             stream=None):
    """The memory update alone over k, v [B, H, L, d] (bf16, segments of N) from
    (M_in, z_in) (None: the zero state); returns (M_out, z_out)."""
    if k.dim() != 4 or k.dtype != torch.bfloat16:
        raise ValueError("k, v must be [B, H, L, d] bf16")
    B, H, L, d = k.shape
    if v.shape != k.shape or v.dtype != k.dtype or not (k.is_cuda and v.is_cuda) or not (
            k.is_contiguous() and v.is_contiguous()):
        raise ValueError("k and v must be contiguous CUDA tensors of the same shape")
    if M_out is None:
        M_out = torch.empty((B, H, d, d), device=k.device, dtype=torch.float32)
        z_out = torch.empty((B, H, d), device=k.device, dtype=torch.float32)
    for t in (M_in, z_in, M_out, z_out):
        if t is not None and (t.dtype != torch.float32 or not t.is_contiguous() or not t.is_cuda):
            raise ValueError("M and z must be contiguous CUDA fp32 tensors")
    _check(_lib.infini_attn_state_update(_ptr(k), _ptr(v), _ptr(M_in), _ptr(z_in), _ptr(M_out),
                                         _ptr(z_out), B, H, L, int(N), d, int(mode),
                                         _stream_handle(stream)))
    return M_out, z_out


def infini_attn_state_sum(dM, dz, M_in=None, z_in=None, M_out=None, z_out=None, stream=None):
    """(M_in, z_in) (None: zero) plus the sum of the blocks dM [count, B, H, d, d],
    dz [count, B, H, d] (fp32, CUDA), in block order; returns (M_out, z_out)."""
    count, B, H, d = dM.shape[0], dM.shape[1], dM.shape[2], dM.shape[3]
    if dM.shape != (count, B, H, d, d) or dz.shape != (count, B, H, d):
        raise ValueError("dM must be [count, B, H, d, d] and dz [count, B, H, d]")
    if M_out is None:
        M_out = torch.empty((B, H, d, d), device=dM.device, dtype=torch.float32)
        z_out = torch.empty((B, H, d), device=dM.device, dtype=torch.float32)
    for t in (dM, dz, M_in, z_in, M_out, z_out):
        if t is not None and (t.dtype != torch.float32 or not t.is_contiguous() or not t.is_cuda):
            raise ValueError("states must be contiguous CUDA fp32 tensors")
    _check(_lib.infini_attn_state_sum(_ptr(dM) if count else None, _ptr(dz) if count else None,
                                      count, _ptr(M_in), _ptr(z_in), _ptr(M_out), _ptr(z_out), B,
                                      H, d, _stream_handle(stream)))
    return M_out, z_out


def infini_attn_backward(q, k, v, beta, N, mode, dout, M_in=None, z_in=None, dM_out=None,
                         dz_out=None, state_grad=True, workspace=None, stage_events=None,
                         stream=None):
    """Gradient of infini_attn_forward (bf16, [B, H, L, 128], N a multiple of 128, L a
    multiple of N) for the loss sum(dout * out) + sum(dM_out * M_out) + sum(dz_out *
    z_out). Returns (dq, dk, dv, dbeta, dM_in, dz_in); dM_in, dz_in are None when
    state_grad is False. workspace: optional uint8 CUDA tensor of at least
    backward_workspace_size(...) bytes; stage_events: up to three torch.cuda.Event
    recorded after the state rebuild, after the dq kernel (with the retrieval's
    backward) and after the dk/dv kernel (with the reverse state chain)."""
    B, H, L, d, _, _, _ = _prepare(q, k, v, beta, M_in, z_in, None, None, None, False)
    if dout.shape != q.shape or dout.dtype != q.dtype or not dout.is_cuda or not dout.is_contiguous():
        raise ValueError("dout must be a contiguous CUDA tensor shaped and typed like q")
    for t in (dM_out, dz_out):
        if t is not None and (t.dtype != torch.float32 or not t.is_contiguous() or not t.is_cuda):
            raise ValueError("dM_out and dz_out must be contiguous CUDA fp32 tensors")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dbeta = torch.empty((H,), device=q.device, dtype=torch.float32)
    dM_in = dz_in = None
    if state_grad:
        dM_in = torch.empty((B, H, d, d), device=q.device, dtype=torch.float32)
        dz_in = torch.empty((B, H, d), device=q.device, dtype=torch.float32)
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(M_in), _ptr(z_in), _ptr(dout),
            _ptr(dM_out), _ptr(dz_out), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dbeta), _ptr(dM_in),
            _ptr(dz_in), B, H, L, int(N), d, int(mode))
    if workspace is None and stage_events is None:
        _check(_lib.infini_attn_backward(*args, _stream_handle(stream)))
    else:
        o = Opts()
        if workspace is not None:
            o.workspace = workspace.data_ptr()
            o.workspace_bytes = workspace.numel() * workspace.element_size()
        for i, ev in enumerate(stage_events or ()):
            o.stage_events[i] = ev.cuda_event if ev is not None else None
        _check(_lib.infini_attn_backward_ex(*args, ctypes.byref(o), _stream_handle(stream)))
    return dq, dk, dv, dbeta, dM_in, dz_in


def infini_attn_gemm_bf16(A, B, out=None, stream=None):
    """A [M, K] @ B [K, N] (bf16 CUDA, row-major; M, N, K multiples of 128) on the
    tensor cores with fp32 accumulation; returns C [M, N] bf16."""
    if A.dim() != 2 or B.dim() != 2 or A.shape[1] != B.shape[0]:
        raise ValueError("A must be [M, K] and B [K, N]")
    for t in (A, B):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("A and B must be contiguous bf16 CUDA tensors")
    M, K = A.shape
    N = B.shape[1]
    if out is None:
        out = torch.empty((M, N), device=A.device, dtype=torch.bfloat16)
    _check(_lib.infini_attn_gemm_bf16(_ptr(A), _ptr(B), _ptr(out), M, N, K,
                                      _stream_handle(stream)))
    return out


def infini_attn_layer_forward(x, Wq, Wk, Wv, Wo, beta, N, mode, H, H_kv=None, M_in=None,
                              z_in=None, out=None, state_out=True, workspace=None,
                              stage_events=None, stream=None):
    """One attention layer: x [B, L, D_model] bf16 -> projections (Wq [D_model, H*128],
    Wk, Wv [D_model, H_kv*128]) -> grouped-head forward -> y = heads @ Wo
    ([H*128, D_model]). Returns (y, M_out, z_out) with the state per key/value head
    (None when state_out is False). workspace: optional uint8 CUDA tensor of at least
    layer_workspace_size(...) bytes; stage_events: up to three torch.cuda.Event recorded
    after the Q/K/V projections, after the forward and after the output projection."""
    H_kv = H if H_kv is None else H_kv
    if x.dim() != 3:
        raise ValueError("x must be [B, L, D_model]")
    B, L, D_model = x.shape
    d = Wq.shape[1] // H
    for t in (x, Wq, Wk, Wv, Wo):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("x and the weights must be contiguous bf16 CUDA tensors")
    if (Wq.shape != (D_model, H * d) or Wk.shape != (D_model, H_kv * d)
            or Wv.shape != (D_model, H_kv * d) or Wo.shape != (H * d, D_model)):
        raise ValueError("weight shapes do not match x, H and H_kv")
    if beta.dtype != torch.float32 or beta.numel() != H or not beta.is_cuda:
        raise ValueError("beta must be a CUDA fp32 tensor with H elements")
    if out is None:
        out = torch.empty_like(x)
    M_out = z_out = None
    if state_out:
        M_out = torch.empty((B, H_kv, d, d), device=x.device, dtype=torch.float32)
        z_out = torch.empty((B, H_kv, d), device=x.device, dtype=torch.float32)
    args = (_ptr(x), _ptr(Wq), _ptr(Wk), _ptr(Wv), _ptr(Wo), _ptr(beta), _ptr(M_in),
            _ptr(z_in), _ptr(out), _ptr(M_out), _ptr(z_out), B, L, D_model, H, H_kv, int(N), d,
            int(mode))
    if workspace is None and stage_events is None:
        _check(_lib.infini_attn_layer_forward(*args, _stream_handle(stream)))
    else:
        o = Opts()
        if workspace is not None:
            o.workspace = workspace.data_ptr()
            o.workspace_bytes = workspace.numel() * workspace.element_size()
        for i, ev in enumerate(stage_events or ()):
            o.stage_events[i] = ev.cuda_event if ev is not None else None
        _check(_lib.infini_attn_layer_forward_ex(*args, ctypes.byref(o), _stream_handle(stream)))
    return out, M_out, z_out


def layer_workspace_size(B, L, D_model, H, H_kv, N, d=128, mode=LINEAR) -> int:
    return int(_lib.infini_attn_layer_workspace_size(B, L, D_model, H, H_kv, N, d, mode))


def backward_workspace_size(B, H, L, N, d, mode=LINEAR) -> int:
    return int(_lib.infini_attn_backward_workspace_size(B, H, L, N, d, mode))


def infini_attn_decode(q, k, v, beta, k_cache, v_cache, M, z, pos, mode=LINEAR, out=None,
                       stream=None):
    """Token-level streaming decode: n new tokens (q, k, v: [B, H, n, d] bf16) join the
    current segment, whose first `pos` tokens are in k_cache / v_cache ([B, H, N, d]
    bf16). Writes the new rows into the caches, returns out ([B, H, n, d] bf16), and
    when pos + n == N folds the segment into M / z ([B, H, d, d] / [B, H, d] fp32) in
    place."""
    if q.dim() != 4 or q.dtype != torch.bfloat16:
        raise ValueError("q, k, v must be [B, H, n, d] bf16")
    B, H, n, d = q.shape
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.shape != q.shape or t.dtype != q.dtype or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor shaped and typed like q")
    if k_cache.dim() != 4 or k_cache.shape[:2] != (B, H) or k_cache.shape[3] != d:
        raise ValueError("k_cache must be [B, H, N, d]")
    for name, t in (("k_cache", k_cache), ("v_cache", v_cache)):
        if (t.shape != k_cache.shape or t.dtype != torch.bfloat16 or not t.is_cuda
                or not t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous CUDA bf16 tensor shaped like k_cache")
    for t in (M, z):
        if t.dtype != torch.float32 or not t.is_contiguous() or not t.is_cuda:
            raise ValueError("M and z must be contiguous CUDA fp32 tensors")
    if beta.dtype != torch.float32 or beta.numel() != H or not beta.is_cuda:
        raise ValueError("beta must be a CUDA fp32 tensor with H elements")
    N = k_cache.shape[2]
    if out is None:
        out = torch.empty_like(q)
    _check(_lib.infini_attn_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(k_cache),
                                   _ptr(v_cache), _ptr(M), _ptr(z), _ptr(out), B, H, n, int(pos),
                                   N, d, int(mode), _stream_handle(stream)))
    return out


def workspace_size(B, H, L, N, d, mode=LINEAR, dtype=DTYPE_BF16) -> int:
    return int(_lib.infini_attn_workspace_size(B, H, L, N, d, mode, dtype))


def device_status() -> int:
    """INFINI_OK (0) or INFINI_ERR_TIMEOUT (-7); synchronises the device."""
    return _lib.infini_attn_device_status()


def selftest_timeout(timeout_ns: int, stream=None) -> None:
    _check(_lib.infini_attn_selftest_timeout(int(timeout_ns), _stream_handle(stream)))


def raw_call(name, *args):
    """Call an exported C function by name with ctypes-compatible arguments."""
    return getattr(_lib, name)(*args)
