"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    import __graft_entry__
    __graft_entry__._build_module().build()
    import compressive_memory_transformer_b200 as m
    return m


def header_functions():
    txt = open(os.path.join(ROOT, "include", "infini_attn.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(infini_attn_\w+)\s*\(", txt)))


def test_header_symbols_exported(lib):
    names = header_functions()
    assert len(names) >= 10
    so = ctypes.CDLL(lib.LIB_PATH)
    for n in names:
        assert hasattr(so, n), f"{n} declared in the header but not exported"
    assert set(names) == set(lib.EXPORTED)


def test_version_and_strerror(lib):
    assert lib.version() >= 100
    for code in range(-9, 1):
        s = lib.strerror(code)
        assert s and s != "unknown status"
    assert lib.strerror(-99) == "unknown status"


FAKE = 1 << 20  # a 16-byte aligned, never dereferenced address


def call_fwd(lib, q=FAKE, k=FAKE + 4096, v=FAKE + 8192, beta=FAKE + 12288, M_in=None, z_in=None,
             out=FAKE * 2, M_out=None, z_out=None, B=1, H=1, L=128, N=128, d=128, mode=0,
             name="infini_attn_forward"):
    return lib.raw_call(name, q, k, v, beta, M_in, z_in, out, M_out, z_out, B, H, L, N, d, mode,
                        None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), -1), (dict(k=None), -1), (dict(v=None), -1), (dict(beta=None), -1),
    (dict(out=None), -1),
    (dict(M_in=FAKE * 4), -1),            # M_in without z_in
    (dict(M_out=FAKE * 4), -1),           # M_out without z_out
    (dict(B=0), -2), (dict(H=-1), -2), (dict(N=0), -2), (dict(L=-5), -2),
    (dict(L=1 << 31), -2),
    (dict(d=64), -3), (dict(d=256), -3), (dict(mode=2), -3),
    (dict(q=FAKE + 2), -4), (dict(out=FAKE * 2 + 8), -4),
    (dict(out=FAKE + 64), -8),            # out overlaps q
])
def test_forward_rejects_bad_arguments(lib, kw, code):
    assert call_fwd(lib, **kw) == code


def test_f32_rejects_wide_heads(lib):
    assert call_fwd(lib, d=129, name="infini_attn_forward_f32") == -3
    assert call_fwd(lib, d=0, name="infini_attn_forward_f32") == -2
    # more heads than the fp32 attention grid's rows hold
    assert call_fwd(lib, B=256, H=256, name="infini_attn_forward_f32") == -2


def test_step_rejects_bad_arguments(lib):
    st = lib.raw_call("infini_attn_step", None, FAKE, FAKE, FAKE, None, None, FAKE * 2, None,
                      None, 1, 1, 128, 128, 0, None)
    assert st == -1
    st = lib.raw_call("infini_attn_step", FAKE, FAKE, FAKE, FAKE, None, None, FAKE * 2, None,
                      None, 1, 1, 128, 64, 0, None)
    assert st == -3


def test_workspace_size_is_host_only(lib):
    assert lib.workspace_size(1, 1, 0, 128, 128) == 0
    w1 = lib.workspace_size(4, 8, 32768, 2048, 128, 0, 0)
    w2 = lib.workspace_size(4, 8, 32768, 2048, 128, 1, 0)
    assert w1 > 0 and w1 == w2
    # per (head, segment): z partials + z_{s-1} + [dM | G] + hi/lo M
    assert w1 >= 32 * 16 * (2 * 128 * 128 * 4 + 2 * 128 * 128 * 2)
    assert lib.workspace_size(1, 2, 256, 64, 64, 0, 1) > 0


def test_package_fails_loudly_without_library(tmp_path):
    import subprocess
    import sys
    code = ("import sys, shutil, os; sys.path.insert(0, %r); "
            "import importlib.util as u; "
            "spec = u.spec_from_file_location('pkgcopy', %r); m = u.module_from_spec(spec); "
            "spec.loader.exec_module(m)") % (
        str(tmp_path), str(tmp_path / "pkgcopy" / "__init__.py"))
    (tmp_path / "pkgcopy").mkdir()
    src = open(os.path.join(ROOT, "compressive_memory_transformer_b200", "__init__.py")).read()
    (tmp_path / "pkgcopy" / "__init__.py").write_text(src)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True)
    assert r.returncode != 0 and "ImportError" in r.stderr and "missing" in r.stderr


def call_decode(lib, q=FAKE, k=FAKE + 4096, v=FAKE + 8192, beta=FAKE + 12288, k_cache=FAKE * 3,
                v_cache=FAKE * 3 + 65536, M=FAKE * 4, z=FAKE * 4 + 65536, out=FAKE * 2, B=1, H=1,
                n=1, pos=0, N=128, d=128, mode=0):
    return lib.raw_call("infini_attn_decode", q, k, v, beta, k_cache, v_cache, M, z, out, B, H,
                        n, pos, N, d, mode, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), -1), (dict(k=None), -1), (dict(v=None), -1), (dict(beta=None), -1),
    (dict(k_cache=None), -1), (dict(v_cache=None), -1), (dict(M=None), -1), (dict(z=None), -1),
    (dict(out=None), -1),
    (dict(B=0), -2), (dict(H=0), -2), (dict(n=0), -2), (dict(pos=-1), -2), (dict(N=0), -2),
    (dict(pos=120, n=9), -2),             # pos + n > N
    (dict(B=256, H=256), -2),             # more heads than the grid's rows hold
    (dict(d=64), -3), (dict(mode=2), -3),
    (dict(q=FAKE + 8), -4), (dict(k_cache=FAKE * 3 + 8), -4), (dict(M=FAKE * 4 + 4), -4),
    (dict(out=FAKE), -8),                 # out is q
    (dict(v_cache=FAKE * 3 + 16384), -8), # the caches overlap
    (dict(out=FAKE * 3 + 256), -8),       # out inside k_cache
    (dict(k=FAKE * 3), -8),               # the new keys inside the cache
    (dict(z=FAKE * 4 + 4096), -8),        # z inside M
])
def test_decode_rejects_bad_arguments(lib, kw, code):
    """Every argument error is reported on the host, before any CUDA call."""
    assert call_decode(lib, **kw) == code


def call_state_update(lib, k=FAKE, v=FAKE + 65536, M_in=None, z_in=None, M_out=FAKE * 4,
                      z_out=FAKE * 4 + 65536, B=1, H=1, L=128, N=128, d=128, mode=0):
    return lib.raw_call("infini_attn_state_update", k, v, M_in, z_in, M_out, z_out, B, H, L, N, d,
                        mode, None)


@pytest.mark.parametrize("kw,code", [
    (dict(k=None), -1), (dict(v=None), -1), (dict(M_out=None), -1), (dict(z_out=None), -1),
    (dict(M_in=FAKE * 8), -1),            # M_in without z_in
    (dict(B=0), -2), (dict(N=0), -2), (dict(L=-1), -2), (dict(L=1 << 31), -2),
    (dict(d=64), -3), (dict(mode=2), -3),
    (dict(k=FAKE + 8), -4), (dict(M_out=FAKE * 4 + 4), -4),
    (dict(M_out=FAKE), -8),               # the state over k
    (dict(z_out=FAKE * 4 + 1024), -8),    # z inside M
])
def test_state_update_rejects_bad_arguments(lib, kw, code):
    assert call_state_update(lib, **kw) == code


def test_state_sum_rejects_bad_arguments(lib):
    ok = dict(dM=FAKE, dz=FAKE * 2, count=2, M_in=None, z_in=None, M_out=FAKE * 4,
              z_out=FAKE * 5, B=1, H=1, d=128)

    def call(**kw):
        a = dict(ok, **kw)
        return lib.raw_call("infini_attn_state_sum", a["dM"], a["dz"], a["count"], a["M_in"],
                            a["z_in"], a["M_out"], a["z_out"], a["B"], a["H"], a["d"], None)
    assert call(M_out=None) == -1
    assert call(dM=None) == -1
    assert call(M_in=FAKE * 6) == -1      # M_in without z_in
    assert call(count=-1) == -2
    assert call(B=0) == -2
    assert call(M_out=FAKE + 4096) == -8  # M_out inside the blocks


@pytest.mark.parametrize("kw,code", [
    (dict(H=4, H_kv=3), -2), (dict(H=4, H_kv=0), -2), (dict(layout=2), -3), (dict(d=64), -3),
    (dict(q=None), -1),
])
def test_forward_gqa_rejects_bad_arguments(lib, kw, code):
    a = dict(q=FAKE, k=FAKE + (1 << 20), v=FAKE + (2 << 20), beta=FAKE + (3 << 20), M_in=None,
             z_in=None, out=FAKE * 8, M_out=None, z_out=None, B=1, H=4, H_kv=2, L=128, N=128,
             d=128, mode=0, layout=0)
    a.update(kw)
    assert lib.raw_call("infini_attn_forward_gqa", a["q"], a["k"], a["v"], a["beta"], a["M_in"],
                        a["z_in"], a["out"], a["M_out"], a["z_out"], a["B"], a["H"], a["H_kv"],
                        a["L"], a["N"], a["d"], a["mode"], a["layout"], None) == code


IN0, OUT0 = 1 << 24, 1 << 28  # inputs and outputs of the gradient, 1 MiB apart each


def call_backward(lib, q=IN0, k=IN0 + (1 << 20), v=IN0 + (2 << 20), beta=IN0 + (3 << 20),
                  M_in=None, z_in=None, dout=IN0 + (4 << 20), dM_out=None, dz_out=None,
                  dq=OUT0, dk=OUT0 + (1 << 20), dv=OUT0 + (2 << 20), dbeta=OUT0 + (3 << 20),
                  dM_in=None, dz_in=None, B=1, H=1, L=256, N=128, d=128, mode=0):
    return lib.raw_call("infini_attn_backward", q, k, v, beta, M_in, z_in, dout, dM_out, dz_out,
                        dq, dk, dv, dbeta, dM_in, dz_in, B, H, L, N, d, mode, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), -1), (dict(dout=None), -1), (dict(dbeta=None), -1), (dict(dq=None), -1),
    (dict(M_in=OUT0 * 2), -1),            # M_in without z_in
    (dict(dM_out=OUT0 * 2), -1),          # dM_out without dz_out
    (dict(dM_in=OUT0 * 2), -1),           # dM_in without dz_in
    (dict(B=0), -2), (dict(N=0), -2), (dict(L=-1), -2),
    (dict(d=64), -3), (dict(mode=2), -3),
    (dict(N=192, L=384), -3),             # N not a multiple of 128
    (dict(L=384, N=256), -3),             # L not a multiple of N
    (dict(dq=OUT0 + 8), -4), (dict(dM_in=OUT0 * 2 + 4, dz_in=OUT0 * 3), -4),
    (dict(dq=IN0), -8),                   # dq is q
    (dict(dk=OUT0 + 4096), -8),           # dk inside dq
    (dict(dbeta=IN0 + (3 << 20)), -8),    # dbeta is beta
    (dict(dM_in=IN0 + (4 << 20), dz_in=OUT0 * 2), -8),  # dM_in over dout
])
def test_backward_rejects_bad_arguments(lib, kw, code):
    """Every argument error of the gradient entry point is reported on the host."""
    assert call_backward(lib, **kw) == code


@pytest.mark.parametrize("kw,code", [
    (dict(A=None), -1), (dict(M=0), -2), (dict(K=-128), -2),
    (dict(M=1 << 31, N=128, K=128), -2),  # rows past 32-bit tensor-map coordinates
    (dict(M=200), -3), (dict(N=96), -3), (dict(K=64), -3),
    (dict(A=IN0 + 8), -4),
    (dict(C=IN0 + 4096), -8),  # C over A
])
def test_gemm_rejects_bad_arguments(lib, kw, code):
    a = dict(A=IN0, B=IN0 + (8 << 20), C=OUT0, M=256, N=256, K=256)
    a.update(kw)
    assert lib.raw_call("infini_attn_gemm_bf16", a["A"], a["B"], a["C"], a["M"], a["N"], a["K"],
                        None) == code


@pytest.mark.parametrize("kw,code", [
    (dict(x=None), -1), (dict(Wo=None), -1), (dict(M_in=OUT0 * 2), -1),
    (dict(B=0), -2), (dict(H=4, H_kv=3), -2), (dict(H_kv=0), -2),
    (dict(B=2, L=1 << 30), -2),  # B * L rows past 32-bit tensor-map coordinates
    (dict(d=64), -3), (dict(D_model=192), -3), (dict(L=100), -3), (dict(mode=2), -3),
    (dict(y=OUT0 + 8), -4),
    (dict(y=IN0), -8),  # y over x
])
def test_layer_forward_rejects_bad_arguments(lib, kw, code):
    a = dict(x=IN0, Wq=IN0 + (8 << 20), Wk=IN0 + (9 << 20), Wv=IN0 + (10 << 20),
             Wo=IN0 + (11 << 20), beta=IN0 + (12 << 20), M_in=None, z_in=None, y=OUT0,
             M_out=None, z_out=None, B=1, L=128, D_model=256, H=2, H_kv=2, N=128, d=128, mode=0)
    a.update(kw)
    assert lib.raw_call("infini_attn_layer_forward", a["x"], a["Wq"], a["Wk"], a["Wv"], a["Wo"],
                        a["beta"], a["M_in"], a["z_in"], a["y"], a["M_out"], a["z_out"], a["B"],
                        a["L"], a["D_model"], a["H"], a["H_kv"], a["N"], a["d"], a["mode"],
                        None) == code


def test_backward_and_layer_workspace_sizes_are_host_only(lib):
    """The scratch-size queries need no device: positive for supported sizes, 0 for
    unsupported ones, and growing with the sequence."""
    b1 = lib.backward_workspace_size(1, 2, 2048, 512, 128, 1)
    b2 = lib.backward_workspace_size(1, 2, 4096, 512, 128, 1)
    assert 0 < b1 < b2
    assert lib.backward_workspace_size(1, 2, 2048, 192, 128, 1) == 0   # N % 128
    assert lib.backward_workspace_size(1, 2, 1000, 512, 128, 1) == 0   # L % N
    assert lib.backward_workspace_size(1, 2, 2048, 512, 64, 1) == 0    # d
    l1 = lib.layer_workspace_size(1, 1024, 256, 2, 1, 256)
    l2 = lib.layer_workspace_size(1, 1024, 256, 2, 2, 256)
    assert 0 < l1 < l2                                                  # more key/value heads
    assert lib.layer_workspace_size(1, 100, 256, 2, 2, 256) == 0        # B * L % 128
    assert lib.layer_workspace_size(1, 1024, 256, 3, 2, 256) == 0       # H % H_kv
    assert lib.layer_workspace_size(2, 1 << 30, 256, 2, 2, 2048) == 0   # B * L >= 2^31


def test_binding_rejects_bad_tensors_before_the_library(lib):
    """The Python binding of the gradient, the layer and the GEMM raises ValueError on
    host tensors, wrong dtypes or mismatched shapes without calling into CUDA."""
    import torch
    bf = torch.zeros((1, 1, 128, 128), dtype=torch.bfloat16)
    beta = torch.zeros(1)
    with pytest.raises(ValueError):
        lib.infini_attn_backward(bf, bf, bf, beta, 128, 0, bf)            # host tensors
    with pytest.raises(ValueError):
        lib.infini_attn_gemm_bf16(torch.zeros((128, 128), dtype=torch.bfloat16),
                                  torch.zeros((256, 128), dtype=torch.bfloat16))  # K mismatch
    with pytest.raises(ValueError):
        lib.infini_attn_gemm_bf16(torch.zeros((128, 128)), torch.zeros((128, 128)))  # fp32
    x = torch.zeros((1, 128, 256), dtype=torch.bfloat16)
    W = torch.zeros((256, 256), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        lib.infini_attn_layer_forward(x, W, W, W, W, torch.zeros(2), 128, 0, 2)  # host tensors
    with pytest.raises(ValueError):
        lib.infini_attn_layer_forward(x[0], W, W, W, W, torch.zeros(2), 128, 0, 2)  # not 3-d


@pytest.mark.parametrize("name", ["infini_attn_step", "infini_attn_step_static"])
@pytest.mark.parametrize("which", ["q", "k", "v", "M_in", "z_in", "M_out", "z_out"])
def test_step_entry_points_reject_the_same_aliasing(lib, name, which):
    """The allocating and the allocation-free step refuse the same overlaps of out with
    an input or a state buffer (INFINI_ERR_ALIAS), on the host, before any launch."""
    gap = 1 << 24                       # B=1, H=1, N=128, d=128: 32 KiB per operand
    args = dict(q=FAKE, k=FAKE + gap, v=FAKE + 2 * gap, beta=FAKE + 3 * gap, M_in=None,
                z_in=None, out=FAKE + 8 * gap, M_out=None, z_out=None)
    inside = args["out"] + 4096         # 16-byte aligned, inside out's 32 KiB
    partner = {"M_in": "z_in", "z_in": "M_in", "M_out": "z_out", "z_out": "M_out"}
    args[which] = inside
    if which in partner:                # state pointers come in pairs
        args[partner[which]] = FAKE + 16 * gap
    st = lib.raw_call(name, args["q"], args["k"], args["v"], args["beta"], args["M_in"],
                      args["z_in"], args["out"], args["M_out"], args["z_out"], 1, 1, 128, 128, 0,
                      None)
    assert st == -8, (name, which, st)
