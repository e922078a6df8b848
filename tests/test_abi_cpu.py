"""The C-ABI library loads without a GPU, exports every symbol the header
declares, sizes workspaces, and rejects bad arguments on the host before any
CUDA call (no compute call is made here)."""
import ctypes
import os
import re

import pytest

from sparse_sliding_window_b200 import build as lfbuild
from sparse_sliding_window_b200 import lf_attn as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    lfbuild.build()
    return L.load()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "lf_attn.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lf_attn_\w+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = declared_symbols()
    assert len(names) >= 9
    for name in names:
        assert hasattr(lib, name), name
    assert sorted(L.EXPORTS) == sorted(n for n in names if n in L.EXPORTS)
    assert set(names) <= set(L.EXPORTS) | {n for n in names if n.startswith("lf_attn_")}
    assert lib.lf_attn_version() == 1


def test_workspace_sizes(lib):
    p = L.make_params(1, 12, 4096, 256, dtype=L.LF_BF16, max_global=65)
    f = L.lf_attn_workspace_size(p, False)
    b = L.lf_attn_workspace_size(p, True)
    assert f > 0 and b > 0 and f % 256 == 0 and b % 256 == 0
    assert b >= 12 * 4096 * 4  # backward holds the per-row deltas
    for bad in (dict(B=0), dict(H=0), dict(n=0), dict(window=-1), dict(dtype=7), dict(kernel=9),
                dict(head_dim=32), dict(H=200)):
        kw = dict(B=1, H=2, n=128, window=4, dtype=L.LF_BF16)
        kw.update(bad)
        hd = kw.pop("head_dim", 64)
        q = L.make_params(head_dim=hd, **kw)
        assert L.lf_attn_workspace_size(q, False) == 0, bad
    q = L.make_params(1, 2, 128, 4, dilation=[1, 0], dtype=L.LF_BF16)
    assert L.lf_attn_workspace_size(q, False) == 0
    q = L.make_params(1, 2, 128, 4, dtype=L.LF_F32, kernel=L.LF_KERNEL_TC)
    assert L.lf_attn_workspace_size(q, False) == 0


def test_host_validation_without_gpu(lib):
    p = L.make_params(1, 2, 128, 4, dtype=L.LF_BF16)
    buf = (ctypes.c_char * 4096)()
    a = ctypes.addressof(buf)
    a16 = (a + 255) & ~255
    vp = ctypes.c_void_p
    # NULL input -> LF_ERR_INVALID, message names it
    rc = lib.lf_attn_fwd(ctypes.byref(p), None, vp(a16), vp(a16), vp(a16), vp(a16), vp(a16),
                         vp(a16), vp(a16), None, vp(a16), 4096, None)
    assert rc == L.LF_ERR_INVALID and b"q_s" in lib.lf_attn_last_error()
    # misaligned pointer
    rc = lib.lf_attn_fwd(ctypes.byref(p), vp(a16 + 2), vp(a16), vp(a16), vp(a16), vp(a16), vp(a16),
                         vp(a16), vp(a16), None, vp(a16), 4096, None)
    assert rc == L.LF_ERR_INVALID and b"aligned" in lib.lf_attn_last_error()
    # workspace too small
    rc = lib.lf_attn_fwd(ctypes.byref(p), *([vp(a16)] * 8), None, vp(a16), 16, None)
    assert rc == L.LF_ERR_INVALID and b"workspace" in lib.lf_attn_last_error()
    # unsupported head_dim
    q = L.make_params(1, 2, 128, 4, dtype=L.LF_BF16, head_dim=128)
    rc = lib.lf_attn_fwd(ctypes.byref(q), *([vp(a16)] * 8), None, vp(a16), 4096, None)
    assert rc == L.LF_ERR_UNSUPPORTED
    # backward needs lse
    rc = lib.lf_attn_bwd(ctypes.byref(p), *([vp(a16)] * 8), None, *([vp(a16)] * 7), vp(a16), 4096, None)
    assert rc == L.LF_ERR_INVALID and b"lse" in lib.lf_attn_last_error()
    # NULL params
    assert lib.lf_attn_count_pairs(None, vp(a16), vp(a16), vp(a16), 4096, None) == L.LF_ERR_INVALID


def test_decode_host_validation_without_gpu(lib):
    """The decode entry refuses a non-causal window and bad pointers on the
    host, before any launch."""
    buf = (ctypes.c_char * 4096)()
    a16 = (ctypes.addressof(buf) + 255) & ~255
    vp = ctypes.c_void_p
    p = L.make_params(1, 2, 128, 4, None, False, 0.0, L.LF_BF16)
    rc = lib.lf_attn_decode(ctypes.byref(p), *([vp(a16)] * 5), None, None)
    assert rc == L.LF_ERR_INVALID and b"causal" in lib.lf_attn_last_error()
    pc = L.make_params(1, 2, 128, 4, None, True, 0.0, L.LF_BF16)
    rc = lib.lf_attn_decode(ctypes.byref(pc), None, *([vp(a16)] * 4), None, None)
    assert rc == L.LF_ERR_INVALID and b"q" in lib.lf_attn_last_error()
    rc = lib.lf_attn_decode(ctypes.byref(pc), vp(a16), vp(a16 + 4), *([vp(a16)] * 3), None, None)
    assert rc == L.LF_ERR_INVALID and b"aligned" in lib.lf_attn_last_error()


def test_projection_abi_exports_and_host_checks(lib):
    """include/lf_proj.h: every declared symbol is exported and bound, the
    workspace is sized, and bad arguments are refused on the host."""
    text = open(os.path.join(ROOT, "include", "lf_proj.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = sorted(set(re.findall(r"\b(lf_proj_\w+)\s*\(", text)))
    assert names == sorted(L.PROJ_EXPORTS)
    for name in names:
        assert hasattr(lib, name), name
    p = L.make_proj_params(2, 4096, 12, L.LF_BF16)
    w0 = L.lf_proj_workspace_size(p, 0)
    w1 = L.lf_proj_workspace_size(p, 65)
    assert 0 < w0 < w1 and w0 % 256 == 0 and w1 % 256 == 0
    assert w1 >= 2 * 65 * 768 * 2  # the gathered rows' hidden states
    for bad in (dict(B=0), dict(n=0), dict(H=6), dict(H=0), dict(dtype=L.LF_F32), dict(head_dim=32)):
        kw = dict(B=1, n=128, H=12, dtype=L.LF_BF16)
        kw.update(bad)
        hd = kw.pop("head_dim", 64)
        assert L.lf_proj_workspace_size(L.make_proj_params(head_dim=hd, **kw), 0) == 0, bad
    buf = (ctypes.c_char * 8192)()
    a = (ctypes.addressof(buf) + 255) & ~255
    outs = (ctypes.c_void_p * 1)(a)
    q = L.make_proj_params(1, 128, 12, L.LF_BF16)
    # NULL x, misaligned weight, nproj out of range, workspace too small: no launch
    assert lib.lf_proj_in(ctypes.byref(q), 1, None, a, None, outs, None, 2, 0, a, 4096, None) == L.LF_ERR_INVALID
    assert lib.lf_proj_in(ctypes.byref(q), 1, a, a + 2, None, outs, None, 2, 0, a, 4096, None) == L.LF_ERR_INVALID
    assert lib.lf_proj_in(ctypes.byref(q), 9, a, a, None, outs, None, 2, 0, a, 4096, None) == L.LF_ERR_INVALID
    assert lib.lf_proj_in(ctypes.byref(q), 1, a, a, None, outs, a, 2, 0, a, 4096, None) == L.LF_ERR_INVALID
    assert lib.lf_proj_out(ctypes.byref(q), a, a, None, a, a, 16, None) == L.LF_ERR_INVALID
    assert lib.lf_proj_out(ctypes.byref(L.make_proj_params(1, 128, 6, L.LF_BF16)), a, a, None, a, a,
                           4096, None) == L.LF_ERR_UNSUPPORTED


def test_cross_attention_workspace_and_host_checks(lib):
    p = L.make_cross_params(2, 16, 1024, 16384, L.LF_BF16)
    w = L.lf_attn_cross_workspace_size(p)
    assert w > 0 and w % 256 == 0
    assert w >= 2 * 16 * 1024 * 64 * 4  # at least one fp32 partial per query row
    for bad in (dict(B=0), dict(H=0), dict(Lq=0), dict(Lk=0), dict(dtype=L.LF_F32), dict(head_dim=32),
                dict(H=200)):
        kw = dict(B=1, H=2, Lq=100, Lk=300, dtype=L.LF_BF16)
        kw.update(bad)
        hd = kw.pop("head_dim", 64)
        assert L.lf_attn_cross_workspace_size(L.make_cross_params(head_dim=hd, **kw)) == 0, bad
    buf = (ctypes.c_char * 8192)()
    a = (ctypes.addressof(buf) + 255) & ~255
    q = L.make_cross_params(1, 2, 100, 300, L.LF_BF16)
    assert lib.lf_attn_cross_fwd(ctypes.byref(q), None, a, a, None, a, None, a, 1 << 20, None) == L.LF_ERR_INVALID
    assert lib.lf_attn_cross_fwd(ctypes.byref(q), a, a + 4, a, None, a, None, a, 1 << 20, None) == L.LF_ERR_INVALID
    assert lib.lf_attn_cross_fwd(ctypes.byref(q), a, a, a, None, a, None, a, 16, None) == L.LF_ERR_INVALID
