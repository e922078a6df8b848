"""Thin ctypes binding of liblf_attn.so (include/lf_attn.h).

Argument marshalling only: torch tensors supply device memory and the CUDA
stream; every step of the attention runs in the library's kernels.  The
functions carry the C names.  There is no fallback of any kind: if the
library cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liblf_attn.so")

LF_OK, LF_ERR_INVALID, LF_ERR_UNSUPPORTED, LF_ERR_CUDA, LF_ERR_DEVICE_TIMEOUT, LF_ERR_DEVICE_INPUT = range(6)
LF_F32, LF_BF16, LF_F16 = 0, 1, 2
LF_KERNEL_AUTO, LF_KERNEL_SIMT, LF_KERNEL_TC = 0, 1, 2
ERROR_NAMES = {1: "LF_ERR_INVALID", 2: "LF_ERR_UNSUPPORTED", 3: "LF_ERR_CUDA",
               4: "LF_ERR_DEVICE_TIMEOUT", 5: "LF_ERR_DEVICE_INPUT"}

# every symbol include/lf_attn.h declares
EXPORTS = ["lf_attn_version", "lf_attn_workspace_size", "lf_attn_fwd", "lf_attn_bwd",
           "lf_attn_count_pairs", "lf_attn_mask_dump", "lf_attn_status",
           "lf_attn_set_timing_events", "lf_attn_launch_count", "lf_attn_last_error",
           "lf_attn_fwd_noalloc", "lf_attn_status_noalloc", "lf_attn_decode",
           "lf_attn_set_test_hooks", "lf_attn_cross_workspace_size", "lf_attn_cross_fwd"]
# every symbol include/lf_proj.h declares
PROJ_EXPORTS = ["lf_proj_workspace_size", "lf_proj_in", "lf_proj_out", "lf_proj_set_timing_events"]
LF_STATIC_WORKSPACE_BYTES = 16 << 20


class LfError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__("%s: %s" % (ERROR_NAMES.get(code, str(code)), msg))
        self.code = code


class lf_attn_params(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("n", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("window", ctypes.c_int),
                ("dilation", ctypes.POINTER(ctypes.c_int32)), ("causal", ctypes.c_int),
                ("scale", ctypes.c_float), ("dtype", ctypes.c_int), ("max_global", ctypes.c_int),
                ("kernel", ctypes.c_int)]


class lf_cross_params(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("Lq", ctypes.c_int), ("Lk", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("scale", ctypes.c_float), ("dtype", ctypes.c_int)]


class lf_proj_params(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("n", ctypes.c_int), ("H", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("dtype", ctypes.c_int)]


_lib = None


def load(path: str = LIB_PATH):
    """Load the library (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError("liblf_attn.so is not built (python -m sparse_sliding_window_b200.build)")
        lib = ctypes.CDLL(path)
        P, sz, i32, vp = ctypes.POINTER(lf_attn_params), ctypes.c_size_t, ctypes.c_int, ctypes.c_void_p
        lib.lf_attn_version.restype = i32
        lib.lf_attn_workspace_size.argtypes = [P, i32]
        lib.lf_attn_workspace_size.restype = sz
        lib.lf_attn_fwd.argtypes = [P] + [vp] * 6 + [vp, vp, vp, vp, sz, vp]
        lib.lf_attn_bwd.argtypes = [P] + [vp] * 6 + [vp, vp, vp, vp] + [vp] * 6 + [vp, sz, vp]
        lib.lf_attn_count_pairs.argtypes = [P, vp, vp, vp, sz, vp]
        lib.lf_attn_mask_dump.argtypes = [P, vp, vp, vp, sz, vp]
        lib.lf_attn_status.argtypes = [vp, vp]
        lib.lf_attn_set_timing_events.argtypes = [vp, vp]
        lib.lf_attn_last_error.restype = ctypes.c_char_p
        lib.lf_attn_launch_count.restype = ctypes.c_uint64
        lib.lf_attn_fwd_noalloc.argtypes = [P] + [vp] * 6 + [vp, vp, vp, vp]
        lib.lf_attn_decode.argtypes = [P, vp, vp, vp, vp, vp, vp, vp]
        lib.lf_attn_decode.restype = i32
        lib.lf_attn_fwd_noalloc.restype = i32
        lib.lf_attn_set_test_hooks.argtypes = [ctypes.c_uint32, i32]
        lib.lf_attn_set_test_hooks.restype = i32
        lib.lf_attn_status_noalloc.argtypes = [vp]
        lib.lf_attn_status_noalloc.restype = i32
        for f in ("fwd", "bwd", "count_pairs", "mask_dump", "status", "set_timing_events"):
            getattr(lib, "lf_attn_" + f).restype = i32
        CP = ctypes.POINTER(lf_cross_params)
        lib.lf_attn_cross_workspace_size.argtypes = [CP]
        lib.lf_attn_cross_workspace_size.restype = sz
        lib.lf_attn_cross_fwd.argtypes = [CP, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        lib.lf_attn_cross_fwd.restype = i32
        PP = ctypes.POINTER(lf_proj_params)
        lib.lf_proj_workspace_size.argtypes = [PP, i32]
        lib.lf_proj_workspace_size.restype = sz
        lib.lf_proj_in.argtypes = [PP, i32, vp, vp, vp, ctypes.POINTER(vp), vp, i32, i32, vp, sz, vp]
        lib.lf_proj_in.restype = i32
        lib.lf_proj_out.argtypes = [PP, vp, vp, vp, vp, vp, sz, vp]
        lib.lf_proj_out.restype = i32
        lib.lf_proj_set_timing_events.argtypes = [vp, vp]
        lib.lf_proj_set_timing_events.restype = i32
        _lib = lib
    return _lib


def _check(code: int):
    if code != LF_OK:
        raise LfError(code, load().lf_attn_last_error().decode())


_DT = {"f32": LF_F32, "bf16": LF_BF16, "f16": LF_F16}


def dtype_code(t) -> int:
    import torch
    return {torch.float32: LF_F32, torch.bfloat16: LF_BF16, torch.float16: LF_F16}[t.dtype]


def make_params(B: int, H: int, n: int, window: int, dilation: Optional[Sequence[int]] = None,
                causal: bool = False, scale: float = 0.0, dtype: int = LF_BF16,
                max_global: int = -1, kernel: int = LF_KERNEL_AUTO, head_dim: int = 64):
    """Build an lf_attn_params (the dilation array is kept alive on it)."""
    p = lf_attn_params()
    p.B, p.H, p.n, p.head_dim, p.window = B, H, n, head_dim, window
    if dilation is not None:
        arr = (ctypes.c_int32 * H)(*[int(x) for x in dilation])
        p._dil_keep = arr  # type: ignore[attr-defined]
        p.dilation = ctypes.cast(arr, ctypes.POINTER(ctypes.c_int32))
    p.causal, p.scale, p.dtype, p.max_global, p.kernel = int(causal), float(scale), dtype, max_global, kernel
    return p


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def lf_attn_workspace_size(p, for_bwd: bool = False) -> int:
    return int(load().lf_attn_workspace_size(ctypes.byref(p), int(for_bwd)))


def workspace(p, for_bwd: bool = False, device="cuda"):
    """Allocate a workspace for params p (a uint8 torch tensor, 256-B aligned)."""
    import torch
    nbytes = lf_attn_workspace_size(p, for_bwd)
    if nbytes == 0:
        _check(LF_ERR_INVALID)
    return torch.zeros(nbytes, dtype=torch.uint8, device=device)  # status words start at zero


def lf_attn_fwd(p, q_s, k_s, v_s, q_g, k_g, v_g, mask, o, lse, ws, stream=None):
    _check(load().lf_attn_fwd(ctypes.byref(p), _ptr(q_s), _ptr(k_s), _ptr(v_s), _ptr(q_g),
                              _ptr(k_g), _ptr(v_g), _ptr(mask), _ptr(o), _ptr(lse), _ptr(ws),
                              ws.numel(), _stream(stream)))


def lf_attn_fwd_noalloc(p, q_s, k_s, v_s, q_g, k_g, v_g, mask, o, lse, stream=None):
    """Forward without a workspace argument (library-internal static scratch);
    for callers that cannot allocate device memory."""
    _check(load().lf_attn_fwd_noalloc(ctypes.byref(p), _ptr(q_s), _ptr(k_s), _ptr(v_s), _ptr(q_g),
                                      _ptr(k_g), _ptr(v_g), _ptr(mask), _ptr(o), _ptr(lse),
                                      _stream(stream)))


def lf_attn_set_test_hooks(wait_limit_us: int = 0, skip_kv_tile: int = 0):
    """Test hook of the device-side failure detection (see lf_attn.h)."""
    _check(load().lf_attn_set_test_hooks(int(wait_limit_us), int(skip_kv_tile)))


def lf_attn_status_noalloc(stream=None):
    """Read and clear the device status word of lf_attn_fwd_noalloc's static
    scratch on the current device (raises LfError on a device-side error)."""
    _check(load().lf_attn_status_noalloc(_stream(stream)))


def lf_attn_decode(p, q, k_cache, v_cache, lengths, o, lse=None, stream=None):
    """Causal-window decode step: q [B,H,64] against the caches [B,H,n,64]
    whose row lengths[b]-1 holds the new token; writes o [B,H,64] (+ lse)."""
    _check(load().lf_attn_decode(ctypes.byref(p), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                 _ptr(lengths), _ptr(o), _ptr(lse), _stream(stream)))


def lf_attn_bwd(p, q_s, k_s, v_s, q_g, k_g, v_g, mask, o, lse, d_o, dq_s, dk_s, dv_s, dq_g, dk_g,
                dv_g, ws, stream=None):
    _check(load().lf_attn_bwd(ctypes.byref(p), _ptr(q_s), _ptr(k_s), _ptr(v_s), _ptr(q_g),
                              _ptr(k_g), _ptr(v_g), _ptr(mask), _ptr(o), _ptr(lse), _ptr(d_o),
                              _ptr(dq_s), _ptr(dk_s), _ptr(dv_s), _ptr(dq_g), _ptr(dk_g),
                              _ptr(dv_g), _ptr(ws), ws.numel(), _stream(stream)))


def lf_attn_count_pairs(p, mask, counts, ws, stream=None):
    _check(load().lf_attn_count_pairs(ctypes.byref(p), _ptr(mask), _ptr(counts), _ptr(ws),
                                      ws.numel(), _stream(stream)))


def lf_attn_mask_dump(p, mask, out, ws, stream=None):
    _check(load().lf_attn_mask_dump(ctypes.byref(p), _ptr(mask), _ptr(out), _ptr(ws), ws.numel(),
                                    _stream(stream)))


def lf_attn_status(ws, stream=None):
    _check(load().lf_attn_status(_ptr(ws), _stream(stream)))


def lf_attn_set_timing_events(ev_start, ev_stop):
    a = None if ev_start is None else ev_start.cuda_event
    b = None if ev_stop is None else ev_stop.cuda_event
    _check(load().lf_attn_set_timing_events(a, b))


def lf_attn_launch_count() -> int:
    return int(load().lf_attn_launch_count())


def make_cross_params(B: int, H: int, Lq: int, Lk: int, dtype: int = LF_BF16, scale: float = 0.0,
                      head_dim: int = 64):
    p = lf_cross_params()
    p.B, p.H, p.Lq, p.Lk, p.head_dim, p.scale, p.dtype = B, H, Lq, Lk, head_dim, float(scale), dtype
    return p


def lf_attn_cross_workspace_size(p) -> int:
    return int(load().lf_attn_cross_workspace_size(ctypes.byref(p)))


def cross_workspace(p, device="cuda"):
    import torch
    nbytes = lf_attn_cross_workspace_size(p)
    if nbytes == 0:
        _check(LF_ERR_INVALID)
    return torch.zeros(nbytes, dtype=torch.uint8, device=device)  # status words start at zero


def lf_attn_cross_fwd(p, q, k, v, key_mask, o, lse, ws, stream=None):
    """LED decoder cross-attention: q [B,H,Lq,64] against k, v [B,H,Lk,64]
    (keys with key_mask != 0; key_mask None: all) -> o [B,H,Lq,64], lse."""
    _check(load().lf_attn_cross_fwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(key_mask), _ptr(o),
                                    _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)))


def make_proj_params(B: int, n: int, H: int, dtype: int = LF_BF16, head_dim: int = 64):
    p = lf_proj_params()
    p.B, p.n, p.H, p.head_dim, p.dtype = B, n, H, head_dim, dtype
    return p


def lf_proj_workspace_size(p, max_rows: int = 0) -> int:
    return int(load().lf_proj_workspace_size(ctypes.byref(p), int(max_rows)))


def proj_workspace(p, max_rows: int = 0, device="cuda"):
    """Allocate a projection workspace (a uint8 torch tensor, 256-B aligned)."""
    import torch
    nbytes = lf_proj_workspace_size(p, max_rows)
    if nbytes == 0:
        _check(LF_ERR_INVALID)
    return torch.zeros(nbytes, dtype=torch.uint8, device=device)  # status words start at zero


def lf_proj_in(p, x, w_in, b_in, outs, ws, rows_mask=None, rows_code: int = 2, max_rows: int = 0,
               stream=None):
    """Input projections: outs[k][b,h,t,:] = x[b,t,:] . w_in[k*D + h*64 + :, :] + b_in[...]
    (only rows with rows_mask == rows_code when a mask is given)."""
    arr = (ctypes.c_void_p * len(outs))(*[o.data_ptr() for o in outs])
    _check(load().lf_proj_in(ctypes.byref(p), len(outs), _ptr(x), _ptr(w_in), _ptr(b_in), arr,
                             _ptr(rows_mask), int(rows_code), int(max_rows), _ptr(ws), ws.numel(),
                             _stream(stream)))


def lf_proj_out(p, o, w_out, b_out, y, ws, stream=None):
    """Output projection: y[b,t,:] = concat_h o[b,h,t,:] . w_out^T + b_out."""
    _check(load().lf_proj_out(ctypes.byref(p), _ptr(o), _ptr(w_out), _ptr(b_out), _ptr(y), _ptr(ws),
                              ws.numel(), _stream(stream)))


def lf_proj_set_timing_events(ev_start, ev_stop):
    a = None if ev_start is None else ev_start.cuda_event
    b = None if ev_stop is None else ev_stop.cuda_event
    _check(load().lf_proj_set_timing_events(a, b))


# ------------------------------------------------------------ convenience --

class LongformerAttention:
    """Holds params + workspace for one problem shape; call fwd / bwd with
    torch tensors [B, H, n, 64] on the GPU and an int32 mask [B, n]."""

    def __init__(self, B, H, n, window, dilation=None, causal=False, scale=0.0, dtype="bf16",
                 max_global=-1, kernel=LF_KERNEL_AUTO, device="cuda"):
        self.p = make_params(B, H, n, window, dilation, causal, scale, _DT[dtype], max_global, kernel)
        self.ws_f = workspace(self.p, False, device)
        self.ws_b = None
        self.device = device

    def fwd(self, q_s, k_s, v_s, q_g, k_g, v_g, mask, o=None, lse=None, stream=None, need_lse=True):
        import torch
        if o is None:
            o = torch.empty_like(q_s)
        if lse is None and need_lse:
            lse = torch.empty(q_s.shape[:3], dtype=torch.float32, device=q_s.device)
        lf_attn_fwd(self.p, q_s, k_s, v_s, q_g, k_g, v_g, mask, o, lse, self.ws_f, stream)
        return o, lse

    def bwd(self, q_s, k_s, v_s, q_g, k_g, v_g, mask, o, lse, d_o, stream=None):
        import torch
        if self.ws_b is None:
            self.ws_b = workspace(self.p, True, self.device)
        grads = [torch.empty_like(q_s) for _ in range(6)]
        lf_attn_bwd(self.p, q_s, k_s, v_s, q_g, k_g, v_g, mask, o, lse, d_o, *grads, self.ws_b, stream)
        return tuple(grads)

    def count_pairs(self, mask, stream=None):
        import torch
        c = torch.empty((self.p.B, self.p.H), dtype=torch.int64, device=mask.device)
        lf_attn_count_pairs(self.p, mask, c, self.ws_f, stream)
        return c

    def mask_dump(self, mask, stream=None):
        import torch
        out = torch.empty((self.p.B, self.p.H, self.p.n, self.p.n), dtype=torch.uint8, device=mask.device)
        lf_attn_mask_dump(self.p, mask, out, self.ws_f, stream)
        return out

    def status(self, bwd=False, stream=None):
        lf_attn_status(self.ws_b if bwd else self.ws_f, stream)
