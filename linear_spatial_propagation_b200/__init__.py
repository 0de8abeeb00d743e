"""libgspn Python binding: the GSPN 2D line scan on B200 (sm_100a).

The compute lives in ``libgspn.so`` (hand-written CUDA behind the C ABI of
``include/gspn.h``).  This module only marshals arguments: it loads the
library with ctypes, exposes its entry points under the same names, and adds
thin torch helpers that allocate outputs / workspace with torch and pass
device pointers and the current stream.  There is no CPU fallback: if the
library cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

from . import _build

DIR_T2B, DIR_B2T, DIR_L2R, DIR_R2L = 1, 2, 4, 8
ALL_DIRS = 15
GSPN_F32, GSPN_BF16 = 0, 1

STATUS = {
    0: "GSPN_OK", 1: "GSPN_ERR_INVALID_ARG", 2: "GSPN_ERR_UNSUPPORTED", 3: "GSPN_ERR_ALIGNMENT",
    4: "GSPN_ERR_WORKSPACE", 5: "GSPN_ERR_CUDA", 6: "GSPN_ERR_TIMEOUT", 7: "GSPN_ERR_SCRATCH_LIMIT",
}

# every symbol include/gspn.h declares
EXPORTS = ("gspn_workspace_size", "gspn_fwd", "gspn_bwd", "gspn_fwd_noalloc", "gspn_device_status",
           "gspn_noalloc_status", "gspn_set_wait_limit_ns", "gspn_set_sync_check", "gspn_set_stall_test",
           "gspn_block_workspace_size", "gspn_block_fwd", "gspn_block_device_status",
           "gspn_launches_per_call", "gspn_variant_name", "gspn_status_string", "gspn_version")


class GspnError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS.get(status, status)} ({gspn_status_string(status)})")
        self.status = status


class gspn_block_desc(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int64), ("C", ctypes.c_int64), ("H", ctypes.c_int64), ("W", ctypes.c_int64),
        ("Cp", ctypes.c_int32), ("groups", ctypes.c_int32), ("norm", ctypes.c_int32), ("eps", ctypes.c_float),
    ]


class gspn_desc(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int64), ("C", ctypes.c_int64), ("H", ctypes.c_int64), ("W", ctypes.c_int64),
        ("dir_mask", ctypes.c_uint32), ("groups", ctypes.c_int32), ("shared_weights", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
    ]


_lib = None


def library_path() -> str:
    return _build.LIB


def load(build_if_missing: bool = True) -> ctypes.CDLL:
    """Load libgspn.so (building it first if it is missing and nvcc exists)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_build.LIB):
        if not build_if_missing:
            raise OSError(f"libgspn.so not built: {_build.LIB}")
        _build.build()
    lib = ctypes.CDLL(_build.LIB)
    vp, sz, dp = ctypes.c_void_p, ctypes.c_size_t, ctypes.POINTER(gspn_desc)
    lib.gspn_workspace_size.argtypes = [dp, ctypes.c_int]
    lib.gspn_workspace_size.restype = sz
    lib.gspn_fwd.argtypes = [dp, vp, vp, vp, vp, vp, sz, vp]
    lib.gspn_fwd.restype = ctypes.c_int
    lib.gspn_bwd.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.gspn_bwd.restype = ctypes.c_int
    lib.gspn_fwd_noalloc.argtypes = [dp, vp, vp, vp, vp, vp]
    lib.gspn_fwd_noalloc.restype = ctypes.c_int
    lib.gspn_device_status.argtypes = [dp, ctypes.c_int, vp, vp]
    lib.gspn_device_status.restype = ctypes.c_int
    lib.gspn_noalloc_status.argtypes = [vp]
    lib.gspn_noalloc_status.restype = ctypes.c_int
    lib.gspn_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    lib.gspn_set_wait_limit_ns.restype = ctypes.c_uint64
    lib.gspn_set_sync_check.argtypes = [ctypes.c_int]
    lib.gspn_set_sync_check.restype = ctypes.c_int
    lib.gspn_set_stall_test.argtypes = [ctypes.c_int]
    lib.gspn_set_stall_test.restype = ctypes.c_int
    bdp = ctypes.POINTER(gspn_block_desc)
    lib.gspn_block_workspace_size.argtypes = [bdp]
    lib.gspn_block_workspace_size.restype = sz
    lib.gspn_block_fwd.argtypes = [bdp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.gspn_block_fwd.restype = ctypes.c_int
    lib.gspn_block_device_status.argtypes = [bdp, vp, vp]
    lib.gspn_block_device_status.restype = ctypes.c_int
    lib.gspn_launches_per_call.argtypes = [dp, ctypes.c_int]
    lib.gspn_launches_per_call.restype = ctypes.c_int
    lib.gspn_variant_name.argtypes = [dp, ctypes.c_int]
    lib.gspn_variant_name.restype = ctypes.c_char_p
    lib.gspn_status_string.argtypes = [ctypes.c_int]
    lib.gspn_status_string.restype = ctypes.c_char_p
    lib.gspn_version.restype = ctypes.c_int
    _lib = lib
    return lib


def make_desc(B, C, H, W, dir_mask=ALL_DIRS, groups=1, shared=False, dtype="bf16") -> gspn_desc:
    dt = {"f32": GSPN_F32, "bf16": GSPN_BF16}.get(dtype, dtype)
    return gspn_desc(int(B), int(C), int(H), int(W), int(dir_mask), int(groups), int(bool(shared)), int(dt))


# ---- the C entry points under their own names (raw pointers) -----------------
def gspn_workspace_size(desc: gspn_desc, backward: int = 0) -> int:
    return int(load().gspn_workspace_size(ctypes.byref(desc), int(backward)))


def gspn_fwd(desc: gspn_desc, x: int, logits: int, lam: int, out: int, workspace: int, ws_bytes: int,
             stream: int) -> int:
    return int(load().gspn_fwd(ctypes.byref(desc), x, logits, lam, out, workspace or None, int(ws_bytes),
                               stream or None))


def gspn_bwd(desc: gspn_desc, x: int, logits: int, lam: int, dout: int, dx: int, dlogits: int, dlam: int,
             workspace: int, ws_bytes: int, stream: int) -> int:
    return int(load().gspn_bwd(ctypes.byref(desc), x, logits, lam, dout, dx, dlogits, dlam, workspace or None,
                               int(ws_bytes), stream or None))


def gspn_fwd_noalloc(desc: gspn_desc, x: int, logits: int, lam: int, out: int, stream: int) -> int:
    """Forward on the library's fixed device scratch: for callers that cannot
    allocate device memory (no workspace argument).  See include/gspn.h."""
    return int(load().gspn_fwd_noalloc(ctypes.byref(desc), x, logits, lam, out, stream or None))


def gspn_device_status(desc: gspn_desc, backward: int, workspace: int, stream: int) -> int:
    """Synchronise `stream`; GSPN_ERR_TIMEOUT if a bounded device wait of the
    last call with this workspace ran out (see include/gspn.h)."""
    return int(load().gspn_device_status(ctypes.byref(desc), int(backward), workspace or None, stream or None))


def gspn_noalloc_status(stream: int) -> int:
    return int(load().gspn_noalloc_status(stream or None))


def gspn_set_wait_limit_ns(limit_ns: int) -> int:
    return int(load().gspn_set_wait_limit_ns(int(limit_ns)))


def gspn_set_sync_check(on: int) -> int:
    return int(load().gspn_set_sync_check(int(on)))


def gspn_set_stall_test(on: int) -> int:
    return int(load().gspn_set_stall_test(int(on)))


def make_block_desc(B, C, H, W, Cp, groups=1, norm=True, eps=1e-6) -> gspn_block_desc:
    return gspn_block_desc(int(B), int(C), int(H), int(W), int(Cp), int(groups), int(bool(norm)), float(eps))


def gspn_block_workspace_size(desc: gspn_block_desc) -> int:
    return int(load().gspn_block_workspace_size(ctypes.byref(desc)))


def gspn_block_fwd(desc: gspn_block_desc, x: int, v_proj: int, logits: int, lam: int, alpha: int, gamma: int,
                   u_proj: int, y: int, workspace: int, ws_bytes: int, stream: int) -> int:
    return int(load().gspn_block_fwd(ctypes.byref(desc), x, v_proj, logits, lam, alpha, gamma, u_proj, y,
                                     workspace or None, int(ws_bytes), stream or None))


def gspn_block_device_status(desc: gspn_block_desc, workspace: int, stream: int) -> int:
    return int(load().gspn_block_device_status(ctypes.byref(desc), workspace or None, stream or None))


def gspn_launches_per_call(desc: gspn_desc, backward: int = 0) -> int:
    return int(load().gspn_launches_per_call(ctypes.byref(desc), int(backward)))


def gspn_variant_name(desc: gspn_desc, backward: int = 0) -> str:
    return load().gspn_variant_name(ctypes.byref(desc), int(backward)).decode()


def gspn_status_string(status: int) -> str:
    try:
        return load().gspn_status_string(int(status)).decode()
    except OSError:
        return "library not loaded"


def gspn_version() -> int:
    return int(load().gspn_version())


# ---- torch helpers (allocation and pointer marshalling only) ---------------
def _torch():
    import torch
    return torch


def _dtype_name(t) -> str:
    torch = _torch()
    if t.dtype == torch.float32:
        return "f32"
    if t.dtype == torch.bfloat16:
        return "bf16"
    raise TypeError(f"unsupported dtype {t.dtype}")


def _check(t, shape, name, dtype, device):
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)} != {tuple(shape)}")
    if t.dtype != dtype or t.device != device:
        raise ValueError(f"{name}: dtype/device {t.dtype}/{t.device} != {dtype}/{device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def desc_for(x, dir_mask=ALL_DIRS, groups=1, shared=False) -> gspn_desc:
    B, C, H, W = x.shape
    return make_desc(B, C, H, W, dir_mask, groups, shared, _dtype_name(x))


def workspace(desc: gspn_desc, backward: int, device) -> Optional["object"]:
    n = gspn_workspace_size(desc, backward)
    if n == 0:
        return None
    return _torch().empty(n, dtype=_torch().uint8, device=device)


def forward(x, logits, lam, dir_mask=ALL_DIRS, groups=1, shared=False, out=None, ws=None, stream=None):
    """out = GSPN forward of torch CUDA tensors (layouts as in include/gspn.h)."""
    torch = _torch()
    desc = desc_for(x, dir_mask, groups, shared)
    B, C, H, W = x.shape
    D = bin(dir_mask).count("1")
    Cw = 1 if shared else C
    _check(x, (B, C, H, W), "x", x.dtype, x.device)
    _check(lam, (D, B, C, H, W), "lam", x.dtype, x.device)
    _check(logits, (D, B, Cw, 3, H, W), "logits", x.dtype, x.device)
    if out is None:
        out = torch.empty_like(x)
    _check(out, (B, C, H, W), "out", x.dtype, x.device)
    if ws is None:
        ws = workspace(desc, 0, x.device)
    s = stream if stream is not None else torch.cuda.current_stream(x.device).cuda_stream
    st = gspn_fwd(desc, x.data_ptr(), logits.data_ptr(), lam.data_ptr(), out.data_ptr(),
                  ws.data_ptr() if ws is not None else 0, ws.numel() if ws is not None else 0, s)
    if st != 0:
        raise GspnError(st, "gspn_fwd")
    return out


def backward(x, logits, lam, dout, dir_mask=ALL_DIRS, groups=1, shared=False, grads=None, ws=None,
             stream=None) -> Tuple[object, object, object]:
    """(dx, dlogits, dlam) of the GSPN forward for upstream gradient dout."""
    torch = _torch()
    desc = desc_for(x, dir_mask, groups, shared)
    B, C, H, W = x.shape
    D = bin(dir_mask).count("1")
    Cw = 1 if shared else C
    for t, shp, n in ((x, (B, C, H, W), "x"), (lam, (D, B, C, H, W), "lam"), (logits, (D, B, Cw, 3, H, W), "logits"),
                      (dout, (B, C, H, W), "dout")):
        _check(t, shp, n, x.dtype, x.device)
    if grads is None:
        grads = (torch.empty_like(x), torch.empty_like(logits), torch.empty_like(lam))
    dx, dlg, dlam = grads
    if ws is None:
        ws = workspace(desc, 1, x.device)
    s = stream if stream is not None else torch.cuda.current_stream(x.device).cuda_stream
    st = gspn_bwd(desc, x.data_ptr(), logits.data_ptr(), lam.data_ptr(), dout.data_ptr(), dx.data_ptr(),
                  dlg.data_ptr(), dlam.data_ptr(), ws.data_ptr() if ws is not None else 0,
                  ws.numel() if ws is not None else 0, s)
    if st != 0:
        raise GspnError(st, "gspn_bwd")
    return dx, dlg, dlam


def block_forward(x, v_proj, logits, lam, alpha, gamma, u_proj, groups=1, norm=True, eps=1e-6, y=None, ws=None,
                  stream=None):
    """y of the compressed propagation block (layouts as in include/gspn.h):
    x [B,C,H,W], v_proj [Cp,C], u_proj [C,Cp], logits [4,B,1,3,H,W],
    lam [4,B,Cp,H,W] (all bf16); alpha [4,Cp], gamma [Cp] (fp32)."""
    torch = _torch()
    B, C, H, W = x.shape
    Cp = v_proj.shape[0]
    desc = make_block_desc(B, C, H, W, Cp, groups, norm, eps)
    bf, f32 = torch.bfloat16, torch.float32
    for t, shp, n, dt in ((x, (B, C, H, W), "x", bf), (v_proj, (Cp, C), "v_proj", bf), (u_proj, (C, Cp), "u_proj", bf),
                          (logits, (4, B, 1, 3, H, W), "logits", bf), (lam, (4, B, Cp, H, W), "lam", bf),
                          (alpha, (4, Cp), "alpha", f32), (gamma, (Cp,), "gamma", f32)):
        _check(t, shp, n, dt, x.device)
    if y is None:
        y = torch.empty_like(x)
    _check(y, (B, C, H, W), "y", bf, x.device)
    if ws is None:
        n = gspn_block_workspace_size(desc)
        if n == 0:
            raise GspnError(2, "gspn_block_workspace_size")
        ws = torch.empty(n, dtype=torch.uint8, device=x.device)
    s = stream if stream is not None else torch.cuda.current_stream(x.device).cuda_stream
    st = gspn_block_fwd(desc, x.data_ptr(), v_proj.data_ptr(), logits.data_ptr(), lam.data_ptr(), alpha.data_ptr(),
                        gamma.data_ptr(), u_proj.data_ptr(), y.data_ptr(), ws.data_ptr(), ws.numel(), s)
    if st != 0:
        raise GspnError(st, "gspn_block_fwd")
    return y
