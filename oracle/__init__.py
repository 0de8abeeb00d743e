"""CPU oracle of the GSPN line scan (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library in
``linear_spatial_propagation_b200``) never touches it.

The arithmetic lives in ``gspn_ref.c`` (plain C, every value in double); this
module compiles it with gcc on first use, widens the stored inputs to double
and calls it through ctypes.  See ``gspn_ref.c`` for what is computed and which
passage of the GSPN / GSPN-2 pages each step follows.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
against closed forms, invariants, brute force and hand-derived values.  The
pages print no worked numeric example, so absolute values are pinned only
through those derivations.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Dict, Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gspn_ref.c")
_LIB = os.path.join(_HERE, "libgspn_ref.so")
_lock = threading.Lock()
_lib = None


class _RefDesc(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int64), ("C", ctypes.c_int64), ("H", ctypes.c_int64), ("W", ctypes.c_int64),
        ("dir_mask", ctypes.c_uint32), ("groups", ctypes.c_int32), ("shared", ctypes.c_int32),
    ]


def build(force: bool = False) -> str:
    """Compile the oracle's C source into ``oracle/libgspn_ref.so``."""
    with _lock:
        if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
            tmp = _LIB + f".tmp{os.getpid()}"
            subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", _SRC,
                                   "-o", tmp, "-lm"])
            os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        dp = ctypes.POINTER(ctypes.c_double)
        lib.gspn_ref_fwd.argtypes = [ctypes.POINTER(_RefDesc), dp, dp, dp, dp, ctypes.c_int]
        lib.gspn_ref_fwd.restype = ctypes.c_int
        lib.gspn_ref_bwd.argtypes = [ctypes.POINTER(_RefDesc), dp, dp, dp, dp, dp, dp, dp, ctypes.c_int]
        lib.gspn_ref_bwd.restype = ctypes.c_int
        lib.gspn_ref_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().gspn_ref_max_threads())


def widen(a: np.ndarray, dtype: str) -> np.ndarray:
    """Stored values -> float64.  bf16 arrives as uint16 bit patterns and is
    widened exactly (its 16 bits become the top half of a float32)."""
    if dtype == "bf16":
        a = np.ascontiguousarray(a, dtype=np.uint16)
        return (a.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return np.ascontiguousarray(a).astype(np.float64)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _desc(B, C, H, W, dir_mask, groups, shared) -> _RefDesc:
    return _RefDesc(int(B), int(C), int(H), int(W), int(dir_mask), int(groups), int(bool(shared)))


def _ndirs(mask: int) -> int:
    return bin(int(mask) & 15).count("1")


def fwd(x: np.ndarray, logits: np.ndarray, lam: np.ndarray, *, dir_mask: int, groups: int = 1,
        shared: bool = False, dtype: str = "f64", nthreads: int = 1) -> np.ndarray:
    """out[B,C,H,W] (float64) of the GSPN forward.

    ``x``: [B,C,H,W]; ``lam``: [D,B,C,H,W]; ``logits``: [D,B,Cw,3,H,W];
    ``dtype`` names how the arrays are stored ("f64", "f32" or "bf16").
    """
    xs = widen(x, dtype) if dtype != "f64" else np.ascontiguousarray(x, dtype=np.float64)
    ls = widen(logits, dtype) if dtype != "f64" else np.ascontiguousarray(logits, dtype=np.float64)
    ms = widen(lam, dtype) if dtype != "f64" else np.ascontiguousarray(lam, dtype=np.float64)
    B, C, H, W = xs.shape
    D = _ndirs(dir_mask)
    Cw = 1 if shared else C
    if ms.shape != (D, B, C, H, W) or ls.shape != (D, B, Cw, 3, H, W):
        raise ValueError(f"bad shapes lam {ms.shape} logits {ls.shape} for x {xs.shape}, D={D}")
    out = np.zeros_like(xs)
    d = _desc(B, C, H, W, dir_mask, groups, shared)
    rc = _load().gspn_ref_fwd(ctypes.byref(d), _ptr(xs), _ptr(ls), _ptr(ms), _ptr(out), int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle forward rejected the arguments (code {rc})")
    return out


def bwd(x: np.ndarray, logits: np.ndarray, lam: np.ndarray, dout: np.ndarray, *, dir_mask: int,
        groups: int = 1, shared: bool = False, dtype: str = "f64",
        nthreads: int = 1) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """(dx, dlogits, dlam) in float64 for upstream gradient ``dout``."""
    conv = (lambda a: widen(a, dtype)) if dtype != "f64" else (lambda a: np.ascontiguousarray(a, dtype=np.float64))
    xs, ls, ms, gs = conv(x), conv(logits), conv(lam), conv(dout)
    B, C, H, W = xs.shape
    D = _ndirs(dir_mask)
    Cw = 1 if shared else C
    if ms.shape != (D, B, C, H, W) or ls.shape != (D, B, Cw, 3, H, W) or gs.shape != xs.shape:
        raise ValueError("bad shapes")
    dx = np.zeros_like(xs)
    dl = np.zeros_like(ls)
    dm = np.zeros_like(ms)
    d = _desc(B, C, H, W, dir_mask, groups, shared)
    rc = _load().gspn_ref_bwd(ctypes.byref(d), _ptr(xs), _ptr(ls), _ptr(ms), _ptr(gs), _ptr(dx), _ptr(dl),
                              _ptr(dm), int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle backward rejected the arguments (code {rc})")
    return dx, dl, dm


def fwd_workload(w, inp: Dict[str, np.ndarray], nthreads: int = 1) -> np.ndarray:
    """Oracle forward of a ``synth.Workload`` on its stored inputs."""
    return fwd(inp["x"], inp["logits"], inp["lam"], dir_mask=w.dir_mask, groups=w.groups, shared=w.shared,
               dtype=w.dtype, nthreads=nthreads)


def bwd_workload(w, inp: Dict[str, np.ndarray], nthreads: int = 1):
    return bwd(inp["x"], inp["logits"], inp["lam"], inp["dout"], dir_mask=w.dir_mask, groups=w.groups,
               shared=w.shared, dtype=w.dtype, nthreads=nthreads)
