"""CPU oracle of the GSPN line scan (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library in
``linear_spatial_propagation_b200``) never touches it.

The arithmetic lives in ``gspn_ref.c`` (plain C, every value in double); this
module compiles it with gcc on first use, widens the stored inputs to double
and calls it through ctypes.  See ``gspn_ref.c`` for what is computed and which
passage of the GSPN / GSPN-2 pages each step follows.

``block_fwd`` adds the compressed propagation block around the scan: the
projection of the C input channels onto C_proxy channels, the four
single-direction scans of those planes, a learnable per-(direction, channel)
merger, an RMS normalisation over the proxy channels of each pixel, and the
projection back to C channels.  Its matrix products are numpy ``einsum`` in
float64; its scans are the C oracle's, one direction at a time.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
and ``tests/test_oracle_block_pins.py`` against closed forms, invariants,
brute force and hand-derived values.  The pages print no worked numeric
example, so absolute values are pinned only through those derivations.
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


# ---------------------------------------------------------------------------
# Compressed propagation block
# ---------------------------------------------------------------------------
_DIR_BITS = (1, 2, 4, 8)  # T2B, B2T, L2R, R2L: the D axis order of lambda, logits and alpha


def block_fwd(x, v_proj, logits, lam, alpha, gamma, u_proj, *, groups: int = 1, norm: bool = True,
              eps: float = 1e-6, dtype: str = "f64", nthreads: int = 1, return_parts: bool = False):
    """y[B,C,H,W] (float64) of the compressed propagation block.

    Steps, each in float64:

    1. proxy projection ("GSPN-2: Efficient Parallel Sequence Modeling",
       OpenReview response, "Relate Compressive Proxy Dimension to Low-rank
       Approximation": x in R^{N x C x H x W} is projected by a linear layer to
       C_proxy channels): xp[b,k] = sum_c v_proj[k,c] x[b,c];
    2. the GSPN line scan of the proxy planes in each of the four directions
       separately ("Parallel Sequence Modeling via Generalized Spatial
       Propagation Network", Key design 2), with channel-shared taps
       (compact mode) and per-channel lambda;
    3. the learnable merger of the four directions (same page, Key design 2:
       "aggregated by a learnable merger"), read as one weight per direction
       and proxy channel: m[b,k] = sum_d alpha[d,k] h_d[b,k];
    4. the fused normalisation ("Scaling Parallel Sequence Models to Vision
       Foundation Models", abstract: a compressed latent-space propagation
       block with fused normalisation), read as an RMS normalisation over the
       proxy channels of each pixel with a per-channel gain:
       n[b,k] = gamma[k] m[b,k] / sqrt(mean_k m[b,k]^2 + eps)  (skipped when
       ``norm`` is false);
    5. the projection back to C channels (the same OpenReview passage):
       y[b,c] = sum_k u_proj[c,k] n[b,k].

    Shapes: x [B,C,H,W]; v_proj [Cp,C]; logits [4,B,1,3,H,W]; lam
    [4,B,Cp,H,W]; alpha [4,Cp]; gamma [Cp]; u_proj [C,Cp].  ``dtype`` names
    how x, v_proj, logits, lam and u_proj are stored ("f64", "f32", "bf16");
    alpha and gamma are float arrays.  With ``return_parts`` the function also
    returns the intermediates (xp, the four h_d, m, n).
    """
    conv = (lambda a: widen(a, dtype)) if dtype != "f64" else (lambda a: np.ascontiguousarray(a, dtype=np.float64))
    xs, vs, ls, ms, us = conv(x), conv(v_proj), conv(logits), conv(lam), conv(u_proj)
    al = np.asarray(alpha, dtype=np.float64)
    ga = np.asarray(gamma, dtype=np.float64)
    B, C, H, W = xs.shape
    Cp = vs.shape[0]
    if vs.shape != (Cp, C) or us.shape != (C, Cp) or ls.shape != (4, B, 1, 3, H, W) or \
            ms.shape != (4, B, Cp, H, W) or al.shape != (4, Cp) or ga.shape != (Cp,):
        raise ValueError("bad block shapes")
    xp = np.einsum("kc,bchw->bkhw", vs, xs)
    hs = []
    for d, bit in enumerate(_DIR_BITS):
        hs.append(fwd(xp, ls[d:d + 1], ms[d:d + 1], dir_mask=bit, groups=groups, shared=True, nthreads=nthreads))
    m = np.zeros_like(xp)
    for d in range(4):
        m += al[d][None, :, None, None] * hs[d]
    if norm:
        r = np.sqrt(np.mean(m * m, axis=1, keepdims=True) + eps)
        n = m / r * ga[None, :, None, None]
    else:
        n = m
    y = np.einsum("ck,bkhw->bchw", us, n)
    if return_parts:
        return y, {"xp": xp, "h": hs, "m": m, "n": n}
    return y
