"""Seeded synthetic inputs for the GSPN line-scan operator.

This module only draws random numbers and lays them out. It holds none of the
operator's arithmetic; both the CPU oracle (``oracle/``) and the CUDA library
(``linear_spatial_propagation_b200``) receive the very same bytes from here.

Tensor layouts (dense, row-major), as the C ABI in ``include/gspn.h`` states:

* ``x``, ``dout``:        ``[B, C, H, W]``
* ``lam`` (lambda):       ``[D, B, C, H, W]``     D = number of directions
* ``logits``:             ``[D, B, Cw, 3, H, W]``  Cw = 1 when taps are shared

Draws (each tensor from its own child stream of ``SeedSequence(seed)``, spawned
in the order x, lambda, logits, dout):

* x ~ N(0, 1), lambda ~ U(0, 1), logits ~ N(0, logit_std), dout ~ N(0, 1),
  all drawn in float32 by numpy's PCG64 generator, in chunks of 2**22
  elements, chunk q from child q of the tensor's stream;
* bf16 tensors are the float32 draws rounded to nearest-even bf16 and are
  stored as ``uint16`` bit patterns (numpy has no bf16 dtype).
"""
from __future__ import annotations

import dataclasses
import os
from typing import Dict, Optional

import numpy as np

DIR_T2B, DIR_B2T, DIR_L2R, DIR_R2L = 1, 2, 4, 8
ALL_DIRS = DIR_T2B | DIR_B2T | DIR_L2R | DIR_R2L
DTYPES = ("f32", "bf16")


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape, mode and input distribution of one GSPN invocation."""

    name: str
    B: int
    C: int
    H: int
    W: int
    dir_mask: int
    groups: int
    shared: bool
    dtype: str
    logit_std: float
    seed: int
    backward: bool = False

    @property
    def D(self) -> int:
        return bin(self.dir_mask).count("1")

    @property
    def Cw(self) -> int:
        return 1 if self.shared else self.C

    @property
    def elt_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def shapes(self) -> Dict[str, tuple]:
        return {
            "x": (self.B, self.C, self.H, self.W),
            "lam": (self.D, self.B, self.C, self.H, self.W),
            "logits": (self.D, self.B, self.Cw, 3, self.H, self.W),
            "dout": (self.B, self.C, self.H, self.W),
        }

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads the operator is specified and measured on.  Names say
# what they are; sizes follow the GSPN / GSPN-2 / C-GSPN pages (tiny-backbone
# stage-1 shape 56x56, 28x28 local stage, the 1K foundation shape B=32 C=1152
# 64x64, and the 2K shape 128x128).
WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in (
        Workload("t2b_f32_b1c4_16x16", 1, 4, 16, 16, DIR_T2B, 1, False, "f32", 1.0, 0),
        Workload("4dir_f32_b8c96_56x56", 8, 96, 56, 56, ALL_DIRS, 1, False, "f32", 1.0, 1),
        Workload("4dir_local4_bf16_b32c192_28x28", 32, 192, 28, 28, ALL_DIRS, 4, False, "bf16", 2.0, 2),
        Workload("compact_4dir_bf16_b32c1152_64x64", 32, 1152, 64, 64, ALL_DIRS, 1, True, "bf16", 1.0, 3),
        Workload("compact_4dir_bf16_b2c1152_128x128_fwdbwd", 2, 1152, 128, 128, ALL_DIRS, 1, True, "bf16", 1.0, 4,
                 backward=True),
    )
}

HEADLINE = "compact_4dir_bf16_b32c1152_64x64"

# Shapes outside the five, timed by the bench only: planes whose sides are not
# multiples of 8 and longer than 64 take the generic kernels (one warp per
# plane, directions in turn); the 256-square compact latent at the 1K channel
# count takes the compact large-plane forward and backward.
EXTRA_WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in (
        Workload("generic_4dir_f32_b2c64_130x70", 2, 64, 130, 70, ALL_DIRS, 1, False, "f32", 1.0, 30),
        Workload("large_compact_4dir_bf16_b2c1152_256x256", 2, 1152, 256, 256, ALL_DIRS, 1, True, "bf16", 1.0, 31),
    )
}


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest-even bf16; return the uint16 bits."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    rounding = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + rounding) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to float32 exactly."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


CHUNK = 1 << 22


def _fill(seq: np.random.SeedSequence, kind: str, shape: tuple, scale: float, bf16: bool) -> np.ndarray:
    """Draw a tensor in chunks of CHUNK elements; chunk q comes from child q of
    ``seq``, so the values do not depend on how many threads draw them."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16 if bf16 else np.float32)
    nchunks = max(1, (n + CHUNK - 1) // CHUNK)
    kids = seq.spawn(nchunks)

    def work(q):
        s, e = q * CHUNK, min(n, (q + 1) * CHUNK)
        if e <= s:
            return
        rng = np.random.Generator(np.random.PCG64(kids[q]))
        if kind == "normal":
            v = rng.standard_normal(e - s, dtype=np.float32)
            if scale != 1.0:
                v *= np.float32(scale)
        else:
            v = rng.random(e - s, dtype=np.float32)
        out[s:e] = f32_to_bf16_bits(v) if bf16 else v

    if nchunks == 1:
        work(0)
    else:
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(max_workers=min(nchunks, os.cpu_count() or 1)) as ex:
            list(ex.map(work, range(nchunks)))
    return out.reshape(shape)


def make_inputs(w: Workload, with_dout: Optional[bool] = None) -> Dict[str, np.ndarray]:
    """Draw the seeded inputs of workload ``w``.

    Returns float32 arrays for ``dtype == 'f32'`` and uint16 bf16 bit patterns
    for ``dtype == 'bf16'``.  ``dout`` is drawn when ``with_dout`` (default:
    ``w.backward``).
    """
    if with_dout is None:
        with_dout = w.backward
    kids = np.random.SeedSequence(w.seed).spawn(4)
    shp = w.shapes()
    bf = w.dtype == "bf16"
    out = {
        "x": _fill(kids[0], "normal", shp["x"], 1.0, bf),
        "lam": _fill(kids[1], "uniform", shp["lam"], 1.0, bf),
        "logits": _fill(kids[2], "normal", shp["logits"], w.logit_std, bf),
    }
    if with_dout:
        out["dout"] = _fill(kids[3], "normal", shp["dout"], 1.0, bf)
    return out


def plane_slice(w: Workload, inp: Dict[str, np.ndarray], b: int, c: int) -> Dict[str, np.ndarray]:
    """Inputs of the single (b, c) plane, as a B=1, C=1 workload's arrays.

    Pure indexing: with shared taps the plane keeps logits channel 0 of batch b.
    """
    cw = 0 if w.shared else c
    sl = {
        "x": inp["x"][b:b + 1, c:c + 1],
        "lam": inp["lam"][:, b:b + 1, c:c + 1],
        "logits": inp["logits"][:, b:b + 1, cw:cw + 1],
    }
    if "dout" in inp:
        sl["dout"] = inp["dout"][b:b + 1, c:c + 1]
    return {k: np.ascontiguousarray(v) for k, v in sl.items()}


# ---------------------------------------------------------------------------
# Compressed propagation block inputs
# ---------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class BlockWorkload:
    """Shape and seed of one compressed-propagation-block invocation (all four
    directions, channel-shared taps over the Cp proxy planes)."""

    name: str
    B: int
    C: int
    H: int
    W: int
    Cp: int
    groups: int
    seed: int
    norm: bool = True
    eps: float = 1e-6

    def replace(self, **kw) -> "BlockWorkload":
        return dataclasses.replace(self, **kw)


# The block at the 1K foundation shape with the proxy width the GSPN-2
# response selects (C_proxy = 2), and at its widest ablation point (32).
BLOCK_WORKLOADS: Dict[str, BlockWorkload] = {
    w.name: w
    for w in (
        BlockWorkload("block_cp2_bf16_b32c1152_64x64", 32, 1152, 64, 64, 2, 1, 20),
        BlockWorkload("block_cp32_bf16_b32c1152_64x64", 32, 1152, 64, 64, 32, 1, 21),
    )
}


def make_block_inputs(w: BlockWorkload) -> Dict[str, np.ndarray]:
    """Seeded inputs of a block workload.  bf16 bit patterns (uint16) for x
    [B,C,H,W] ~ N(0,1), v_proj [Cp,C] ~ N(0, 1/C), u_proj [C,Cp] ~ N(0, 1/Cp),
    lam [4,B,Cp,H,W] ~ U(0,1), logits [4,B,1,3,H,W] ~ N(0,1); float32 alpha
    [4,Cp] ~ N(0,1) and gamma [Cp] ~ 0.5 + U(0,1).  Every tensor has its own
    child of SeedSequence(seed), in the order listed."""
    kids = np.random.SeedSequence(w.seed).spawn(7)
    return {
        "x": _fill(kids[0], "normal", (w.B, w.C, w.H, w.W), 1.0, True),
        "v_proj": _fill(kids[1], "normal", (w.Cp, w.C), float(1.0 / np.sqrt(w.C)), True),
        "u_proj": _fill(kids[2], "normal", (w.C, w.Cp), float(1.0 / np.sqrt(w.Cp)), True),
        "lam": _fill(kids[3], "uniform", (4, w.B, w.Cp, w.H, w.W), 1.0, True),
        "logits": _fill(kids[4], "normal", (4, w.B, 1, 3, w.H, w.W), 1.0, True),
        "alpha": _fill(kids[5], "normal", (4, w.Cp), 1.0, False),
        "gamma": (0.5 + _fill(kids[6], "uniform", (w.Cp,), 1.0, False)).astype(np.float32),
    }
