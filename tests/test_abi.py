"""CPU checks of the C-ABI library: it loads, exports every symbol that
include/gspn.h declares, and rejects bad arguments on the host (no GPU, no
compute)."""
import ctypes
import os
import re

import pytest

import linear_spatial_propagation_b200 as lsp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gspn.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gspn_\w+)\s*\(", src)))


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(lsp.EXPORTS)


def test_library_loads_and_exports_every_declared_symbol():
    lib = lsp.load()
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_version_and_status_strings():
    assert lsp.gspn_version() >= 100
    assert lsp.gspn_status_string(0) == "ok"
    for s in range(1, 8):
        assert lsp.gspn_status_string(s) and lsp.gspn_status_string(s) != "unknown status"
    assert "timed out" in lsp.gspn_status_string(6)
    assert lsp.gspn_status_string(99) == "unknown status"


def test_wait_settings_round_trip():
    """The process-wide wait limit, stall hook and sync-check switch return
    their previous values; a limit of 0 restores the 2 s default."""
    assert lsp.gspn_set_wait_limit_ns(12345) == 2_000_000_000
    assert lsp.gspn_set_wait_limit_ns(0) == 12345
    assert lsp.gspn_set_wait_limit_ns(0) == 2_000_000_000
    assert lsp.gspn_set_stall_test(1) == 0
    assert lsp.gspn_set_stall_test(0) == 1
    assert lsp.gspn_set_sync_check(7) == 0
    assert lsp.gspn_set_sync_check(0) == 1


def test_device_status_rejects_a_bad_descriptor():
    assert lsp.gspn_device_status(lsp.make_desc(0, 1, 8, 8), 0, 0, 0) == 1
    assert lsp.gspn_device_status(lsp.make_desc(1, 1, 8, 8, dir_mask=0), 1, 0, 0) == 1


A = 1 << 20  # a 16-byte aligned fake device address: never dereferenced on rejected calls


def fwd(desc, x=A, lg=A, lam=A, out=A, ws=0, nbytes=0):
    return lsp.gspn_fwd(desc, x, lg, lam, out, ws, nbytes, 0)


def bwd(desc, ptrs=(A,) * 7):
    return lsp.gspn_bwd(desc, *ptrs, 0, 0, 0)


@pytest.mark.parametrize("kw", [
    dict(B=0), dict(C=0), dict(H=0), dict(W=-1), dict(dir_mask=0), dict(dir_mask=16), dict(dir_mask=33),
    dict(groups=0), dict(groups=3),                      # 3 does not divide 8
    dict(H=6, W=8, groups=4, dir_mask=1),                # T2B needs g | H
    dict(H=8, W=6, groups=4, dir_mask=4),                # L2R needs g | W
    dict(H=1 << 21),
])
def test_invalid_descriptors_are_rejected_before_launch(kw):
    base = dict(B=2, C=3, H=8, W=8, dir_mask=15, groups=1, shared=False, dtype="bf16")
    base.update(kw)
    d = lsp.make_desc(**base)
    assert fwd(d) == 1
    assert bwd(d) == 1
    assert lsp.gspn_workspace_size(d, 0) == 0 and lsp.gspn_workspace_size(d, 1) == 0
    assert lsp.gspn_launches_per_call(d, 0) == 0
    assert lsp.gspn_variant_name(d, 0) == "invalid"


def test_groups_only_constrain_enabled_scan_axes():
    # g = 4 divides H = 8 but not W = 6; a column-free direction set is fine
    d = lsp.make_desc(1, 1, 8, 6, dir_mask=1 | 2, groups=4)
    assert lsp.gspn_launches_per_call(d, 0) >= 1


def test_unknown_dtype_is_unsupported():
    d = lsp.make_desc(1, 1, 4, 4, 15, 1, False, 7)
    assert fwd(d) == 2


def test_null_descriptor_and_pointers():
    lib = lsp.load()
    assert lib.gspn_fwd(None, A, A, A, A, None, 0, None) == 1
    d = lsp.make_desc(1, 2, 4, 4)
    assert fwd(d, x=0) == 1
    assert fwd(d, out=0) == 1
    for q in range(7):
        p = [A] * 7
        p[q] = 0
        assert bwd(d, tuple(p)) == 1


def test_misaligned_pointers():
    d = lsp.make_desc(1, 2, 4, 4)
    assert fwd(d, lam=A + 8) == 3
    assert fwd(d, out=A + 2) == 3
    p = [A] * 7
    p[5] = A + 4
    assert bwd(d, tuple(p)) == 3


def test_python_helpers_raise_on_error():
    with pytest.raises(lsp.GspnError) as e:
        st = fwd(lsp.make_desc(1, 1, 4, 4, dir_mask=0))
        raise lsp.GspnError(st, "gspn_fwd")
    assert e.value.status == 1


@pytest.mark.parametrize("args, fwd, bwd", [
    # planes of at most 64x64 in any mode: one CTA per plane, one warp per direction
    ((8, 96, 56, 56, 15, 1, False, "f32"), ("small_plane_fwd", 1), ("small_plane_bwd", 1)),
    ((1, 2, 64, 64, 5, 2, False, "bf16"), ("small_plane_fwd", 1), ("small_plane_bwd", 1)),
    ((3, 9, 64, 64, 15, 1, True, "bf16"), ("small_plane_fwd", 1), ("small_plane_bwd", 3)),  # C % 8 != 0
    ((1, 1, 16, 16, 1, 1, False, "f32"), ("small_plane_fwd", 1), ("small_plane_bwd", 1)),
    # longer lines with H, W multiples of 8 (up to 512): the large-plane forward
    ((2, 6, 128, 128, 15, 1, True, "bf16"), ("large_plane_fwd", 2), ("generic_bwd", 3)),  # C % 4 != 0; taps kernel
    ((1, 4, 512, 256, 15, 1, True, "bf16"), ("large_plane_fwd", 2), ("generic_bwd", 3)),
    ((1, 2, 72, 320, 5, 1, False, "f32"), ("large_plane_fwd", 1), ("generic_bwd", 1)),
    # anything else: the generic kernels
    ((1, 2, 65, 64, 15, 1, False, "f32"), ("generic_fwd", 1), ("generic_bwd", 1)),
    ((1, 2, 97, 41, 9, 1, False, "f32"), ("generic_fwd", 1), ("generic_bwd", 1)),
    ((1, 2, 1024, 8, 15, 1, True, "bf16"), ("generic_fwd", 1), ("generic_bwd", 3)),  # lines above 512
])
def test_path_chooser(args, fwd, bwd):
    d = lsp.make_desc(*args)
    assert (lsp.gspn_variant_name(d, 0), lsp.gspn_launches_per_call(d, 0)) == fwd
    assert (lsp.gspn_variant_name(d, 1), lsp.gspn_launches_per_call(d, 1)) == bwd


@pytest.mark.parametrize("args, fast", [
    ((32, 1152, 64, 64, 15, 1, True, "bf16"), "compact64_tma"),
    ((2, 1152, 128, 128, 15, 1, True, "bf16"), "compact128_tma"),
    ((1, 4, 128, 128, 15, 4, True, "bf16"), "compact128_tma"),
])
def test_compact_shapes_take_the_tma_kernels_when_the_encoder_is_there(args, fast):
    """The compact shapes run on the TMA-fed kernels wherever the driver's
    tensor-map encoder is available (a GPU host); without it the chooser falls
    back to the small-plane, large-plane (forward) or generic kernels, which
    also cover them."""
    d = lsp.make_desc(*args)
    small = max(args[2], args[3]) <= 64
    for bwd, launches in ((0, 2), (1, 3)):
        name = lsp.gspn_variant_name(d, bwd)
        suffix = "_bwd" if bwd else "_fwd"
        if name == fast + suffix:
            assert lsp.gspn_launches_per_call(d, bwd) == launches
        else:
            fallback = "small_plane" if small else ("generic" if bwd else "large_plane")
            assert name == fallback + suffix


@pytest.mark.parametrize("args", [
    (2, 1152, 256, 256, 15, 1, True, "bf16"),
    (1, 16, 136, 200, 15, 2, True, "bf16"),
    (1, 8, 256, 168, 10, 4, True, "bf16"),
    (1, 8, 144, 256, 1, 1, True, "bf16"),
])
def test_compact_large_planes_take_the_warp_per_plane_kernel_when_the_encoder_is_there(args):
    """Compact bf16 planes with lines of 129..256 positions, whole groups of 8
    channels and a row direction run on the compact large-plane kernels (the
    forward in two launches: the taps table, then the scan) where the
    tensor-map encoder is available, else on the general large-plane forward."""
    d = lsp.make_desc(*args)
    name = lsp.gspn_variant_name(d, 0)
    assert name in ("large_compact_fwd", "large_plane_fwd")
    assert lsp.gspn_launches_per_call(d, 0) == 2
    if name == "large_compact_fwd":
        # and its backward: states pass, adjoint pass, dlogits, after the taps table
        assert lsp.gspn_variant_name(d, 1) == "large_compact_bwd"
        assert lsp.gspn_launches_per_call(d, 1) == 4


@pytest.mark.parametrize("args", [
    (1, 4, 256, 256, 15, 1, True, "bf16"),     # C % 8 != 0
    (1, 8, 256, 256, 15, 1, False, "bf16"),    # per-channel taps
    (1, 8, 256, 256, 15, 1, True, "f32"),      # fp32
    (1, 8, 256, 256, 12, 1, True, "bf16"),     # column scans only: the output would be written by columns
    (1, 8, 512, 256, 15, 1, True, "bf16"),     # lines above 256
    (1, 8, 128, 96, 15, 1, True, "bf16"),      # no line above 128
])
def test_other_large_planes_stay_off_the_compact_kernel(args):
    d = lsp.make_desc(*args)
    assert lsp.gspn_variant_name(d, 0) != "large_compact_fwd"
    assert lsp.gspn_variant_name(d, 1) != "large_compact_bwd"


# ---- the compressed propagation block ---------------------------------------------

def _block_fwd(desc, ptr=A):
    return lsp.gspn_block_fwd(desc, ptr, ptr, ptr, ptr, ptr, ptr, ptr, ptr, 0, 0, 0)


@pytest.mark.parametrize("args, status", [
    ((0, 64, 16, 16, 2), 1),        # B < 1
    ((1, 0, 16, 16, 2), 1),         # C < 1
    ((1, 64, 16, 16, 0), 1),        # C_proxy < 1
    ((1, 64, 18, 16, 2, 4), 1),     # groups not dividing H
    ((1, 64, 16, 16, 33), 2),       # C_proxy above 32
    ((1, 64, 136, 16, 2), 2),       # lines above 128
    ((1, 60, 16, 16, 2), 2),        # C not a multiple of 8
    ((1, 64, 12, 16, 2), 2),        # H not a multiple of 8
    ((1, 3072 + 8, 16, 16, 2), 2),  # U beyond shared memory at C_proxy <= 16
    ((1, 1536 + 8, 16, 16, 32), 2),  # and at C_proxy 32
])
def test_block_rejects_descriptors_on_the_host(args, status):
    """Dimension and limit checks come before any device query, so the same
    status holds with or without a GPU; a rejected descriptor also has no
    workspace size."""
    d = lsp.make_block_desc(*args)
    assert _block_fwd(d) == status
    assert lsp.gspn_block_workspace_size(d) == 0


def test_block_rejects_a_bad_eps():
    for eps in (-1.0, 2.0, float("nan")):
        assert _block_fwd(lsp.make_block_desc(1, 64, 16, 16, 2, eps=eps)) == 1


def test_block_null_descriptor_and_status():
    lib = lsp.load()
    assert lib.gspn_block_fwd(None, *([None] * 8), None, 0, None) == 1
    assert lib.gspn_block_workspace_size(None) == 0
    assert lib.gspn_block_device_status(None, None, None) == 1
