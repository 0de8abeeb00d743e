"""GPU parity of the large-plane kernels against the oracle: the compact
forward and backward for channel-shared bf16 planes with lines of 129..256
positions (one warp per plane, groups of 8 channels), the general forward
(lines of 65..512 positions, one CTA streaming a plane line by line), and the
backward of the other large planes (the generic kernels, pipelined up to 256
positions per line).

Shapes: 256x256 and 512x512 compact bf16 (the planes beyond the on-chip
kernels), rectangular planes whose two scan directions use different warp
counts, per-channel fp32 taps, local groups and partial direction sets.
Canaries around the output catch stores outside it.  Tolerances as
everywhere: 1e-5 (fp32) and 1e-2 (bf16) of max|reference|.
"""
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

gu = pytest.importorskip("gpu_util")

CASES = [
    # B, C, H, W, dir_mask, groups, shared, dtype
    (1, 4, 256, 256, 15, 1, True, "bf16"),
    (1, 2, 512, 512, 15, 1, True, "bf16"),
    (2, 3, 200, 136, 15, 1, False, "bf16"),   # 4 warps for column lines, 3 for row lines
    (1, 3, 128, 96, 15, 4, False, "f32"),     # per-channel fp32, local groups
    (1, 2, 72, 320, 5, 1, True, "f32"),       # T2B + L2R only
    (1, 2, 264, 80, 10, 2, True, "bf16"),     # B2T + R2L, groups of 132 / 40 lines
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c)))
def test_large_plane_forward_matches_oracle(case):
    import linear_spatial_propagation_b200 as lsp
    t = gu.torch()
    B, C, H, W, mask, g, shared, dtype = case
    w = synth.Workload(f"large_{'x'.join(map(str, case))}", B, C, H, W, mask, g, shared, dtype, 1.0,
                       4000 + H + W + C)
    d = lsp.make_desc(B, C, H, W, mask, g, shared, dtype)
    assert lsp.gspn_variant_name(d, 0) == "large_plane_fwd"
    inp = synth.make_inputs(w, with_dout=False)
    dinp = gu.dev_inputs(w, inp)
    guard = 4096
    buf = t.full((dinp["x"].numel() + 2 * guard,), -3.0, dtype=dinp["x"].dtype, device="cuda")
    out = buf[guard:guard + dinp["x"].numel()].view(dinp["x"].shape)
    gu.run_fwd(w, dinp, out=out)
    t.cuda.synchronize()
    assert bool((buf[:guard] == -3.0).all()) and bool((buf[guard + out.numel():] == -3.0).all())
    gu.assert_close(gu.from_dev(out), oracle.fwd_workload(w, inp, nthreads=8), dtype, w.name)


def test_large_plane_forward_is_deterministic():
    t = gu.torch()
    w = synth.Workload("large_det", 1, 4, 256, 256, 15, 1, True, "bf16", 1.0, 4100)
    dinp = gu.dev_inputs(w, synth.make_inputs(w, with_dout=False))
    o1 = gu.run_fwd(w, dinp)
    o2 = gu.run_fwd(w, dinp)
    t.cuda.synchronize()
    assert bool(t.equal(o1, o2))


BWD_CASES = [
    # B, C, H, W, dir_mask, groups, shared, dtype, backward variant
    (1, 2, 256, 256, 15, 1, True, "bf16", "generic_bwd"),    # lines of 256: the pipelined kernel, 8 per lane
    (1, 2, 200, 136, 15, 2, False, "f32", "generic_bwd"),    # per-channel, local groups, two line lengths
    (1, 1, 512, 512, 15, 1, True, "bf16", "generic_bwd"),    # lines of 512: the kernel without prefetch
]


@pytest.mark.parametrize("case", BWD_CASES, ids=lambda c: "x".join(map(str, c[:8])))
def test_large_plane_backward_matches_oracle(case):
    """Backward of planes above 64x64 (other than the compact 64x64 / 128x128
    ones): dx, dlambda and dlogits against the oracle's adjoint."""
    import linear_spatial_propagation_b200 as lsp
    B, C, H, W, mask, g, shared, dtype, variant = case
    w = synth.Workload(f"large_bwd_{'x'.join(map(str, case[:8]))}", B, C, H, W, mask, g, shared, dtype, 1.0,
                       4200 + H + W + C, backward=True)
    assert lsp.gspn_variant_name(lsp.make_desc(B, C, H, W, mask, g, shared, dtype), 1) == variant
    inp = synth.make_inputs(w, with_dout=True)
    dinp = gu.dev_inputs(w, inp)
    dx, dlg, dlam = (gu.from_dev(t) for t in gu.run_bwd(w, dinp))
    rdx, rdlg, rdlam = oracle.bwd_workload(w, inp, nthreads=8)
    gu.assert_close(dx, rdx, dtype, f"{w.name} dx")
    gu.assert_close(dlam, rdlam, dtype, f"{w.name} dlam")
    gu.assert_close(dlg, rdlg, dtype, f"{w.name} dlogits")


LC_CASES = [
    # B, C, H, W, dir_mask, groups: compact bf16, whole groups of 8 channels
    (1, 8, 256, 256, 15, 1),
    (2, 16, 136, 200, 15, 2),   # H != W, local groups of 68 / 100 lines, 2 images
    (1, 8, 200, 256, 5, 1),     # top->bottom + left->right
    (1, 8, 256, 168, 10, 4),    # bottom->top + right->left (the transposed read in reverse), groups
    (1, 8, 256, 256, 3, 1),     # row scans only (no column sums)
    (1, 8, 144, 256, 1, 1),     # top->bottom only: straight to the output
    (1, 8, 256, 248, 2, 1),     # bottom->top only
    (1, 16, 248, 136, 11, 2),   # top->bottom + bottom->top + right->left
    (1, 8, 64, 144, 12 | 1, 1), # short columns (lanes beyond the line idle), all but bottom->top
    (1, 8, 8, 256, 15, 1),      # 8-row planes: row chunks of 4 lines, one lane per column line
    (1, 8, 256, 8, 15, 2),      # 8-column planes: one column chunk per direction, local groups
    (1, 8, 16, 144, 13, 1),     # top->bottom + left->right + right->left on a flat plane
]


@pytest.mark.parametrize("case", LC_CASES, ids=lambda c: "x".join(map(str, c)))
def test_large_compact_forward_matches_oracle(case):
    import linear_spatial_propagation_b200 as lsp
    t = gu.torch()
    B, C, H, W, mask, g = case
    w = synth.Workload(f"lc_{'x'.join(map(str, case))}", B, C, H, W, mask, g, True, "bf16", 1.0, 4400 + H + W + mask)
    d = lsp.make_desc(B, C, H, W, mask, g, True, "bf16")
    assert lsp.gspn_variant_name(d, 0) == "large_compact_fwd"
    assert lsp.gspn_launches_per_call(d, 0) == 2
    inp = synth.make_inputs(w, with_dout=False)
    dinp = gu.dev_inputs(w, inp)
    guard = 4096
    buf = t.full((dinp["x"].numel() + 2 * guard,), -3.0, dtype=dinp["x"].dtype, device="cuda")
    out = buf[guard:guard + dinp["x"].numel()].view(dinp["x"].shape)
    ws = t.empty(lsp.gspn_workspace_size(d, 0), dtype=t.uint8, device="cuda")
    gu.run_fwd(w, dinp, out=out, ws=ws)
    stream = t.cuda.current_stream().cuda_stream
    assert lsp.gspn_device_status(d, 0, ws.data_ptr(), stream) == 0
    assert bool((buf[:guard] == -3.0).all()) and bool((buf[guard + out.numel():] == -3.0).all())
    gu.assert_close(gu.from_dev(out), oracle.fwd_workload(w, inp, nthreads=8), "bf16", w.name)


def test_large_compact_forward_is_deterministic():
    t = gu.torch()
    w = synth.Workload("lc_det", 1, 16, 256, 256, 15, 1, True, "bf16", 1.0, 4500)
    dinp = gu.dev_inputs(w, synth.make_inputs(w, with_dout=False))
    o1 = gu.run_fwd(w, dinp)
    o2 = gu.run_fwd(w, dinp)
    t.cuda.synchronize()
    assert bool(t.equal(o1, o2))


def test_large_compact_forward_full_size_sampled_planes():
    """2 x 1152 x 256 x 256 (the 256-square latent at the 1K channel count) in
    the launch configuration the bench times; the oracle checks sampled planes."""
    import numpy as np
    import linear_spatial_propagation_b200 as lsp
    w = synth.Workload("lc_full", 2, 1152, 256, 256, 15, 1, True, "bf16", 1.0, 4600)
    assert lsp.gspn_variant_name(lsp.make_desc(2, 1152, 256, 256, 15, 1, True, "bf16"), 0) == "large_compact_fwd"
    inp = synth.make_inputs(w, with_dout=False)
    out = gu.run_fwd(w, gu.dev_inputs(w, inp))
    rng = np.random.default_rng(5)
    picks = {(0, 0), (1, 1151), (0, 577)}
    while len(picks) < 6:
        picks.add((int(rng.integers(2)), int(rng.integers(1152))))
    one = w.replace(B=1, C=1)
    for b, c in sorted(picks):
        got = gu.from_dev(out[b:b + 1, c:c + 1])
        gu.assert_close(got, oracle.fwd_workload(one, synth.plane_slice(w, inp, b, c)), "bf16", f"plane ({b},{c})")


LCB_CASES = [
    # B, C, H, W, dir_mask, groups: compact bf16 backward, whole groups of 8 channels
    (1, 8, 256, 256, 15, 1),
    (2, 16, 136, 200, 15, 2),   # H != W, local groups, 2 images (2 CTAs per image)
    (1, 8, 200, 256, 5, 1),     # top->bottom + left->right
    (1, 8, 256, 168, 10, 4),    # bottom->top + right->left, groups
    (1, 8, 256, 256, 3, 1),     # row scans only
    (1, 8, 144, 256, 1, 1),     # top->bottom only
    (1, 16, 248, 136, 11, 2),   # three directions
    (1, 8, 8, 256, 15, 1),      # 8-row planes
    (1, 8, 256, 8, 15, 2),      # 8-column planes, groups
]


@pytest.mark.parametrize("case", LCB_CASES, ids=lambda c: "x".join(map(str, c)))
def test_large_compact_backward_matches_oracle(case):
    """The compact large-plane backward (a states pass, the adjoint pass, the
    dlogits kernel): dx, dlambda and the channel-summed dlogits against the
    oracle's adjoint."""
    import linear_spatial_propagation_b200 as lsp
    t = gu.torch()
    B, C, H, W, mask, g = case
    w = synth.Workload(f"lcb_{'x'.join(map(str, case))}", B, C, H, W, mask, g, True, "bf16", 1.0, 4700 + H + W + mask,
                       backward=True)
    d = lsp.make_desc(B, C, H, W, mask, g, True, "bf16")
    assert lsp.gspn_variant_name(d, 1) == "large_compact_bwd"
    assert lsp.gspn_launches_per_call(d, 1) == 4
    inp = synth.make_inputs(w, with_dout=True)
    dinp = gu.dev_inputs(w, inp)
    ws = t.empty(lsp.gspn_workspace_size(d, 1), dtype=t.uint8, device="cuda")
    dx, dlg, dlam = lsp.backward(dinp["x"], dinp["logits"], dinp["lam"], dinp["dout"], dir_mask=mask, groups=g,
                                 shared=True, ws=ws)
    assert lsp.gspn_device_status(d, 1, ws.data_ptr(), t.cuda.current_stream().cuda_stream) == 0
    rdx, rdlg, rdlam = oracle.bwd_workload(w, inp, nthreads=8)
    gu.assert_close(gu.from_dev(dx), rdx, "bf16", f"{w.name} dx")
    gu.assert_close(gu.from_dev(dlam), rdlam, "bf16", f"{w.name} dlam")
    gu.assert_close(gu.from_dev(dlg), rdlg, "bf16", f"{w.name} dlogits")


def test_large_compact_backward_2x64_256_square():
    """256-square planes, 2 images of 64 channels (8 CTAs per image add their
    tap values into the same sums), checked whole against the oracle."""
    w = synth.Workload("lcb_2x64_256", 2, 64, 256, 256, 15, 1, True, "bf16", 1.0, 4800, backward=True)
    inp = synth.make_inputs(w, with_dout=True)
    dx, dlg, dlam = (gu.from_dev(x) for x in gu.run_bwd(w, gu.dev_inputs(w, inp)))
    rdx, rdlg, rdlam = oracle.bwd_workload(w, inp, nthreads=8)
    gu.assert_close(dx, rdx, "bf16", "dx")
    gu.assert_close(dlam, rdlam, "bf16", "dlam")
    gu.assert_close(dlg, rdlg, "bf16", "dlogits")


def test_large_compact_backward_repeats():
    """dx and dlambda repeat bit for bit; dlogits are fp32 sums of the warps'
    tap values in arrival order, so they repeat to within rounding."""
    t = gu.torch()
    w = synth.Workload("lcb_det", 1, 16, 136, 144, 15, 1, True, "bf16", 1.0, 4900, backward=True)
    d = gu.dev_inputs(w, synth.make_inputs(w, with_dout=True))
    r1 = tuple(x.clone() for x in gu.run_bwd(w, d))
    r2 = gu.run_bwd(w, d)
    t.cuda.synchronize()
    assert bool(t.equal(r1[0], r2[0])) and bool(t.equal(r1[2], r2[2]))
    a, b = r1[1].float(), r2[1].float()
    assert float((a - b).abs().max()) <= 1e-2 * float(a.abs().max())


def test_large_compact_backward_writes_only_its_outputs():
    """Guard bands around dx, dlogits and dlambda stay untouched (column
    directions write dlambda as 4-column pieces per row)."""
    import linear_spatial_propagation_b200 as lsp
    t = gu.torch()
    w = synth.Workload("lcb_guard", 1, 8, 144, 136, 15, 2, True, "bf16", 1.0, 4950, backward=True)
    d = gu.dev_inputs(w, synth.make_inputs(w, with_dout=True))
    guard = 4096

    def framed(like):
        buf = t.full((like.numel() + 2 * guard,), -5.0, dtype=like.dtype, device="cuda")
        return buf, buf[guard:guard + like.numel()].view(like.shape)

    (bx, dx), (bg, dlg), (bl, dlam) = framed(d["x"]), framed(d["logits"]), framed(d["lam"])
    lsp.backward(d["x"], d["logits"], d["lam"], d["dout"], dir_mask=15, groups=2, shared=True, grads=(dx, dlg, dlam))
    t.cuda.synchronize()
    for name, buf, inner in (("dx", bx, dx), ("dlogits", bg, dlg), ("dlambda", bl, dlam)):
        assert bool((buf[:guard] == -5.0).all()) and bool((buf[guard + inner.numel():] == -5.0).all()), name
