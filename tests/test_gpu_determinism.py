"""Repeat-determinism of the backward: two calls on the same inputs give
bit-identical dx, dlogits and dlambda.

dx and dlambda never depend on timing.  The channel-shared tap gradients of
the small-plane and generic kernels sum over channels with order-independent
fixed-point atomics, so they repeat bit for bit at any size.  The compact
TMA kernels sum each CTA's share in a fixed order and then add the CTAs'
shares into global fp32 sums; the cases here have two CTAs per batch image,
where fp32 addition (commutative) still gives one result."""
import pytest

import synth

pytestmark = pytest.mark.gpu

gu = pytest.importorskip("gpu_util")

CASES = [
    # B, C, H, W, dir_mask, groups, shared, dtype: expected backward variant
    ((2, 24, 56, 56, 15, 1, True, "bf16"), "small_plane_bwd"),
    ((1, 16, 28, 28, 15, 4, True, "f32"), "small_plane_bwd"),
    ((1, 6, 96, 72, 15, 1, True, "bf16"), "generic_bwd"),
    ((1, 3, 80, 40, 15, 2, True, "f32"), "generic_bwd"),
    ((2, 8, 64, 64, 15, 1, False, "bf16"), "small_plane_bwd"),
    ((2, 16, 64, 64, 15, 1, True, "bf16"), "compact64_tma_bwd"),    # 2 CTAs per image
    ((1, 8, 128, 128, 15, 1, True, "bf16"), "compact128_tma_bwd"),  # 2 CTAs per image
]


@pytest.mark.parametrize("case,variant", CASES, ids=lambda c: "x".join(map(str, c)) if isinstance(c, tuple) else c)
def test_backward_repeats_bit_for_bit(case, variant):
    import linear_spatial_propagation_b200 as lsp
    t = gu.torch()
    B, C, H, W, mask, g, shared, dtype = case
    w = synth.Workload("det_" + "x".join(map(str, case)), B, C, H, W, mask, g, shared, dtype, 1.0, 5000 + H + C)
    assert lsp.gspn_variant_name(lsp.make_desc(*case), 1) == variant
    d = gu.dev_inputs(w, synth.make_inputs(w, with_dout=True))
    r1 = gu.run_bwd(w, d)
    r1 = tuple(x.clone() for x in r1)
    r2 = gu.run_bwd(w, d)
    t.cuda.synchronize()
    for name, a, b in zip(("dx", "dlogits", "dlambda"), r1, r2):
        assert bool(t.equal(a, b)), f"{name} differs between two identical calls"
