"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle on
identical seeded inputs, element by element.

* every workload at a reduced batch/channel count (same planes, modes and
  distributions) that the oracle finishes in seconds;
* every workload at its full size, on sampled (b, c) planes the oracle
  computes one by one (the backward workload in full: its channel-summed
  tap gradients need every channel);
* random shapes and edge cases: W = 1, H = 1, odd and prime sizes, g = L,
  single directions, ragged channel counts;
* guard bands around every output (compute-sanitizer is not available, so
  out-of-bounds stores are caught by canaries).
"""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

gu = pytest.importorskip("gpu_util")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    t = pytest.importorskip("torch")
    if not t.cuda.is_available():
        pytest.skip("no CUDA device")
    import linear_spatial_propagation_b200 as lsp
    lsp.load(build_if_missing=False)
    yield


REDUCED = {
    "t2b_f32_b1c4_16x16": dict(),
    "4dir_f32_b8c96_56x56": dict(B=2, C=10),
    "4dir_local4_bf16_b32c192_28x28": dict(B=2, C=18),
    "compact_4dir_bf16_b32c1152_64x64": dict(B=3, C=40),
    "compact_4dir_bf16_b2c1152_128x128_fwdbwd": dict(B=1, C=7),
}


def check_fwd(w, inp=None, nthreads=8):
    inp = inp if inp is not None else synth.make_inputs(w, with_dout=False)
    got = gu.from_dev(gu.run_fwd(w, gu.dev_inputs(w, inp)))
    want = oracle.fwd_workload(w, inp, nthreads=nthreads)
    return gu.assert_close(got, want, w.dtype, f"{w.name} fwd")


def check_bwd(w, inp=None, nthreads=8):
    inp = inp if inp is not None else synth.make_inputs(w, with_dout=True)
    dinp = gu.dev_inputs(w, inp)
    dx, dlg, dlam = (gu.from_dev(t) for t in gu.run_bwd(w, dinp))
    rdx, rdlg, rdlam = oracle.bwd_workload(w, inp, nthreads=nthreads)
    gu.assert_close(dx, rdx, w.dtype, f"{w.name} dx")
    gu.assert_close(dlam, rdlam, w.dtype, f"{w.name} dlam")
    gu.assert_close(dlg, rdlg, w.dtype, f"{w.name} dlogits")


@pytest.mark.parametrize("name", list(REDUCED))
def test_workload_reduced_forward(name):
    w = synth.WORKLOADS[name].replace(**REDUCED[name])
    check_fwd(w)


@pytest.mark.parametrize("name", list(REDUCED))
def test_workload_reduced_backward(name):
    w = synth.WORKLOADS[name].replace(**REDUCED[name])
    check_bwd(w)


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_workload_full_size_sampled_planes(name):
    w = synth.WORKLOADS[name]
    inp = synth.make_inputs(w, with_dout=False)
    out = gu.run_fwd(w, gu.dev_inputs(w, inp))
    rng = np.random.default_rng(7)
    picks = {(0, 0), (w.B - 1, w.C - 1)}
    while len(picks) < min(12, w.B * w.C):
        picks.add((int(rng.integers(w.B)), int(rng.integers(w.C))))
    one = w.replace(B=1, C=1)
    for b, c in sorted(picks):
        sl = synth.plane_slice(w, inp, b, c)
        got = gu.from_dev(out[b:b + 1, c:c + 1])
        gu.assert_close(got, oracle.fwd_workload(one, sl), w.dtype, f"{name} plane ({b},{c})")


def test_backward_workload_full_size():
    w = synth.WORKLOADS["compact_4dir_bf16_b2c1152_128x128_fwdbwd"]
    check_bwd(w, nthreads=max(1, oracle.max_threads()))


def test_headline_backward_full_size_sampled():
    """The 32x1152x64x64 backward in its bench launch configuration.  dx and
    dlambda of sampled planes against the oracle plane by plane; dlogits (a
    sum over all channels) through a second full-size launch whose upstream
    gradient is zero outside the sampled planes, so that the oracle needs only
    those planes: planes with a zero gradient contribute nothing to any
    gradient."""
    t = gu.torch()
    w = synth.WORKLOADS["compact_4dir_bf16_b32c1152_64x64"].replace(backward=True)
    inp = synth.make_inputs(w, with_dout=True)
    rng = np.random.default_rng(11)
    picks = {(0, 0), (w.B - 1, w.C - 1), (5, 17)}
    while len(picks) < 8:
        picks.add((int(rng.integers(w.B)), int(rng.integers(w.C))))
    one = w.replace(B=1, C=1)
    dinp = gu.dev_inputs(w, inp)
    dx, _, dlam = gu.run_bwd(w, dinp)
    for b, c in sorted(picks):
        rdx, _, rdlam = oracle.bwd_workload(one, synth.plane_slice(w, inp, b, c))
        gu.assert_close(gu.from_dev(dx[b:b + 1, c:c + 1]), rdx, w.dtype, f"dx plane ({b},{c})")
        gu.assert_close(gu.from_dev(dlam[:, b:b + 1, c:c + 1]), rdlam, w.dtype, f"dlam plane ({b},{c})")
    # dlogits with the upstream gradient restricted to the sampled planes
    mask = np.zeros((w.B, w.C, 1, 1), dtype=bool)
    for b, c in picks:
        mask[b, c] = True
    sparse = dict(inp)
    sparse["dout"] = np.where(mask, inp["dout"], np.zeros_like(inp["dout"]))
    dinp["dout"] = gu.to_dev(sparse["dout"], w.dtype)
    dx2, dlg2, _ = gu.run_bwd(w, dinp)
    want = np.zeros(tuple(dlg2.shape))
    for b, c in sorted(picks):
        _, rdlg, _ = oracle.bwd_workload(one, synth.plane_slice(w, sparse, b, c))
        want[:, b:b + 1] += rdlg
    gu.assert_close(gu.from_dev(dlg2), want, w.dtype, "dlogits (sampled upstream gradient)")
    # and a plane outside the sample gets no gradient
    b, c = next((b, c) for b in range(w.B) for c in range(w.C) if (b, c) not in picks)
    assert float(t.count_nonzero(dx2[b, c]).item()) == 0.0


SHAPES = [
    # B, C, H, W, mask, groups, shared, dtype
    (1, 1, 1, 1, 15, 1, False, "f32"),
    (1, 2, 1, 9, 15, 1, False, "f32"),
    (1, 2, 9, 1, 15, 1, True, "bf16"),
    (2, 3, 2, 2, 15, 2, False, "f32"),
    (1, 3, 7, 13, 1, 1, False, "f32"),
    (1, 3, 13, 7, 2, 1, True, "f32"),
    (1, 3, 5, 31, 4, 1, False, "bf16"),
    (1, 3, 31, 5, 8, 1, True, "bf16"),
    (2, 5, 33, 65, 15, 1, True, "f32"),
    (1, 4, 64, 64, 15, 64, True, "bf16"),
    (1, 4, 64, 64, 15, 16, False, "bf16"),
    (3, 9, 64, 64, 15, 1, True, "bf16"),
    (1, 6, 64, 64, 5, 2, True, "f32"),
    (1, 2, 97, 41, 9, 1, False, "f32"),
    (2, 37, 64, 64, 15, 1, True, "bf16"),
    (2, 16, 64, 64, 15, 1, True, "bf16"),
    (1, 8, 64, 64, 15, 4, True, "bf16"),
    (3, 24, 64, 64, 15, 64, True, "bf16"),
    (5, 8, 64, 64, 15, 2, True, "bf16"),
    (1, 2, 130, 70, 15, 1, True, "bf16"),
    (1, 2, 150, 90, 15, 3, False, "f32"),  # lines of 129..256 positions: 8 positions per lane
    # 128x128 compact bf16 with C % 4 == 0: the TMA-fed 128x128 forward
    (1, 4, 128, 128, 15, 1, True, "bf16"),
    (2, 12, 128, 128, 15, 1, True, "bf16"),
    (1, 8, 128, 128, 15, 4, True, "bf16"),
    (1, 4, 128, 128, 15, 128, True, "bf16"),
    (1, 600, 128, 128, 15, 2, True, "bf16"),  # 150 groups of 4 planes: CTAs take more than one
    (1, 1, 257, 33, 3, 1, False, "f32"),
]


def shape_workload(B, C, H, W, mask, g, shared, dt, seed):
    return synth.Workload(f"shape_{B}x{C}x{H}x{W}_m{mask}_g{g}_{'s' if shared else 'p'}_{dt}", B, C, H, W, mask,
                          g, shared, dt, 1.5, seed)


@pytest.mark.parametrize("case", SHAPES, ids=lambda c: "x".join(map(str, c)))
def test_random_shapes_forward(case):
    check_fwd(shape_workload(*case, seed=100 + sum(case[:4])))


@pytest.mark.parametrize("case", SHAPES, ids=lambda c: "x".join(map(str, c)))
def test_random_shapes_backward(case):
    check_bwd(shape_workload(*case, seed=200 + sum(case[:4])))


def test_guard_bands_untouched():
    t = gu.torch()
    w = shape_workload(2, 5, 64, 64, 15, 1, True, "bf16", 301)
    inp = synth.make_inputs(w, with_dout=True)
    d = gu.dev_inputs(w, inp)
    guard = 4096
    n = w.B * w.C * w.H * w.W
    buf = t.full((n + 2 * guard,), 7.0, dtype=t.bfloat16, device="cuda")
    out = buf[guard:guard + n].view(w.B, w.C, w.H, w.W)
    gu.run_fwd(w, d, out=out)
    t.cuda.synchronize()
    assert bool((buf[:guard] == 7.0).all()) and bool((buf[guard + n:] == 7.0).all())
    want = oracle.fwd_workload(w, inp)
    gu.assert_close(gu.from_dev(out), want, w.dtype, "guarded out")
    # backward outputs
    import linear_spatial_propagation_b200 as lsp
    bufs = [t.full((x.numel() + 2 * guard,), -3.0, dtype=t.bfloat16, device="cuda") for x in
            (d["x"], d["logits"], d["lam"])]
    views = [b[guard:guard + x.numel()].view(x.shape) for b, x in zip(bufs, (d["x"], d["logits"], d["lam"]))]
    lsp.backward(d["x"], d["logits"], d["lam"], d["dout"], dir_mask=15, shared=True, grads=tuple(views))
    t.cuda.synchronize()
    for b, v in zip(bufs, views):
        assert bool((b[:guard] == -3.0).all()) and bool((b[guard + v.numel():] == -3.0).all())


def test_non_default_stream_and_repeat_calls_are_deterministic_forward():
    t = gu.torch()
    w = shape_workload(2, 9, 64, 64, 15, 1, True, "bf16", 401)
    inp = synth.make_inputs(w, with_dout=False)
    d = gu.dev_inputs(w, inp)
    s = t.cuda.Stream()
    with t.cuda.stream(s):
        a = gu.run_fwd(w, d)
        b = gu.run_fwd(w, d)
    s.synchronize()
    assert bool(t.equal(a, b))


def test_workspace_errors_on_gpu():
    import linear_spatial_propagation_b200 as lsp
    t = gu.torch()
    w = synth.WORKLOADS["compact_4dir_bf16_b2c1152_128x128_fwdbwd"].replace(C=4)
    d = lsp.make_desc(w.B, w.C, w.H, w.W, w.dir_mask, w.groups, w.shared, w.dtype)
    need = lsp.gspn_workspace_size(d, 1)
    if need == 0:
        pytest.skip("no workspace needed")
    x = t.zeros(w.B, w.C, w.H, w.W, dtype=t.bfloat16, device="cuda")
    st = lsp.gspn_bwd(d, *(x.data_ptr(),) * 7, 0, 0, 0)
    assert st == 4
    ws = t.empty(need, dtype=t.uint8, device="cuda")
    st = lsp.gspn_bwd(d, *(x.data_ptr(),) * 7, ws.data_ptr(), need - 1, 0)
    assert st == 4


def test_compact128_forward_dispatch_guards_and_repeats():
    """The 128x128 compact forward: its dispatch, out-of-bounds canaries around
    the output and after the exact workspace (which holds its row-sum scratch
    planes), and bit-identical repeats on a side stream."""
    import linear_spatial_propagation_b200 as lsp
    t = gu.torch()
    w = shape_workload(1, 8, 128, 128, 15, 1, True, "bf16", 501)
    d = lsp.make_desc(w.B, w.C, w.H, w.W, w.dir_mask, w.groups, w.shared, w.dtype)
    assert lsp.gspn_variant_name(d, 0) == "compact128_tma_fwd"
    assert lsp.gspn_launches_per_call(d, 0) == 2
    inp = synth.make_inputs(w, with_dout=False)
    dinp = gu.dev_inputs(w, inp)
    guard = 4096
    n = w.B * w.C * w.H * w.W
    buf = t.full((n + 2 * guard,), 7.0, dtype=t.bfloat16, device="cuda")
    out = buf[guard:guard + n].view(w.B, w.C, w.H, w.W)
    need = lsp.gspn_workspace_size(d, 0)
    wsbuf = t.full((need + guard,), 0x5A, dtype=t.uint8, device="cuda")
    s = t.cuda.Stream()
    s.wait_stream(t.cuda.current_stream())  # the inputs and canaries are written on the default stream
    with t.cuda.stream(s):
        lsp.forward(dinp["x"], dinp["logits"], dinp["lam"], dir_mask=15, shared=True, out=out, ws=wsbuf[:need])
        again = lsp.forward(dinp["x"], dinp["logits"], dinp["lam"], dir_mask=15, shared=True)
    s.synchronize()
    assert bool((buf[:guard] == 7.0).all()) and bool((buf[guard + n:] == 7.0).all())
    assert bool((wsbuf[need:] == 0x5A).all())
    assert bool(t.equal(out, again))
    gu.assert_close(gu.from_dev(out), oracle.fwd_workload(w, inp), w.dtype, "128x128 compact forward")


def test_compact128_backward_dispatch_and_guards():
    """The 128x128 compact backward: its dispatch, canaries around every
    gradient and after the exact workspace (tap table, tap sums and the
    per-warp dx and a_B scratch planes), and the oracle's gradients."""
    import linear_spatial_propagation_b200 as lsp
    t = gu.torch()
    w = shape_workload(1, 8, 128, 128, 15, 1, True, "bf16", 601)
    d = lsp.make_desc(w.B, w.C, w.H, w.W, w.dir_mask, w.groups, w.shared, w.dtype)
    assert lsp.gspn_variant_name(d, 1) == "compact128_tma_bwd"
    assert lsp.gspn_launches_per_call(d, 1) == 3
    inp = synth.make_inputs(w, with_dout=True)
    dinp = gu.dev_inputs(w, inp)
    guard = 4096
    bufs = [t.full((x.numel() + 2 * guard,), -3.0, dtype=t.bfloat16, device="cuda") for x in
            (dinp["x"], dinp["logits"], dinp["lam"])]
    views = [b[guard:guard + x.numel()].view(x.shape) for b, x in zip(bufs, (dinp["x"], dinp["logits"], dinp["lam"]))]
    need = lsp.gspn_workspace_size(d, 1)
    wsbuf = t.full((need + guard,), 0x5A, dtype=t.uint8, device="cuda")
    lsp.backward(dinp["x"], dinp["logits"], dinp["lam"], dinp["dout"], dir_mask=15, shared=True, grads=tuple(views),
                 ws=wsbuf[:need])
    t.cuda.synchronize()
    for b, v in zip(bufs, views):
        assert bool((b[:guard] == -3.0).all()) and bool((b[guard + v.numel():] == -3.0).all())
    assert bool((wsbuf[need:] == 0x5A).all())
    assert int(wsbuf[:4].view(t.int32).item()) == 0  # no device-side wait gave up
    rdx, rdlg, rdlam = oracle.bwd_workload(w, inp, nthreads=8)
    gu.assert_close(gu.from_dev(views[0]), rdx, w.dtype, "dx")
    gu.assert_close(gu.from_dev(views[1]), rdlg, w.dtype, "dlogits")
    gu.assert_close(gu.from_dev(views[2]), rdlam, w.dtype, "dlam")


@pytest.mark.parametrize("case", [(1, 3, 56, 56, 15, 1, False, "f32"), (2, 5, 40, 24, 15, 4, True, "bf16"),
                                  (1, 4, 28, 28, 5, 7, False, "bf16"), (1, 2, 64, 64, 10, 1, False, "f32")],
                         ids=lambda c: "x".join(map(str, c)))
def test_small_plane_dispatch_guards_and_parity(case):
    """Planes of at most 64x64 run on the one-CTA-per-plane kernels: their
    dispatch, canaries around every output, and the oracle's results (both
    passes, per-channel and shared taps, local groups, partial direction sets,
    aligned and unaligned rows)."""
    import linear_spatial_propagation_b200 as lsp
    t = gu.torch()
    w = shape_workload(*case, seed=700 + sum(case[:4]))
    d = lsp.make_desc(w.B, w.C, w.H, w.W, w.dir_mask, w.groups, w.shared, w.dtype)
    assert lsp.gspn_variant_name(d, 0) == "small_plane_fwd"
    assert lsp.gspn_variant_name(d, 1) == "small_plane_bwd"
    inp = synth.make_inputs(w, with_dout=True)
    dinp = gu.dev_inputs(w, inp)
    tdt = dinp["x"].dtype
    guard = 4096

    def guarded(like):
        buf = t.full((like.numel() + 2 * guard,), -3.0, dtype=tdt, device="cuda")
        return buf, buf[guard:guard + like.numel()].view(like.shape)

    ob, out = guarded(dinp["x"])
    lsp.forward(dinp["x"], dinp["logits"], dinp["lam"], dir_mask=w.dir_mask, groups=w.groups, shared=w.shared,
                out=out)
    grads = [guarded(x) for x in (dinp["x"], dinp["logits"], dinp["lam"])]
    lsp.backward(dinp["x"], dinp["logits"], dinp["lam"], dinp["dout"], dir_mask=w.dir_mask, groups=w.groups,
                 shared=w.shared, grads=tuple(v for _, v in grads))
    t.cuda.synchronize()
    for b, v in [(ob, out)] + grads:
        assert bool((b[:guard] == -3.0).all()) and bool((b[guard + v.numel():] == -3.0).all())
    gu.assert_close(gu.from_dev(out), oracle.fwd_workload(w, inp), w.dtype, "small-plane forward")
    rdx, rdlg, rdlam = oracle.bwd_workload(w, inp)
    gu.assert_close(gu.from_dev(grads[0][1]), rdx, w.dtype, "dx")
    gu.assert_close(gu.from_dev(grads[1][1]), rdlg, w.dtype, "dlogits")
    gu.assert_close(gu.from_dev(grads[2][1]), rdlam, w.dtype, "dlam")
