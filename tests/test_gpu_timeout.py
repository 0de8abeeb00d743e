"""Device-side timeouts reach the caller.

The TMA-fed kernels (compact 64x64 and 128x128, and the compact large-plane
kernels, forward and backward) hand
data between warps through shared-memory barriers, and every wait is bounded.
These tests make one wait run out without any fault: gspn_set_stall_test(1)
makes one warp wait on a barrier that only its own final arrival can complete,
with the wait limit shortened to a few milliseconds.  The kernel then records
its error word and ends through its error path.  The tests check that
gspn_device_status (and, in synchronous-check mode, the launching call itself)
reports GSPN_ERR_TIMEOUT, that the GPU still answers, and that the next
normal call is correct.
"""
import contextlib

import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

gu = pytest.importorskip("gpu_util")

TIMEOUT = 6
LIMIT_NS = 2_000_000  # 2 ms


@pytest.fixture(scope="module")
def lsp():
    t = pytest.importorskip("torch")
    if not t.cuda.is_available():
        pytest.skip("no CUDA device")
    import linear_spatial_propagation_b200 as m
    m.load(build_if_missing=False)
    return m


@contextlib.contextmanager
def stalled(lsp, sync=False):
    prev_limit = lsp.gspn_set_wait_limit_ns(LIMIT_NS)
    prev_stall = lsp.gspn_set_stall_test(1)
    prev_sync = lsp.gspn_set_sync_check(1 if sync else 0)
    try:
        yield
    finally:
        lsp.gspn_set_stall_test(prev_stall)
        lsp.gspn_set_sync_check(prev_sync)
        lsp.gspn_set_wait_limit_ns(prev_limit)


def _case(B, C, S, seed):
    return synth.Workload(f"timeout_compact_bf16_b{B}c{C}_{S}x{S}", B, C, S, S, 15, 1, True, "bf16", 1.0, seed,
                          backward=True)


def _fwd_raw(lsp, w, d, out, ws):
    t = gu.torch()
    desc = lsp.make_desc(w.B, w.C, w.H, w.W, w.dir_mask, w.groups, w.shared, w.dtype)
    return desc, lsp.gspn_fwd(desc, d["x"].data_ptr(), d["logits"].data_ptr(), d["lam"].data_ptr(), out.data_ptr(),
                              ws.data_ptr(), ws.numel(), t.cuda.current_stream().cuda_stream)


def _bwd_raw(lsp, w, d, grads, ws):
    t = gu.torch()
    desc = lsp.make_desc(w.B, w.C, w.H, w.W, w.dir_mask, w.groups, w.shared, w.dtype)
    dx, dlg, dlam = grads
    return desc, lsp.gspn_bwd(desc, d["x"].data_ptr(), d["logits"].data_ptr(), d["lam"].data_ptr(),
                              d["dout"].data_ptr(), dx.data_ptr(), dlg.data_ptr(), dlam.data_ptr(), ws.data_ptr(),
                              ws.numel(), t.cuda.current_stream().cuda_stream)


def _gpu_answers():
    t = gu.torch()
    a = t.arange(1 << 20, device="cuda", dtype=t.float32)
    assert float((a * 2).sum().item()) == float(2 * (1 << 20) * ((1 << 20) - 1) / 2)


@pytest.mark.parametrize("S,variant", [(64, "compact64_tma_fwd"), (128, "compact128_tma_fwd"),
                                       (136, "large_compact_fwd")])
def test_forward_timeout_is_reported_and_the_next_call_is_clean(lsp, S, variant):
    t = gu.torch()
    w = _case(2, 16 if S == 64 else 8, S, 900 + S)
    inp = synth.make_inputs(w, with_dout=False)
    d = gu.dev_inputs(w, inp)
    desc = lsp.make_desc(w.B, w.C, w.H, w.W, w.dir_mask, w.groups, w.shared, w.dtype)
    assert lsp.gspn_variant_name(desc, 0) == variant
    ws = t.empty(lsp.gspn_workspace_size(desc, 0), dtype=t.uint8, device="cuda")
    out = t.empty_like(d["x"])
    stream = t.cuda.current_stream().cuda_stream
    with stalled(lsp):
        _, st = _fwd_raw(lsp, w, d, out, ws)
        assert st == 0, "the launch itself succeeds; the timeout is found on the device"
        assert lsp.gspn_device_status(desc, 0, ws.data_ptr(), stream) == TIMEOUT
    _gpu_answers()
    _, st = _fwd_raw(lsp, w, d, out, ws)
    assert st == 0
    assert lsp.gspn_device_status(desc, 0, ws.data_ptr(), stream) == 0
    gu.assert_close(gu.from_dev(out), oracle.fwd_workload(w, inp), w.dtype, f"{variant} after a timeout")


@pytest.mark.parametrize("S,variant", [(64, "compact64_tma_bwd"), (128, "compact128_tma_bwd"),
                                       (136, "large_compact_bwd")])
def test_backward_timeout_is_reported_and_the_next_call_is_clean(lsp, S, variant):
    t = gu.torch()
    w = _case(1, 16 if S == 64 else 8, S, 910 + S)
    inp = synth.make_inputs(w, with_dout=True)
    d = gu.dev_inputs(w, inp)
    desc = lsp.make_desc(w.B, w.C, w.H, w.W, w.dir_mask, w.groups, w.shared, w.dtype)
    assert lsp.gspn_variant_name(desc, 1) == variant
    ws = t.empty(lsp.gspn_workspace_size(desc, 1), dtype=t.uint8, device="cuda")
    grads = (t.empty_like(d["x"]), t.empty_like(d["logits"]), t.empty_like(d["lam"]))
    stream = t.cuda.current_stream().cuda_stream
    with stalled(lsp):
        _, st = _bwd_raw(lsp, w, d, grads, ws)
        assert st == 0
        assert lsp.gspn_device_status(desc, 1, ws.data_ptr(), stream) == TIMEOUT
    _gpu_answers()
    _, st = _bwd_raw(lsp, w, d, grads, ws)
    assert st == 0
    assert lsp.gspn_device_status(desc, 1, ws.data_ptr(), stream) == 0
    rdx, rdlg, rdlam = oracle.bwd_workload(w, inp, nthreads=8)
    gu.assert_close(gu.from_dev(grads[0]), rdx, w.dtype, "dx after a timeout")
    gu.assert_close(gu.from_dev(grads[1]), rdlg, w.dtype, "dlogits after a timeout")
    gu.assert_close(gu.from_dev(grads[2]), rdlam, w.dtype, "dlambda after a timeout")


def test_sync_check_mode_returns_the_timeout_from_the_call(lsp):
    t = gu.torch()
    w = _case(1, 8, 64, 920)
    inp = synth.make_inputs(w, with_dout=False)
    d = gu.dev_inputs(w, inp)
    desc = lsp.make_desc(w.B, w.C, w.H, w.W, w.dir_mask, w.groups, w.shared, w.dtype)
    ws = t.empty(lsp.gspn_workspace_size(desc, 0), dtype=t.uint8, device="cuda")
    out = t.empty_like(d["x"])
    with stalled(lsp, sync=True):
        _, st = _fwd_raw(lsp, w, d, out, ws)
        assert st == TIMEOUT
    prev = lsp.gspn_set_sync_check(1)
    try:
        _, st = _fwd_raw(lsp, w, d, out, ws)
        assert st == 0
    finally:
        lsp.gspn_set_sync_check(prev)
    gu.assert_close(gu.from_dev(out), oracle.fwd_workload(w, inp), w.dtype, "forward in sync-check mode")


def test_noalloc_timeout_is_reported_through_its_status_call(lsp):
    t = gu.torch()
    w = _case(2, 8, 64, 930)
    inp = synth.make_inputs(w, with_dout=False)
    d = gu.dev_inputs(w, inp)
    desc = lsp.make_desc(w.B, w.C, w.H, w.W, w.dir_mask, w.groups, w.shared, w.dtype)
    out = t.empty_like(d["x"])
    stream = t.cuda.current_stream().cuda_stream
    args = (desc, d["x"].data_ptr(), d["logits"].data_ptr(), d["lam"].data_ptr(), out.data_ptr(), stream)
    with stalled(lsp):
        assert lsp.gspn_fwd_noalloc(*args) == 0
        assert lsp.gspn_noalloc_status(stream) == TIMEOUT
    _gpu_answers()
    assert lsp.gspn_fwd_noalloc(*args) == 0
    assert lsp.gspn_noalloc_status(stream) == 0
    gu.assert_close(gu.from_dev(out), oracle.fwd_workload(w, inp), w.dtype, "noalloc forward after a timeout")


def test_paths_without_device_waits_report_ok(lsp):
    t = gu.torch()
    w = synth.Workload("timeout_small_f32_b1c2_16x16", 1, 2, 16, 16, 15, 1, False, "f32", 1.0, 940)
    d = gu.dev_inputs(w, synth.make_inputs(w, with_dout=False))
    desc = lsp.make_desc(w.B, w.C, w.H, w.W, w.dir_mask, w.groups, w.shared, w.dtype)
    assert not lsp.gspn_variant_name(desc, 0).startswith("compact")
    with stalled(lsp):
        gu.run_fwd(w, d)
        assert lsp.gspn_device_status(desc, 0, 0, t.cuda.current_stream().cuda_stream) == 0
