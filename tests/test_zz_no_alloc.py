"""gspn_fwd_noalloc: the forward for callers that cannot allocate device memory.

Some callers have no way to allocate: a host framework that owns all device
memory through its own pool, a latency-critical path where cudaMalloc would
block or synchronise, a plugin that is handed only its input and output
tensors.  gspn_fwd_noalloc serves them from a fixed scratch array inside the
library, so they pass inputs and outputs only.  These tests call it through
the C ABI and check it against gspn_fwd (which takes a caller workspace),
on two calls in a row and across problems that share the one scratch array.
This file is collected last on purpose.
"""
import pytest

import synth

pytestmark = pytest.mark.gpu

gu = pytest.importorskip("gpu_util")


@pytest.fixture(scope="module")
def lib():
    t = pytest.importorskip("torch")
    if not t.cuda.is_available():
        pytest.skip("no CUDA device")
    import linear_spatial_propagation_b200 as lsp
    lsp.load(build_if_missing=False)
    return lsp


def _case(B, C, groups, seed):
    return synth.Workload(f"noalloc_compact_bf16_b{B}c{C}_g{groups}_64x64", B, C, 64, 64, 15, groups, True, "bf16",
                          1.0, seed)


def _noalloc(lsp, w, d):
    t = gu.torch()
    desc = lsp.make_desc(w.B, w.C, w.H, w.W, w.dir_mask, w.groups, w.shared, w.dtype)
    out = t.full_like(d["x"], float("nan"))
    st = lsp.gspn_fwd_noalloc(desc, d["x"].data_ptr(), d["logits"].data_ptr(), d["lam"].data_ptr(),
                              out.data_ptr(), t.cuda.current_stream().cuda_stream)
    assert st == 0, lsp.gspn_status_string(st)
    return out


def test_noalloc_matches_workspace_forward_on_two_calls_in_a_row(lib):
    t = gu.torch()
    w = _case(3, 24, 1, 515)
    d = gu.dev_inputs(w, synth.make_inputs(w, with_dout=False))
    ref = gu.from_dev(gu.run_fwd(w, d))
    for _ in range(2):
        got = _noalloc(lib, w, d)
        t.cuda.synchronize()
        gu.assert_close(gu.from_dev(got), ref, w.dtype, "noalloc vs workspace forward")


def test_noalloc_calls_on_different_problems_do_not_leak_state(lib):
    t = gu.torch()
    cases = [_case(32, 8, 1, 516), _case(2, 16, 4, 517), _case(1, 8, 64, 518)]
    data = [(w, gu.dev_inputs(w, synth.make_inputs(w, with_dout=False))) for w in cases]
    refs = [gu.from_dev(gu.run_fwd(w, d)) for w, d in data]
    for (w, d), ref in zip(data + data[:1], refs + refs[:1]):
        got = _noalloc(lib, w, d)
        t.cuda.synchronize()
        gu.assert_close(gu.from_dev(got), ref, w.dtype, f"noalloc {w.name}")


def test_noalloc_rejects_what_the_fixed_scratch_cannot_hold(lib):
    t = gu.torch()
    x = t.zeros(16, dtype=t.bfloat16, device="cuda")  # never read: the calls are rejected before launch
    p = x.data_ptr()
    too_big = lib.make_desc(33, 8, 64, 64, 15, 1, True, "bf16")
    assert lib.gspn_fwd_noalloc(too_big, p, p, p, p, 0) == 7
    other = lib.make_desc(2, 8, 56, 56, 15, 1, True, "bf16")
    assert lib.gspn_fwd_noalloc(other, p, p, p, p, 0) == 2
    bad = lib.make_desc(2, 8, 64, 64, 0, 1, True, "bf16")
    assert lib.gspn_fwd_noalloc(bad, p, p, p, p, 0) == 1
