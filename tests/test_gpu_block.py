"""GPU parity of the compressed propagation block (gspn_block_fwd) against the
oracle (``oracle.block_fwd``, float64).

The block: proxy projection C -> C_proxy on the tensor cores, the four
single-direction scans of the proxy planes, the learnable merger and RMS
normalisation fused into the back-projection's prologue, and the projection
back to C channels on the tensor cores.  Tolerance: bf16 storage, so the
maximum absolute error over y must stay within 1e-2 * max|y_oracle|.  Shapes
cover several 128-pixel tiles and a ragged last tile, channel counts that are
not multiples of the 64-channel K block or of the 128-channel output chunk,
odd and maximal proxy widths, local groups and the block without its
normalisation; canaries around y catch stores outside it.
"""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

gu = pytest.importorskip("gpu_util")


@pytest.fixture(scope="module")
def lsp():
    t = pytest.importorskip("torch")
    if not t.cuda.is_available():
        pytest.skip("no CUDA device")
    import linear_spatial_propagation_b200 as m
    m.load(build_if_missing=False)
    return m


def _dev(inp):
    t = gu.torch()
    out = {}
    for k, v in inp.items():
        if v.dtype == np.uint16:
            out[k] = t.from_numpy(np.ascontiguousarray(v)).view(t.bfloat16).cuda()
        else:
            out[k] = t.from_numpy(np.ascontiguousarray(v, dtype=np.float32)).cuda()
    return out


def _oracle(w, inp):
    return oracle.block_fwd(inp["x"], inp["v_proj"], inp["logits"], inp["lam"], inp["alpha"], inp["gamma"],
                            inp["u_proj"], groups=w.groups, norm=w.norm, eps=w.eps, dtype="bf16", nthreads=8)


def _run(lsp, w, d, guard=4096):
    t = gu.torch()
    buf = t.full((w.B * w.C * w.H * w.W + 2 * guard,), -7.0, dtype=t.bfloat16, device="cuda")
    y = buf[guard:guard + w.B * w.C * w.H * w.W].view(w.B, w.C, w.H, w.W)
    lsp.block_forward(d["x"], d["v_proj"], d["logits"], d["lam"], d["alpha"], d["gamma"], d["u_proj"],
                      groups=w.groups, norm=w.norm, eps=w.eps, y=y)
    t.cuda.synchronize()
    assert bool((buf[:guard] == -7.0).all()) and bool((buf[guard + y.numel():] == -7.0).all()), "store outside y"
    return y


CASES = [
    # B, C, H, W, Cp, groups, norm
    (2, 64, 16, 16, 2, 1, True),      # 2 pixel tiles per image, one K block, one output chunk
    (2, 1152, 64, 64, 2, 1, True),    # the 1K shape at a batch of 2
    (1, 200, 24, 40, 3, 1, True),     # ragged pixel tile (960 px), ragged K block and chunk, odd Cp
    (2, 256, 32, 32, 16, 2, True),    # Cp = 16, local groups
    (1, 320, 64, 64, 32, 1, True),    # Cp = 32 (the second MMA K step)
    (1, 128, 48, 56, 5, 4, False),    # without normalisation, local groups of 12 / 14 lines
    (1, 136, 128, 128, 2, 1, True),   # 128-wide lines (P = 4 per lane), ragged output chunk
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "b{}c{}_{}x{}_cp{}_g{}_{}".format(*c[:6],
                                                                                    "norm" if c[6] else "raw"))
def test_block_matches_oracle(lsp, case):
    B, C, H, W, Cp, g, norm = case
    w = synth.BlockWorkload(f"block_case_b{B}c{C}_{H}x{W}_cp{Cp}", B, C, H, W, Cp, g, 3000 + C + Cp, norm=norm)
    inp = synth.make_block_inputs(w)
    d = _dev(inp)
    y = _run(lsp, w, d)
    gu.assert_close(gu.from_dev(y), _oracle(w, inp), "bf16", f"block {w.name}")


def test_block_is_deterministic_and_reports_no_timeout(lsp):
    t = gu.torch()
    w = synth.BlockWorkload("block_det", 2, 384, 32, 32, 4, 1, 3100)
    d = _dev(synth.make_block_inputs(w))
    desc = lsp.make_block_desc(w.B, w.C, w.H, w.W, w.Cp, w.groups, w.norm, w.eps)
    ws = t.empty(lsp.gspn_block_workspace_size(desc), dtype=t.uint8, device="cuda")
    y1 = lsp.block_forward(d["x"], d["v_proj"], d["logits"], d["lam"], d["alpha"], d["gamma"], d["u_proj"], ws=ws)
    assert lsp.gspn_block_device_status(desc, ws.data_ptr(), t.cuda.current_stream().cuda_stream) == 0
    y2 = lsp.block_forward(d["x"], d["v_proj"], d["logits"], d["lam"], d["alpha"], d["gamma"], d["u_proj"], ws=ws)
    t.cuda.synchronize()
    assert bool(t.equal(y1, y2))


def test_block_full_size_sampled_images(lsp):
    """The 1K block workload (B = 32, C = 1152, 64x64, C_proxy = 2) at full
    size in the launch configuration the bench times; the oracle checks three
    of its batch images (the block is independent per image)."""
    w = synth.BLOCK_WORKLOADS["block_cp2_bf16_b32c1152_64x64"]
    inp = synth.make_block_inputs(w)
    d = _dev(inp)
    y = _run(lsp, w, d)
    got = gu.from_dev(y)
    for b in (0, 17, 31):
        sub = dict(inp)
        sub["x"] = inp["x"][b:b + 1]
        sub["lam"] = inp["lam"][:, b:b + 1]
        sub["logits"] = inp["logits"][:, b:b + 1]
        want = _oracle(w.replace(B=1), sub)
        gu.assert_close(got[b:b + 1], want, "bf16", f"block 1K image {b}")
