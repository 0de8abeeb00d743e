"""The C-ABI calls only enqueue work on the stream they are given, so a whole
forward + backward can be captured once into a CUDA graph and replayed (the
launch form `bench.py --graph` times).  Each case runs the calls directly,
then captures them with the same buffers and replays the graph twice; the
replay must give the direct results: the forward, dx and dlambda bit for bit
(every path sums in a fixed order), dlogits within 1e-5 of max|dlogits| (the
channel-shared TMA paths add their per-CTA tap sums with fp32 reductions
whose order may vary; the compact large-plane backward adds every warp's tap
values that way, so there one bf16 step, within 1e-2).  One case per kernel family: small plane, compact
64x64 and 128x128, both large-plane forwards (the compact one with its own
backward, the general one with the generic backward), generic,
and the compressed propagation block.
"""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu

gu = pytest.importorskip("gpu_util")

CASES = [
    # B, C, H, W, dir_mask, groups, shared, dtype, forward variant
    (1, 4, 28, 28, 15, 4, False, "f32", "small_plane_fwd"),
    (2, 16, 64, 64, 15, 1, True, "bf16", "compact64_tma_fwd"),
    (1, 8, 128, 128, 15, 1, True, "bf16", "compact128_tma_fwd"),
    (1, 2, 256, 256, 15, 1, True, "bf16", "large_plane_fwd"),
    (1, 8, 136, 136, 15, 1, True, "bf16", "large_compact_fwd"),
    (1, 2, 97, 41, 15, 1, False, "f32", None),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c[:8])))
def test_captured_step_replays_the_direct_results(case):
    import linear_spatial_propagation_b200 as lsp
    t = gu.torch()
    B, C, H, W, mask, g, shared, dtype, variant = case
    w = synth.Workload(f"graph_{'x'.join(map(str, case[:8]))}", B, C, H, W, mask, g, shared, dtype, 1.0,
                       5000 + H + W + C)
    desc = lsp.make_desc(B, C, H, W, mask, g, shared, dtype)
    if variant is not None:
        assert lsp.gspn_variant_name(desc, 0) == variant
    d = gu.dev_inputs(w, synth.make_inputs(w, with_dout=True))
    wsf = lsp.workspace(desc, 0, "cuda")
    wsb = lsp.workspace(desc, 1, "cuda")

    def step(out, grads, stream):
        lsp.forward(d["x"], d["logits"], d["lam"], mask, g, shared, out=out, ws=wsf, stream=stream)
        lsp.backward(d["x"], d["logits"], d["lam"], d["dout"], mask, g, shared, grads=grads, ws=wsb, stream=stream)

    out_d = t.empty_like(d["x"])
    grads_d = (t.empty_like(d["x"]), t.empty_like(d["logits"]), t.empty_like(d["lam"]))
    step(out_d, grads_d, t.cuda.current_stream().cuda_stream)
    t.cuda.synchronize()

    out_g = t.full_like(d["x"], 7.0)
    grads_g = tuple(t.full_like(x, 7.0) for x in grads_d)
    s = t.cuda.Stream()
    s.wait_stream(t.cuda.current_stream())
    graph = t.cuda.CUDAGraph()
    with t.cuda.graph(graph, stream=s):
        step(out_g, grads_g, s.cuda_stream)
    for _ in range(2):
        graph.replay()
    t.cuda.synchronize()
    assert bool(t.equal(out_g, out_d)), "forward"
    assert bool(t.equal(grads_g[0], grads_d[0])), "dx"
    assert bool(t.equal(grads_g[2], grads_d[2])), "dlambda"
    a, b = gu.from_dev(grads_g[1]), gu.from_dev(grads_d[1])
    scale = max(float(np.max(np.abs(b))), 1e-30)
    # the compact large-plane backward adds every warp's tap values into fp32
    # sums in arrival order, so a sum can round to the neighbouring bf16 value
    tol = 1e-2 if lsp.gspn_variant_name(desc, 1) == "large_compact_bwd" else 1e-5
    assert float(np.max(np.abs(a - b))) <= tol * scale, "dlogits"
    del graph


def test_captured_block_replays_the_direct_result():
    import linear_spatial_propagation_b200 as lsp
    t = gu.torch()
    w = synth.BlockWorkload("graph_block", 2, 256, 32, 32, 4, 1, 5100)
    inp = synth.make_block_inputs(w)
    d = {}
    for k, v in inp.items():
        if v.dtype == np.uint16:
            d[k] = t.from_numpy(np.ascontiguousarray(v)).view(t.bfloat16).cuda()
        else:
            d[k] = t.from_numpy(np.ascontiguousarray(v, dtype=np.float32)).cuda()
    desc = lsp.make_block_desc(w.B, w.C, w.H, w.W, w.Cp, w.groups, w.norm, w.eps)
    ws = t.empty(lsp.gspn_block_workspace_size(desc), dtype=t.uint8, device="cuda")
    args = (d["x"], d["v_proj"], d["logits"], d["lam"], d["alpha"], d["gamma"], d["u_proj"])
    y_d = lsp.block_forward(*args, groups=w.groups, norm=w.norm, eps=w.eps, ws=ws)
    t.cuda.synchronize()
    y_g = t.full_like(y_d, 7.0)
    s = t.cuda.Stream()
    s.wait_stream(t.cuda.current_stream())
    graph = t.cuda.CUDAGraph()
    with t.cuda.graph(graph, stream=s):
        lsp.block_forward(*args, groups=w.groups, norm=w.norm, eps=w.eps, y=y_g, ws=ws, stream=s.cuda_stream)
    graph.replay()
    t.cuda.synchronize()
    assert bool(t.equal(y_g, y_d))
    del graph
