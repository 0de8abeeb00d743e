"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each test fixes one part of what the GSPN pages define, so that a plausible
mistake in the oracle (a dropped term, a swapped tap, a wrong direction
mapping, a missed group reset, a sign error in a gradient) fails at least one:

* hand-derived values (tests/golden) -- gate normalisation, border taps, the
  lambda*x term ("Parallel Sequence Modeling via Generalized Spatial
  Propagation Network", Key design 1 and 2);
* the closed form h_i = sum_j W_ij lambda_j x_j, W_ij = prod w_tau, by dense
  products of explicit tridiagonal matrices built from chosen weights (Key
  design 1);
* Theorem 1 (rows of W_ij sum to 1: a constant field is carried unchanged)
  and Theorem 2 (no blow-up: |h_i| <= sum_j max|lambda_j x_j|) (Key design 1);
* W = 1 reduces to a prefix sum; g = L reduces to h = lambda*x (Key design 3);
* reverse / transposed scans equal the top-to-bottom scan of the flipped /
  transposed input (Key design 2, four directions);
* compact mode equals per-channel mode with the taps broadcast over channels
  ("GSPN-2: Efficient Parallel Sequence Modeling", Justification for
  Channel-Agnostic Propagation, W kron I(C));
* backward against central finite differences of the forward.
"""
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
T2B, B2T, L2R, R2L = 1, 2, 4, 8


def rnd(shape, seed, kind="normal", scale=1.0):
    rng = np.random.default_rng(seed)
    if kind == "normal":
        return rng.standard_normal(shape) * scale
    return rng.random(shape)


def inputs(B, C, H, W, mask, shared=False, seed=0, lscale=1.0):
    D = bin(mask).count("1")
    Cw = 1 if shared else C
    x = rnd((B, C, H, W), seed)
    lam = rnd((D, B, C, H, W), seed + 1, "uniform")
    lg = rnd((D, B, Cw, 3, H, W), seed + 2, scale=lscale)
    return x, lg, lam


# --------------------------------------------------------------------------
# hand-derived values
# --------------------------------------------------------------------------
def test_golden_hand_t2b():
    g = json.load(open(os.path.join(GOLDEN, "hand_t2b_2x3.json")))
    H, W = g["H"], g["W"]
    x = np.array(g["x"]).reshape(1, 1, H, W)
    lam = np.array(g["lam"]).reshape(1, 1, 1, H, W)
    lg = np.zeros((1, 1, 1, 3, H, W))
    lg[0, 0, 0, :, 0, :] = np.array(g["logits_row0"])
    for k in range(3):
        lg[0, 0, 0, k, 1, :] = g["logits_row1_by_tap"][f"tap{k}"]
    out = oracle.fwd(x, lg, lam, dir_mask=g["dir_mask"], groups=g["groups"])
    np.testing.assert_allclose(out[0, 0], np.array(g["expected_out"]), rtol=0, atol=g["tolerance"])


def test_equal_logits_give_thirds_and_halves():
    # all logits equal: interior rows average 3 neighbours, border rows 2
    H, W = 2, 5
    x = np.zeros((1, 1, H, W))
    x[0, 0, 0] = [1, 2, 3, 4, 5]
    lam = np.zeros((1, 1, 1, H, W))
    lam[0, 0, 0, 0] = 1.0
    lg = np.full((1, 1, 1, 3, H, W), 0.7)
    out = oracle.fwd(x, lg, lam, dir_mask=T2B)
    want = [(1 + 2) / 2, (1 + 2 + 3) / 3, (2 + 3 + 4) / 3, (3 + 4 + 5) / 3, (4 + 5) / 2]
    np.testing.assert_allclose(out[0, 0, 1], want, rtol=0, atol=1e-14)


# --------------------------------------------------------------------------
# closed form by dense matrix products (T2B)
# --------------------------------------------------------------------------
def logits_for_weights(w):
    """Logits whose sigmoid-then-normalise gives weights w (last axis = taps).

    Uses the inverse of the sigmoid, s = w * c with c = 0.9 / max(w), so the
    test never evaluates the forward gate formula."""
    c = 0.9 / w.max(axis=-1, keepdims=True)
    s = np.clip(w * c, 1e-300, None)
    return np.log(s) - np.log1p(-s)


def random_row_stochastic(L, N, seed):
    rng = np.random.default_rng(seed)
    w = rng.random((L, N, 3)) + 0.05
    w[:, 0, 0] = 0.0          # tap 0 of position 0 reads position -1
    w[:, N - 1, 2] = 0.0      # tap 2 of position N-1 reads position N
    if N == 1:
        w[:, 0, :] = [0.0, 1.0, 0.0]
    return w / w.sum(axis=-1, keepdims=True)


def tridiag(wl):
    N = wl.shape[0]
    M = np.zeros((N, N))
    for j in range(N):
        for k in range(3):
            q = j + k - 1
            if 0 <= q < N:
                M[j, q] = wl[j, k]
    return M


@pytest.mark.parametrize("H,W,groups", [(6, 5, 1), (8, 7, 2), (4, 4, 4), (7, 1, 1), (1, 6, 1), (9, 3, 3)])
def test_closed_form_dense_products(H, W, groups):
    w = random_row_stochastic(H, W, seed=H * 31 + W)
    lg_t = logits_for_weights(w)                        # [L=H][N=W][3]
    lg = np.transpose(lg_t, (2, 0, 1))[None, None, None]  # [1,1,1,3,H,W]
    x = rnd((1, 1, H, W), 5)
    lam = rnd((1, 1, 1, H, W), 6, "uniform")
    out = oracle.fwd(x, lg, lam, dir_mask=T2B, groups=groups)[0, 0]
    seg = H // groups
    v = lam[0, 0, 0] * x[0, 0]
    mats = [tridiag(w[i]) for i in range(H)]
    for i in range(H):
        h = np.zeros(W)
        g0 = (i // seg) * seg
        for j in range(g0, i + 1):
            P = np.eye(W)
            for t in range(j + 1, i + 1):     # W_ij = w_i ... w_{j+1}
                P = mats[t] @ P
            # Theorem 1: each row of the cumulative product sums to 1
            np.testing.assert_allclose(P.sum(axis=1), 1.0, atol=1e-12)
            h += P @ v[j]
        np.testing.assert_allclose(out[i], h, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# Theorem 1 / Theorem 2
# --------------------------------------------------------------------------
@pytest.mark.parametrize("mask", [T2B, B2T, L2R, R2L])
def test_theorem1_constant_field_is_carried(mask):
    H, W = 7, 9
    _, lg, _ = inputs(1, 1, H, W, mask, seed=11, lscale=3.0)
    x = np.full((1, 1, H, W), 2.5)
    lam = np.zeros((1, 1, 1, H, W))
    first = {T2B: (slice(0, 1), slice(None)), B2T: (slice(H - 1, H), slice(None)),
             L2R: (slice(None), slice(0, 1)), R2L: (slice(None), slice(W - 1, W))}[mask]
    lam[(0, 0, 0) + first] = 1.0
    out = oracle.fwd(x, lg, lam, dir_mask=mask)
    np.testing.assert_allclose(out, 2.5, rtol=0, atol=1e-13)


@pytest.mark.parametrize("mask", [T2B, B2T, L2R, R2L])
def test_theorem2_no_blowup(mask):
    H, W = 10, 8
    x, lg, lam = inputs(1, 1, H, W, mask, seed=21, lscale=4.0)
    out = oracle.fwd(x, lg, lam, dir_mask=mask)[0, 0]
    v = np.abs(lam[0, 0, 0] * x[0, 0])
    if mask in (T2B, B2T):
        per_line = v.max(axis=1)
        order = range(H) if mask == T2B else range(H - 1, -1, -1)
        bound, acc = np.zeros(H), 0.0
        for r in order:
            acc += per_line[r]
            bound[r] = acc
        assert np.all(np.abs(out) <= bound[:, None] + 1e-12)
    else:
        per_line = v.max(axis=0)
        order = range(W) if mask == L2R else range(W - 1, -1, -1)
        bound, acc = np.zeros(W), 0.0
        for c in order:
            acc += per_line[c]
            bound[c] = acc
        assert np.all(np.abs(out) <= bound[None, :] + 1e-12)


# --------------------------------------------------------------------------
# special cases
# --------------------------------------------------------------------------
def test_width_one_is_prefix_sum():
    H = 13
    x, lg, lam = inputs(2, 3, H, 1, T2B, seed=31)
    out = oracle.fwd(x, lg, lam, dir_mask=T2B)
    np.testing.assert_allclose(out, np.cumsum(lam[0] * x, axis=2), rtol=1e-13, atol=1e-13)


def test_groups_equal_length_is_lambda_x():
    H, W = 6, 6
    x, lg, lam = inputs(1, 2, H, W, 15, seed=41)
    out = oracle.fwd(x, lg, lam, dir_mask=15, groups=6)
    np.testing.assert_allclose(out, lam.sum(axis=0) * x, rtol=1e-14, atol=1e-14)


@pytest.mark.parametrize("mask", [T2B, B2T, L2R, R2L])
def test_group_is_fresh_scan_of_its_slab(mask):
    H, W, g = 8, 12, 4
    x, lg, lam = inputs(1, 2, H, W, mask, seed=51)
    out = oracle.fwd(x, lg, lam, dir_mask=mask, groups=g)
    if mask in (T2B, B2T):
        s = H // g
        for q in range(g):
            sl = slice(q * s, (q + 1) * s)
            part = oracle.fwd(x[:, :, sl], lg[..., sl, :], lam[..., sl, :], dir_mask=mask)
            np.testing.assert_allclose(out[:, :, sl], part, rtol=1e-13, atol=1e-13)
    else:
        s = W // g
        for q in range(g):
            sl = slice(q * s, (q + 1) * s)
            part = oracle.fwd(x[..., sl], lg[..., sl], lam[..., sl], dir_mask=mask)
            np.testing.assert_allclose(out[..., sl], part, rtol=1e-13, atol=1e-13)


def test_groups_one_is_global():
    x, lg, lam = inputs(1, 2, 6, 6, 15, seed=61)
    a = oracle.fwd(x, lg, lam, dir_mask=15, groups=1)
    b = oracle.fwd(x, lg, lam, dir_mask=15)
    np.testing.assert_array_equal(a, b)


# --------------------------------------------------------------------------
# direction mapping
# --------------------------------------------------------------------------
def test_b2t_is_t2b_of_row_flip():
    x, lg, lam = inputs(2, 2, 7, 5, T2B, seed=71)
    a = oracle.fwd(x, lg, lam, dir_mask=B2T)
    b = oracle.fwd(x[:, :, ::-1], lg[..., ::-1, :], lam[..., ::-1, :], dir_mask=T2B)[:, :, ::-1]
    np.testing.assert_allclose(a, b, rtol=1e-14, atol=1e-14)


def test_l2r_is_t2b_of_transpose():
    x, lg, lam = inputs(2, 2, 7, 5, T2B, seed=81)
    a = oracle.fwd(x, lg, lam, dir_mask=L2R)
    tr = lambda t: np.swapaxes(t, -1, -2)
    b = tr(oracle.fwd(tr(x), tr(lg), tr(lam), dir_mask=T2B))
    np.testing.assert_allclose(a, b, rtol=1e-14, atol=1e-14)


def test_r2l_is_l2r_of_column_flip():
    x, lg, lam = inputs(2, 2, 7, 5, T2B, seed=91)
    a = oracle.fwd(x, lg, lam, dir_mask=R2L)
    b = oracle.fwd(x[..., ::-1], lg[..., ::-1], lam[..., ::-1], dir_mask=L2R)[..., ::-1]
    np.testing.assert_allclose(a, b, rtol=1e-14, atol=1e-14)


def test_merge_is_sum_of_single_directions():
    x, lg, lam = inputs(2, 3, 6, 7, 15, seed=101)
    full = oracle.fwd(x, lg, lam, dir_mask=15, groups=1)
    acc = np.zeros_like(full)
    for slot, m in enumerate([T2B, B2T, L2R, R2L]):
        acc += oracle.fwd(x, lg[slot:slot + 1], lam[slot:slot + 1], dir_mask=m)
    np.testing.assert_allclose(full, acc, rtol=1e-14, atol=1e-14)
    # a subset of directions keeps its slots in bit order
    sub = oracle.fwd(x, lg[[1, 3]], lam[[1, 3]], dir_mask=B2T | R2L)
    ref = oracle.fwd(x, lg[1:2], lam[1:2], dir_mask=B2T) + oracle.fwd(x, lg[3:4], lam[3:4], dir_mask=R2L)
    np.testing.assert_allclose(sub, ref, rtol=1e-14, atol=1e-14)


# --------------------------------------------------------------------------
# compact mode, linearity
# --------------------------------------------------------------------------
def test_compact_equals_broadcast_per_channel():
    x, lg, lam = inputs(2, 4, 6, 5, 15, shared=True, seed=111)
    a = oracle.fwd(x, lg, lam, dir_mask=15, shared=True)
    b = oracle.fwd(x, np.repeat(lg, 4, axis=2), lam, dir_mask=15, shared=False)
    np.testing.assert_allclose(a, b, rtol=1e-14, atol=1e-14)


def test_linear_in_x():
    x1, lg, lam = inputs(1, 2, 6, 6, 15, seed=121)
    x2 = rnd(x1.shape, 122)
    f = lambda x: oracle.fwd(x, lg, lam, dir_mask=15, groups=2)
    np.testing.assert_allclose(f(2.0 * x1 - 3.0 * x2), 2.0 * f(x1) - 3.0 * f(x2), rtol=1e-12, atol=1e-12)


def test_stored_dtypes_are_widened_exactly():
    import synth
    w = synth.WORKLOADS["t2b_f32_b1c4_16x16"].replace(dtype="bf16")
    inp = synth.make_inputs(w)
    a = oracle.fwd_workload(w, inp)
    b = oracle.fwd(synth.bf16_bits_to_f32(inp["x"]).astype(np.float64),
                   synth.bf16_bits_to_f32(inp["logits"]).astype(np.float64),
                   synth.bf16_bits_to_f32(inp["lam"]).astype(np.float64), dir_mask=w.dir_mask)
    np.testing.assert_array_equal(a, b)


def test_rejects_bad_arguments():
    x, lg, lam = inputs(1, 1, 6, 6, T2B, seed=1)
    with pytest.raises(ValueError):
        oracle.fwd(x, lg, lam, dir_mask=T2B, groups=4)   # 4 does not divide 6
    with pytest.raises(ValueError):
        oracle.fwd(x, lg, lam, dir_mask=T2B | B2T)      # lam has one slot only


def test_threads_do_not_change_results():
    x, lg, lam = inputs(3, 5, 9, 7, 15, shared=True, seed=131)
    a = oracle.fwd(x, lg, lam, dir_mask=15, shared=True, nthreads=1)
    b = oracle.fwd(x, lg, lam, dir_mask=15, shared=True, nthreads=4)
    np.testing.assert_array_equal(a, b)


# --------------------------------------------------------------------------
# backward
# --------------------------------------------------------------------------
def fd_grad(f, a, eps=1e-6):
    g = np.zeros_like(a)
    flat = a.reshape(-1)
    gf = g.reshape(-1)
    for q in range(flat.size):
        old = flat[q]
        flat[q] = old + eps
        fp = f()
        flat[q] = old - eps
        fm = f()
        flat[q] = old
        gf[q] = (fp - fm) / (2 * eps)
    return g


@pytest.mark.parametrize("mask,groups,shared,H,W", [
    (T2B, 1, False, 4, 5), (B2T, 2, False, 4, 3), (L2R, 1, True, 3, 4), (R2L, 2, True, 5, 4),
    (15, 1, False, 4, 4), (15, 2, True, 4, 6), (15, 1, True, 1, 3), (T2B | L2R, 1, False, 3, 1),
])
def test_backward_matches_finite_differences(mask, groups, shared, H, W):
    B, C = 2, 2
    x, lg, lam = inputs(B, C, H, W, mask, shared=shared, seed=141 + H + 10 * W)
    dout = rnd((B, C, H, W), 999)
    kw = dict(dir_mask=mask, groups=groups, shared=shared)
    loss = lambda: float(np.sum(dout * oracle.fwd(x, lg, lam, **kw)))
    dx, dlg, dlam = oracle.bwd(x, lg, lam, dout, **kw)
    np.testing.assert_allclose(dx, fd_grad(loss, x), rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(dlam, fd_grad(loss, lam), rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(dlg, fd_grad(loss, lg), rtol=1e-6, atol=1e-7)


def test_backward_zero_on_unused_logits():
    H, W, g = 6, 9, 3
    x, lg, lam = inputs(1, 2, H, W, 15, seed=151)
    dout = rnd((1, 2, H, W), 152)
    _, dlg, _ = oracle.bwd(x, lg, lam, dout, dir_mask=15, groups=g)
    # T2B: group-start rows 0, 2, 4; tap 0 at column 0 and tap 2 at column W-1
    assert np.all(dlg[0, :, :, :, 0::H // g, :] == 0)
    assert np.all(dlg[0, :, :, 0, :, 0] == 0) and np.all(dlg[0, :, :, 2, :, W - 1] == 0)
    # B2T: group starts are the last row of each group
    assert np.all(dlg[1, :, :, :, H // g - 1::H // g, :] == 0)
    # L2R: group-start columns; taps read rows, so tap 0 at row 0 is unused
    assert np.all(dlg[2, :, :, :, :, 0::W // g] == 0)
    # R2L: group starts are the last column of each group
    assert np.all(dlg[3, :, :, :, :, W // g - 1::W // g] == 0)
    # and the rest of the logits do receive gradient
    assert np.count_nonzero(dlg[0, :, :, 1, 1, :]) == dlg[0, :, :, 1, 1, :].size
    assert np.all(dlg[2, :, :, 0, 0, :] == 0) and np.all(dlg[2, :, :, 2, H - 1, :] == 0)


def test_backward_adjoint_identity_lambda_x():
    # out is linear in x for fixed (logits, lambda): <dout, J v> = <J^T dout, v>
    x, lg, lam = inputs(1, 3, 5, 6, 15, shared=True, seed=161)
    v = rnd(x.shape, 162)
    dout = rnd(x.shape, 163)
    Jv = oracle.fwd(v, lg, lam, dir_mask=15, shared=True)
    dx, _, _ = oracle.bwd(x, lg, lam, dout, dir_mask=15, shared=True)
    assert abs(np.sum(dout * Jv) - np.sum(dx * v)) < 1e-11 * max(1.0, abs(np.sum(dout * Jv)))


def test_backward_compact_is_channel_sum_of_per_channel():
    x, lg, lam = inputs(1, 3, 5, 4, 15, shared=True, seed=171)
    dout = rnd(x.shape, 172)
    _, dl_shared, _ = oracle.bwd(x, lg, lam, dout, dir_mask=15, shared=True, nthreads=3)
    _, dl_per, _ = oracle.bwd(x, np.repeat(lg, 3, axis=2), lam, dout, dir_mask=15, shared=False)
    np.testing.assert_allclose(dl_shared, dl_per.sum(axis=2, keepdims=True), rtol=1e-12, atol=1e-13)
