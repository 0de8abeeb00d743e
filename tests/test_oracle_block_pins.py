"""Pins of the compressed-propagation-block oracle (``oracle.block_fwd``).

The block: proxy projection C -> C_proxy, the four single-direction GSPN scans
of the proxy planes, a learnable per-(direction, channel) merger, an RMS
normalisation over the proxy channels of each pixel, and the projection back
to C channels ("GSPN-2: Efficient Parallel Sequence Modeling", OpenReview
response, "Relate Compressive Proxy Dimension to Low-rank Approximation";
"Parallel Sequence Modeling via Generalized Spatial Propagation Network", Key
design 2, learnable merger; "Scaling Parallel Sequence Models to Vision
Foundation Models", abstract, fused normalisation).

Each test fixes a part of that composition with something that is not the
oracle's own formula: brute-force loops over explicit tridiagonal products,
the reduction to the plain scan, invariants of the normalisation, and the
low-rank identity y = (U V) scan(x) that holds when the merger and lambda do
not depend on the proxy channel.  A swapped einsum index, a transposed
projection, a merger weight indexed by the wrong axis or direction order, or
a normalisation over the wrong axis fails at least one of them.
"""
import numpy as np
import pytest

import oracle
from test_oracle_pins import logits_for_weights, random_row_stochastic, tridiag

T2B, B2T, L2R, R2L = 1, 2, 4, 8


def block_inputs(B, C, Cp, H, W, seed):
    rng = np.random.default_rng(seed)
    return dict(
        x=rng.standard_normal((B, C, H, W)),
        v_proj=rng.standard_normal((Cp, C)) / np.sqrt(C),
        logits=rng.standard_normal((4, B, 1, 3, H, W)),
        lam=rng.random((4, B, Cp, H, W)),
        alpha=rng.standard_normal((4, Cp)),
        gamma=rng.random(Cp) + 0.5,
        u_proj=rng.standard_normal((C, Cp)),
    )


def run(inp, **kw):
    return oracle.block_fwd(inp["x"], inp["v_proj"], inp["logits"], inp["lam"], inp["alpha"], inp["gamma"],
                            inp["u_proj"], **kw)


# --------------------------------------------------------------------------
# brute force: loops and dense tridiagonal products
# --------------------------------------------------------------------------
def scan_dense(plane, lam, w_dir, d):
    """One direction's scan of an H x W plane by dense products of explicit
    tridiagonal matrices.  w_dir[i][j][k] are the taps of scan line i,
    position j (scan coordinates).  The plane is first mapped to scan
    coordinates (rows = lines): T2B as is, B2T flipped along H, L2R
    transposed, R2L transposed then flipped along the scan axis."""
    def to_scan(a):
        if d == T2B:
            return a
        if d == B2T:
            return a[::-1, :]
        if d == L2R:
            return a.T
        return a.T[::-1, :]

    def from_scan(a):
        if d == T2B:
            return a
        if d == B2T:
            return a[::-1, :]
        if d == L2R:
            return a.T
        return a[::-1, :].T

    u = to_scan(plane) * to_scan(lam)
    L, N = u.shape
    h = np.zeros((L, N))
    for i in range(L):
        acc = u[i].copy()
        for j0 in range(i):  # h_i = sum_j0 (w_i ... w_{j0+1}) u_j0 + u_i
            Wm = np.eye(N)
            for tau in range(j0 + 1, i + 1):
                Wm = tridiag(w_dir[tau]) @ Wm
            acc += Wm @ u[j0]
        h[i] = acc
    return from_scan(h)


def logits_from_dir_weights(w_dirs, H, W):
    """[4,1,1,3,H,W] logits (pixel-stored, image coordinates) whose normalised
    sigmoids are the chosen scan-coordinate weights of each direction."""
    lg = np.zeros((4, 1, 1, 3, H, W))
    for slot, d in enumerate((T2B, B2T, L2R, R2L)):
        lt = logits_for_weights(w_dirs[slot])  # [L][N][3] in scan coordinates
        for i in range(lt.shape[0]):
            for j in range(lt.shape[1]):
                r, c = {T2B: (i, j), B2T: (H - 1 - i, j), L2R: (j, i), R2L: (j, W - 1 - i)}[d]
                lg[slot, 0, 0, :, r, c] = lt[i, j]
    return lg


@pytest.mark.parametrize("C,Cp,H,W", [(3, 2, 4, 3), (5, 3, 3, 5), (2, 2, 1, 4)])
def test_block_against_brute_force_loops(C, Cp, H, W):
    rng = np.random.default_rng(100 + C * 7 + H)
    w_dirs = [random_row_stochastic(H, W, 11 + s) if d < L2R else random_row_stochastic(W, H, 11 + s)
              for s, d in enumerate((T2B, B2T, L2R, R2L))]
    lg = logits_from_dir_weights(w_dirs, H, W)
    x = rng.standard_normal((1, C, H, W))
    V = rng.standard_normal((Cp, C))
    lam = rng.random((4, 1, Cp, H, W))
    alpha = rng.standard_normal((4, Cp))
    gamma = rng.random(Cp) + 0.5
    U = rng.standard_normal((C, Cp))
    eps = 1e-6
    # loops
    xp = np.zeros((Cp, H, W))
    for k in range(Cp):
        for c in range(C):
            for r in range(H):
                for q in range(W):
                    xp[k, r, q] += V[k, c] * x[0, c, r, q]
    m = np.zeros((Cp, H, W))
    for slot, d in enumerate((T2B, B2T, L2R, R2L)):
        for k in range(Cp):
            m[k] += alpha[slot, k] * scan_dense(xp[k], lam[slot, 0, k], w_dirs[slot], d)
    n = np.zeros_like(m)
    for r in range(H):
        for q in range(W):
            ms = sum(m[k, r, q] ** 2 for k in range(Cp)) / Cp
            for k in range(Cp):
                n[k, r, q] = gamma[k] * m[k, r, q] / np.sqrt(ms + eps)
    y = np.zeros((C, H, W))
    for c in range(C):
        for k in range(Cp):
            y[c] += U[c, k] * n[k]
    got = oracle.block_fwd(x, V, lg, lam, alpha, gamma, U, eps=eps)
    np.testing.assert_allclose(got[0], y, rtol=1e-10, atol=1e-10)


# --------------------------------------------------------------------------
# reductions and identities
# --------------------------------------------------------------------------
def test_identity_projections_and_unit_merger_give_the_plain_scan():
    B, C, H, W = 2, 3, 6, 5
    inp = block_inputs(B, C, C, H, W, 1)
    inp["v_proj"] = np.eye(C)
    inp["u_proj"] = np.eye(C)
    inp["alpha"] = np.ones((4, C))
    got = run(inp, norm=False)
    want = oracle.fwd(inp["x"], inp["logits"], inp["lam"], dir_mask=15, shared=True)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("slot,bit", [(0, T2B), (1, B2T), (2, L2R), (3, R2L)])
def test_one_hot_merger_selects_its_direction(slot, bit):
    B, C, H, W = 1, 2, 5, 6
    inp = block_inputs(B, C, C, H, W, 2 + slot)
    inp["v_proj"] = np.eye(C)
    inp["u_proj"] = np.eye(C)
    alpha = np.zeros((4, C))
    alpha[slot] = [2.0, -0.5]  # distinct per proxy channel: pins alpha's channel axis too
    inp["alpha"] = alpha
    got = run(inp, norm=False)
    h = oracle.fwd(inp["x"], inp["logits"][slot:slot + 1], inp["lam"][slot:slot + 1], dir_mask=bit, shared=True)
    np.testing.assert_allclose(got, h * alpha[slot][None, :, None, None], rtol=1e-12, atol=1e-12)


def test_low_rank_identity():
    """With lambda and the merger weights the same for every proxy channel,
    the block without normalisation is the rank-Cp matrix U V applied over
    channels to the (alpha-merged) scan of x itself."""
    B, C, Cp, H, W = 2, 5, 2, 4, 6
    inp = block_inputs(B, C, Cp, H, W, 7)
    lam0 = np.random.default_rng(8).random((4, B, 1, H, W))
    inp["lam"] = np.repeat(lam0, Cp, axis=2)
    a = np.array([0.3, -1.2, 0.8, 2.0])
    inp["alpha"] = np.repeat(a[:, None], Cp, axis=1)
    got = run(inp, norm=False)
    s = np.zeros_like(inp["x"])
    for slot, bit in enumerate((T2B, B2T, L2R, R2L)):
        s += a[slot] * oracle.fwd(inp["x"], inp["logits"][slot:slot + 1], np.repeat(lam0[slot:slot + 1], C, axis=2),
                                  dir_mask=bit, shared=True)
    want = np.einsum("cd,bdhw->bchw", inp["u_proj"] @ inp["v_proj"], s)
    np.testing.assert_allclose(got, want, rtol=1e-11, atol=1e-11)


def test_rms_norm_invariants():
    """gamma = 1 and eps = 0: every pixel's normalised proxy vector has mean
    square 1 (read through U = I), the output does not change when x is
    scaled (the scan is linear), and gamma scales its channel."""
    B, C, H, W = 2, 4, 5, 5
    inp = block_inputs(B, C, C, H, W, 9)
    inp["v_proj"] = np.eye(C)
    inp["u_proj"] = np.eye(C)
    inp["gamma"] = np.ones(C)
    y = run(inp, eps=0.0)
    np.testing.assert_allclose(np.mean(y * y, axis=1), 1.0, rtol=1e-12)
    scaled = dict(inp, x=inp["x"] * 3.7)
    np.testing.assert_allclose(run(scaled, eps=0.0), y, rtol=1e-11, atol=1e-12)
    g = np.array([0.5, 2.0, 1.0, 3.0])
    np.testing.assert_allclose(run(dict(inp, gamma=g), eps=0.0), y * g[None, :, None, None], rtol=1e-12)


def test_linear_without_norm():
    B, C, Cp, H, W = 1, 3, 2, 4, 4
    i1 = block_inputs(B, C, Cp, H, W, 10)
    x2 = np.random.default_rng(11).standard_normal(i1["x"].shape)
    y1 = run(i1, norm=False)
    y2 = run(dict(i1, x=x2), norm=False)
    y12 = run(dict(i1, x=2.0 * i1["x"] - 0.5 * x2), norm=False)
    np.testing.assert_allclose(y12, 2.0 * y1 - 0.5 * y2, rtol=1e-11, atol=1e-11)


def test_local_groups_pass_through_to_the_scans():
    B, C, H, W = 1, 2, 6, 6
    inp = block_inputs(B, C, C, H, W, 12)
    inp["v_proj"] = np.eye(C)
    inp["u_proj"] = np.eye(C)
    inp["alpha"] = np.ones((4, C))
    got = run(inp, norm=False, groups=3)
    want = oracle.fwd(inp["x"], inp["logits"], inp["lam"], dir_mask=15, groups=3, shared=True)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)
