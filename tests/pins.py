"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each ``pin_*`` function takes an oracle object (``oracle.Oracle``) and raises
AssertionError when the oracle disagrees.  ``test_oracle_pins.py`` runs them on the
oracle as built; ``test_oracle_mutants.py`` runs them on copies of the oracle with a
planted mistake and requires every copy to fail at least one of them.

The equations cited are those of the page "Vision Mamba Guide: Efficient
Bidirectional SSM & VMamba" (aifetchly-blog); section names are given per pin.
"""
import math
import os

import numpy as np

import brute

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _vim_case(rng, batch=2, L=7, Di=3, N=4, separate_bc=True):
    """Random Vim inputs with every parameter different per direction and channel."""
    u = rng.normal(size=(batch, L, Di))
    delta = rng.uniform(0.01, 0.6, size=(batch, L, Di))          # post-softplus Delta
    z = rng.normal(size=(batch, L, Di))
    nb = 2 if separate_bc else 1
    B = rng.normal(size=(nb, batch, L, N))
    C = rng.normal(size=(nb, batch, L, N))
    A = -rng.uniform(0.2, 3.0, size=(2, Di, N))
    D = rng.normal(size=(2, Di))
    bias = rng.normal(size=(2, Di))
    stride = batch * L * N if separate_bc else 0
    return dict(u=u, delta=delta, z=z, B=B, C=C, A=A, D=D, bias=bias, stride=stride)


def _vim(orc, c, *, gate=True, raw=False, **over):
    c = {**c, **over}
    return orc.vim_bidir(c["u"], c["delta"], c["z"] if gate else None, c["B"], c["C"], c["A"], c["D"],
                         c["bias"], bc_dir_stride=c["stride"], delta_is_raw=raw)


def pin_delta_zero(orc):
    """Delta = 0 gives Abar = 1 and Bbar = 0: h stays at 0, so y = (D_f + D_b) u.

    Sections "Discretization via Zero-Order Hold (ZOH)" and "Continuous-Time State
    Space Equations" (the D x skip).
    """
    c = _vim_case(_rng(1))
    y = _vim(orc, c, gate=False, delta=np.zeros_like(c["delta"]))
    expect = (c["D"][0] + c["D"][1])[None, None, :] * c["u"]
    np.testing.assert_allclose(y, expect, rtol=1e-14, atol=1e-14)


def pin_constant_input_geometric(orc):
    """Constant Delta, u, B and C: h after k steps is the geometric series
    Delta B u (1 - Abar^k) / (1 - Abar); the forward pass has taken t+1 steps at
    token t and the backward pass L-t steps.

    Sections "Discretization via Zero-Order Hold (ZOH)" and "2. The Bidirectional
    Mamba Block" (forward over 1..N+1, backward from N+1 down to 1).
    """
    rng = _rng(2)
    batch, L, Di, N = 1, 23, 3, 5
    dlt, uu = 0.37, -1.3
    B = np.broadcast_to(rng.normal(size=(2, 1, 1, N)), (2, batch, L, N)).copy()
    C = np.broadcast_to(rng.normal(size=(2, 1, 1, N)), (2, batch, L, N)).copy()
    A = -rng.uniform(0.1, 2.0, size=(2, Di, N))
    D = rng.normal(size=(2, Di))
    u = np.full((batch, L, Di), uu)
    delta = np.full((batch, L, Di), dlt)
    y = orc.vim_bidir(u, delta, None, B, C, A, D, None, bc_dir_stride=batch * L * N,
                      delta_is_raw=False)
    t = np.arange(L)[:, None, None]
    steps = (t + 1, L - t)
    expect = np.zeros((L, Di))
    for k in range(2):
        abar = np.exp(dlt * A[k])[None]                      # [1, Di, N]
        geo = -np.expm1(steps[k] * np.log(abar)) / -np.expm1(np.log(abar))
        h = dlt * B[k, 0, 0][None, None, :] * uu * geo        # [L, Di, N]
        expect += (h * C[k, 0, 0][None, None, :]).sum(-1) + D[k][None, :] * uu
    np.testing.assert_allclose(y[0], expect, rtol=1e-12, atol=1e-12)


def pin_reverse_symmetry(orc):
    """Reversing the token sequence and swapping the forward/backward parameters
    reverses the output: the backward pathway is the forward pathway run on the
    reversed sequence with its output flipped back (section "2. The Bidirectional
    Mamba Block").  Checked both for one direction alone and for the gated pair.
    """
    rng = _rng(3)
    c = _vim_case(rng, L=9)
    # one direction: the reversed order on x equals flip(forward(flip(x)))
    u, dl, B, C = c["u"], c["delta"], c["B"][0], c["C"][0]
    L = u.shape[1]
    rev = np.arange(L)[::-1]
    yb = orc.s6_direction(u, dl, B, C, c["A"][1], c["D"][1], c["bias"][1], rev, delta_is_raw=True)
    yf = orc.s6_direction(u[:, ::-1], dl[:, ::-1], B[:, ::-1], C[:, ::-1], c["A"][1], c["D"][1],
                          c["bias"][1], np.arange(L), delta_is_raw=True)
    np.testing.assert_allclose(yb, yf[:, ::-1], rtol=1e-13, atol=1e-13)
    # the whole gated block, raw Delta through the bias
    y = _vim(orc, c, raw=True)
    flip = lambda a: a[..., ::-1, :]
    swapped = dict(u=flip(c["u"]), delta=flip(c["delta"]), z=flip(c["z"]),
                   B=flip(c["B"][::-1]), C=flip(c["C"][::-1]), A=c["A"][::-1], D=c["D"][::-1],
                   bias=c["bias"][::-1])
    y2 = _vim(orc, c, raw=True, **{k: np.ascontiguousarray(v) for k, v in swapped.items()})
    np.testing.assert_allclose(y, flip(y2), rtol=1e-12, atol=1e-12)


def pin_brute_force(orc):
    """Explicit unrolled sums (tests/brute.py) agree on tiny inputs, L = 1..8."""
    rng = _rng(4)
    for L in (1, 2, 3, 5, 8):
        c = _vim_case(rng, batch=1, L=L, Di=2, N=3)
        y = _vim(orc, c, gate=False)
        Bf, Bb = c["B"][0, 0].tolist(), c["B"][1, 0].tolist()
        Cf, Cb = c["C"][0, 0].tolist(), c["C"][1, 0].tolist()
        ref = brute.bidir_ungated(c["u"][0].tolist(), c["delta"][0].tolist(), Bf, Cf,
                                  c["A"].tolist(), c["D"].tolist(), Bb, Cb)
        np.testing.assert_allclose(y[0], np.array(ref), rtol=1e-12, atol=1e-12)


def pin_prefix_sum(orc):
    """A = 0, N = 1, B = C = 1, D = 0: Abar = 1, so the forward output is the prefix
    sum of Delta u and the backward output the suffix sum (math.fsum)."""
    rng = _rng(5)
    L = 57
    u = rng.normal(size=(1, L, 1))
    delta = rng.uniform(0, 1, size=(1, L, 1))
    ones = np.ones((1, L, 1))
    y = orc.vim_bidir(u, delta, None, ones, ones, np.zeros((2, 1, 1)), np.zeros((2, 1)), None,
                      delta_is_raw=False)
    du = (u * delta)[0, :, 0].tolist()
    expect = [math.fsum(du[: t + 1]) + math.fsum(du[t:]) for t in range(L)]
    np.testing.assert_allclose(y[0, :, 0], expect, rtol=1e-13, atol=1e-13)


def pin_linearity(orc):
    """At fixed Delta, B and C the recurrence and readout are linear in u."""
    rng = _rng(6)
    c = _vim_case(rng, L=11)
    u2 = rng.normal(size=c["u"].shape)
    a, b = 0.7, -1.9
    y1 = _vim(orc, c, gate=False)
    y2 = _vim(orc, c, gate=False, u=u2)
    y12 = _vim(orc, c, gate=False, u=a * c["u"] + b * u2)
    np.testing.assert_allclose(y12, a * y1 + b * y2, rtol=1e-11, atol=1e-11)


def pin_softplus(orc):
    """Delta = softplus(delta_raw + bias) (section "The Selective State Space (S6)
    Mechanism").  With L = 1, N = 1, A = 0, B = C = u = 1 and D = 0 each direction
    outputs its Delta, so one pass reads softplus off.  Checked against properties
    that fix it: softplus(0) = ln 2, softplus(x) - softplus(-x) = x, softplus(x) ->
    e^x - e^{2x}/2 for x -> -inf, and softplus(x) = x above the cut at 20.
    """
    def sp1(x):
        ones = np.ones((1, 1, 1))
        bias = np.array([[x], [-40.0]])                 # backward direction: Delta ~ e^-40
        y = orc.vim_bidir(ones, ones * 0.0, None, ones, ones, np.zeros((2, 1, 1)),
                          np.zeros((2, 1)), bias, delta_is_raw=True)
        return float(y[0, 0, 0]) - math.exp(-40.0)

    assert abs(sp1(0.0) - math.log(2.0)) < 1e-15
    for x in (0.5, 3.0, 7.25, 15.0):
        assert abs((sp1(x) - sp1(-x)) - x) < 1e-13 * max(1.0, x)
    for x in (-12.0, -25.0, -30.0):
        e = math.exp(x)
        assert abs(sp1(x) - (e - e * e / 2 + e * e * e / 3)) <= 1e-13 * e
    assert sp1(25.0) == 25.0 and sp1(21.0) == 21.0


def pin_gate_is_silu(orc):
    """The fused output is multiplied by silu(z) = z * sigmoid(z) (section "2. The
    Bidirectional Mamba Block").  Pinned by silu(z) - silu(-z) = z: the gated
    outputs for z and -z differ by z times the ungated output, and silu(0) = 0."""
    c = _vim_case(_rng(7))
    y0 = _vim(orc, c, gate=False)
    yp = _vim(orc, c, gate=True)
    ym = orc.vim_bidir(c["u"], c["delta"], -c["z"], c["B"], c["C"], c["A"], c["D"], c["bias"],
                       bc_dir_stride=c["stride"], delta_is_raw=False)
    np.testing.assert_allclose(yp - ym, c["z"] * y0, rtol=1e-12, atol=1e-12)
    yz = orc.vim_bidir(c["u"], c["delta"], np.zeros_like(c["z"]), c["B"], c["C"], c["A"], c["D"],
                       c["bias"], bc_dir_stride=c["stride"], delta_is_raw=False)
    assert np.all(yz == 0.0)
    # large |z|: silu(z) -> z, silu(-z) -> 0
    big = np.full_like(c["z"], 40.0)
    yb = orc.vim_bidir(c["u"], c["delta"], big, c["B"], c["C"], c["A"], c["D"], c["bias"],
                       bc_dir_stride=c["stride"], delta_is_raw=False)
    np.testing.assert_allclose(yb, 40.0 * y0, rtol=1e-15, atol=1e-15)


def _golden_orders():
    rows = []
    with open(os.path.join(GOLDEN, "cross_scan_orders.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                v = [int(x) for x in line.split()]
                rows.append((v[0], v[1], v[2], v[3:]))
    return rows


def pin_cross_orders_golden(orc):
    """The four traversal orders match the hand-written fixture (section "1.
    Cross-Scan Traversal (CS-Traverse)")."""
    rows = _golden_orders()
    assert len(rows) >= 12
    for H, W, k, order in rows:
        assert orc.cross_order(k - 1, H, W).tolist() == order, (H, W, k)


def _traverse(x):
    """Explicit CS-Traverse of a channels-last grid x [B, H, W, C] into the four
    sequences [4, B, H*W, C]: row-major, its reverse, column-major (transpose, then
    flatten), its reverse."""
    b, H, W, c = x.shape
    s1 = x.reshape(b, H * W, c)
    s3 = x.transpose(0, 2, 1, 3).reshape(b, W * H, c)
    return np.stack([s1, s1[:, ::-1], s3, s3[:, ::-1]])


def _untraverse(ys, H, W):
    """Inverse of _traverse for one direction each: [4, B, H*W, C] -> 4 grids."""
    _, b, L, c = ys.shape
    g1 = ys[0].reshape(b, H, W, c)
    g2 = ys[1][:, ::-1].reshape(b, H, W, c)
    g3 = ys[2].reshape(b, W, H, c).transpose(0, 2, 1, 3)
    g4 = ys[3][:, ::-1].reshape(b, W, H, c).transpose(0, 2, 1, 3)
    return [g1, g2, g3, g4]


def pin_cross_scan_is_transpose_and_flip(orc):
    """The four-direction scan equals: explicit transpose/flip of the grid into four
    sequences, four plain forward scans (each with its own parameters and its own
    B/C, gathered the same way), the inverse maps, the sum and the gate (sections
    "1. Cross-Scan Traversal", "2. Parallel S6 State Space Processing",
    "3. Cross-Merge Reversal").  H != W so a transposed index cannot pass."""
    rng = _rng(8)
    b, H, W, c, N = 2, 3, 5, 4, 3
    u = rng.normal(size=(b, H, W, c))
    dr = rng.normal(size=(b, H, W, c)) * 0.5
    z = rng.normal(size=(b, H, W, c))
    B = rng.normal(size=(4, b, H * W, N))
    C = rng.normal(size=(4, b, H * W, N))
    A = -rng.uniform(0.1, 2.0, size=(4, c, N))
    D = rng.normal(size=(4, c))
    bias = rng.normal(size=(4, c))
    y = orc.cross_scan4(u, dr, z, B, C, A, D, bias, delta_is_raw=True)
    seq_u, seq_d = _traverse(u), _traverse(dr)
    outs = []
    for k in range(4):
        Bk = _traverse(B[k].reshape(b, H, W, N))[k]
        Ck = _traverse(C[k].reshape(b, H, W, N))[k]
        outs.append(orc.s6_direction(np.ascontiguousarray(seq_u[k]), np.ascontiguousarray(seq_d[k]),
                                     np.ascontiguousarray(Bk), np.ascontiguousarray(Ck),
                                     A[k], D[k], bias[k], np.arange(H * W), delta_is_raw=True))
    grids = _untraverse(np.stack(outs), H, W)
    gate = orc.cross_scan4(u, dr, None, B, C, A, D, bias, delta_is_raw=True)
    np.testing.assert_allclose(gate, sum(grids), rtol=1e-12, atol=1e-12)
    # the gate, through the silu(z) - silu(-z) = z identity
    ym = orc.cross_scan4(u, dr, -z, B, C, A, D, bias, delta_is_raw=True)
    np.testing.assert_allclose(y - ym, z * gate, rtol=1e-12, atol=1e-12)


def pin_cross_merge(orc):
    """CS-Merge maps each scan back to (h, w) and sums (section "3. Cross-Merge
    Reversal"): merging the explicit traversal of a grid gives 4x the grid, and
    one-hot scans land where the inverse maps say.  Shapes follow the page's
    verification block: a (2, 64, 16, 16) map traverses to (4, 2, 256, 64) and
    merges back to (2, 64, 16, 16) (channels last here)."""
    rng = _rng(9)
    shapes = {}
    with open(os.path.join(GOLDEN, "page_shapes.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                k, *v = line.split()
                shapes[k] = tuple(int(x) for x in v)
    b, c, H, W = shapes["cross_in_bchw"]
    x = rng.normal(size=(b, H, W, c))
    scans = _traverse(x)
    assert scans.shape == shapes["cross_scans"]
    merged = orc.cross_merge4(np.ascontiguousarray(scans), None, H, W)
    assert merged.transpose(0, 3, 1, 2).shape == shapes["cross_merged_bchw"]
    np.testing.assert_allclose(merged, 4 * x, rtol=1e-14, atol=1e-14)
    # non-square, per-direction distinct inputs
    H, W = 2, 3
    ys = rng.normal(size=(4, 1, H * W, 2))
    got = orc.cross_merge4(ys, None, H, W)
    want = sum(_untraverse(ys, H, W))
    np.testing.assert_allclose(got, want, rtol=1e-14, atol=1e-14)
    z = rng.normal(size=(1, H, W, 2))
    gz = orc.cross_merge4(ys, z, H, W)
    gm = orc.cross_merge4(ys, -z, H, W)
    np.testing.assert_allclose(gz - gm, z * want, rtol=1e-13, atol=1e-13)


def pin_separate_bc(orc):
    """With bc_dir_stride the backward direction reads its own B and C: running the
    pair with swapped copies equals the brute force with swapped copies."""
    rng = _rng(10)
    c = _vim_case(rng, batch=1, L=4, Di=2, N=2)
    y = _vim(orc, c, gate=False)
    ref = brute.bidir_ungated(c["u"][0].tolist(), c["delta"][0].tolist(), c["B"][0, 0].tolist(),
                              c["C"][0, 0].tolist(), c["A"].tolist(), c["D"].tolist(),
                              c["B"][1, 0].tolist(), c["C"][1, 0].tolist())
    np.testing.assert_allclose(y[0], np.array(ref), rtol=1e-12, atol=1e-12)


def pin_conv_front_is_correlation(orc):
    """The convolution in front of each pathway (section "2. The Bidirectional Mamba
    Block": "1D Conv -> SiLU"; a depthwise kernel-3 convolution with padding 1, the
    backward one on the reversed sequence).  With a large bias the SiLU is the
    identity to within e^-40, so the pre-activation is read off and compared with
    numpy's 'same'-mode correlation: directly for the forward pathway, and on the
    reversed sequence, flipped back, for the backward one."""
    rng = _rng(11)
    b, L, Di = 2, 13, 3
    x = rng.normal(size=(b, L, Di))
    w = rng.normal(size=(Di, 3))
    big = 60.0
    cb = np.full(Di, big)
    uf = orc.conv_silu(x, w, cb) - big
    ub = orc.conv_silu(x, w, cb, reversed=True) - big
    for bi in range(b):
        for d in range(Di):
            ref_f = np.correlate(x[bi, :, d], w[d], mode="same")
            ref_b = np.correlate(x[bi, ::-1, d], w[d], mode="same")[::-1]
            np.testing.assert_allclose(uf[bi, :, d], ref_f, rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(ub[bi, :, d], ref_b, rtol=1e-12, atol=1e-12)
    # the activation is silu: the identity silu(v) - silu(-v) = v with w = (0, 1, 0)
    e = np.zeros((Di, 3)); e[:, 1] = 1.0
    np.testing.assert_allclose(orc.conv_silu(x, e, np.zeros(Di)) - orc.conv_silu(-x, e, np.zeros(Di)), x,
                               rtol=1e-12, atol=1e-12)


def pin_conv_scan_composition(orc):
    """The scan with the convolution front is the plain bidirectional scan with each
    direction fed its own smoothed input; and reversing the sequence while swapping
    every per-direction parameter (weights, biases, B/C copies) reverses the output."""
    rng = _rng(12)
    c = _vim_case(rng, L=10)
    x = rng.normal(size=c["u"].shape)
    cw = rng.normal(size=(2, 3, 3))
    cbias = rng.normal(size=(2, 3))
    y = orc.vim_bidir_conv(x, cw, cbias, c["delta"], c["z"], c["B"], c["C"], c["A"], c["D"], c["bias"],
                           bc_dir_stride=c["stride"], delta_is_raw=True)
    uf = orc.conv_silu(x, cw[0], cbias[0])
    ub = orc.conv_silu(x, cw[1], cbias[1], reversed=True)
    L = x.shape[1]
    yf = orc.s6_direction(uf, c["delta"], c["B"][0], c["C"][0], c["A"][0], c["D"][0], c["bias"][0],
                          np.arange(L), delta_is_raw=True)
    yb = orc.s6_direction(ub, c["delta"], c["B"][1], c["C"][1], c["A"][1], c["D"][1], c["bias"][1],
                          np.arange(L)[::-1], delta_is_raw=True)
    gate_ref = orc.vim_bidir(np.ones_like(x), np.zeros_like(x), c["z"], c["B"], c["C"], c["A"],
                             np.stack([np.ones(3), np.zeros(3)]), c["bias"], bc_dir_stride=c["stride"],
                             delta_is_raw=False)   # = silu(z): Delta = 0, D_f = 1, u = 1
    np.testing.assert_allclose(y, (yf + yb) * gate_ref, rtol=1e-12, atol=1e-12)
    flip = lambda a: np.ascontiguousarray(a[..., ::-1, :])
    y2 = orc.vim_bidir_conv(flip(x), cw[::-1].copy(), cbias[::-1].copy(), flip(c["delta"]), flip(c["z"]),
                            flip(c["B"][::-1]), flip(c["C"][::-1]), c["A"][::-1].copy(), c["D"][::-1].copy(),
                            c["bias"][::-1].copy(), bc_dir_stride=c["stride"], delta_is_raw=True)
    np.testing.assert_allclose(y, flip(y2), rtol=1e-12, atol=1e-12)


def pin_zoh_matches_ode(orc):
    """The exact zero-order hold is exact for inputs held over each step: with
    Delta_t, u_t and B_t constant on a step of length Delta_t, integrating the
    continuous system h' = A h + B x (section "Continuous-Time State Space
    Equations") over that step gives h_t = Abar h_{t-1} + Bbar x_t with Abar =
    exp(Delta A) and Bbar = (Delta A)^-1 (exp(Delta A) - I) Delta B (section
    "Discretization via Zero-Order Hold (ZOH)").  The reference here is a numerical
    ODE solver (scipy's DOP853 at rtol 1e-12), independent of the closed form; the
    first-order form Delta B must differ from it by far more than the tolerance.
    """
    from scipy.integrate import solve_ivp

    rng = _rng(91)
    batch, L, Di, N = 1, 6, 2, 4
    u = rng.normal(size=(batch, L, Di))
    delta = rng.uniform(0.05, 0.9, size=(batch, L, Di))
    B = rng.normal(size=(batch, L, N))
    C = rng.normal(size=(batch, L, N))
    A = -rng.uniform(0.2, 3.0, size=(Di, N))
    D = rng.normal(size=Di)
    order = np.arange(L)
    expect = np.zeros((batch, L, Di))
    for b in range(batch):
        for d in range(Di):
            h = np.zeros(N)
            for t in range(L):
                drive = B[b, t] * u[b, t, d]
                sol = solve_ivp(lambda _s, hh: A[d] * hh + drive, (0.0, delta[b, t, d]), h,
                                method="DOP853", rtol=1e-12, atol=1e-14)
                h = sol.y[:, -1]
                expect[b, t, d] = C[b, t] @ h + D[d] * u[b, t, d]
    got = orc.s6_direction(u, delta, B, C, A, D, None, order, delta_is_raw=False, zoh=True)
    np.testing.assert_allclose(got, expect, rtol=1e-9, atol=1e-11)
    euler = orc.s6_direction(u, delta, B, C, A, D, None, order, delta_is_raw=False, zoh=False)
    assert np.max(np.abs(euler - expect)) > 1e-3


def pin_zoh_fixed_point_and_limits(orc):
    """Three consequences of the exact form, each checked through the two-direction
    scan (section "Discretization via Zero-Order Hold (ZOH)"):
    - constant input: h tends to the continuous system's rest point -B u / A,
      whatever Delta is, so both directions end at y = sum_k (C (-B u / A_k) + D_k u);
    - A = 0: Bbar is its limit Delta B, so the exact and first-order forms agree;
    - small Delta: the two forms differ by O(Delta^2) per step, so halving Delta
      quarters the gap (ratio within 3.5 .. 4.5).
    """
    rng = _rng(92)
    batch, L, Di, N = 1, 400, 3, 4
    u0 = rng.normal(size=Di)
    Bc, Cc = rng.normal(size=N), rng.normal(size=N)
    A = -rng.uniform(0.3, 2.0, size=(2, Di, N))
    D = rng.normal(size=(2, Di))
    u = np.broadcast_to(u0, (batch, L, Di)).copy()
    B = np.broadcast_to(Bc, (batch, L, N)).copy()
    Cm = np.broadcast_to(Cc, (batch, L, N)).copy()
    delta = np.full((batch, L, Di), 0.7)
    y = orc.vim_bidir(u, delta, None, B, Cm, A, D, None, delta_is_raw=False, zoh=True)
    rest = sum(((-Bc[None, :] / A[k]) @ Cc) * u0 + D[k] * u0 for k in range(2))
    # forward has taken L steps at the last token, backward L steps at the first;
    # only the sum at the middle has both near rest, so check y at L/2 against it
    np.testing.assert_allclose(y[0, L // 2], rest, rtol=1e-12, atol=1e-12)

    c = _vim_case(_rng(93))
    A0 = np.zeros_like(c["A"])
    ye = _vim(orc, c, gate=False, A=A0)
    yz = orc.vim_bidir(c["u"], c["delta"], None, c["B"], c["C"], A0, c["D"], c["bias"],
                       bc_dir_stride=c["stride"], delta_is_raw=False, zoh=True)
    np.testing.assert_allclose(yz, ye, rtol=1e-14, atol=1e-14)

    gaps = []
    for scale in (1e-3, 5e-4):
        dl = np.full_like(c["delta"], scale)
        y1 = _vim(orc, c, gate=False, delta=dl)
        y2 = orc.vim_bidir(c["u"], dl, None, c["B"], c["C"], c["A"], c["D"], c["bias"],
                           bc_dir_stride=c["stride"], delta_is_raw=False, zoh=True)
        gaps.append(np.max(np.abs(y2 - y1)))
    assert 3.5 < gaps[0] / gaps[1] < 4.5, gaps


def pin_zoh_reaches_every_entry(orc):
    """The exact-ZOH choice reaches every direction of every entry: the
    two-direction scan (with and without the convolution front) and the
    four-direction scan each equal their explicit composition from single exact-ZOH
    directions (the single direction itself is pinned by pin_zoh_matches_ode)."""
    rng = _rng(94)
    c = _vim_case(rng, L=9)
    L = c["u"].shape[1]
    yf = orc.s6_direction(c["u"], c["delta"], c["B"][0], c["C"][0], c["A"][0], c["D"][0], None,
                          np.arange(L), delta_is_raw=False, zoh=True)
    yb = orc.s6_direction(c["u"], c["delta"], c["B"][1], c["C"][1], c["A"][1], c["D"][1], None,
                          np.arange(L)[::-1], delta_is_raw=False, zoh=True)
    y = orc.vim_bidir(c["u"], c["delta"], None, c["B"], c["C"], c["A"], c["D"], None,
                      bc_dir_stride=c["stride"], delta_is_raw=False, zoh=True)
    np.testing.assert_allclose(y, yf + yb, rtol=1e-12, atol=1e-12)

    x = rng.normal(size=c["u"].shape)
    cw, cbias = rng.normal(size=(2, 3, 3)), rng.normal(size=(2, 3))
    uf, ub = orc.conv_silu(x, cw[0], cbias[0]), orc.conv_silu(x, cw[1], cbias[1], reversed=True)
    yf = orc.s6_direction(uf, c["delta"], c["B"][0], c["C"][0], c["A"][0], c["D"][0], None,
                          np.arange(L), delta_is_raw=False, zoh=True)
    yb = orc.s6_direction(ub, c["delta"], c["B"][1], c["C"][1], c["A"][1], c["D"][1], None,
                          np.arange(L)[::-1], delta_is_raw=False, zoh=True)
    y = orc.vim_bidir_conv(x, cw, cbias, c["delta"], None, c["B"], c["C"], c["A"], c["D"], None,
                           bc_dir_stride=c["stride"], delta_is_raw=False, zoh=True)
    np.testing.assert_allclose(y, yf + yb, rtol=1e-12, atol=1e-12)

    b, H, W, ch, N = 1, 3, 4, 2, 3
    u = rng.normal(size=(b, H, W, ch))
    dl = rng.uniform(0.05, 0.8, size=(b, H, W, ch))
    B = rng.normal(size=(4, b, H * W, N))
    C = rng.normal(size=(4, b, H * W, N))
    A = -rng.uniform(0.1, 2.0, size=(4, ch, N))
    D = rng.normal(size=(4, ch))
    y = orc.cross_scan4(u, dl, None, B, C, A, D, None, delta_is_raw=False, zoh=True)
    seq_u, seq_d = _traverse(u), _traverse(dl)
    outs = []
    for k in range(4):
        Bk = _traverse(B[k].reshape(b, H, W, N))[k]
        Ck = _traverse(C[k].reshape(b, H, W, N))[k]
        outs.append(orc.s6_direction(np.ascontiguousarray(seq_u[k]), np.ascontiguousarray(seq_d[k]),
                                     np.ascontiguousarray(Bk), np.ascontiguousarray(Ck), A[k], D[k], None,
                                     np.arange(H * W), delta_is_raw=False, zoh=True))
    np.testing.assert_allclose(y, sum(_untraverse(np.stack(outs), H, W)), rtol=1e-12, atol=1e-12)


def _bwd_case(rng, batch=1, L=5, Di=2, N=3, separate_bc=True):
    c = _vim_case(rng, batch=batch, L=L, Di=Di, N=N, separate_bc=separate_bc)
    c["delta"] = rng.normal(size=c["u"].shape) * 0.8          # raw delta
    c["dout"] = rng.normal(size=c["u"].shape)
    return c


def _loss(orc, c, zoh=False, **over):
    c = {**c, **over}
    y = orc.vim_bidir(c["u"], c["delta"], c["z"], c["B"], c["C"], c["A"], c["D"], c["bias"],
                      bc_dir_stride=c["stride"], delta_is_raw=True, zoh=zoh)
    return float(np.sum(c["dout"] * y))


def _bwd_fd(orc, c, zoh):
    g = orc.vim_bidir_bwd(c["u"], c["delta"], c["z"], c["B"], c["C"], c["A"], c["D"], c["bias"], c["dout"],
                          bc_dir_stride=c["stride"], zoh=zoh)
    for name, key in (("u", "du"), ("delta", "ddelta"), ("z", "dz"), ("B", "dB"), ("C", "dC"),
                      ("A", "dA"), ("D", "dD"), ("bias", "dbias")):
        arr, eps = c[name], 1e-6
        fd = np.zeros_like(arr)
        for i in np.ndindex(arr.shape):
            up, dn = arr.copy(), arr.copy()
            up[i] += eps
            dn[i] -= eps
            fd[i] = (_loss(orc, c, zoh, **{name: up}) - _loss(orc, c, zoh, **{name: dn})) / (2 * eps)
        err = np.max(np.abs(fd - g[key])) / np.max(np.abs(fd))
        assert err < 1e-7, (name, zoh, err)


def pin_bwd_finite_differences(orc):
    """Every derivative of the two-direction scan (u, raw delta, z, per-direction B
    and C, A, D, delta bias) against central finite differences of the loss
    sum(dout * y) computed with the forward oracle alone (sections "Discretization
    via Zero-Order Hold (ZOH)", "The Selective State Space (S6) Mechanism", "2. The
    Bidirectional Mamba Block").  Step 1e-6 in fp64: truncation and rounding stay
    near 1e-9 of the gradient's size."""
    _bwd_fd(orc, _bwd_case(_rng(101)), zoh=False)


def pin_zoh_bwd_finite_differences(orc):
    """The same check for the exact zero-order hold (section "Discretization via
    Zero-Order Hold (ZOH)": Bbar_n = (exp(Delta A_n) - 1) / A_n B_n), with A spanning
    small |Delta A_n| (the oracle's series for dBbar/dA), large ones (its closed form)
    and one A_n = 0 (the limit Delta B_n, whose A-derivative is Delta^2 B_n / 2)."""
    c = _bwd_case(_rng(131))
    A = -np.exp(_rng(132).uniform(np.log(0.005), np.log(4.0), size=c["A"].shape))
    A[0, 1, 2] = 0.0
    c["A"] = A
    _bwd_fd(orc, c, zoh=True)


def pin_bwd_homogeneity(orc):
    """Identities of the loss's derivative at a larger size, with B and C shared by
    the directions: the output is linear in u, in B and in C (Delta fixed), so by
    Euler's theorem sum(du*u) = ell, sum(dB*B) = sum(dC*C) = ell minus the D u part,
    and sum(dD*D) = the D u part (each direction's D enters linearly)."""
    rng = _rng(102)
    c = _bwd_case(rng, batch=2, L=40, Di=5, N=4, separate_bc=False)
    g = orc.vim_bidir_bwd(c["u"], c["delta"], c["z"], c["B"], c["C"], c["A"], c["D"], c["bias"], c["dout"],
                          bc_dir_stride=0)
    ell = _loss(orc, c)
    silu = c["z"] / (1 + np.exp(-c["z"]))
    ell_D = float(np.sum(c["dout"] * silu * (c["D"][0] + c["D"][1])[None, None, :] * c["u"]))
    np.testing.assert_allclose(np.sum(g["du"] * c["u"]), ell, rtol=1e-11)
    np.testing.assert_allclose(np.sum(g["dB"] * c["B"]), ell - ell_D, rtol=1e-11)
    np.testing.assert_allclose(np.sum(g["dC"] * c["C"]), ell - ell_D, rtol=1e-11)
    np.testing.assert_allclose(np.sum(g["dD"] * c["D"]), ell_D, rtol=1e-11)


def pin_xproj_is_matmul(orc):
    """x_proj is a plain matrix product (the PyTorch SimpleSelectiveSSM's
    nn.Linear without bias, page "Vision Mamba Guide"): checked against numpy's
    matmul on a non-square weight, so a transposed index cannot pass."""
    rng = _rng(111)
    u = rng.normal(size=(2, 7, 6))
    Wx = rng.normal(size=(6, 9))
    np.testing.assert_allclose(orc.xproj(u, Wx), np.matmul(u, Wx), rtol=1e-13, atol=1e-13)


def pin_block_scan_composition(orc):
    """The Vim block scan with its projections equals its steps done separately:
    each pathway's smoothed input by numpy correlation (the conv pin's method), its
    projection by numpy matmul split as the page's module splits it (B = columns
    0..N-1, C = N..2N-1, the step input = column 2N), dt_proj as the outer product of
    that column with the pathway's weights, the two directions by single-direction
    scans (pinned separately), then the gate."""
    rng = _rng(112)
    batch, L, Di, N = 2, 9, 3, 4
    x = rng.normal(size=(batch, L, Di))
    z = rng.normal(size=(batch, L, Di))
    Wx = rng.normal(size=(2, Di, 2 * N + 1)) * 0.5
    Wdt = rng.normal(size=(2, Di))
    bias = rng.normal(size=(2, Di))
    A = -rng.uniform(0.2, 2.0, size=(2, Di, N))
    D = rng.normal(size=(2, Di))
    cw = rng.normal(size=(2, Di, 3))
    cb = rng.normal(size=(2, Di))
    y = orc.vim_block_scan(x, Wx, Wdt, A, D, bias, z, conv_w=cw, conv_b=cb)
    silu = lambda v: v / (1 + np.exp(-v))
    total = np.zeros_like(x)
    for k in range(2):
        u = np.zeros_like(x)
        for b in range(batch):
            for d in range(Di):
                seq = x[b, :, d] if k == 0 else x[b, ::-1, d]
                sm = np.correlate(np.pad(seq, 1), cw[k, d], mode="valid") + cb[k, d]
                u[b, :, d] = silu(sm) if k == 0 else silu(sm)[::-1]
        P = np.matmul(u, Wx[k])
        Bk, Ck, s = P[..., :N], P[..., N:2 * N], P[..., 2 * N]
        draw = s[..., None] * Wdt[k][None, None, :]
        order = np.arange(L) if k == 0 else np.arange(L)[::-1]
        total += orc.s6_direction(u, draw, np.ascontiguousarray(Bk), np.ascontiguousarray(Ck), A[k], D[k],
                                  bias[k], order, delta_is_raw=True)
    np.testing.assert_allclose(y, total * silu(z), rtol=1e-11, atol=1e-11)
    # without the convolution the pathways see x itself
    y0 = orc.vim_block_scan(x, Wx, Wdt, A, D, bias, None)
    P0 = [np.matmul(x, Wx[k]) for k in range(2)]
    ref0 = sum(orc.s6_direction(x, P0[k][..., 2 * N][..., None] * Wdt[k][None, None, :],
                                np.ascontiguousarray(P0[k][..., :N]), np.ascontiguousarray(P0[k][..., N:2 * N]),
                                A[k], D[k], bias[k], np.arange(L) if k == 0 else np.arange(L)[::-1],
                                delta_is_raw=True) for k in range(2))
    np.testing.assert_allclose(y0, ref0, rtol=1e-11, atol=1e-11)


def _cross_bwd_fd(orc, seed, zoh):
    rng = _rng(seed)
    b, H, W, c, N = 1, 2, 3, 2, 2
    x = dict(u=rng.normal(size=(b, H, W, c)), delta=rng.normal(size=(b, H, W, c)) * 0.8,
             z=rng.normal(size=(b, H, W, c)), B=rng.normal(size=(4, b, H * W, N)),
             C=rng.normal(size=(4, b, H * W, N)), A=-rng.uniform(0.2, 2.0, size=(4, c, N)),
             D=rng.normal(size=(4, c)), bias=rng.normal(size=(4, c)))
    dout = rng.normal(size=(b, H, W, c))
    loss = lambda **o: float(np.sum(dout * orc.cross_scan4(*[{**x, **o}[k] for k in
                                                               ("u", "delta", "z", "B", "C", "A", "D", "bias")],
                                                             zoh=zoh)))
    g = orc.cross_scan4_bwd(x["u"], x["delta"], x["z"], x["B"], x["C"], x["A"], x["D"], x["bias"], dout, zoh=zoh)
    for name, key in (("u", "du"), ("delta", "ddelta"), ("z", "dz"), ("B", "dB"), ("C", "dC"), ("A", "dA"),
                      ("D", "dD"), ("bias", "dbias")):
        arr, eps = x[name], 1e-6
        fd = np.zeros_like(arr)
        for i in np.ndindex(arr.shape):
            up, dn = arr.copy(), arr.copy()
            up[i] += eps
            dn[i] -= eps
            fd[i] = (loss(**{name: up}) - loss(**{name: dn})) / (2 * eps)
        err = np.max(np.abs(fd - g[key])) / np.max(np.abs(fd))
        assert err < 1e-7, (name, zoh, err)


def pin_cross_bwd_finite_differences(orc):
    """Every derivative of the four-direction scan against central finite differences
    of the forward oracle's loss sum(dout * y) on a 2 x 3 grid (H != W, so a transposed
    traversal cannot pass), with per-direction B, C, A, D and bias (sections "1.
    Cross-Scan Traversal" to "3. Cross-Merge Reversal"); first-order and exact hold."""
    _cross_bwd_fd(orc, 121, zoh=False)
    _cross_bwd_fd(orc, 122, zoh=True)


def _conv_bwd_case(rng, batch=1, L=6, Di=2, N=3):
    c = _bwd_case(rng, batch=batch, L=L, Di=Di, N=N, separate_bc=True)
    c["x"] = c.pop("u")
    c["conv_w"] = rng.normal(size=(2, Di, 3)) * 0.7
    c["conv_b"] = rng.normal(size=(2, Di)) * 0.5
    return c


def _conv_loss(orc, c, zoh=False, **over):
    c = {**c, **over}
    y = orc.vim_bidir_conv(c["x"], c["conv_w"], c["conv_b"], c["delta"], c["z"], c["B"], c["C"], c["A"], c["D"],
                           c["bias"], bc_dir_stride=c["stride"], delta_is_raw=True, zoh=zoh)
    return float(np.sum(c["dout"] * y))


def pin_conv_bwd_finite_differences(orc):
    """Every derivative of the scan with its convolution front (x, both pathways'
    taps and biases, raw delta, z, per-direction B and C, A, D, delta bias) against
    central finite differences of the forward oracle's loss sum(dout * y) (section "2.
    The Bidirectional Mamba Block": each pathway's "1D Conv -> SiLU" in front of its
    SSM); first-order and exact hold.  Step 1e-6 in fp64."""
    for seed, zoh in ((141, False), (142, True)):
        c = _conv_bwd_case(_rng(seed))
        g = orc.vim_bidir_conv_bwd(c["x"], c["conv_w"], c["conv_b"], c["delta"], c["z"], c["B"], c["C"], c["A"],
                                   c["D"], c["bias"], c["dout"], bc_dir_stride=c["stride"], zoh=zoh)
        for name, key in (("x", "dx"), ("conv_w", "dconv_w"), ("conv_b", "dconv_b"), ("delta", "ddelta"),
                          ("z", "dz"), ("B", "dB"), ("C", "dC"), ("A", "dA"), ("D", "dD"), ("bias", "dbias")):
            arr, eps = c[name], 1e-6
            fd = np.zeros_like(arr)
            for i in np.ndindex(arr.shape):
                up, dn = arr.copy(), arr.copy()
                up[i] += eps
                dn[i] -= eps
                fd[i] = (_conv_loss(orc, c, zoh, **{name: up}) - _conv_loss(orc, c, zoh, **{name: dn})) / (2 * eps)
            err = np.max(np.abs(fd - g[key])) / np.max(np.abs(fd))
            assert err < 1e-7, (name, zoh, err)


def pin_conv_bwd_identity_taps(orc):
    """With taps (0, 1, 0) and zero biases both pathways see u = silu(x), so the
    front's derivative reduces to the plain scan's by the chain rule: dx = du silu'(x)
    with du from the scan's derivative at u = silu(x); every other derivative equals
    the scan's; summed over the two pathways, the bias derivatives are the token sums
    of du silu'(x) and the middle taps' those of du silu'(x) x."""
    rng = _rng(143)
    c = _conv_bwd_case(rng, batch=2, L=9, Di=3, N=4)
    c["conv_w"] = np.zeros((2, 3, 3))
    c["conv_w"][:, :, 1] = 1.0
    c["conv_b"] = np.zeros((2, 3))
    x = c["x"]
    u = x / (1 + np.exp(-x))
    sg = 1 / (1 + np.exp(-x))
    dsilu = sg * (1 + x * (1 - sg))
    g = orc.vim_bidir_conv_bwd(x, c["conv_w"], c["conv_b"], c["delta"], c["z"], c["B"], c["C"], c["A"], c["D"],
                               c["bias"], c["dout"], bc_dir_stride=c["stride"])
    r = orc.vim_bidir_bwd(u, c["delta"], c["z"], c["B"], c["C"], c["A"], c["D"], c["bias"], c["dout"],
                          bc_dir_stride=c["stride"])
    np.testing.assert_allclose(g["dx"], r["du"] * dsilu, rtol=1e-11, atol=1e-13)
    for k in ("ddelta", "dz", "dB", "dC", "dA", "dD", "dbias"):
        np.testing.assert_allclose(g[k], r[k], rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(g["dconv_b"].sum(axis=0), (r["du"] * dsilu).sum(axis=(0, 1)), rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(g["dconv_w"][:, :, 1].sum(axis=0), (r["du"] * dsilu * x).sum(axis=(0, 1)),
                               rtol=1e-11, atol=1e-13)


def pin_block_bwd_finite_differences(orc):
    """Every derivative of the block scan with its projections (x, both pathways'
    taps and biases, x_proj's Wx, dt_proj's Wdt and bias, A, D, z) against central
    finite differences of the forward oracle's loss sum(dout * y) (page "Vision Mamba
    Guide": the SSM module derives B, C and Delta from its input by x_proj and dt_proj,
    section "The Selective State Space (S6) Mechanism"; the pathways' "1D Conv -> SiLU",
    section "2. The Bidirectional Mamba Block"), with and without the convolution front."""
    for seed, conv in ((151, True), (152, False)):
        rng = _rng(seed)
        b, L, Di, N = 1, 5, 3, 2
        c = dict(x=rng.normal(size=(b, L, Di)), Wx=rng.normal(size=(2, Di, 2 * N + 1)) * 0.6,
                 Wdt=rng.normal(size=(2, Di)) * 0.8, A=-rng.uniform(0.2, 2.0, size=(2, Di, N)),
                 D=rng.normal(size=(2, Di)), bias=rng.normal(size=(2, Di)) * 0.5, z=rng.normal(size=(b, L, Di)),
                 conv_w=rng.normal(size=(2, Di, 3)) * 0.7 if conv else None,
                 conv_b=rng.normal(size=(2, Di)) * 0.5 if conv else None)
        dout = rng.normal(size=(b, L, Di))

        def loss(**over):
            d = {**c, **over}
            y = orc.vim_block_scan(d["x"], d["Wx"], d["Wdt"], d["A"], d["D"], d["bias"], d["z"],
                                   conv_w=d["conv_w"], conv_b=d["conv_b"])
            return float(np.sum(dout * y))

        g = orc.vim_block_scan_bwd(c["x"], c["Wx"], c["Wdt"], c["A"], c["D"], c["bias"], c["z"], dout,
                                   conv_w=c["conv_w"], conv_b=c["conv_b"])
        names = [("x", "dx"), ("Wx", "dWx"), ("Wdt", "dWdt"), ("bias", "dbias"), ("A", "dA"), ("D", "dD"),
                 ("z", "dz")] + ([("conv_w", "dconv_w"), ("conv_b", "dconv_b")] if conv else [])
        for name, key in names:
            arr, eps = c[name], 1e-6
            fd = np.zeros_like(arr)
            for i in np.ndindex(arr.shape):
                up, dn = arr.copy(), arr.copy()
                up[i] += eps
                dn[i] -= eps
                fd[i] = (loss(**{name: up}) - loss(**{name: dn})) / (2 * eps)
            err = np.max(np.abs(fd - g[key])) / np.max(np.abs(fd))
            assert err < 1e-7, (name, conv, err)


ALL_PINS = [
    pin_delta_zero,
    pin_constant_input_geometric,
    pin_reverse_symmetry,
    pin_brute_force,
    pin_prefix_sum,
    pin_linearity,
    pin_softplus,
    pin_gate_is_silu,
    pin_cross_orders_golden,
    pin_cross_scan_is_transpose_and_flip,
    pin_cross_merge,
    pin_separate_bc,
    pin_conv_front_is_correlation,
    pin_conv_scan_composition,
    pin_zoh_matches_ode,
    pin_zoh_fixed_point_and_limits,
    pin_zoh_reaches_every_entry,
    pin_bwd_finite_differences,
    pin_zoh_bwd_finite_differences,
    pin_bwd_homogeneity,
    pin_xproj_is_matmul,
    pin_cross_bwd_finite_differences,
    pin_block_scan_composition,
    pin_conv_bwd_finite_differences,
    pin_conv_bwd_identity_taps,
    pin_block_bwd_finite_differences,
]
