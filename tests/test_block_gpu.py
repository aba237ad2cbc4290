"""Parity of vim_block_scan (x_proj on the tensor cores, dt_proj inside the scan,
optional convolution front; through the C ABI) with the oracle's composition of the
same steps in fp64.

bf16 I/O: tolerance 2e-2 normwise, as for the scan; the elementwise error is recorded
(tests/gates.py) but not gated.  The kernel rounds each pathway's
smoothed input to bf16 before x_proj and B, C to bf16 after it (the scan's input
type); the oracle takes both exactly.
"""
import os

import numpy as np
import pytest
import torch

import gates
import oracle
from vision_mamba_selective_b200 import workloads as wl

pytestmark = pytest.mark.gpu
TOL = 2e-2


@pytest.fixture(scope="module")
def vs():
    from vision_mamba_selective_b200 import vimscan

    return vimscan


def block_inputs(batch, L, Di, N, seed, conv):
    """x, z ~ N(0, 1); Wx ~ N(0, 1/Di) so that B, C and the step input are O(1); dt_proj
    weights ~ N(0, 0.5) and biases log(expm1(s)), s log-uniform in [1e-3, 1e-1], so that
    delta_raw is spread like the scan workloads'; A = -(n+1); D ~ N(0, 1); the
    convolution front drawn like a default Conv1d (uniform in +-1/sqrt(3))."""
    g = torch.Generator().manual_seed(seed)
    r = lambda *s: torch.randn(s, generator=g)
    x = r(batch, L, Di).to(torch.bfloat16)
    z = r(batch, L, Di).to(torch.bfloat16)
    Wx = (r(2, Di, 2 * N + 1) / np.sqrt(Di)).to(torch.bfloat16)
    Wdt = r(2, Di) * 0.5
    s = torch.exp(np.log(1e-3) + (np.log(1e-1) - np.log(1e-3)) * torch.rand((2, Di), generator=g, dtype=torch.float64))
    bias = torch.log(torch.expm1(s)).float()
    A = -torch.arange(1, N + 1, dtype=torch.float32).repeat(2, Di, 1)
    D = r(2, Di)
    cw = cb = None
    if conv:
        k = 1 / np.sqrt(3)
        cw = ((torch.rand((2, Di, 3), generator=g) * 2 - 1) * k).contiguous()
        cb = ((torch.rand((2, Di), generator=g) * 2 - 1) * k).contiguous()
    return dict(x=x, z=z, Wx=Wx.contiguous(), Wdt=Wdt.contiguous(), bias=bias.contiguous(), A=A.contiguous(),
                D=D.contiguous(), cw=cw, cb=cb)


def run(vs, p, gate=True):
    c = lambda t: None if t is None else t.cuda()
    y = vs.vim_block_scan(c(p["x"]), c(p["Wx"]), c(p["Wdt"]), c(p["bias"]), c(p["A"]), c(p["D"]),
                          c(p["z"]) if gate else None, conv_w=c(p["cw"]), conv_b=c(p["cb"]))
    torch.cuda.synchronize()
    return y


def ref(p, gate=True):
    return oracle.vim_block_scan(p["x"], p["Wx"], p["Wdt"], p["A"], p["D"], p["bias"], p["z"] if gate else None,
                                 conv_w=p["cw"], conv_b=p["cb"])


CASES = [
    # batch, L, Di, N, conv, gate
    (1, 1, 16, 16, False, True),
    (2, 33, 64, 16, True, True),
    (1, 197, 72, 8, True, True),       # partial 64-channel slice of the projection
    (2, 300, 128, 16, True, False),
    (1, 500, 64, 4, False, True),
    (2, 257, 200, 2, True, True),
    (3, 65, 64, 16, True, True),        # projection tiles across batch boundaries
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"b{c[0]}_L{c[1]}_D{c[2]}_N{c[3]}"
                         f"{'_conv' if c[4] else ''}{'' if c[5] else '_nogate'}")
def test_block_small(vs, case):
    batch, L, Di, N, conv, gate = case
    p = block_inputs(batch, L, Di, N, seed=L * 5 + Di, conv=conv)
    gates.gate(f"block_{case}", run(vs, p, gate), ref(p, gate), torch.bfloat16, norm_tol=TOL, elementwise=False)


# Sequence ends at every offset within the projection's 16-row groups: the front's
# outer taps meet the zero padding at t = 0 and t = L - 1, so those rows (and rows past
# the data) are formed with masks, all other groups without.  (L 49: a group ends just
# before the last row; L 48: a group ends on it; L 17: both ends in one group; L 100 with
# no front: the unmasked copy of u.)
EDGE_CASES = [
    (2, 49, 64, 16, True),
    (1, 48, 64, 16, True),
    (3, 17, 64, 16, True),
    (2, 161, 128, 16, True),
    (1, 100, 64, 16, False),
]


@pytest.mark.parametrize("case", EDGE_CASES, ids=lambda c: f"b{c[0]}_L{c[1]}_D{c[2]}_N{c[3]}"
                         f"{'_conv' if c[4] else ''}")
def test_block_sequence_ends_per_token(vs, case):
    """Each token's error against the oracle, normwise over its channels with the floor
    sqrt(d_inner) rms(y): a token whose front took a wrong neighbour differs by O(1)
    there, which the gate over the whole output could dilute."""
    batch, L, Di, N, conv = case
    p = block_inputs(batch, L, Di, N, seed=7 * L + Di, conv=conv)
    y, r = gates.as_np(run(vs, p)), gates.as_np(ref(p))
    floor = np.sqrt(Di) * np.sqrt(np.mean(r * r))
    err = np.linalg.norm(y - r, axis=-1) / np.maximum(np.linalg.norm(r, axis=-1), floor)
    worst = np.unravel_index(np.argmax(err), err.shape)
    assert err.max() <= TOL, f"token (b, t) = {worst}: error {err.max():.3e} > {TOL:.0e}"


def test_block_rejects_fp32(vs):
    p = block_inputs(1, 10, 16, 16, seed=1, conv=False)
    with pytest.raises(vs.VimScanError):
        vs.vim_block_scan(p["x"].float().cuda(), p["Wx"].float().cuda(), p["Wdt"].cuda(), p["bias"].cuda(),
                          p["A"].cuda(), p["D"].cuda(), p["z"].float().cuda())


def test_block_full_size(vs):
    """The 1024 px Vim-Ti size (batch 8, L 4097, d_inner 384, d_state 16) with the
    convolution front, against the oracle on every output."""
    w = wl.BY_NAME["vim_tiny_1024px_bf16"]
    p = block_inputs(w.batch, w.L, w.channels, w.d_state, seed=4097, conv=True)
    oracle.set_threads(max(1, len(os.sched_getaffinity(0))))
    gates.gate("block_full_vim_tiny_1024px_bf16", run(vs, p), ref(p), torch.bfloat16, norm_tol=TOL, elementwise=False)


# ---------------------------------------------------------------------------
# the derivative (vim_block_scan_bwd)
# ---------------------------------------------------------------------------
BWD_KEYS = ["dx", "dz", "dWx", "dWdt", "ddt_bias", "dA", "dD", "dconv_w", "dconv_b"]
REF_KEY = {"ddt_bias": "dbias"}


def run_bwd(vs, p, dout, gate=True):
    c = lambda t: None if t is None else t.cuda()
    out = vs.vim_block_scan_bwd(c(p["x"]), c(p["Wx"]), c(p["Wdt"]), c(p["bias"]), c(p["A"]), c(p["D"]),
                                c(p["z"]) if gate else None, c(dout), conv_w=c(p["cw"]), conv_b=c(p["cb"]))
    torch.cuda.synchronize()
    return out


def ref_bwd(p, dout, gate=True):
    return oracle.vim_block_scan_bwd(p["x"], p["Wx"], p["Wdt"], p["A"], p["D"], p["bias"], p["z"] if gate else None,
                                     dout, conv_w=p["cw"], conv_b=p["cb"])


BWD_CASES = [
    # batch, L, Di, N, conv, gate
    (1, 5, 16, 16, True, True),
    (2, 33, 64, 16, True, True),        # 2 chunks of the derivative, the last 1 token
    (1, 197, 72, 8, True, True),        # partial channel slices
    (2, 100, 64, 4, False, True),       # no convolution front
    (1, 300, 128, 16, True, False),
    (3, 65, 64, 16, True, True),        # projection tiles across batch boundaries
    (1, 700, 64, 2, False, False),
]


@pytest.mark.parametrize("case", BWD_CASES, ids=lambda c: f"b{c[0]}_L{c[1]}_D{c[2]}_N{c[3]}"
                         f"{'_conv' if c[4] else ''}{'' if c[5] else '_nogate'}")
def test_block_bwd(vs, case):
    """Every derivative against the oracle's, normwise within the bf16 tolerance: the
    kernel takes B and C rounded to bf16 (as the forward call does); the oracle exactly."""
    batch, L, Di, N, conv, gate = case
    p = block_inputs(batch, L, Di, N, seed=L * 3 + Di, conv=conv)
    g = torch.Generator().manual_seed(L + 1)
    dout = torch.randn((batch, L, Di), generator=g).to(torch.bfloat16)
    got, want = run_bwd(vs, p, dout, gate), ref_bwd(p, dout, gate)
    for k in BWD_KEYS:
        w = want[REF_KEY.get(k, k)]
        if w is None:
            assert got[k] is None, k
            continue
        gates.gate(f"block_bwd_{case}:{k}", got[k], w, torch.bfloat16, norm_tol=TOL, elementwise=False)


def test_block_bwd_deterministic(vs):
    p = block_inputs(2, 300, 64, 16, seed=4, conv=True)
    dout = torch.randn((2, 300, 64), generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    a, b = run_bwd(vs, p, dout), run_bwd(vs, p, dout)
    for k in BWD_KEYS:
        assert torch.equal(a[k], b[k]), k


def test_block_bwd_larger(vs):
    """4097 tokens, batch 2, d_inner 128 with the convolution front, against the oracle."""
    p = block_inputs(2, 4097, 128, 16, seed=44, conv=True)
    dout = torch.randn((2, 4097, 128), generator=torch.Generator().manual_seed(45)).to(torch.bfloat16)
    oracle.set_threads(max(1, len(os.sched_getaffinity(0))))
    got, want = run_bwd(vs, p, dout), ref_bwd(p, dout)
    for k in BWD_KEYS:
        gates.gate(f"block_bwd_4097:{k}", got[k], want[REF_KEY.get(k, k)], torch.bfloat16, norm_tol=TOL,
                   elementwise=False)


def test_block_bwd_exact_projection(vs):
    """Inputs whose projections are exact in bf16 (no convolution front; x in {0, +-1/2},
    Wx with at most four entries of +-1/8 per column), so the kernel's B and C equal the
    oracle's and every fp32 derivative must agree to fp32 accuracy: this isolates the
    chain through dt_proj and x_proj from the bf16 rounding the other cases allow for."""
    batch, L, Di, N = 2, 200, 64, 16
    g = torch.Generator().manual_seed(61)
    p = block_inputs(batch, L, Di, N, seed=61, conv=False)
    p["x"] = (torch.randint(-1, 2, (batch, L, Di), generator=g).float() * 0.5).to(torch.bfloat16)
    Wx = torch.zeros(2, Di, 2 * N + 1)
    for k in range(2):
        for j in range(2 * N + 1):
            rows = torch.randperm(Di, generator=g)[:4]
            Wx[k, rows, j] = (torch.randint(0, 2, (4,), generator=g).float() * 2 - 1) * 0.125
    p["Wx"] = Wx.to(torch.bfloat16).contiguous()
    dout = torch.randn((batch, L, Di), generator=g).to(torch.bfloat16)
    got, want = run_bwd(vs, p, dout), ref_bwd(p, dout)
    for k in BWD_KEYS:
        w = want[REF_KEY.get(k, k)]
        if w is None:
            assert got[k] is None, k
            continue
        if k in ("dx", "dz"):   # bf16 outputs, rounded once
            gates.gate(f"block_bwd_exact:{k}", got[k], w, torch.bfloat16)
        else:
            gates.gate(f"block_bwd_exact:{k}", got[k], w, torch.float32, norm_tol=5e-5, elementwise=False)
