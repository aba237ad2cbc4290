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
