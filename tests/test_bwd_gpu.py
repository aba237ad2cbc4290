"""Parity of the scan's derivative (vim_scan_bidir_bwd, through the C ABI) with the
fp64 oracle's reverse-mode derivative (itself pinned against finite differences).

Gates: the per-element derivatives du, d delta_raw and dz take the forward's (those
of tests/gates.py: normwise 1e-5 for fp32 I/O and 2e-2 for bf16 I/O, whose outputs are
rounded to bf16, and every element within rtol |r| + 1e-3 rms(r)); the fp32 sums over
channels (dB, dC) and over tokens (dA, dD, d delta_bias) take normwise 1e-5 on the
small cases and 5e-5 at full size: they add up to batch*L terms of both signs in
fp32, and a cancelling sum's rounding error is relative to its terms, not to the
result (measured at most 1.4e-6 and 4.6e-6).
"""
import os

import numpy as np
import pytest
import torch

import gates
import oracle
from vision_mamba_selective_b200 import workloads as wl

pytestmark = pytest.mark.gpu

SUM_TOL = 1e-5        # sums on the small cases (measured: at most 1.4e-6)
SUM_TOL_FULL = 5e-5   # sums over the full-size workloads (measured: at most 4.6e-6)
KEYS = [("du", "du"), ("ddelta", "ddelta"), ("dz", "dz"), ("dB", "dB"), ("dC", "dC"), ("dA", "dA"),
        ("dD", "dD"), ("ddelta_bias", "dbias")]


@pytest.fixture(scope="module")
def vs():
    from vision_mamba_selective_b200 import vimscan

    return vimscan


def inputs(batch, L, Di, N, dtype, seed, *, separate_bc=False, generic_A=False):
    g = torch.Generator().manual_seed(seed)
    r = lambda *s, std=1.0: torch.randn(s, generator=g) * std
    u, dr, z, dout = r(batch, L, Di), r(batch, L, Di, std=0.5), r(batch, L, Di), r(batch, L, Di)
    nb = 2 if separate_bc else 1
    B, C = r(nb, batch, L, N), r(nb, batch, L, N)
    if not separate_bc:
        B, C = B[0], C[0]
    if generic_A:
        A = -(0.05 + 3 * torch.rand((2, Di, N), generator=g))
    else:
        A = -torch.arange(1, N + 1, dtype=torch.float32).repeat(2, Di, 1)
    D = r(2, Di)
    s = torch.exp(np.log(1e-3) + (np.log(1e-1) - np.log(1e-3)) * torch.rand((2, Di), generator=g, dtype=torch.float64))
    bias = torch.log(torch.expm1(s)).float()
    t = lambda x: x.to(dtype).contiguous()
    return dict(u=t(u), delta=t(dr), z=t(z), dout=t(dout), B=t(B), C=t(C), A=A.contiguous(), D=D.contiguous(),
                bias=bias.contiguous(), stride=batch * L * N if separate_bc else 0)


def run(vs, x, gate=True):
    c = lambda k: x[k].cuda()
    out = vs.vim_scan_bidir_bwd(c("u"), c("delta"), c("z") if gate else None, c("B"), c("C"), c("A"), c("D"),
                                c("bias"), c("dout"), bc_dir_stride=x["stride"])
    torch.cuda.synchronize()
    return out


def ref(x, gate=True):
    return oracle.vim_bidir_bwd(x["u"], x["delta"], x["z"] if gate else None, x["B"], x["C"], x["A"], x["D"],
                                x["bias"], x["dout"], bc_dir_stride=x["stride"])


def check_all(name, got, want, dtype, sum_tol=SUM_TOL):
    """Per-element derivatives (du, d delta_raw, dz): both gates of tests/gates.py.
    Sums over channels or tokens (dB, dC, dA, dD, d delta_bias): normwise within
    sum_tol."""
    errs = {}
    for k_got, k_ref in KEYS:
        if want[k_ref] is None:
            assert got[k_got] is None
            continue
        g = got[k_got]
        if k_got in ("du", "ddelta", "dz"):
            m = gates.gate(f"{name}:{k_got}", g, want[k_ref], dtype)
        else:
            m = gates.gate(f"{name}:{k_got}", g, want[k_ref], dtype, norm_tol=sum_tol, elementwise=False)
        errs[k_got] = m["normwise"]
    return errs


CASES = [
    # batch, L, Di, N, dtype, separate_bc, generic_A, gate
    (1, 1, 16, 16, torch.float32, False, False, True),
    (1, 5, 16, 4, torch.float32, True, False, True),
    (2, 31, 24, 16, torch.float32, False, False, True),      # partial channel block
    (1, 32, 16, 8, torch.float32, False, True, True),        # one whole chunk
    (2, 33, 64, 16, torch.float32, True, False, True),       # 2 chunks, the last 1 token
    (1, 100, 40, 2, torch.float32, False, False, False),
    (2, 197, 64, 16, torch.bfloat16, False, False, True),
    (1, 300, 72, 8, torch.bfloat16, True, True, True),
    (2, 300, 200, 16, torch.float32, False, False, True),
    (1, 1000, 64, 16, torch.float32, True, False, True),
    (1, 777, 48, 4, torch.bfloat16, False, True, False),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"b{c[0]}_L{c[1]}_D{c[2]}_N{c[3]}_{str(c[4])[6:]}"
                         f"{'_sepBC' if c[5] else ''}{'_genA' if c[6] else ''}{'' if c[7] else '_nogate'}")
def test_bwd_small(vs, case):
    batch, L, Di, N, dtype, sep, gen, gate = case
    x = inputs(batch, L, Di, N, dtype, seed=L * 3 + Di, separate_bc=sep, generic_A=gen)
    check_all(f"bwd_{case}", run(vs, x, gate), ref(x, gate), dtype)


def test_bwd_long_carry_chains(vs):
    # 17000 tokens are 532 chunks of 32, for both folds (the forward state and the adjoint)
    x = inputs(1, 17000, 32, 16, torch.float32, seed=17)
    check_all("bwd_long_L17000", run(vs, x), ref(x), torch.float32, sum_tol=SUM_TOL_FULL)


def offset_copy(t):
    """A copy of t one element past the start of a device allocation, so that its address
    is not a multiple of 8 bytes (bf16) or 16 bytes (fp32)."""
    flat = torch.empty(t.numel() + 1, dtype=t.dtype, device="cuda")
    v = flat[1:].view(t.shape)
    v.copy_(t)
    return v


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["fp32", "bf16"])
def test_bwd_unaligned(vs, dtype):
    """dout, z, B, C and the per-element outputs at addresses that rule out the kernels'
    vector loads and stores (the entry point asks only for element alignment of these):
    the element-wise paths give the same derivatives.  Three 32-token chunks, so the
    summary kernels run too."""
    batch, L, Di, N = 2, 70, 32, 16
    x = inputs(batch, L, Di, N, dtype, seed=70)
    c = lambda k: x[k].cuda()
    u = c("u")
    f32 = lambda *s: torch.zeros(s, dtype=torch.float32, device="cuda")
    out = dict(du=offset_copy(torch.zeros_like(u)), ddelta=offset_copy(torch.zeros_like(u)),
               dz=offset_copy(torch.zeros_like(u)), dB=f32(batch, L, N), dC=f32(batch, L, N), dA=f32(2, Di, N),
               dD=f32(2, Di), ddelta_bias=f32(2, Di))
    got = vs.vim_scan_bidir_bwd(u, c("delta"), offset_copy(c("z")), offset_copy(c("B")), offset_copy(c("C")),
                                c("A"), c("D"), c("bias"), offset_copy(c("dout")), out=out)
    torch.cuda.synchronize()
    check_all(f"bwd_unaligned_{dtype}", got, ref(x), dtype)


def test_bwd_deterministic(vs):
    x = inputs(2, 500, 64, 16, torch.float32, seed=8)
    a, b = run(vs, x), run(vs, x)
    for k, _ in KEYS:
        assert torch.equal(a[k], b[k]), k


def test_bwd_full_size(vs):
    """The 1024 px Vim-Ti workload (bf16, batch 8, L 4097, d_inner 384) against the
    oracle on every output, with dout drawn like the inputs."""
    w = wl.BY_NAME["vim_tiny_1024px_bf16"]
    x = wl.make_inputs(w)
    g = torch.Generator().manual_seed(777)
    dout = torch.randn(x["u"].shape, generator=g).to(x["u"].dtype)
    oracle.set_threads(max(1, len(os.sched_getaffinity(0))))
    d = {k: v.cuda() for k, v in x.items()}
    got = vs.vim_scan_bidir_bwd(d["u"], d["delta"], d["z"], d["B"], d["C"], d["A"], d["D"], d["delta_bias"],
                                dout.cuda())
    torch.cuda.synchronize()
    want = oracle.vim_bidir_bwd(x["u"], x["delta"], x["z"], x["B"], x["C"], x["A"], x["D"], x["delta_bias"], dout)
    check_all("bwd_full", got, want, torch.bfloat16, sum_tol=SUM_TOL_FULL)


# ---------------------------------------------------------------------------
# the exact zero-order hold (vim_scan_bidir_bwd_ex with VIM_FLAG_ZOH_EXACT)
# ---------------------------------------------------------------------------
ZOH_CASES = [
    # batch, L, Di, N, dtype, separate_bc, generic_A
    (1, 5, 16, 16, torch.float32, False, False),
    (2, 70, 32, 16, torch.float32, True, True),          # 3 chunks, general A
    (1, 33, 16, 8, torch.float32, False, False),          # 2 chunks, the last 1 token
    (2, 100, 24, 4, torch.float32, False, True),
    (1, 300, 64, 16, torch.bfloat16, False, False),
    (1, 97, 40, 2, torch.bfloat16, True, True),
]


def run_zoh(vs, x):
    c = lambda k: x[k].cuda()
    out = vs.vim_scan_bidir_bwd(c("u"), c("delta"), c("z"), c("B"), c("C"), c("A"), c("D"), c("bias"), c("dout"),
                                bc_dir_stride=x["stride"], zoh=True)
    torch.cuda.synchronize()
    return out


def ref_zoh(x):
    return oracle.vim_bidir_bwd(x["u"], x["delta"], x["z"], x["B"], x["C"], x["A"], x["D"], x["bias"], x["dout"],
                                bc_dir_stride=x["stride"], zoh=True)


@pytest.mark.parametrize("case", ZOH_CASES, ids=lambda c: f"b{c[0]}_L{c[1]}_D{c[2]}_N{c[3]}_{str(c[4])[6:]}"
                         f"{'_sepBC' if c[5] else ''}{'_genA' if c[6] else ''}")
def test_bwd_zoh(vs, case):
    """The exact hold's derivative against the oracle's (pinned by finite differences);
    Delta A_n spans both sides of the kernels' series/closed-form switch at 1/2."""
    batch, L, Di, N, dtype, sep, gen = case
    x = inputs(batch, L, Di, N, dtype, seed=L * 7 + Di, separate_bc=sep, generic_A=gen)
    check_all(f"bwd_zoh_{case}", run_zoh(vs, x), ref_zoh(x), dtype)


def test_bwd_zoh_a_zero(vs):
    """A_n = 0 for some states: the hold's gain is its limit Delta and its A-derivative
    Delta^2 / 2."""
    x = inputs(1, 50, 16, 16, torch.float32, seed=50, generic_A=True)
    x["A"] = x["A"].clone()
    x["A"][0, 3, :] = 0.0
    x["A"][1, 5, 7] = 0.0
    check_all("bwd_zoh_a_zero", run_zoh(vs, x), ref_zoh(x), torch.float32)


def test_bwd_zoh_first_order_unchanged(vs):
    """Without the flag the _ex entry point is the first-order derivative, bit for bit."""
    x = inputs(2, 70, 32, 16, torch.float32, seed=71)
    c = lambda k: x[k].cuda()
    a = vs.vim_scan_bidir_bwd(c("u"), c("delta"), c("z"), c("B"), c("C"), c("A"), c("D"), c("bias"), c("dout"))
    b = run(vs, x)
    for k, _ in KEYS:
        assert torch.equal(a[k], b[k]), k


def test_bwd_zoh_full_size(vs):
    """The 1024 px Vim-Ti workload with the exact hold, against the oracle on every
    output."""
    w = wl.BY_NAME["vim_tiny_1024px_bf16"]
    x = wl.make_inputs(w)
    g = torch.Generator().manual_seed(778)
    dout = torch.randn(x["u"].shape, generator=g).to(x["u"].dtype)
    oracle.set_threads(max(1, len(os.sched_getaffinity(0))))
    d = {k: v.cuda() for k, v in x.items()}
    got = vs.vim_scan_bidir_bwd(d["u"], d["delta"], d["z"], d["B"], d["C"], d["A"], d["D"], d["delta_bias"],
                                dout.cuda(), zoh=True)
    torch.cuda.synchronize()
    want = oracle.vim_bidir_bwd(x["u"], x["delta"], x["z"], x["B"], x["C"], x["A"], x["D"], x["delta_bias"], dout,
                                zoh=True)
    check_all("bwd_zoh_full", got, want, torch.bfloat16, sum_tol=SUM_TOL_FULL)


# ---------------------------------------------------------------------------
# the four-direction cross-scan
# ---------------------------------------------------------------------------
def cross_inputs(batch, H, W, Ch, N, dtype, seed, generic_A=False):
    g = torch.Generator().manual_seed(seed)
    r = lambda *s, std=1.0: torch.randn(s, generator=g) * std
    u, dr, z, dout = r(batch, H, W, Ch), r(batch, H, W, Ch, std=0.5), r(batch, H, W, Ch), r(batch, H, W, Ch)
    B, C = r(4, batch, H * W, N), r(4, batch, H * W, N)
    if generic_A:
        A = -(0.05 + 3 * torch.rand((4, Ch, N), generator=g))
    else:
        A = -torch.arange(1, N + 1, dtype=torch.float32).repeat(4, Ch, 1)
    D = r(4, Ch)
    s = torch.exp(np.log(1e-3) + (np.log(1e-1) - np.log(1e-3)) * torch.rand((4, Ch), generator=g, dtype=torch.float64))
    bias = torch.log(torch.expm1(s)).float()
    t = lambda x: x.to(dtype).contiguous()
    return dict(u=t(u), delta=t(dr), z=t(z), dout=t(dout), B=t(B), C=t(C), A=A.contiguous(), D=D.contiguous(),
                bias=bias.contiguous())


CROSS_CASES = [
    # batch, H, W, C, N, dtype, generic_A, gate
    (1, 1, 1, 16, 16, torch.float32, False, True),
    (1, 3, 5, 16, 16, torch.float32, False, True),
    (2, 5, 3, 24, 8, torch.float32, True, True),
    (1, 7, 40, 64, 16, torch.float32, False, True),     # 280 tokens: several 32-token chunks
    (1, 40, 7, 32, 4, torch.float32, True, False),
    (2, 16, 16, 64, 16, torch.bfloat16, False, True),
    (1, 127, 3, 32, 16, torch.float32, False, True),    # tall grid: chunks span column ends at odd H
]


@pytest.mark.parametrize("case", CROSS_CASES, ids=lambda c: f"b{c[0]}_{c[1]}x{c[2]}_C{c[3]}_N{c[4]}_"
                         f"{str(c[5])[6:]}{'_genA' if c[6] else ''}{'' if c[7] else '_nogate'}")
def test_cross_bwd_small(vs, case):
    batch, H, W, Ch, N, dtype, gen, gate = case
    x = cross_inputs(batch, H, W, Ch, N, dtype, seed=H * 17 + W, generic_A=gen)
    c = lambda k: x[k].cuda()
    got = vs.vmamba_cross_scan4_bwd(c("u"), c("delta"), c("z") if gate else None, c("B"), c("C"), c("A"), c("D"),
                                    c("bias"), c("dout"))
    torch.cuda.synchronize()
    want = oracle.cross_scan4_bwd(x["u"], x["delta"], x["z"] if gate else None, x["B"], x["C"], x["A"], x["D"],
                                  x["bias"], x["dout"])
    check_all(f"cross_bwd_{case}", got, want, dtype)


def test_cross_bwd_full_size(vs):
    """The 64 x 64 VMamba workload (bf16, batch 16, 192 channels) against the oracle."""
    w = wl.BY_NAME["vmamba_64x64_bf16"]
    x = wl.make_inputs(w)
    g = torch.Generator().manual_seed(778)
    dout = torch.randn(x["u"].shape, generator=g).to(x["u"].dtype)
    oracle.set_threads(max(1, len(os.sched_getaffinity(0))))
    d = {k: v.cuda() for k, v in x.items()}
    got = vs.vmamba_cross_scan4_bwd(d["u"], d["delta"], d["z"], d["B"], d["C"], d["A"], d["D"], d["delta_bias"],
                                    dout.cuda())
    torch.cuda.synchronize()
    want = oracle.cross_scan4_bwd(x["u"], x["delta"], x["z"], x["B"], x["C"], x["A"], x["D"], x["delta_bias"], dout)
    check_all("cross_bwd_full", got, want, torch.bfloat16, sum_tol=SUM_TOL_FULL)


CROSS_ZOH_CASES = [
    # batch, H, W, C, N, dtype, generic_A
    (1, 3, 5, 16, 16, torch.float32, False),
    (2, 5, 3, 24, 8, torch.float32, True),
    (1, 7, 40, 64, 16, torch.float32, False),     # several 32-token chunks in both orders
    (2, 16, 16, 64, 16, torch.bfloat16, False),
]


@pytest.mark.parametrize("case", CROSS_ZOH_CASES, ids=lambda c: f"b{c[0]}_{c[1]}x{c[2]}_C{c[3]}_N{c[4]}_"
                         f"{str(c[5])[6:]}{'_genA' if c[6] else ''}")
def test_cross_bwd_zoh(vs, case):
    """The cross-scan's derivative with the exact hold (vmamba_cross_scan4_bwd_ex)
    against the oracle's."""
    batch, H, W, Ch, N, dtype, gen = case
    x = cross_inputs(batch, H, W, Ch, N, dtype, seed=H * 19 + W, generic_A=gen)
    c = lambda k: x[k].cuda()
    got = vs.vmamba_cross_scan4_bwd(c("u"), c("delta"), c("z"), c("B"), c("C"), c("A"), c("D"), c("bias"),
                                    c("dout"), zoh=True)
    torch.cuda.synchronize()
    want = oracle.cross_scan4_bwd(x["u"], x["delta"], x["z"], x["B"], x["C"], x["A"], x["D"], x["bias"], x["dout"],
                                  zoh=True)
    check_all(f"cross_bwd_zoh_{case}", got, want, dtype)


# ---------------------------------------------------------------------------
# the scan with its convolution front (vim_scan_bidir_conv_bwd)
# ---------------------------------------------------------------------------
CONV_KEYS = [("dx", "dx"), ("ddelta", "ddelta"), ("dz", "dz"), ("dconv_w", "dconv_w"), ("dconv_b", "dconv_b"),
             ("dB", "dB"), ("dC", "dC"), ("dA", "dA"), ("dD", "dD"), ("ddelta_bias", "dbias")]


def conv_inputs(batch, L, Di, N, dtype, seed, separate_bc=False, generic_A=False):
    x = inputs(batch, L, Di, N, dtype, seed, separate_bc=separate_bc, generic_A=generic_A)
    x["x"] = x.pop("u")
    g = torch.Generator().manual_seed(seed + 1)
    k = 1.0 / np.sqrt(3.0)   # the kernel-3 depthwise convolution's default init bound
    x["conv_w"] = ((torch.rand((2, Di, 3), generator=g) * 2 - 1) * k).contiguous()
    x["conv_b"] = ((torch.rand((2, Di), generator=g) * 2 - 1) * k).contiguous()
    return x


def run_conv(vs, x, gate=True, zoh=False):
    c = lambda k: x[k].cuda()
    out = vs.vim_scan_bidir_conv_bwd(c("x"), c("conv_w"), c("conv_b"), c("delta"), c("z") if gate else None, c("B"),
                                     c("C"), c("A"), c("D"), c("bias"), c("dout"), bc_dir_stride=x["stride"], zoh=zoh)
    torch.cuda.synchronize()
    return out


def ref_conv(x, gate=True, zoh=False):
    return oracle.vim_bidir_conv_bwd(x["x"], x["conv_w"], x["conv_b"], x["delta"], x["z"] if gate else None, x["B"],
                                     x["C"], x["A"], x["D"], x["bias"], x["dout"], bc_dir_stride=x["stride"], zoh=zoh)


def check_conv(name, got, want, dtype, sum_tol=SUM_TOL):
    """dx, d delta_raw, dz: both gates; the sums (the taps' and biases' over tokens,
    dB, dC over channels, dA, dD, d delta_bias): normwise within sum_tol."""
    for k_got, k_ref in CONV_KEYS:
        if want[k_ref] is None:
            assert got[k_got] is None
            continue
        if k_got in ("dx", "ddelta", "dz"):
            gates.gate(f"{name}:{k_got}", got[k_got], want[k_ref], dtype)
        else:
            gates.gate(f"{name}:{k_got}", got[k_got], want[k_ref], dtype, norm_tol=sum_tol, elementwise=False)


CONV_CASES = [
    # batch, L, Di, N, dtype, separate_bc, generic_A, gate, zoh
    (1, 1, 16, 16, torch.float32, False, False, True, False),
    (1, 5, 16, 4, torch.float32, True, False, True, False),
    (2, 33, 64, 16, torch.float32, True, False, True, False),     # 2 chunks, the last 1 token
    (1, 100, 40, 8, torch.float32, False, True, False, False),    # 2 front tiles, a partial channel tile
    (2, 128, 48, 16, torch.float32, False, False, True, False),   # 2 whole front tiles, half a channel tile
    (2, 197, 64, 16, torch.bfloat16, False, False, True, False),
    (1, 300, 72, 16, torch.bfloat16, True, False, True, False),
    (1, 1000, 64, 16, torch.float32, False, False, True, False),
    (2, 70, 32, 16, torch.float32, True, True, True, True),        # exact hold, general A
    (1, 300, 64, 16, torch.bfloat16, False, False, True, True),
]


@pytest.mark.parametrize("case", CONV_CASES, ids=lambda c: f"b{c[0]}_L{c[1]}_D{c[2]}_N{c[3]}_{str(c[4])[6:]}"
                         f"{'_sepBC' if c[5] else ''}{'_genA' if c[6] else ''}{'' if c[7] else '_nogate'}"
                         f"{'_zoh' if c[8] else ''}")
def test_conv_bwd(vs, case):
    batch, L, Di, N, dtype, sep, gen, gate, zoh = case
    x = conv_inputs(batch, L, Di, N, dtype, seed=L * 5 + Di, separate_bc=sep, generic_A=gen)
    check_conv(f"conv_bwd_{case}", run_conv(vs, x, gate, zoh), ref_conv(x, gate, zoh), dtype)


def test_conv_bwd_identity_taps_is_the_scan_derivative(vs):
    # taps (0, 1, 0), zero biases: every derivative but dx and the front's own equals the
    # scan derivative at u = silu(x), and dx = du silu'(x)
    x = conv_inputs(2, 300, 64, 16, torch.float32, seed=9)
    x["conv_w"].zero_()
    x["conv_w"][:, :, 1] = 1.0
    x["conv_b"].zero_()
    got = run_conv(vs, x)
    u = torch.nn.functional.silu(x["x"])
    c = lambda t: t.cuda()
    plain = vs.vim_scan_bidir_bwd(c(u), c(x["delta"]), c(x["z"]), c(x["B"]), c(x["C"]), c(x["A"]), c(x["D"]),
                                  c(x["bias"]), c(x["dout"]))
    torch.cuda.synchronize()
    s = torch.sigmoid(x["x"].double())
    dsilu = (s * (1 + x["x"].double() * (1 - s))).cuda()
    gates.gate("conv_identity:dx", got["dx"], plain["du"].double() * dsilu, torch.float32)
    for k in ("ddelta", "dz"):
        gates.gate(f"conv_identity:{k}", got[k], plain[k], torch.float32)
    for k in ("dB", "dC", "dA", "dD", "ddelta_bias"):
        gates.gate(f"conv_identity:{k}", got[k], plain[k], torch.float32, norm_tol=SUM_TOL, elementwise=False)


def test_conv_bwd_larger(vs):
    """4097 tokens (129 chunks, 65 runs of the front's walk) at bf16, batch 2, against
    the oracle."""
    x = conv_inputs(2, 4097, 128, 16, torch.bfloat16, seed=31)
    oracle.set_threads(max(1, len(os.sched_getaffinity(0))))
    check_conv("conv_bwd_4097", run_conv(vs, x), ref_conv(x), torch.bfloat16, sum_tol=SUM_TOL_FULL)


def test_conv_bwd_deterministic(vs):
    x = conv_inputs(2, 500, 64, 16, torch.float32, seed=12)
    a, b = run_conv(vs, x), run_conv(vs, x)
    for k, _ in CONV_KEYS:
        assert torch.equal(a[k], b[k]), k


# the training pair: the forward scan keeping the derivative's chunk states
# (vim_scan_bidir(ckpt=...)) and the derivative that takes them
CKPT_CASES = [
    # batch, L, Di, N, dtype, separate_bc, generic_A, gate, zoh
    (1, 1, 16, 16, torch.float32, False, False, True, False),
    (2, 31, 16, 4, torch.float32, True, False, True, False),       # one partial chunk
    (1, 64, 64, 16, torch.float32, False, True, True, False),      # two whole chunks
    (2, 100, 40, 8, torch.float32, False, False, False, False),    # the forward's 32-token chunks
    (1, 240, 72, 16, torch.bfloat16, False, False, True, False),   # the forward's single chunk (L <= 256)
    (1, 300, 64, 16, torch.float32, True, False, True, False),     # 96-token chunks, a ragged last one
    (2, 1000, 64, 16, torch.bfloat16, False, False, True, False),
    (1, 333, 64, 16, torch.float32, False, True, True, True),      # exact hold, general A
    (1, 500, 64, 16, torch.bfloat16, False, False, True, True),
]


def ckpt_pair(vs, x, gate=True, zoh=False):
    c = lambda k: x[k].cuda()
    batch, L, Di = x["u"].shape
    N = x["B"].shape[-1]
    ck = torch.full(vs.ckpt_shape(batch, L, Di, N), float("nan"), device="cuda")
    y = vs.vim_scan_bidir(c("u"), c("delta"), c("z") if gate else None, c("B"), c("C"), c("A"), c("D"), c("bias"),
                          bc_dir_stride=x["stride"], zoh=zoh, ckpt=ck)
    y_plain = vs.vim_scan_bidir(c("u"), c("delta"), c("z") if gate else None, c("B"), c("C"), c("A"), c("D"),
                                c("bias"), bc_dir_stride=x["stride"], zoh=zoh)
    got = vs.vim_scan_bidir_bwd(c("u"), c("delta"), c("z") if gate else None, c("B"), c("C"), c("A"), c("D"),
                                c("bias"), c("dout"), bc_dir_stride=x["stride"], zoh=zoh, ckpt=ck)
    torch.cuda.synchronize()
    return y, y_plain, ck, got


@pytest.mark.parametrize("case", CKPT_CASES, ids=lambda c: f"b{c[0]}_L{c[1]}_D{c[2]}_N{c[3]}_{str(c[4])[6:]}"
                         f"{'_sepBC' if c[5] else ''}{'_genA' if c[6] else ''}{'' if c[7] else '_nogate'}"
                         f"{'_zoh' if c[8] else ''}")
def test_ckpt_pair(vs, case):
    batch, L, Di, N, dtype, sep, gen, gate, zoh = case
    x = inputs(batch, L, Di, N, dtype, seed=L * 11 + Di, separate_bc=sep, generic_A=gen)
    y, y_plain, ck, got = ckpt_pair(vs, x, gate, zoh)
    # keeping the states changes nothing in y; every entry is written, and the chunk each
    # direction visits first starts from zero
    assert torch.equal(y, y_plain)
    assert torch.isfinite(ck).all()
    assert (ck[:, 0, 0] == 0).all() and (ck[:, -1, 1] == 0).all()
    want = oracle.vim_bidir_bwd(x["u"], x["delta"], x["z"] if gate else None, x["B"], x["C"], x["A"], x["D"],
                                x["bias"], x["dout"], bc_dir_stride=x["stride"], zoh=zoh)
    check_all(f"bwd_ckpt_{case}", got, want, dtype)


def test_ckpt_pair_full_size(vs):
    """The 1024 px Vim-Ti workload: the derivative from the forward's states against the
    oracle, and against the derivative that forms its own."""
    w = wl.BY_NAME["vim_tiny_1024px_bf16"]
    x = wl.make_inputs(w)
    g = torch.Generator().manual_seed(779)
    x["dout"] = torch.randn(x["u"].shape, generator=g).to(x["u"].dtype)
    x["bias"], x["stride"] = x["delta_bias"], 0
    oracle.set_threads(max(1, len(os.sched_getaffinity(0))))
    y, y_plain, ck, got = ckpt_pair(vs, x)
    assert torch.equal(y, y_plain)
    c = lambda k: x[k].cuda()
    own = vs.vim_scan_bidir_bwd(c("u"), c("delta"), c("z"), c("B"), c("C"), c("A"), c("D"), c("bias"), c("dout"))
    torch.cuda.synchronize()
    for k in ("dA", "dD", "ddelta_bias", "dB", "dC"):
        gates.gate(f"bwd_ckpt_vs_own:{k}", got[k], own[k].double(), torch.float32, norm_tol=SUM_TOL_FULL,
                   elementwise=False)
    want = oracle.vim_bidir_bwd(x["u"], x["delta"], x["z"], x["B"], x["C"], x["A"], x["D"], x["bias"], x["dout"])
    check_all("bwd_ckpt_full", got, want, torch.bfloat16, sum_tol=SUM_TOL_FULL)


# the training pair with the convolution front
CONV_CKPT_CASES = [
    # batch, L, Di, N, dtype, gate, zoh
    (1, 5, 16, 4, torch.float32, True, False),
    (2, 100, 40, 8, torch.float32, False, False),   # the forward's 32-token chunks
    (1, 300, 72, 16, torch.bfloat16, True, False),  # 96-token chunks, a ragged last one
    (1, 333, 64, 16, torch.float32, True, True),     # exact hold
]


@pytest.mark.parametrize("case", CONV_CKPT_CASES, ids=lambda c: f"b{c[0]}_L{c[1]}_D{c[2]}_N{c[3]}_"
                         f"{str(c[4])[6:]}{'' if c[5] else '_nogate'}{'_zoh' if c[6] else ''}")
def test_conv_ckpt_pair(vs, case):
    batch, L, Di, N, dtype, gate, zoh = case
    x = conv_inputs(batch, L, Di, N, dtype, seed=L * 13 + Di)
    c = lambda k: x[k].cuda()
    ck = torch.full(vs.ckpt_shape(batch, L, Di, N), float("nan"), device="cuda")
    zz = c("z") if gate else None
    y = vs.vim_scan_bidir_conv(c("x"), c("conv_w"), c("conv_b"), c("delta"), zz, c("B"), c("C"), c("A"), c("D"),
                               c("bias"), zoh=zoh, ckpt=ck)
    y_plain = vs.vim_scan_bidir_conv(c("x"), c("conv_w"), c("conv_b"), c("delta"), zz, c("B"), c("C"), c("A"),
                                     c("D"), c("bias"), zoh=zoh)
    got = vs.vim_scan_bidir_conv_bwd(c("x"), c("conv_w"), c("conv_b"), c("delta"), zz, c("B"), c("C"), c("A"),
                                     c("D"), c("bias"), c("dout"), zoh=zoh, ckpt=ck)
    torch.cuda.synchronize()
    assert torch.equal(y, y_plain)
    assert torch.isfinite(ck).all() and (ck[:, 0, 0] == 0).all() and (ck[:, -1, 1] == 0).all()
    check_conv(f"conv_bwd_ckpt_{case}", got, ref_conv(x, gate, zoh), dtype)


# the training pair of the cross-scan
CROSS_CKPT_CASES = [
    # batch, H, W, C, N, dtype, generic_A, zoh
    (1, 3, 5, 16, 16, torch.float32, False, False),
    (1, 7, 40, 64, 16, torch.float32, True, False),    # several chunks, tiles across column ends
    (2, 16, 16, 64, 16, torch.bfloat16, False, False),
    (1, 20, 17, 32, 8, torch.float32, False, True),    # exact hold
]


@pytest.mark.parametrize("case", CROSS_CKPT_CASES, ids=lambda c: f"b{c[0]}_{c[1]}x{c[2]}_C{c[3]}_N{c[4]}_"
                         f"{str(c[5])[6:]}{'_genA' if c[6] else ''}{'_zoh' if c[7] else ''}")
def test_cross_ckpt_pair(vs, case):
    batch, H, W, Ch, N, dtype, gen, zoh = case
    x = cross_inputs(batch, H, W, Ch, N, dtype, seed=H * 19 + W, generic_A=gen)
    c = lambda k: x[k].cuda()
    ck = torch.full(vs.cross_ckpt_shape(batch, H, W, Ch, N), float("nan"), device="cuda")
    y = vs.vmamba_cross_scan4(c("u"), c("delta"), c("z"), c("B"), c("C"), c("A"), c("D"), c("bias"), zoh=zoh,
                              ckpt=ck)
    y_plain = vs.vmamba_cross_scan4(c("u"), c("delta"), c("z"), c("B"), c("C"), c("A"), c("D"), c("bias"), zoh=zoh)
    got = vs.vmamba_cross_scan4_bwd(c("u"), c("delta"), c("z"), c("B"), c("C"), c("A"), c("D"), c("bias"),
                                    c("dout"), zoh=zoh, ckpt=ck)
    torch.cuda.synchronize()
    assert torch.equal(y, y_plain)
    assert torch.isfinite(ck).all() and (ck[:, :, 0, 0] == 0).all() and (ck[:, :, -1, 1] == 0).all()
    want = oracle.cross_scan4_bwd(x["u"], x["delta"], x["z"], x["B"], x["C"], x["A"], x["D"], x["bias"], x["dout"],
                                  zoh=zoh)
    check_all(f"cross_bwd_ckpt_{case}", got, want, dtype)
