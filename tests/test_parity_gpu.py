"""Parity of the CUDA path (through the C ABI) with the fp64 CPU oracle.

Both sides get the same seeded input bits (bf16 or fp32; the oracle reads them
exactly in fp64).  The gates are those of tests/gates.py: normwise max_i |y_i - r_i| / max_i |r_i|
within the target's tolerances (1e-5 for fp32 I/O, 2e-2 for bf16 I/O, fp32 state in
both), and every element within rtol |r_i| + 1e-3 rms(r) (rtol 1e-5 fp32, 1e-2
bf16).  Shapes cover several chunks and tiles with ragged tails, channel
counts that leave a partial block of 64, d_state 2..16, general (not S4D-real) A,
the softplus cut at 20, large |z|, empty inputs, and the five full-size workloads
in the launch configuration the benchmark times, and the same over the fused
convolution front.
"""
import os

import numpy as np
import pytest
import torch

import gates
import oracle
from vision_mamba_selective_b200 import workloads as wl

pytestmark = pytest.mark.gpu

TOL = gates.NORM_TOL


@pytest.fixture(scope="module")
def vs():
    from vision_mamba_selective_b200 import vimscan

    return vimscan


def normwise(y, ref):
    return gates.measures(y, ref)["normwise"]


def check(name, y, ref, dtype):
    """Both gates of tests/gates.py: normwise within the target tolerance, every
    element within rtol |r| + 1e-3 rms(r)."""
    return gates.gate(name, y, ref, dtype)["normwise"]


def vim_inputs(batch, L, Di, N, dtype, seed, *, generic_A=False, separate_bc=False, delta_scale=0.5):
    g = torch.Generator().manual_seed(seed)
    r = lambda *s, std=1.0: (torch.randn(s, generator=g) * std)
    u, dr, z = r(batch, L, Di), r(batch, L, Di, std=delta_scale), r(batch, L, Di)
    nb = 2 if separate_bc else 1
    B, C = r(nb, batch, L, N), r(nb, batch, L, N)
    if generic_A:
        A = -(0.05 + 3 * torch.rand((2, Di, N), generator=g))
    else:
        A = -torch.arange(1, N + 1, dtype=torch.float32).repeat(2, Di, 1)
    D = r(2, Di)
    s = torch.exp(np.log(1e-3) + (np.log(1e-1) - np.log(1e-3)) * torch.rand((2, Di), generator=g, dtype=torch.float64))
    bias = torch.log(torch.expm1(s)).float()
    t = lambda x: x.to(dtype).contiguous()
    return dict(u=t(u), delta=t(dr), z=t(z), B=t(B), C=t(C), A=A.contiguous(), D=D.contiguous(),
                bias=bias.contiguous(), stride=batch * L * N if separate_bc else 0)


def run_vim(vs, x, gate=True, zoh=False):
    dev = lambda t: t.cuda()
    y = vs.vim_scan_bidir(dev(x["u"]), dev(x["delta"]), dev(x["z"]) if gate else None,
                          dev(x["B"]), dev(x["C"]), dev(x["A"]), dev(x["D"]), dev(x["bias"]),
                          bc_dir_stride=x["stride"], zoh=zoh)
    torch.cuda.synchronize()
    return y


def ref_vim(x, gate=True, zoh=False):
    return oracle.vim_bidir(x["u"], x["delta"], x["z"] if gate else None, x["B"], x["C"], x["A"],
                            x["D"], x["bias"], bc_dir_stride=x["stride"], zoh=zoh)


VIM_CASES = [
    # batch, L, Di, N, dtype, generic_A, separate_bc, gate
    (1, 1, 8, 16, torch.float32, False, False, True),
    (2, 2, 64, 16, torch.float32, False, False, True),
    (1, 7, 72, 16, torch.bfloat16, False, False, True),
    (3, 16, 64, 8, torch.float32, True, True, True),
    (2, 17, 136, 16, torch.bfloat16, False, True, False),
    (1, 33, 64, 4, torch.float32, False, False, True),
    (2, 197, 200, 16, torch.float32, False, False, True),
    (1, 197, 64, 2, torch.bfloat16, True, False, True),
    (1, 256, 64, 16, torch.float32, False, False, True),      # longest single chunk
    (2, 257, 72, 16, torch.float32, False, False, True),      # 3 chunks, last one 1 token
    (1, 300, 64, 16, torch.float32, True, True, True),        # chunks with general A
    (1, 1000, 128, 16, torch.bfloat16, False, False, True),
    (2, 1111, 64, 8, torch.float32, False, True, True),
    (2, 50, 12, 16, torch.float32, False, False, True),       # fp32: channels a multiple of 4 only
    (1, 400, 36, 16, torch.float32, True, False, True),
]


@pytest.mark.parametrize("case", VIM_CASES, ids=lambda c: f"b{c[0]}_L{c[1]}_D{c[2]}_N{c[3]}_{str(c[4])[6:]}"
                         f"{'_genA' if c[5] else ''}{'_sepBC' if c[6] else ''}{'' if c[7] else '_nogate'}")
def test_vim_small(vs, case):
    batch, L, Di, N, dtype, gen, sep, gate = case
    x = vim_inputs(batch, L, Di, N, dtype, seed=L * 7 + Di, generic_A=gen, separate_bc=sep)
    check(f"vim_{case}", run_vim(vs, x, gate), ref_vim(x, gate), dtype)


@pytest.mark.parametrize("L", [12000, 50000], ids=["G125", "G521"])
def test_vim_long_carry_chains(vs, L):
    # long chains of chunk summaries: 125 and 521 chunks of 96 tokens, folded 16 loads at
    # a time
    x = vim_inputs(1, L, 64, 16, torch.float32, seed=L % 997)
    check(f"vim_long_L{L}", run_vim(vs, x), ref_vim(x), torch.float32)


def test_vim_softplus_cut_and_large_gate(vs):
    x = vim_inputs(2, 40, 64, 16, torch.float32, seed=5)
    x["delta"] = (x["delta"] * 0 + torch.linspace(-30, 30, 40)[None, :, None]).contiguous()
    x["z"] = (x["z"] * 40).contiguous()
    check("vim_extreme", run_vim(vs, x), ref_vim(x), torch.float32)


def test_vim_empty(vs):
    x = vim_inputs(1, 5, 64, 16, torch.float32, seed=1)
    for k in ("u", "delta", "z"):
        x[k] = x[k][:0]
    y = run_vim(vs, x)
    assert y.shape == (0, 5, 64)
    x = vim_inputs(1, 0, 64, 16, torch.bfloat16, seed=1)
    assert run_vim(vs, x).shape == (1, 0, 64)


def test_vim_output_written_once_and_inputs_untouched(vs):
    x = vim_inputs(2, 300, 72, 16, torch.bfloat16, seed=9)
    dev = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in x.items()}
    before = {k: v.clone() for k, v in dev.items() if torch.is_tensor(v)}
    y = torch.full_like(dev["u"], float("nan"))
    vs.vim_scan_bidir(dev["u"], dev["delta"], dev["z"], dev["B"], dev["C"], dev["A"], dev["D"],
                      dev["bias"], y=y)
    torch.cuda.synchronize()
    assert torch.isfinite(y.float()).all()
    for k, v in before.items():
        assert torch.equal(v, dev[k]), k
    check("vim_prefilled", y, ref_vim(x), torch.bfloat16)


def test_vim_deterministic(vs):
    x = vim_inputs(2, 600, 64, 16, torch.float32, seed=3)
    y1, y2 = run_vim(vs, x), run_vim(vs, x)
    assert torch.equal(y1, y2)


def conv_params(Di, seed):
    """Depthwise kernel-3 weights and biases of the two pathways, drawn like a
    default-initialised Conv1d (uniform in +-1/sqrt(3), fan-in 3)."""
    g = torch.Generator().manual_seed(seed)
    k = 1 / np.sqrt(3)
    w = (torch.rand((2, Di, 3), generator=g) * 2 - 1) * k
    b = (torch.rand((2, Di), generator=g) * 2 - 1) * k
    return w.contiguous(), b.contiguous()


def run_vim_conv(vs, x, w, b, gate=True, zoh=False):
    dev = lambda t: t.cuda()
    y = vs.vim_scan_bidir_conv(dev(x["u"]), dev(w), dev(b), dev(x["delta"]), dev(x["z"]) if gate else None,
                               dev(x["B"]), dev(x["C"]), dev(x["A"]), dev(x["D"]), dev(x["bias"]),
                               bc_dir_stride=x["stride"], zoh=zoh)
    torch.cuda.synchronize()
    return y


def ref_vim_conv(x, w, b, gate=True, zoh=False):
    return oracle.vim_bidir_conv(x["u"], w, b, x["delta"], x["z"] if gate else None, x["B"], x["C"], x["A"],
                                 x["D"], x["bias"], bc_dir_stride=x["stride"], zoh=zoh)


CONV_CASES = [
    # batch, L, Di, N, dtype, generic_A, separate_bc, gate
    (1, 1, 8, 16, torch.float32, False, False, True),        # both taps fall in the padding
    (1, 2, 64, 16, torch.float32, False, False, True),
    (2, 17, 72, 16, torch.bfloat16, False, True, True),      # tile edge + 1 token
    (1, 32, 64, 8, torch.float32, True, False, False),       # two whole tiles
    (2, 197, 200, 16, torch.float32, False, False, True),
    (1, 256, 64, 16, torch.bfloat16, False, False, True),    # longest single chunk
    (2, 257, 72, 16, torch.float32, False, True, True),      # chunk edges with 1-token tail
    (1, 300, 64, 4, torch.float32, True, False, True),
    (1, 1000, 136, 16, torch.bfloat16, False, False, True),
    (2, 1111, 64, 16, torch.float32, False, False, True),
    (1, 400, 36, 16, torch.float32, True, True, True),
]


@pytest.mark.parametrize("case", CONV_CASES, ids=lambda c: f"b{c[0]}_L{c[1]}_D{c[2]}_N{c[3]}_{str(c[4])[6:]}"
                         f"{'_genA' if c[5] else ''}{'_sepBC' if c[6] else ''}{'' if c[7] else '_nogate'}")
def test_vim_conv(vs, case):
    """The convolution front fused into the scan: every output against the oracle's
    conv + SiLU followed by the two-direction scan, over chunk and tile edges (the
    taps read one token across each)."""
    batch, L, Di, N, dtype, gen, sep, gate = case
    x = vim_inputs(batch, L, Di, N, dtype, seed=L * 11 + Di, generic_A=gen, separate_bc=sep)
    w, b = conv_params(Di, seed=L + Di)
    check(f"vim_conv_{case}", run_vim_conv(vs, x, w, b, gate), ref_vim_conv(x, w, b, gate), dtype)


def test_vim_conv_identity_taps_is_plain_scan(vs):
    """Taps (0, 1, 0) with a bias that makes SiLU the identity on the inputs' range are
    the plain scan of x + bias: the fused path and vim_scan_bidir on x + bias agree."""
    x = vim_inputs(2, 300, 64, 16, torch.float32, seed=21)
    w = torch.zeros(2, 64, 3)
    w[:, :, 1] = 1
    b = torch.full((2, 64), 40.0)
    y_conv = run_vim_conv(vs, x, w, b)
    x2 = dict(x, u=(x["u"] + 40.0).contiguous())
    y_plain = run_vim(vs, x2)
    err = normwise(y_conv, y_plain.double().cpu().numpy())
    assert err < 1e-6, err


def test_vim_conv_rejects_missing_weights(vs):
    x = vim_inputs(1, 20, 64, 16, torch.float32, seed=2)
    w, b = conv_params(64, seed=2)
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in x.items()}
    with pytest.raises(vs.VimScanError):
        vs.vim_scan_bidir_conv(d["u"], w.cuda(), None, d["delta"], d["z"], d["B"], d["C"], d["A"], d["D"],
                               d["bias"])


def cross_inputs(batch, H, W, Ch, N, dtype, seed, generic_A=False):
    g = torch.Generator().manual_seed(seed)
    r = lambda *s, std=1.0: (torch.randn(s, generator=g) * std)
    u, dr, z = r(batch, H, W, Ch), r(batch, H, W, Ch, std=0.5), r(batch, H, W, Ch)
    B, C = r(4, batch, H * W, N), r(4, batch, H * W, N)
    if generic_A:
        A = -(0.05 + 3 * torch.rand((4, Ch, N), generator=g))
    else:
        A = -torch.arange(1, N + 1, dtype=torch.float32).repeat(4, Ch, 1)
    D = r(4, Ch)
    s = torch.exp(np.log(1e-3) + (np.log(1e-1) - np.log(1e-3)) * torch.rand((4, Ch), generator=g, dtype=torch.float64))
    bias = torch.log(torch.expm1(s)).float()
    t = lambda x: x.to(dtype).contiguous()
    return dict(u=t(u), delta=t(dr), z=t(z), B=t(B), C=t(C), A=A, D=D.contiguous(), bias=bias)


def run_cross(vs, x, gate=True, zoh=False):
    c = lambda t: t.cuda()
    y = vs.vmamba_cross_scan4(c(x["u"]), c(x["delta"]), c(x["z"]) if gate else None, c(x["B"]),
                              c(x["C"]), c(x["A"]), c(x["D"]), c(x["bias"]), zoh=zoh)
    torch.cuda.synchronize()
    return y


def ref_cross(x, gate=True, zoh=False):
    return oracle.cross_scan4(x["u"], x["delta"], x["z"] if gate else None, x["B"], x["C"], x["A"],
                              x["D"], x["bias"], zoh=zoh)


CROSS_CASES = [
    # batch, H, W, C, N, dtype, generic_A, gate
    (1, 1, 1, 8, 16, torch.float32, False, True),
    (2, 3, 5, 64, 16, torch.float32, False, True),
    (1, 5, 3, 72, 8, torch.bfloat16, True, True),
    (2, 16, 16, 64, 16, torch.bfloat16, False, False),
    (1, 7, 40, 64, 16, torch.float32, False, True),     # 280 tokens: several chunks
    (1, 40, 7, 64, 4, torch.float32, True, True),
    (2, 32, 48, 72, 16, torch.bfloat16, False, True),
    (1, 127, 3, 64, 16, torch.float32, False, True),    # tall: a tile spans column ends at odd H
    (1, 2, 300, 64, 16, torch.float32, False, True),    # H = 2: every other token starts a column
]


@pytest.mark.parametrize("case", CROSS_CASES, ids=lambda c: f"b{c[0]}_{c[1]}x{c[2]}_C{c[3]}_N{c[4]}_{str(c[5])[6:]}"
                         f"{'_genA' if c[6] else ''}{'' if c[7] else '_nogate'}")
def test_cross_small(vs, case):
    batch, H, W, Ch, N, dtype, gen, gate = case
    x = cross_inputs(batch, H, W, Ch, N, dtype, seed=H * 100 + W, generic_A=gen)
    check(f"cross_{case}", run_cross(vs, x, gate), ref_cross(x, gate), dtype)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("hw", [(1, 1), (3, 5), (16, 16), (9, 33)])
def test_merge(vs, dtype, hw):
    H, W = hw
    g = torch.Generator().manual_seed(H * W)
    ys = torch.randn((4, 2, H * W, 24), generator=g).to(dtype)
    z = torch.randn((2, H, W, 24), generator=g).to(dtype)
    for zz in (None, z):
        y = vs.cross_merge4(ys.cuda(), None if zz is None else zz.cuda(), H, W)
        torch.cuda.synchronize()
        check(f"merge_{hw}_{zz is not None}", y, oracle.cross_merge4(ys, zz, H, W), dtype)


def test_merge_then_is_cross_scan(vs):
    """The unfused path: four single-direction scans (each run as a pair's forward
    half on its traversal) merged by cross_merge4 equal the fused cross-scan."""
    x = cross_inputs(1, 6, 10, 64, 16, torch.float32, seed=77)
    yfused = run_cross(vs, x)
    H, W = 6, 10
    ys = []
    for k in range(4):
        order = oracle.cross_order(k, H, W)
        seq = lambda t: t.reshape(1, H * W, -1)[:, order].contiguous()
        Bk, Ck = x["B"][k][:, order].contiguous(), x["C"][k][:, order].contiguous()
        # a pair whose backward half sees B = C = 0 and D = 0 contributes nothing
        Bp = torch.stack([Bk, torch.zeros_like(Bk)]).contiguous()
        Cp = torch.stack([Ck, torch.zeros_like(Ck)]).contiguous()
        A = torch.stack([x["A"][k], x["A"][k]]).contiguous()
        D = torch.stack([x["D"][k], torch.zeros_like(x["D"][k])]).contiguous()
        bias = torch.stack([x["bias"][k], x["bias"][k]]).contiguous()
        yk = vs.vim_scan_bidir(seq(x["u"]).cuda(), seq(x["delta"]).cuda(), None, Bp.cuda(), Cp.cuda(),
                               A.cuda(), D.cuda(), bias.cuda(), bc_dir_stride=Bk.numel())
        ys.append(yk)
    ym = vs.cross_merge4(torch.stack(ys).contiguous(), x["z"].cuda(), H, W)
    torch.cuda.synchronize()
    err = normwise(ym, yfused.double().cpu().numpy())
    assert err < 1e-5, err


@pytest.mark.parametrize("w", wl.WORKLOADS, ids=lambda w: w.name)
def test_full_size(vs, w):
    """Every workload at full size, in the launch configuration the benchmark
    times, against the oracle on every output."""
    x = wl.make_inputs(w)
    oracle.set_threads(max(1, len(os.sched_getaffinity(0))))
    dev = {k: v.cuda() for k, v in x.items()}
    if w.kind == "vim":
        y = vs.vim_scan_bidir(dev["u"], dev["delta"], dev["z"], dev["B"], dev["C"], dev["A"], dev["D"],
                              dev["delta_bias"])
        ref = oracle.vim_bidir(x["u"], x["delta"], x["z"], x["B"], x["C"], x["A"], x["D"], x["delta_bias"])
    else:
        y = vs.vmamba_cross_scan4(dev["u"], dev["delta"], dev["z"], dev["B"], dev["C"], dev["A"], dev["D"],
                                  dev["delta_bias"])
        ref = oracle.cross_scan4(x["u"], x["delta"], x["z"], x["B"], x["C"], x["A"], x["D"], x["delta_bias"])
    torch.cuda.synchronize()
    check(f"full_{w.name}", y, ref, w.torch_dtype())


def test_full_size_conv(vs):
    """The fused convolution front at the full size of the 1024 px Vim-Ti workload
    (bf16), against the oracle on every output."""
    w = wl.BY_NAME["vim_tiny_1024px_bf16"]
    x = wl.make_inputs(w)
    cw, cb = conv_params(w.channels, seed=4242)
    oracle.set_threads(max(1, len(os.sched_getaffinity(0))))
    dev = {k: v.cuda() for k, v in x.items()}
    y = vs.vim_scan_bidir_conv(dev["u"], cw.cuda(), cb.cuda(), dev["delta"], dev["z"], dev["B"], dev["C"],
                               dev["A"], dev["D"], dev["delta_bias"])
    torch.cuda.synchronize()
    ref = oracle.vim_bidir_conv(x["u"], cw, cb, x["delta"], x["z"], x["B"], x["C"], x["A"], x["D"],
                                x["delta_bias"])
    check("full_conv_vim_tiny_1024px_bf16", y, ref, w.torch_dtype())


# ---------------------------------------------------------------------------
# exact zero-order hold (VIM_FLAG_ZOH_EXACT)
# ---------------------------------------------------------------------------
ZOH_VIM_CASES = [
    # batch, L, Di, N, dtype, generic_A, separate_bc, delta_scale
    (1, 1, 8, 16, torch.float32, False, False, 0.5),
    (2, 17, 64, 16, torch.float32, False, True, 0.5),
    (1, 33, 72, 8, torch.bfloat16, False, False, 0.5),
    (2, 197, 200, 16, torch.float32, False, False, 3.0),    # Delta A_0 on both sides of -1/2
    (1, 197, 64, 2, torch.bfloat16, True, False, 0.5),
    (2, 257, 72, 16, torch.float32, False, True, 0.5),      # 3 chunks
    (1, 300, 64, 4, torch.float32, True, True, 3.0),        # chunks with general A
    (1, 1000, 128, 16, torch.bfloat16, False, False, 0.5),
    (2, 1111, 64, 8, torch.float32, False, False, 3.0),
    (1, 400, 36, 16, torch.float32, True, False, 0.5),
]


@pytest.mark.parametrize("case", ZOH_VIM_CASES, ids=lambda c: f"b{c[0]}_L{c[1]}_D{c[2]}_N{c[3]}_{str(c[4])[6:]}"
                         f"{'_genA' if c[5] else ''}{'_sepBC' if c[6] else ''}_ds{c[7]}")
def test_vim_zoh(vs, case):
    """The exact zero-order-hold Bbar through the two-direction scan, against the
    oracle's expm1(Delta A) / A * B; delta scale 3 puts Delta A_0 on both sides of the
    kernel's switch between its series and exp - 1."""
    batch, L, Di, N, dtype, gen, sep, ds = case
    x = vim_inputs(batch, L, Di, N, dtype, seed=L * 13 + Di, generic_A=gen, separate_bc=sep, delta_scale=ds)
    check(f"vim_zoh_{case}", run_vim(vs, x, zoh=True), ref_vim(x, zoh=True), dtype)


def test_vim_zoh_differs_from_first_order(vs):
    """The flag reaches the kernels: at Delta near 1 the two forms differ by far more
    than the tolerance, and each side matches its own oracle."""
    x = vim_inputs(1, 300, 64, 16, torch.float32, seed=44, delta_scale=3.0)
    x["delta"] = (x["delta"].abs() + 4.0).contiguous()        # Delta about 4 .. 10
    y_e, y_z = run_vim(vs, x), run_vim(vs, x, zoh=True)
    r_e, r_z = ref_vim(x), ref_vim(x, zoh=True)
    check("vim_zoh_big_delta", y_z, r_z, torch.float32)
    check("vim_euler_big_delta", y_e, r_e, torch.float32)
    assert normwise(y_z, r_e) > 1e-2


def test_vim_zoh_zero_A(vs):
    """A = 0 in one direction (structured, A_0 = 0): Bbar is its limit Delta B there."""
    x = vim_inputs(2, 300, 64, 16, torch.float32, seed=45)
    x["A"] = x["A"].clone()
    x["A"][1] = 0.0
    check("vim_zoh_zero_A", run_vim(vs, x, zoh=True), ref_vim(x, zoh=True), torch.float32)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_vim_conv_zoh(vs, dtype):
    x = vim_inputs(2, 300, 72, 16, dtype, seed=46, separate_bc=True)
    w, b = conv_params(72, seed=46)
    check(f"vim_conv_zoh_{dtype}", run_vim_conv(vs, x, w, b, zoh=True), ref_vim_conv(x, w, b, zoh=True), dtype)


ZOH_CROSS_CASES = [
    # batch, H, W, C, N, dtype, generic_A
    (1, 3, 5, 64, 16, torch.float32, False),
    (1, 5, 3, 72, 8, torch.bfloat16, True),
    (1, 7, 40, 64, 16, torch.float32, False),
    (2, 32, 48, 72, 16, torch.bfloat16, False),
]


@pytest.mark.parametrize("case", ZOH_CROSS_CASES, ids=lambda c: f"b{c[0]}_{c[1]}x{c[2]}_C{c[3]}_N{c[4]}_"
                         f"{str(c[5])[6:]}{'_genA' if c[6] else ''}")
def test_cross_zoh(vs, case):
    batch, H, W, Ch, N, dtype, gen = case
    x = cross_inputs(batch, H, W, Ch, N, dtype, seed=H * 31 + W, generic_A=gen)
    check(f"cross_zoh_{case}", run_cross(vs, x, zoh=True), ref_cross(x, zoh=True), dtype)


@pytest.mark.parametrize("name", ["vim_tiny_1024px_bf16", "vmamba_64x64_bf16"])
def test_full_size_zoh(vs, name):
    """The exact hold at full size, in the benchmark's launch configuration."""
    w = wl.BY_NAME[name]
    x = wl.make_inputs(w)
    oracle.set_threads(max(1, len(os.sched_getaffinity(0))))
    dev = {k: v.cuda() for k, v in x.items()}
    args = [dev[k] for k in ("u", "delta", "z", "B", "C", "A", "D", "delta_bias")]
    refargs = [x[k] for k in ("u", "delta", "z", "B", "C", "A", "D", "delta_bias")]
    if w.kind == "vim":
        y = vs.vim_scan_bidir(*args, zoh=True)
        ref = oracle.vim_bidir(*refargs, zoh=True)
    else:
        y = vs.vmamba_cross_scan4(*args, zoh=True)
        ref = oracle.cross_scan4(*refargs, zoh=True)
    torch.cuda.synchronize()
    check(f"full_zoh_{name}", y, ref, w.torch_dtype())


def test_vim_cuda_graph(vs):
    """The entry points only enqueue work on the given stream, so a call can be captured
    into a CUDA graph and replayed; the replay matches the oracle on new inputs copied
    into the captured buffers (here with PDL-chained kernels: L = 1111, several chunks)."""
    x = vim_inputs(2, 1111, 64, 16, torch.bfloat16, seed=31)
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in x.items()}
    ws = torch.empty(vs.vim_scan_workspace_bytes(0, 2, 1111, 0, 64, 16), dtype=torch.uint8, device="cuda")
    y = torch.empty_like(d["u"])
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):      # first call outside capture (attribute set-up)
        vs.vim_scan_bidir(d["u"], d["delta"], d["z"], d["B"], d["C"], d["A"], d["D"], d["bias"], y=y, workspace=ws)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        vs.vim_scan_bidir(d["u"], d["delta"], d["z"], d["B"], d["C"], d["A"], d["D"], d["bias"], y=y, workspace=ws)
    x2 = vim_inputs(2, 1111, 64, 16, torch.bfloat16, seed=32)
    for k in ("u", "delta", "z", "B", "C"):
        d[k].copy_(x2[k])
    g.replay()
    torch.cuda.synchronize()
    ref_in = dict(x, **{k: x2[k] for k in ("u", "delta", "z", "B", "C")})   # captured parameters stay
    check("vim_graph_replay", y, ref_vim(ref_in), torch.bfloat16)
