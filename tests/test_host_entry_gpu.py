"""vim_scan_bidir_host: the bidirectional scan with its activations in host memory.

The call cuts the batch into pieces and pipelines each piece's upload, scan and
download over three streams.  For sequences longer than one chunk the scan of a piece
runs the same kernels on the same data as the device entry point, so the result must
equal vim_scan_bidir bit for bit, whatever the piece count (including counts that do
not divide the batch), with pinned or pageable host memory, with a separate backward
B/C copy and without a gate.  Short sequences may take another chunking per piece, so
they are checked against the oracle.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vs():
    from vision_mamba_selective_b200 import vimscan

    return vimscan


def make(batch, L, Di, N, dtype, seed, two_bc=False, gate=True):
    g = torch.Generator().manual_seed(seed)
    r = lambda *s, std=1.0: torch.randn(s, generator=g) * std
    nbc = 2 if two_bc else 1
    x = dict(u=r(batch, L, Di), delta=r(batch, L, Di, std=0.5), z=r(batch, L, Di) if gate else None,
             B=r(nbc * batch, L, N), C=r(nbc * batch, L, N))
    x = {k: (None if v is None else v.to(dtype).contiguous()) for k, v in x.items()}
    s = torch.exp(np.log(1e-3) + (np.log(1e-1) - np.log(1e-3)) * torch.rand((2, Di), generator=g, dtype=torch.float64))
    x["A"] = (-torch.arange(1, N + 1, dtype=torch.float32).repeat(2, Di, 1)).cuda()
    x["D"] = r(2, Di).cuda()
    x["bias"] = torch.log(torch.expm1(s)).float().cuda()
    x["stride"] = batch * L * N if two_bc else 0
    return x


def on_device(vs, x, zoh=False):
    dev = {k: (None if x[k] is None else x[k].cuda()) for k in ("u", "delta", "z", "B", "C")}
    return vs.vim_scan_bidir(dev["u"], dev["delta"], dev["z"], dev["B"], dev["C"], x["A"], x["D"], x["bias"],
                             bc_dir_stride=x["stride"], zoh=zoh).cpu()


def on_host(vs, x, slices, pinned=True, zoh=False):
    h = {k: (None if x[k] is None else (x[k].pin_memory() if pinned else x[k])) for k in ("u", "delta", "z", "B", "C")}
    y = torch.full(x["u"].shape, float("nan"), dtype=x["u"].dtype)
    if pinned:
        y = y.pin_memory()
    out = vs.vim_scan_bidir_host(h["u"], h["delta"], h["z"], h["B"], h["C"], x["A"], x["D"], x["bias"], y=y,
                                 bc_dir_stride=x["stride"], slices=slices, zoh=zoh)
    torch.cuda.current_stream().synchronize()
    assert out is y
    return y


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("slices", [1, 2, 3, 5, 8])
def test_equals_the_device_entry(vs, dtype, slices):
    x = make(5, 1000, 64, 16, dtype, 31)
    y = on_host(vs, x, slices)
    assert torch.isfinite(y.float()).all()
    assert torch.equal(y, on_device(vs, x))


@pytest.mark.parametrize("pinned", [True, False])
def test_two_bc_copies_no_gate_pageable(vs, pinned):
    x = make(4, 700, 128, 16, torch.bfloat16, 32, two_bc=True, gate=False)
    assert torch.equal(on_host(vs, x, 3, pinned=pinned), on_device(vs, x))


def test_exact_hold(vs):
    x = make(3, 600, 64, 16, torch.float32, 33)
    assert torch.equal(on_host(vs, x, 2, zoh=True), on_device(vs, x, zoh=True))


def test_consecutive_calls_reuse_the_streams(vs):
    # the second call's uploads must wait for the first call's downloads (same workspace)
    ws = torch.empty(vs.vim_scan_host_workspace_bytes(4, 900, 64, 16, vs.VIM_BF16, 4, False), dtype=torch.uint8,
                     device="cuda")
    xs = [make(4, 900, 64, 16, torch.bfloat16, 40 + i) for i in range(3)]
    # the pinned copies must outlive the queued copies that read them
    hs = [{k: x[k].pin_memory() for k in ("u", "delta", "z", "B", "C")} for x in xs]
    ys = []
    for x, h in zip(xs, hs):
        ys.append(vs.vim_scan_bidir_host(h["u"], h["delta"], h["z"], h["B"], h["C"], x["A"], x["D"], x["bias"],
                                         slices=4, workspace=ws))
    torch.cuda.current_stream().synchronize()
    for x, y in zip(xs, ys):
        assert torch.equal(y, on_device(vs, x))


def test_short_sequences_against_the_oracle(vs):
    import gates
    import oracle

    x = make(6, 197, 64, 16, torch.float32, 34)
    y = on_host(vs, x, 4)
    want = oracle.vim_bidir(x["u"], x["delta"], x["z"], x["B"], x["C"], x["A"].cpu(), x["D"].cpu(), x["bias"].cpu())
    gates.gate("host_entry_L197", y, want, torch.float32)


def test_refusals_leave_the_output(vs):
    x = make(2, 300, 64, 16, torch.bfloat16, 35)
    y = torch.full(x["u"].shape, float("nan"), dtype=torch.bfloat16)
    with pytest.raises(TypeError):   # device activations belong to vim_scan_bidir
        vs.vim_scan_bidir_host(x["u"].cuda(), x["delta"], x["z"], x["B"], x["C"], x["A"], x["D"], x["bias"], y=y)
    with pytest.raises(ValueError):
        vs.vim_scan_bidir_host(x["u"], x["delta"][:, :200], x["z"], x["B"], x["C"], x["A"], x["D"], x["bias"], y=y)
    with pytest.raises(vs.VimScanError):
        vs.vim_scan_bidir_host(x["u"], x["delta"], x["z"], x["B"], x["C"], x["A"], x["D"], x["bias"], y=y, slices=0)
    assert torch.isnan(y.float()).all()
