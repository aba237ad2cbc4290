"""The Python binding refuses tensors the kernels could not address safely, before any
launch: wrong shapes (a short output, a flat or transposed parameter), a short B/C
buffer for the given per-direction stride, tensors on different devices.  Each
refusal leaves the output untouched.
"""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vs():
    from vision_mamba_selective_b200 import vimscan

    return vimscan


def vim_args(batch=2, L=40, Di=64, N=16, dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(3)
    r = lambda *s: torch.randn(s, generator=g)
    d = dict(u=r(batch, L, Di), delta=r(batch, L, Di) * 0.5, z=r(batch, L, Di), B=r(batch, L, N), C=r(batch, L, N))
    d = {k: v.to(dtype).cuda() for k, v in d.items()}
    d["A"] = (-torch.arange(1, N + 1, dtype=torch.float32).repeat(2, Di, 1)).cuda()
    d["D"] = torch.ones(2, Di, device="cuda")
    d["bias"] = torch.full((2, Di), -3.0, device="cuda")
    return d


def call(vs, d, **kw):
    return vs.vim_scan_bidir(d["u"], d["delta"], d["z"], d["B"], d["C"], d["A"], d["D"], d["bias"], **kw)


@pytest.mark.parametrize("key,shape", [
    ("delta", (2, 40, 32)),          # fewer channels than u
    ("z", (2, 39, 64)),              # fewer tokens
    ("B", (2, 39, 16)),              # a short B
    ("C", (2, 40, 8)),               # wrong d_state
    ("A", (2, 16, 64)),              # transposed A
    ("D", (2 * 64,)),                # flat D
    ("bias", (1, 64)),               # one direction only
])
def test_wrong_shapes_are_refused(vs, key, shape):
    d = vim_args()
    d[key] = torch.zeros(shape, dtype=d[key].dtype, device="cuda")
    y = torch.full_like(d["u"], float("nan"))
    with pytest.raises(ValueError):
        call(vs, d, y=y)
    torch.cuda.synchronize()
    assert torch.isnan(y.float()).all()


def test_short_output_is_refused(vs):
    d = vim_args()
    y = torch.full((2, 40, 32), float("nan"), dtype=d["u"].dtype, device="cuda")
    with pytest.raises(ValueError):
        call(vs, d, y=y)


def test_bc_stride_needs_a_second_copy(vs):
    d = vim_args()
    y = torch.full_like(d["u"], float("nan"))
    with pytest.raises(ValueError):
        call(vs, d, y=y, bc_dir_stride=d["B"].numel())   # B holds one copy only
    torch.cuda.synchronize()
    assert torch.isnan(y.float()).all()


def test_cross_scan_shapes(vs):
    batch, H, W, Ch, N = 1, 4, 6, 64, 16
    u = torch.randn(batch, H, W, Ch, device="cuda").to(torch.bfloat16)
    B = torch.randn(4, batch, H * W, N, device="cuda").to(torch.bfloat16)
    A = (-torch.arange(1, N + 1, dtype=torch.float32).repeat(4, Ch, 1)).cuda()
    D = torch.ones(4, Ch, device="cuda")
    bias = torch.full((4, Ch), -3.0, device="cuda")
    y = torch.full_like(u, float("nan"))
    with pytest.raises(ValueError):   # B/C for two directions only
        vs.vmamba_cross_scan4(u, u, u, B[:2].contiguous(), B[:2].contiguous(), A, D, bias, y=y)
    with pytest.raises(ValueError):   # Vim-style parameters
        vs.vmamba_cross_scan4(u, u, u, B, B, A[:2].contiguous(), D[:2].contiguous(), bias[:2].contiguous(), y=y)
    torch.cuda.synchronize()
    assert torch.isnan(y.float()).all()


def test_derivative_output_shapes(vs):
    d = vim_args(dtype=torch.float32)
    dout = torch.randn_like(d["u"])
    good = vs.vim_scan_bidir_bwd(d["u"], d["delta"], d["z"], d["B"], d["C"], d["A"], d["D"], d["bias"], dout)
    bad = dict(good)
    bad["dA"] = torch.zeros(2, 64, device="cuda")
    with pytest.raises(ValueError):
        vs.vim_scan_bidir_bwd(d["u"], d["delta"], d["z"], d["B"], d["C"], d["A"], d["D"], d["bias"], dout, out=bad)


def test_other_device_is_refused(vs):
    if torch.cuda.device_count() < 2:
        pytest.skip("one GPU: the cross-device case needs two")
    d = vim_args()
    d["z"] = d["z"].to("cuda:1")
    with pytest.raises(ValueError):
        call(vs, d)
