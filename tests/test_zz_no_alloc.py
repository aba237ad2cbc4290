"""vim_scan_bidir_noalloc: the bidirectional scan for callers that cannot allocate.

Some callers cannot give the scan a workspace (code that must not call cudaMalloc, for
example inside a capture that may not allocate, or under an allocator that owns all
device memory).  The no-allocation entry point keeps the chunk carries in a buffer
built into the library instead.  Its results must match vim_scan_bidir with a
caller-provided workspace, on consecutive calls that reuse the built-in buffer, and
problems too large for the buffer must be refused without touching the output.

This file is collected last on purpose: if it fails, a run stopping at the first
failure has already run every other test.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vs():
    from vision_mamba_selective_b200 import vimscan

    return vimscan


def make(batch, L, Di, N, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    r = lambda *s, std=1.0: torch.randn(s, generator=g) * std
    x = dict(u=r(batch, L, Di), delta=r(batch, L, Di, std=0.5), z=r(batch, L, Di), B=r(batch, L, N),
             C=r(batch, L, N))
    x = {k: v.to(dtype).cuda().contiguous() for k, v in x.items()}
    s = torch.exp(np.log(1e-3) + (np.log(1e-1) - np.log(1e-3)) * torch.rand((2, Di), generator=g, dtype=torch.float64))
    x["A"] = (-torch.arange(1, N + 1, dtype=torch.float32).repeat(2, Di, 1)).cuda()
    x["D"] = r(2, Di).cuda()
    x["bias"] = torch.log(torch.expm1(s)).float().cuda()
    return x


def normwise(y, ref):
    y, ref = y.double(), ref.double()
    return float((y - ref).abs().max() / ref.abs().max())


def run_both(vs, x):
    args = (x["u"], x["delta"], x["z"], x["B"], x["C"], x["A"], x["D"], x["bias"])
    ref = vs.vim_scan_bidir(*args)
    y = vs.vim_scan_bidir_noalloc(*args, y=torch.full_like(x["u"], float("nan")))
    torch.cuda.synchronize()
    return y, ref


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_matches_workspace_entry_point_on_consecutive_calls(vs, dtype):
    # 1000 tokens span several chunks, so the carries go through the built-in buffer;
    # the second call uses different data, so nothing may leak from the first.  Both
    # entry points run the same kernels in the same order: the outputs are equal bit
    # for bit.
    for call, seed in enumerate((11, 12)):
        x = make(2, 1000, 128, 16, dtype, seed)
        y, ref = run_both(vs, x)
        assert torch.isfinite(y.float()).all(), call
        assert torch.equal(y, ref), (call, normwise(y, ref))


def test_matches_the_oracle(vs):
    import gates
    import oracle

    x = make(1, 700, 64, 16, torch.float32, 21)
    y, _ = run_both(vs, x)
    c = {k: v.cpu() for k, v in x.items()}
    want = oracle.vim_bidir(c["u"], c["delta"], c["z"], c["B"], c["C"], c["A"], c["D"], c["bias"])
    gates.gate("noalloc_vs_oracle", y, want, torch.float32)


def test_single_chunk_needs_no_scratch(vs):
    x = make(3, 197, 64, 16, torch.bfloat16, 5)
    y, ref = run_both(vs, x)
    assert torch.equal(y, ref)


def test_too_large_is_refused(vs):
    # the smallest batch of 16385-token, 256-channel sequences whose carries do not fit
    L, Di, N = 16385, 256, 16
    batch = 1
    while vs.vim_scan_workspace_bytes(0, batch, L, 0, Di, N) <= vs.VIM_NOALLOC_SCRATCH_BYTES:
        batch += 1
    x = make(batch, L, Di, N, torch.bfloat16, 7)
    y = torch.full_like(x["u"], float("nan"))
    with pytest.raises(vs.VimScanError) as e:
        vs.vim_scan_bidir_noalloc(x["u"], x["delta"], x["z"], x["B"], x["C"], x["A"], x["D"], x["bias"], y=y)
    assert e.value.status == vs.VIM_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.isnan(y.float()).all()
