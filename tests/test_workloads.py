"""Seeded synthetic inputs: determinism, shapes and value distributions (CPU)."""
import math

import torch

from vision_mamba_selective_b200 import workloads as wl


def test_table():
    assert [w.index for w in wl.WORKLOADS] == [0, 1, 2, 3, 4]
    assert [w.tokens for w in wl.WORKLOADS] == [197, 197, 4097, 4096, 16385]
    assert wl.WORKLOADS[0].dtype == "f32" and all(w.dtype == "bf16" for w in wl.WORKLOADS[1:])
    assert wl.WORKLOADS[2].tok_ch == 12_585_984


def test_deterministic_and_shaped():
    w = wl.WORKLOADS[0].scaled(L=33, channels=16)
    a, b = wl.make_inputs(w), wl.make_inputs(w)
    for k in a:
        assert torch.equal(a[k], b[k]), k
    assert a["u"].shape == (1, 33, 16) and a["B"].shape == (1, 33, 16)
    assert a["A"].shape == (2, 16, 16) and a["D"].shape == (2, 16)
    assert torch.equal(a["A"][1, 3], -torch.arange(1, 17, dtype=torch.float32))
    v = wl.WORKLOADS[3].scaled(batch=2, H=5, W=7, channels=8)
    c = wl.make_inputs(v)
    assert c["u"].shape == (2, 5, 7, 8) and c["B"].shape == (4, 2, 35, 16)
    assert c["u"].dtype == torch.bfloat16 and c["A"].dtype == torch.float32


def test_distributions():
    w = wl.WORKLOADS[1].scaled(batch=4)
    x = wl.make_inputs(w)
    assert abs(x["u"].float().std().item() - 1.0) < 0.01
    assert abs(x["delta"].float().std().item() - 0.5) < 0.01
    sp = torch.nn.functional.softplus(x["delta_bias"].double())
    assert sp.min().item() >= 1e-3 * (1 - 1e-5) and sp.max().item() <= 1e-1 * (1 + 1e-5)
    lg = torch.log(sp)
    assert abs(lg.mean().item() - 0.5 * (math.log(1e-3) + math.log(1e-1))) < 0.1
    assert torch.all(x["D"] == 1)
    # bf16 rounding happened after drawing: the values are exactly representable
    assert torch.equal(x["u"].float().to(torch.bfloat16).float(), x["u"].float())


def test_byte_counts():
    w = wl.WORKLOADS[2]
    assert wl.output_bytes(w) == 2 * w.tok_ch
    assert wl.input_bytes(w) == 3 * 2 * w.tok_ch + 2 * 2 * 8 * 4097 * 16 + 2 * 384 * 18 * 4
