"""Seeded synthetic inputs for the selective-scan workloads.

This module holds no arithmetic of the scan itself: it only draws random tensors
with the shapes and value distributions of the workloads the pages measure, so that
the CUDA path and the CPU oracle can be fed the same bits.

Token counts follow the page "Vision Mamba Guide: Efficient Bidirectional SSM &
VMamba", section "The Quadratic Bottleneck in Vision Transformers (ViT)" (224, 1024
and 2048 px images at patch 16 give 196, 4,096 and 16,384 patches), plus the class
token that section "1. Patch Tokenization and Position Embedding" prepends.

Recipe (one ``torch.Generator`` on the CPU, seeded ``1000 + index``, drawn in this
order): u, delta_raw (std 0.5), z ~ N(0, 1) over [batch, L, channels]; then B and C
~ N(0, 1) over [batch, L, d_state] (one shared pair for the bidirectional scan, one
pair per direction for the cross-scan); then per direction the Delta bias
log(expm1(s)) with s = exp(U(ln 1e-3, ln 1e-1)) so that softplus(bias) is
log-uniform in [1e-3, 1e-1]; A[d, n] = -(n + 1) (S4D-real); D = 1.  Tensors of a
bf16 workload are rounded to bf16 (round-to-nearest-even) after drawing; A, D and
the bias stay fp32.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    index: int
    name: str
    kind: str            # "vim" (bidirectional) or "vmamba" (four-direction cross-scan)
    dtype: str           # "f32" or "bf16": dtype of u, delta, z, B, C and y
    batch: int
    channels: int        # d_inner (Vim) or C (VMamba)
    d_state: int
    L: int = 0           # tokens (Vim)
    H: int = 0           # grid rows (VMamba)
    W: int = 0           # grid columns (VMamba)

    @property
    def tokens(self) -> int:
        return self.L if self.kind == "vim" else self.H * self.W

    @property
    def directions(self) -> int:
        return 2 if self.kind == "vim" else 4

    @property
    def tok_ch(self) -> int:
        """Token-channels per pass: the unit of the throughput metric."""
        return self.batch * self.tokens * self.channels

    @property
    def seed(self) -> int:
        return 1000 + self.index

    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = [
    Workload(0, "vim_tiny_224px_fp32", "vim", "f32", batch=1, channels=384, d_state=16, L=197),
    Workload(1, "vim_small_224px_bf16", "vim", "bf16", batch=64, channels=768, d_state=16, L=197),
    Workload(2, "vim_tiny_1024px_bf16", "vim", "bf16", batch=8, channels=384, d_state=16, L=4097),
    Workload(3, "vmamba_64x64_bf16", "vmamba", "bf16", batch=16, channels=192, d_state=16, H=64, W=64),
    Workload(4, "vim_tiny_2048px_bf16", "vim", "bf16", batch=4, channels=384, d_state=16, L=16385),
]

BY_NAME = {w.name: w for w in WORKLOADS}


def _normal(g, shape, std=1.0):
    return torch.randn(shape, generator=g, dtype=torch.float32) * std


def make_inputs(w: Workload, seed: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """Draw the inputs of workload ``w`` on the CPU (see the module docstring).

    Returns a dict of CPU tensors:
      u, delta, z : [batch, L, ch] (Vim) or [batch, H, W, ch] (VMamba), dtype of w
      B, C        : [batch, L, N] (Vim) or [4, batch, H*W, N] (VMamba), dtype of w
      A           : [dirs, ch, N] fp32;  D, delta_bias : [dirs, ch] fp32
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed if seed is None else seed)
    dirs, ch, N = w.directions, w.channels, w.d_state
    grid = (w.batch, w.L, ch) if w.kind == "vim" else (w.batch, w.H, w.W, ch)
    u = _normal(g, grid)
    delta = _normal(g, grid, std=0.5)
    z = _normal(g, grid)
    if w.kind == "vim":
        B = _normal(g, (w.batch, w.L, N))
        C = _normal(g, (w.batch, w.L, N))
    else:
        Bs, Cs = [], []
        for _ in range(dirs):
            Bs.append(_normal(g, (w.batch, w.H * w.W, N)))
            Cs.append(_normal(g, (w.batch, w.H * w.W, N)))
        B, C = torch.stack(Bs), torch.stack(Cs)
    lo, hi = math.log(1e-3), math.log(1e-1)
    biases = []
    for _ in range(dirs):
        s = torch.exp(lo + (hi - lo) * torch.rand((ch,), generator=g, dtype=torch.float64))
        biases.append(torch.log(torch.expm1(s)).to(torch.float32))
    delta_bias = torch.stack(biases)
    A = -torch.arange(1, N + 1, dtype=torch.float32).repeat(dirs, ch, 1)
    D = torch.ones((dirs, ch), dtype=torch.float32)
    dt = w.torch_dtype()
    out = dict(u=u, delta=delta, z=z, B=B, C=C)
    out = {k: v.to(dt).contiguous() for k, v in out.items()}
    out.update(A=A.contiguous(), D=D, delta_bias=delta_bias.contiguous())
    return out


def input_bytes(w: Workload) -> int:
    """Bytes of the step's inputs (u, delta, z, B, C and the fp32 parameters)."""
    el = 4 if w.dtype == "f32" else 2
    n_bc = w.batch * w.tokens * w.d_state * (1 if w.kind == "vim" else w.directions)
    params = w.directions * w.channels * (w.d_state + 2) * 4
    return 3 * w.tok_ch * el + 2 * n_bc * el + params


def output_bytes(w: Workload) -> int:
    el = 4 if w.dtype == "f32" else 2
    return w.tok_ch * el
