"""fp64 CPU oracle of the Vision Mamba / VMamba selective scan.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library never
calls it, and it never calls the CUDA library.

Every function converts its inputs to contiguous float64 arrays (bf16 and fp32
values are represented exactly), runs the plain sequential recurrence of
``oracle.c`` and returns float64 numpy arrays.  The equations followed are those of
the page "Vision Mamba Guide: Efficient Bidirectional SSM & VMamba": sections
"Discretization via Zero-Order Hold (ZOH)", "The Selective State Space (S6)
Mechanism", "2. The Bidirectional Mamba Block", "1. Cross-Scan Traversal
(CS-Traverse)" and "3. Cross-Merge Reversal (CS-Merge)".
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_HERE = os.path.dirname(os.path.abspath(__file__))

_D = ctypes.POINTER(ctypes.c_double)
_I64 = ctypes.POINTER(ctypes.c_int64)


def _f64(x):
    """Contiguous float64 copy of a numpy array or a (CPU or CUDA) torch tensor."""
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor
        import torch

        x = x.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _p(a):
    return None if a is None else a.ctypes.data_as(_D)


class Oracle:
    """ctypes view of one build of ``oracle.c``.

    The module-level functions use the default build next to this file; the test
    suite also loads deliberately broken copies (built in a temporary directory)
    to show that the pins catch a planted mistake.
    """

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        lib.oracle_s6_direction.argtypes = [_D, _D, _D, _D, _D, _D, _D, _I64, _D] + [ctypes.c_int] * 7
        lib.oracle_vim_bidir.argtypes = [_D, _D, _D, _D, _D, ctypes.c_int64, _D, _D, _D, _D] + [ctypes.c_int] * 6
        lib.oracle_cross_scan4.argtypes = [_D] * 9 + [ctypes.c_int] * 7
        lib.oracle_cross_merge4.argtypes = [_D, _D, _D] + [ctypes.c_int] * 4
        lib.oracle_cross_order.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, _I64]
        lib.oracle_conv_silu.argtypes = [_D, _D, _D, _D] + [ctypes.c_int] * 4
        lib.oracle_vim_bidir_conv.argtypes = [_D, _D, _D, _D, _D, _D, _D, ctypes.c_int64, _D, _D, _D, _D] + [ctypes.c_int] * 6
        lib.oracle_s6_direction_bwd.argtypes = [_D] * 7 + [_I64] + [_D] * 8 + [ctypes.c_int] * 6
        lib.oracle_vim_bidir_bwd.argtypes = [_D, _D, _D, _D, _D, ctypes.c_int64] + [_D] * 12 + [ctypes.c_int] * 6
        lib.oracle_cross_scan4_bwd.argtypes = [_D] * 17 + [ctypes.c_int] * 7
        lib.oracle_vim_bidir_conv_bwd.argtypes = [_D] * 7 + [ctypes.c_int64] + [_D] * 14 + [ctypes.c_int] * 6
        lib.oracle_vim_block_scan_bwd.argtypes = [_D] * 19 + [ctypes.c_int] * 4
        lib.oracle_xproj.argtypes = [_D, _D, _D, ctypes.c_int64, ctypes.c_int, ctypes.c_int]
        lib.oracle_set_threads.argtypes = [ctypes.c_int]
        lib.oracle_max_threads.restype = ctypes.c_int
        self.lib = lib
        self.path = path

    def set_threads(self, n: int) -> None:
        """Number of OpenMP threads (parallel over independent sequences only)."""
        self.lib.oracle_set_threads(int(n))

    def max_threads(self) -> int:
        return int(self.lib.oracle_max_threads())

    def cross_order(self, k: int, H: int, W: int) -> np.ndarray:
        """Grid position (p = h*W + w) visited at each step of CS-Traverse scan k+1."""
        out = np.zeros(H * W, dtype=np.int64)
        if self.lib.oracle_cross_order(int(k), int(H), int(W), out.ctypes.data_as(_I64)):
            raise ValueError("bad direction index")
        return out

    def s6_direction(self, u, delta, B, C, A, D, bias, order, *, delta_is_raw=True, zoh=False):
        """One S6 direction (no gate) over tokens visited in ``order``.

        u, delta: [batch, L, Di]; B, C: [batch, L, N] (by position); A: [Di, N];
        D, bias: [Di]; order: [L] permutation.  Returns y [batch, L, Di] with
        y[b, order[t], d] = C_t . h_t + D u_t.  zoh=True takes the exact zero-order-hold
        Bbar = expm1(Delta A) / A * B instead of Delta B.
        """
        u, delta, B, C, A, D, bias = map(_f64, (u, delta, B, C, A, D, bias))
        batch, L, Di = u.shape
        N = B.shape[-1]
        order = np.ascontiguousarray(np.asarray(order, dtype=np.int64))
        assert sorted(order.tolist()) == list(range(L)), "order must be a permutation"
        if bias is None:
            bias = np.zeros(Di)
        y = np.zeros((batch, L, Di))
        rc = self.lib.oracle_s6_direction(_p(u), _p(delta), _p(B), _p(C), _p(A), _p(D), _p(bias),
                                          order.ctypes.data_as(_I64), _p(y),
                                          batch, L, Di, N, int(bool(delta_is_raw)), 0, int(bool(zoh)))
        if rc:
            raise ValueError("oracle_s6_direction: bad sizes")
        return y

    def vim_bidir(self, u, delta, z, B, C, A, D, bias, *, bc_dir_stride=0, delta_is_raw=True, zoh=False):
        """Vim bidirectional scan: (y^f + y^b) * silu(z); z=None gives the ungated sum.

        u, delta, z: [batch, L, Di]; B, C: [batch, L, N] shared by both directions,
        or a larger buffer whose backward copy starts ``bc_dir_stride`` elements in;
        A: [2, Di, N]; D, bias: [2, Di].
        """
        u, delta, z, B, C, A, D, bias = map(_f64, (u, delta, z, B, C, A, D, bias))
        batch, L, Di = u.shape
        N = B.shape[-1]
        if bias is None:
            bias = np.zeros((2, Di))
        y = np.zeros((batch, L, Di))
        rc = self.lib.oracle_vim_bidir(_p(u), _p(delta), _p(z), _p(B), _p(C), int(bc_dir_stride),
                                       _p(A), _p(D), _p(bias), _p(y), batch, L, Di, N,
                                       int(bool(delta_is_raw)), int(bool(zoh)))
        if rc:
            raise ValueError("oracle_vim_bidir: bad sizes")
        return y

    def vim_bidir_bwd(self, u, delta, z, B, C, A, D, bias, dout, *, bc_dir_stride=0, delta_is_raw=True,
                      zoh=False):
        """Derivatives of vim_bidir (first-order Bbar, or the exact hold with zoh) for
        the loss sum(dout * y).

        Returns a dict of fp64 arrays: du, ddelta (w.r.t. the raw delta when
        delta_is_raw), dz (None without a gate), dB and dC shaped like B and C, dA
        [2, Di, N], dD and dbias [2, Di] (dbias zero when not delta_is_raw).
        """
        u, delta, z, B, C, A, D, bias, dout = map(_f64, (u, delta, z, B, C, A, D, bias, dout))
        batch, L, Di = u.shape
        N = B.shape[-1]
        if bias is None:
            bias = np.zeros((2, Di))
        out = dict(du=np.zeros((batch, L, Di)), ddelta=np.zeros((batch, L, Di)),
                   dz=np.zeros((batch, L, Di)) if z is not None else None,
                   dB=np.zeros(B.shape), dC=np.zeros(C.shape), dA=np.zeros((2, Di, N)),
                   dD=np.zeros((2, Di)), dbias=np.zeros((2, Di)))
        rc = self.lib.oracle_vim_bidir_bwd(_p(u), _p(delta), _p(z), _p(B), _p(C), int(bc_dir_stride),
                                           _p(A), _p(D), _p(bias), _p(dout), _p(out["du"]),
                                           _p(out["ddelta"]), _p(out["dz"]), _p(out["dB"]), _p(out["dC"]),
                                           _p(out["dA"]), _p(out["dD"]), _p(out["dbias"]),
                                           batch, L, Di, N, int(bool(delta_is_raw)), int(bool(zoh)))
        if rc:
            raise ValueError("oracle_vim_bidir_bwd: bad sizes")
        return out

    def vim_bidir_conv_bwd(self, x, conv_w, conv_b, delta, z, B, C, A, D, bias, dout, *, bc_dir_stride=0,
                           delta_is_raw=True, zoh=False):
        """Derivatives of vim_bidir_conv for the loss sum(dout * y).

        Returns a dict of fp64 arrays: dx [batch, L, Di], dconv_w [2, Di, 3], dconv_b
        [2, Di], and ddelta, dz (None without a gate), dB, dC, dA, dD, dbias as in
        vim_bidir_bwd.
        """
        x, conv_w, conv_b, delta, z, B, C, A, D, bias, dout = map(
            _f64, (x, conv_w, conv_b, delta, z, B, C, A, D, bias, dout))
        batch, L, Di = x.shape
        N = B.shape[-1]
        if bias is None:
            bias = np.zeros((2, Di))
        out = dict(dx=np.zeros((batch, L, Di)), dconv_w=np.zeros((2, Di, 3)), dconv_b=np.zeros((2, Di)),
                   ddelta=np.zeros((batch, L, Di)), dz=np.zeros((batch, L, Di)) if z is not None else None,
                   dB=np.zeros(B.shape), dC=np.zeros(C.shape), dA=np.zeros((2, Di, N)),
                   dD=np.zeros((2, Di)), dbias=np.zeros((2, Di)))
        rc = self.lib.oracle_vim_bidir_conv_bwd(
            _p(x), _p(conv_w), _p(conv_b), _p(delta), _p(z), _p(B), _p(C), int(bc_dir_stride), _p(A), _p(D),
            _p(bias), _p(dout), _p(out["dx"]), _p(out["dconv_w"]), _p(out["dconv_b"]), _p(out["ddelta"]),
            _p(out["dz"]), _p(out["dB"]), _p(out["dC"]), _p(out["dA"]), _p(out["dD"]), _p(out["dbias"]),
            batch, L, Di, N, int(bool(delta_is_raw)), int(bool(zoh)))
        if rc:
            raise ValueError("oracle_vim_bidir_conv_bwd: bad sizes")
        return out

    def cross_scan4_bwd(self, u, delta, z, B, C, A, D, bias, dout, *, delta_is_raw=True, zoh=False):
        """Derivatives of cross_scan4 (first-order Bbar, or the exact hold with zoh) for
        the loss sum(dout * y).

        u, delta, z, dout: [batch, H, W, Ci]; B, C: [4, batch, H*W, N]; A [4, Ci, N];
        D, bias [4, Ci].  Returns a dict of fp64 arrays shaped like the inputs: du,
        ddelta, dz (None without a gate), dB, dC, dA, dD, dbias.
        """
        u, delta, z, B, C, A, D, bias, dout = map(_f64, (u, delta, z, B, C, A, D, bias, dout))
        batch, H, W, Ci = u.shape
        N = B.shape[-1]
        if bias is None:
            bias = np.zeros((4, Ci))
        out = dict(du=np.zeros(u.shape), ddelta=np.zeros(u.shape), dz=np.zeros(u.shape) if z is not None else None,
                   dB=np.zeros(B.shape), dC=np.zeros(C.shape), dA=np.zeros((4, Ci, N)), dD=np.zeros((4, Ci)),
                   dbias=np.zeros((4, Ci)))
        rc = self.lib.oracle_cross_scan4_bwd(_p(u), _p(delta), _p(z), _p(B), _p(C), _p(A), _p(D), _p(bias), _p(dout),
                                             _p(out["du"]), _p(out["ddelta"]), _p(out["dz"]), _p(out["dB"]),
                                             _p(out["dC"]), _p(out["dA"]), _p(out["dD"]), _p(out["dbias"]),
                                             batch, H, W, Ci, N, int(bool(delta_is_raw)), int(bool(zoh)))
        if rc:
            raise ValueError("oracle_cross_scan4_bwd: bad sizes")
        return out

    def xproj(self, u, Wx):
        """x_proj of the S6 module: P = u @ Wx, u [..., Di], Wx [Di, NO] -> P [..., NO]."""
        u, Wx = _f64(u), _f64(Wx)
        Di, NO = Wx.shape
        lead = u.shape[:-1]
        M = int(np.prod(lead)) if lead else 1
        P = np.zeros(lead + (NO,))
        if self.lib.oracle_xproj(_p(np.ascontiguousarray(u)), _p(Wx), _p(P), M, Di, NO):
            raise ValueError("oracle_xproj: bad sizes")
        return P

    def vim_block_scan(self, x, Wx, Wdt, A, D, bias, z, *, conv_w=None, conv_b=None):
        """The Vim block's two S6 modules from their common input, each with its own
        projections (page "Vision Mamba Guide": the block runs "1D Conv -> SiLU -> SSM"
        per pathway, the backward one on the reversed sequence; each SSM derives B, C
        and Delta from its own input by x_proj and dt_proj):
          u_k   = silu(conv_k(x)) (conv_w given) or x
          P_k   = u_k @ Wx[k];  B_k = P_k[..., :N], C_k = P_k[..., N:2N], s_k = P_k[..., 2N]
          delta_raw_k[t, d] = s_k[t] * Wdt[k, d]   (dt_proj; its bias is `bias`, inside softplus)
          y = (S6_f(u_f) + S6_b(u_b)) * silu(z)
        x, z: [batch, L, Di]; Wx [2, Di, 2N+1]; Wdt, bias, D [2, Di]; A [2, Di, N].
        """
        x, Wx, Wdt, A, D, bias, z = map(_f64, (x, Wx, Wdt, A, D, bias, z))
        batch, L, Di = x.shape
        N = A.shape[-1]
        y = np.zeros((batch, L, Di))
        for k in range(2):
            if conv_w is not None:
                u = self.conv_silu(x, _f64(conv_w)[k], _f64(conv_b)[k], reversed=bool(k))
            else:
                u = x
            P = self.xproj(u, Wx[k])
            Bk, Ck = np.ascontiguousarray(P[..., :N]), np.ascontiguousarray(P[..., N:2 * N])
            draw = P[..., 2 * N][..., None] * Wdt[k][None, None, :]
            order = np.arange(L) if k == 0 else np.arange(L)[::-1].copy()
            y += self.s6_direction(u, draw, Bk, Ck, A[k], D[k], bias[k], order, delta_is_raw=True)
        if z is not None:
            y *= z / (1.0 + np.exp(-z))
        return y

    def vim_block_scan_bwd(self, x, Wx, Wdt, A, D, bias, z, dout, *, conv_w=None, conv_b=None):
        """Derivatives of vim_block_scan (first-order Bbar) for the loss sum(dout * y).

        Returns a dict of fp64 arrays: dx [batch, L, Di], dz (None without a gate), dWx
        [2, Di, 2N+1], dWdt, dbias, dD [2, Di], dA [2, Di, N], and with the convolution
        front dconv_w [2, Di, 3], dconv_b [2, Di] (else None).
        """
        x, Wx, Wdt, A, D, bias, z, dout, conv_w, conv_b = map(_f64, (x, Wx, Wdt, A, D, bias, z, dout, conv_w, conv_b))
        batch, L, Di = x.shape
        N = A.shape[-1]
        conv = conv_w is not None
        out = dict(dx=np.zeros((batch, L, Di)), dz=np.zeros((batch, L, Di)) if z is not None else None,
                   dWx=np.zeros((2, Di, 2 * N + 1)), dWdt=np.zeros((2, Di)), dbias=np.zeros((2, Di)),
                   dD=np.zeros((2, Di)), dA=np.zeros((2, Di, N)),
                   dconv_w=np.zeros((2, Di, 3)) if conv else None, dconv_b=np.zeros((2, Di)) if conv else None)
        rc = self.lib.oracle_vim_block_scan_bwd(
            _p(x), _p(conv_w), _p(conv_b), _p(Wx), _p(Wdt), _p(A), _p(D), _p(bias), _p(z), _p(dout), _p(out["dx"]),
            _p(out["dz"]), _p(out["dWx"]), _p(out["dWdt"]), _p(out["dbias"]), _p(out["dD"]), _p(out["dA"]),
            _p(out["dconv_w"]), _p(out["dconv_b"]), batch, L, Di, N)
        if rc:
            raise ValueError("oracle_vim_block_scan_bwd: bad sizes")
        return out

    def conv_silu(self, x, w, cb, *, reversed=False):
        """silu of the kernel-3 depthwise convolution (zero padding 1) in front of a
        pathway; reversed=True for the backward pathway (taps x[t+1], x[t], x[t-1]).

        x: [batch, L, Di]; w: [Di, 3]; cb: [Di].  Returns u [batch, L, Di].
        """
        x, w, cb = map(_f64, (x, w, cb))
        batch, L, Di = x.shape
        u = np.zeros((batch, L, Di))
        if self.lib.oracle_conv_silu(_p(x), _p(w), _p(cb), _p(u), batch, L, Di, int(bool(reversed))):
            raise ValueError("oracle_conv_silu: bad sizes")
        return u

    def vim_bidir_conv(self, x, conv_w, conv_b, delta, z, B, C, A, D, bias, *, bc_dir_stride=0,
                       delta_is_raw=True, zoh=False):
        """Vim scan with its convolution front: u_f = silu(conv_f(x)), u_b = silu of
        conv_b on the reversed sequence; then (y^f + y^b) * silu(z).

        x, delta, z: [batch, L, Di]; conv_w: [2, Di, 3]; conv_b: [2, Di]; the rest as
        in vim_bidir.
        """
        x, conv_w, conv_b, delta, z, B, C, A, D, bias = map(
            _f64, (x, conv_w, conv_b, delta, z, B, C, A, D, bias))
        batch, L, Di = x.shape
        N = B.shape[-1]
        if bias is None:
            bias = np.zeros((2, Di))
        y = np.zeros((batch, L, Di))
        rc = self.lib.oracle_vim_bidir_conv(_p(x), _p(conv_w), _p(conv_b), _p(delta), _p(z), _p(B), _p(C),
                                            int(bc_dir_stride), _p(A), _p(D), _p(bias), _p(y), batch, L, Di,
                                            N, int(bool(delta_is_raw)), int(bool(zoh)))
        if rc:
            raise ValueError("oracle_vim_bidir_conv: bad sizes")
        return y

    def cross_scan4(self, u, delta, z, B, C, A, D, bias, *, delta_is_raw=True, zoh=False):
        """VMamba four-direction scan with CS-Merge: (sum_k y_k) * silu(z).

        u, delta, z: [batch, H, W, Ci]; B, C: [4, batch, H*W, N] in grid order;
        A: [4, Ci, N]; D, bias: [4, Ci].
        """
        u, delta, z, B, C, A, D, bias = map(_f64, (u, delta, z, B, C, A, D, bias))
        batch, H, W, Ci = u.shape
        N = B.shape[-1]
        if bias is None:
            bias = np.zeros((4, Ci))
        y = np.zeros((batch, H, W, Ci))
        rc = self.lib.oracle_cross_scan4(_p(u), _p(delta), _p(z), _p(B), _p(C), _p(A), _p(D),
                                         _p(bias), _p(y), batch, H, W, Ci, N, int(bool(delta_is_raw)),
                                         int(bool(zoh)))
        if rc:
            raise ValueError("oracle_cross_scan4: bad sizes")
        return y

    def cross_merge4(self, ys, z, H, W):
        """CS-Merge alone: ys [4, batch, H*W, Ci] in scan order -> [batch, H, W, Ci]."""
        ys, z = _f64(ys), _f64(z)
        _, batch, L, Ci = ys.shape
        assert L == H * W
        y = np.zeros((batch, H, W, Ci))
        rc = self.lib.oracle_cross_merge4(_p(ys), _p(z), _p(y), batch, H, W, Ci)
        if rc:
            raise ValueError("oracle_cross_merge4: bad sizes")
        return y


_default = None


def default() -> Oracle:
    """The oracle built from ``oracle.c`` next to this file (built on first use)."""
    global _default
    if _default is None:
        _default = Oracle(_build.build())
    return _default


def set_threads(n):
    default().set_threads(n)


def max_threads():
    return default().max_threads()


def cross_order(k, H, W):
    return default().cross_order(k, H, W)


def s6_direction(*a, **k):
    return default().s6_direction(*a, **k)


def vim_bidir(*a, **k):
    return default().vim_bidir(*a, **k)


def cross_scan4(*a, **k):
    return default().cross_scan4(*a, **k)


def conv_silu(*a, **k):
    return default().conv_silu(*a, **k)


def vim_bidir_bwd(*a, **k):
    return default().vim_bidir_bwd(*a, **k)


def xproj(*a, **k):
    return default().xproj(*a, **k)


def cross_scan4_bwd(*a, **k):
    return default().cross_scan4_bwd(*a, **k)


def vim_block_scan(*a, **k):
    return default().vim_block_scan(*a, **k)


def vim_bidir_conv(*a, **k):
    return default().vim_bidir_conv(*a, **k)


def vim_bidir_conv_bwd(*a, **k):
    return default().vim_bidir_conv_bwd(*a, **k)


def vim_block_scan_bwd(*a, **k):
    return default().vim_block_scan_bwd(*a, **k)


def cross_merge4(*a, **k):
    return default().cross_merge4(*a, **k)
