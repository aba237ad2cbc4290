"""Thin ctypes binding of libvimscan.so (declared in include/vimscan.h).

Argument marshalling only: every tensor is checked for device (the current CUDA
device), dtype, shape and contiguity before the library is called, then turned into
raw device pointers and handed to the C ABI together with
the current torch CUDA stream.  Every step of the scan runs in the library's sm_100a
kernels; there is no fallback of any kind, and a missing library is an ImportError.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libvimscan.so")

VIM_OK, VIM_ERR_INVALID_ARG, VIM_ERR_UNSUPPORTED, VIM_ERR_WORKSPACE, VIM_ERR_CUDA, VIM_ERR_TIMEOUT = range(6)
VIM_F32, VIM_BF16 = 0, 1

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m vision_mamba_selective_b200.build` "
        "(nvcc, sm_100a); the selective scan has no other implementation")

lib = ctypes.CDLL(LIB_PATH)

_vp, _i, _i64, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
lib.vim_scan_bidir.argtypes = [_vp, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp,
                               _i, _i, _i, _i, _i, _vp, _sz, _vp]
lib.vim_scan_bidir.restype = _i
lib.vmamba_cross_scan4.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                   _i, _i, _i, _i, _i, _i, _vp, _sz, _vp]
lib.vmamba_cross_scan4.restype = _i
lib.vim_scan_bidir_events.argtypes = lib.vim_scan_bidir.argtypes + [_vp]
lib.vim_scan_bidir_events.restype = _i
lib.vmamba_cross_scan4_events.argtypes = lib.vmamba_cross_scan4.argtypes + [_vp]
lib.vmamba_cross_scan4_events.restype = _i
lib.vim_scan_bidir_conv.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp,
                                    _i, _i, _i, _i, _i, _vp, _sz, _vp]
lib.vim_scan_bidir_conv.restype = _i
lib.vim_scan_bidir_conv_events.argtypes = lib.vim_scan_bidir_conv.argtypes + [_vp]
lib.vim_scan_bidir_conv_events.restype = _i
_u = ctypes.c_uint
lib.vim_scan_bidir_ex.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp,
                                  _i, _i, _i, _i, _i, _u, _vp, _sz, _vp, _vp]
lib.vim_scan_bidir_ex.restype = _i
lib.vmamba_cross_scan4_ex.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                      _i, _i, _i, _i, _i, _i, _u, _vp, _sz, _vp, _vp]
lib.vmamba_cross_scan4_ex.restype = _i
VIM_FLAG_ZOH_EXACT = 1
lib.vim_scan_bidir_bwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                   _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _sz, _vp]
lib.vim_scan_bidir_bwd.restype = _i
lib.vim_scan_bidir_bwd_events.argtypes = lib.vim_scan_bidir_bwd.argtypes + [_vp]
lib.vim_scan_bidir_bwd_events.restype = _i
# the _bwd arguments with `flags` before the workspace, then the events
lib.vim_scan_bidir_bwd_ex.argtypes = (lib.vim_scan_bidir_bwd.argtypes[:23] + [ctypes.c_uint]
                                      + lib.vim_scan_bidir_bwd.argtypes[23:] + [_vp])
lib.vim_scan_bidir_bwd_ex.restype = _i
# the training pair: the forward scan keeping the derivative's chunk states, and the
# derivative that takes them
lib.vim_scan_bidir_ckpt.argtypes = [_vp, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp,
                                    _i, _i, _i, _i, _i, _u, _vp, _sz, _vp, _vp]
lib.vim_scan_bidir_ckpt.restype = _i
lib.vim_scan_bidir_bwd_ckpt.argtypes = (lib.vim_scan_bidir_bwd_ex.argtypes[:9] + [_vp]
                                        + lib.vim_scan_bidir_bwd_ex.argtypes[9:])
lib.vim_scan_bidir_bwd_ckpt.restype = _i
lib.vim_scan_ckpt_bytes.argtypes = [_i, _i, _i, _i]
lib.vim_scan_ckpt_bytes.restype = _sz
lib.vim_scan_bwd_workspace_bytes.argtypes = [_i, _i, _i, _i, _i]
lib.vim_scan_bwd_workspace_bytes.restype = _sz
lib.vim_block_scan.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i,
                               _vp, _sz, _vp, _vp]
lib.vim_block_scan.restype = _i
lib.vim_block_workspace_bytes.argtypes = [_i, _i, _i, _i]
lib.vim_block_workspace_bytes.restype = _sz
lib.vmamba_cross_scan4_bwd.argtypes = [_vp] * 17 + [_i, _i, _i, _i, _i, _i, _vp, _sz, _vp]
lib.vmamba_cross_scan4_bwd_ex.argtypes = [_vp] * 17 + [_i, _i, _i, _i, _i, _i, ctypes.c_uint, _vp, _sz, _vp]
lib.vmamba_cross_scan4_bwd_ex.restype = _i
lib.vmamba_cross_scan4_bwd.restype = _i
lib.vmamba_cross_scan4_bwd_workspace_bytes.argtypes = [_i, _i, _i, _i, _i]
lib.vmamba_cross_scan4_bwd_workspace_bytes.restype = _sz
lib.vim_scan_bidir_noalloc.argtypes = [_vp, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp,
                                       _i, _i, _i, _i, _i, _vp]
lib.vim_scan_bidir_noalloc.restype = _i
VIM_NOALLOC_SCRATCH_BYTES = 8 << 20
lib.vim_scan_bidir_conv_bwd_ex.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp,
                                           _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                           _i, _i, _i, _i, _i, _u, _vp, _sz, _vp]
lib.vim_scan_bidir_conv_bwd_ex.restype = _i
lib.vim_scan_bidir_conv_bwd.argtypes = (lib.vim_scan_bidir_conv_bwd_ex.argtypes[:27]
                                        + lib.vim_scan_bidir_conv_bwd_ex.argtypes[28:])
lib.vim_scan_bidir_conv_bwd.restype = _i
# the training pair with the convolution front
lib.vim_scan_bidir_conv_ckpt.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp,
                                         _i, _i, _i, _i, _i, _u, _vp, _sz, _vp, _vp]
lib.vim_scan_bidir_conv_ckpt.restype = _i
lib.vim_scan_bidir_conv_bwd_ckpt.argtypes = (lib.vim_scan_bidir_conv_bwd_ex.argtypes[:11] + [_vp]
                                             + lib.vim_scan_bidir_conv_bwd_ex.argtypes[11:])
lib.vim_scan_bidir_conv_bwd_ckpt.restype = _i
# the training pair of the cross-scan
lib.vmamba_cross_scan4_ckpt.argtypes = [_vp] * 10 + [_i, _i, _i, _i, _i, _i, _u, _vp, _sz, _vp, _vp]
lib.vmamba_cross_scan4_ckpt.restype = _i
lib.vmamba_cross_scan4_bwd_ckpt.argtypes = [_vp] * 18 + [_i, _i, _i, _i, _i, _i, _u, _vp, _sz, _vp]
lib.vmamba_cross_scan4_bwd_ckpt.restype = _i
lib.vmamba_cross_ckpt_bytes.argtypes = [_i, _i, _i, _i, _i]
lib.vmamba_cross_ckpt_bytes.restype = _sz
lib.vim_scan_conv_bwd_workspace_bytes.argtypes = [_i, _i, _i, _i, _i, _i]
lib.vim_scan_conv_bwd_workspace_bytes.restype = _sz
lib.vim_block_scan_bwd.argtypes = [_vp] * 19 + [_i, _i, _i, _i, _i, _vp, _sz, _vp]
lib.vim_block_scan_bwd.restype = _i
lib.vim_block_bwd_workspace_bytes.argtypes = [_i, _i, _i, _i]
lib.vim_block_bwd_workspace_bytes.restype = _sz
lib.vim_scan_bidir_host.argtypes = [_vp, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp,
                                    _i, _i, _i, _i, _i, _u, _i, _vp, _sz, _vp, _vp, _vp]
lib.vim_scan_bidir_host.restype = _i
lib.vim_scan_host_workspace_bytes.argtypes = [_i, _i, _i, _i, _i, _i, _i]
lib.vim_scan_host_workspace_bytes.restype = _sz
lib.cross_merge4.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _i, _vp]
lib.cross_merge4.restype = _i
lib.vim_scan_workspace_bytes.argtypes = [_i, _i, _i, _i, _i, _i]
lib.vim_scan_workspace_bytes.restype = _sz
lib.vim_status_string.argtypes = [_i]
lib.vim_status_string.restype = ctypes.c_char_p


class VimScanError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


def status_string(status: int) -> str:
    return lib.vim_status_string(int(status)).decode()


def vim_scan_workspace_bytes(which: int, batch: int, L_or_H: int, W: int, channels: int, d_state: int) -> int:
    return int(lib.vim_scan_workspace_bytes(which, batch, L_or_H, W, channels, d_state))


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return VIM_F32
    if t.dtype == torch.bfloat16:
        return VIM_BF16
    raise TypeError(f"unsupported dtype {t.dtype}: fp32 or bf16")


def _ptrs(where, ref, specs):
    """Check every tensor the kernels will address and return their data pointers, in
    the order of ``specs`` (None for an absent tensor), before the library is called.

    ``ref`` fixes the device; it must be the current CUDA device (the stream the library
    launches on belongs to it).  ``specs`` holds (name, tensor or None, dtype or None,
    rule) with rule either an exact shape tuple or ("numel", n, last): at least n
    elements with last dimension ``last`` (buffers such as B/C with a per-direction
    stride).  Every tensor must be contiguous.  Raises TypeError (not a CUDA tensor, a
    wrong dtype) or ValueError (device, shape, layout).  One pass per tensor, integer
    device indices and direct size comparisons: this runs on every call, so its cost
    is part of a small problem's launch latency.
    """
    if not isinstance(ref, torch.Tensor) or not ref.is_cuda:
        raise TypeError(f"{where}: inputs must be CUDA tensors")
    dev = ref.get_device()
    cur = torch.cuda.current_device()
    if dev != cur:
        raise ValueError(f"{where}: tensors are on {ref.device} but the current device is cuda:{cur}")
    out = []
    for name, t, dtype, rule in specs:
        if t is None:
            out.append(None)
            continue
        if not isinstance(t, torch.Tensor) or t.get_device() != dev:
            if not isinstance(t, torch.Tensor) or not t.is_cuda:
                raise TypeError(f"{where}: {name} must be a CUDA tensor")
            raise ValueError(f"{where}: {name} is on {t.device}, the other inputs on {ref.device}")
        if dtype is not None and t.dtype != dtype:
            raise TypeError(f"{where}: {name} must be {dtype}, got {t.dtype}")
        if rule[0] == "numel":
            _, n, last = rule
            if t.numel() < n or t.dim() == 0 or t.shape[-1] != last:
                raise ValueError(f"{where}: {name} has shape {tuple(t.shape)}; it needs at least {n} "
                                 f"elements with last dimension {last}")
        elif t.shape != rule:
            raise ValueError(f"{where}: {name} has shape {tuple(t.shape)}, expected {tuple(rule)}")
        if not t.is_contiguous():
            raise ValueError(f"{where}: {name} must be contiguous")
        out.append(t.data_ptr())
    return out


def _out_specs(out, io, act, bc, a_shape, d_shape):
    """The derivative outputs as _ptrs specs, in the library's argument order (none when
    there is no output dict: the inputs were refused before it could be allocated)."""
    if out is None:
        return []
    f32 = torch.float32
    return [("out['du']", out["du"], io, act), ("out['ddelta']", out["ddelta"], io, act),
            ("out['dz']", out["dz"], io, act), ("out['dB']", out["dB"], f32, bc), ("out['dC']", out["dC"], f32, bc),
            ("out['dA']", out["dA"], f32, a_shape), ("out['dD']", out["dD"], f32, d_shape),
            ("out['ddelta_bias']", out["ddelta_bias"], f32, d_shape)]


def _bc_rule(batch, L, N, bc_dir_stride):
    if bc_dir_stride < 0:
        raise ValueError("bc_dir_stride must be >= 0")
    return ("numel", int(bc_dir_stride) + batch * L * N, N)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _workspace(nbytes, workspace, device):
    if nbytes == 0:
        return None, 0
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
    if workspace.numel() * workspace.element_size() < nbytes:
        raise ValueError(f"workspace too small: need {nbytes} bytes")
    return workspace, workspace.numel() * workspace.element_size()


def _events(events):
    """Raw cudaEvent_t handles of torch CUDA events (created by recording them once)."""
    handles = []
    for e in events:
        if e.cuda_event == 0:
            e.record()
        handles.append(e.cuda_event)
    return (ctypes.c_void_p * len(handles))(*handles)


def _bidir(name, u, conv_w, conv_b, delta, z, B, C, A, D, delta_bias, y, bc_dir_stride, workspace, stream,
           events, zoh, ckpt=None):
    batch, L, Di = u.shape
    N = B.shape[-1]
    dt = _dtype_code(u)
    act = (batch, L, Di)
    bc = _bc_rule(batch, L, N, bc_dir_stride)
    if y is None:
        y = torch.empty_like(u)
    conv = conv_w is not None or conv_b is not None
    f32, io = torch.float32, u.dtype
    pu, pcw, pcb, pdelta, pz, pB, pC, pA, pD, pbias, py = _ptrs(name, u, [
        ("x" if conv else "u", u, None, act), ("conv_w", conv_w, f32, (2, Di, 3)), ("conv_b", conv_b, f32, (2, Di)),
        ("delta", delta, io, act), ("z", z, io, act), ("B", B, io, bc), ("C", C, io, bc),
        ("A", A, f32, (2, Di, N)), ("D", D, f32, (2, Di)), ("delta_bias", delta_bias, f32, (2, Di)),
        ("y", y, io, act)])
    ws, ws_bytes = _workspace(vim_scan_workspace_bytes(0, batch, L, 0, Di, N), workspace, u.device)
    if ckpt is not None:
        (pk,) = _ptrs(name, u, [("ckpt", ckpt, f32, ckpt_shape(batch, L, Di, N))])
        tail = (batch, L, Di, N, dt, VIM_FLAG_ZOH_EXACT if zoh else 0, None if ws is None else ws.data_ptr(),
                ws_bytes, _stream(stream), None if events is None else _events(events))
        if conv:
            st = lib.vim_scan_bidir_conv_ckpt(pu, pcw, pcb, pdelta, pz, pB, pC, int(bc_dir_stride), pA, pD, pbias,
                                              py, pk, *tail)
        else:
            st = lib.vim_scan_bidir_ckpt(pu, pdelta, pz, pB, pC, int(bc_dir_stride), pA, pD, pbias, py, pk, *tail)
        if st != VIM_OK:
            raise VimScanError(st, name)
        return y
    pre = (pu, pcw, pcb) if conv or zoh else (pu,)
    args = pre + (pdelta, pz, pB, pC, int(bc_dir_stride), pA, pD, pbias, py, batch, L, Di, N, dt)
    tail = (None if ws is None else ws.data_ptr(), ws_bytes, _stream(stream))
    ev = None if events is None else _events(events)
    if zoh:
        st = lib.vim_scan_bidir_ex(*args, VIM_FLAG_ZOH_EXACT, *tail, ev)
    elif conv:
        st = (lib.vim_scan_bidir_conv(*args, *tail) if ev is None
              else lib.vim_scan_bidir_conv_events(*args, *tail, ev))
    else:
        st = lib.vim_scan_bidir(*args, *tail) if ev is None else lib.vim_scan_bidir_events(*args, *tail, ev)
    if st != VIM_OK:
        raise VimScanError(st, name)
    return y


def ckpt_shape(batch, L, d_inner, d_state):
    """Shape of the checkpoints vim_scan_bidir(ckpt=...) writes and
    vim_scan_bidir_bwd(ckpt=...) reads: [batch, ceil(L / 32), 2, d_state, d_inner]."""
    return (batch, (L + 31) // 32, 2, d_state, d_inner)


def vim_scan_bidir(u, delta, z, B, C, A, D, delta_bias, *, y=None, bc_dir_stride=0,
                   workspace=None, stream=None, events=None, zoh=False, ckpt=None):
    """Vim bidirectional selective scan, (y^f + y^b) * silu(z); see include/vimscan.h.

    u, delta, z: [batch, L, d_inner]; B, C: [batch, L, d_state] (or a larger buffer
    whose backward copy starts ``bc_dir_stride`` elements in); A: [2, d_inner,
    d_state] fp32; D, delta_bias: [2, d_inner] fp32.  Returns y [batch, L, d_inner].
    zoh=True takes the exact zero-order-hold Bbar (VIM_FLAG_ZOH_EXACT).  ``ckpt``, an
    fp32 tensor of ckpt_shape(...), receives the states the derivative needs
    (vim_scan_bidir_ckpt) for vim_scan_bidir_bwd(ckpt=...).
    """
    return _bidir("vim_scan_bidir", u, None, None, delta, z, B, C, A, D, delta_bias, y, bc_dir_stride,
                  workspace, stream, events, zoh, ckpt)


def vim_scan_bidir_conv(x, conv_w, conv_b, delta, z, B, C, A, D, delta_bias, *, y=None, bc_dir_stride=0,
                        workspace=None, stream=None, events=None, zoh=False, ckpt=None):
    """vim_scan_bidir with the pathways' kernel-3 convolution + SiLU front fused in.

    x, delta, z: [batch, L, d_inner]; conv_w: [2, d_inner, 3] fp32; conv_b: [2, d_inner]
    fp32; the rest as in vim_scan_bidir.  Returns y [batch, L, d_inner].  A missing
    half of the front (conv_w or conv_b None) is rejected by the library.  ``ckpt`` as in
    vim_scan_bidir (vim_scan_bidir_conv_ckpt), for vim_scan_bidir_conv_bwd(ckpt=...).
    """
    return _bidir("vim_scan_bidir_conv", x, conv_w, conv_b, delta, z, B, C, A, D, delta_bias, y,
                  bc_dir_stride, workspace, stream, events, zoh, ckpt)


def vim_scan_bwd_workspace_bytes(batch, L, d_inner, d_state, separate_bc):
    return int(lib.vim_scan_bwd_workspace_bytes(batch, L, d_inner, d_state, int(bool(separate_bc))))


def vim_scan_bidir_bwd(u, delta, z, B, C, A, D, delta_bias, dout, *, bc_dir_stride=0, workspace=None,
                       stream=None, out=None, events=None, zoh=False, ckpt=None):
    """Derivatives of vim_scan_bidir (first-order Bbar, or with ``zoh`` the exact
    zero-order hold) for a loss whose derivative with respect to y is ``dout``; see
    include/vimscan.h.

    Returns a dict: du, ddelta (w.r.t. the raw delta), dz (None without z), in the
    input dtype; dB and dC (fp32, shaped like B and C); dA [2, d_inner, d_state], dD
    and ddelta_bias [2, d_inner] (fp32).  ``out`` may hold those tensors from an
    earlier call to be written again; ``events`` 4 CUDA events (see
    vim_scan_bidir_bwd_events).  ``ckpt``: the checkpoints vim_scan_bidir(ckpt=...) wrote
    for the same inputs (vim_scan_bidir_bwd_ckpt), which replace the derivative's own
    forward summaries.
    """
    batch, L, Di = u.shape
    N = B.shape[-1]
    dt = _dtype_code(u)
    dev = u.device
    act = (batch, L, Di)
    bc = _bc_rule(batch, L, N, bc_dir_stride)
    if out is not None:
        if z is not None and out["dz"] is None:
            raise ValueError("vim_scan_bidir_bwd: out['dz'] is needed when z is given")
    elif isinstance(u, torch.Tensor) and u.is_cuda:
        out = dict(du=torch.empty_like(u), ddelta=torch.empty_like(u),
                   dz=torch.empty_like(u) if z is not None else None,
                   dB=torch.zeros(B.shape, dtype=torch.float32, device=dev),
                   dC=torch.zeros(C.shape, dtype=torch.float32, device=dev),
                   dA=torch.empty((2, Di, N), dtype=torch.float32, device=dev),
                   dD=torch.empty((2, Di), dtype=torch.float32, device=dev),
                   ddelta_bias=torch.empty((2, Di), dtype=torch.float32, device=dev))
    f32, io = torch.float32, u.dtype
    ptrs = _ptrs("vim_scan_bidir_bwd", u, [
        ("u", u, None, act), ("delta", delta, io, act), ("z", z, io, act), ("B", B, io, bc), ("C", C, io, bc),
        ("A", A, f32, (2, Di, N)), ("D", D, f32, (2, Di)), ("delta_bias", delta_bias, f32, (2, Di)),
        ("dout", dout, io, act)] + _out_specs(out, io, act, bc, (2, Di, N), (2, Di)))
    ws, ws_bytes = _workspace(vim_scan_bwd_workspace_bytes(batch, L, Di, N, bc_dir_stride > 0), workspace, dev)
    if ckpt is not None:
        (pk,) = _ptrs("vim_scan_bidir_bwd", u, [("ckpt", ckpt, f32, ckpt_shape(batch, L, Di, N))])
        st = lib.vim_scan_bidir_bwd_ckpt(
            *ptrs[:5], int(bc_dir_stride), *ptrs[5:8], pk, *ptrs[8:], batch, L, Di, N, dt,
            VIM_FLAG_ZOH_EXACT if zoh else 0, None if ws is None else ws.data_ptr(), ws_bytes, _stream(stream),
            None if events is None else _events(events))
        if st != VIM_OK:
            raise VimScanError(st, "vim_scan_bidir_bwd")
        return out
    if zoh:
        fn = lib.vim_scan_bidir_bwd_ex
        flags, extra = (VIM_FLAG_ZOH_EXACT,), (None if events is None else _events(events),)
    else:
        fn = lib.vim_scan_bidir_bwd if events is None else lib.vim_scan_bidir_bwd_events
        flags, extra = (), (() if events is None else (_events(events),))
    st = fn(
        *ptrs[:5], int(bc_dir_stride), *ptrs[5:],
        batch, L, Di, N, dt, *flags, None if ws is None else ws.data_ptr(), ws_bytes, _stream(stream), *extra)
    if st != VIM_OK:
        raise VimScanError(st, "vim_scan_bidir_bwd")
    return out


def vim_scan_conv_bwd_workspace_bytes(batch, L, d_inner, d_state, dtype_code, separate_bc):
    return int(lib.vim_scan_conv_bwd_workspace_bytes(batch, L, d_inner, d_state, dtype_code, int(bool(separate_bc))))


def vim_scan_bidir_conv_bwd(x, conv_w, conv_b, delta, z, B, C, A, D, delta_bias, dout, *, bc_dir_stride=0,
                            workspace=None, stream=None, out=None, zoh=False, ckpt=None):
    """Derivatives of vim_scan_bidir_conv (first-order Bbar, or with ``zoh`` the exact
    hold) for a loss whose derivative with respect to y is ``dout``; see
    include/vimscan.h.

    Returns a dict: dx, ddelta (w.r.t. the raw delta), dz (None without z) in the input
    dtype; dconv_w [2, d_inner, 3] and dconv_b [2, d_inner] fp32; dB, dC (fp32, shaped
    like B and C), dA [2, d_inner, d_state], dD and ddelta_bias [2, d_inner] fp32.
    ``out`` may hold those tensors from an earlier call to be written again.  ``ckpt``: the
    checkpoints vim_scan_bidir_conv(ckpt=...) wrote for the same inputs
    (vim_scan_bidir_conv_bwd_ckpt).
    """
    batch, L, Di = x.shape
    N = B.shape[-1]
    dt = _dtype_code(x)
    dev = x.device
    act = (batch, L, Di)
    bc = _bc_rule(batch, L, N, bc_dir_stride)
    if out is not None:
        if z is not None and out["dz"] is None:
            raise ValueError("vim_scan_bidir_conv_bwd: out['dz'] is needed when z is given")
    elif isinstance(x, torch.Tensor) and x.is_cuda:
        e32 = lambda *shape: torch.empty(shape, dtype=torch.float32, device=dev)
        out = dict(dx=torch.empty_like(x), ddelta=torch.empty_like(x), dz=torch.empty_like(x) if z is not None else None,
                   dconv_w=e32(2, Di, 3), dconv_b=e32(2, Di),
                   dB=torch.zeros(B.shape, dtype=torch.float32, device=dev),
                   dC=torch.zeros(C.shape, dtype=torch.float32, device=dev),
                   dA=e32(2, Di, N), dD=e32(2, Di), ddelta_bias=e32(2, Di))
    f32, io = torch.float32, x.dtype
    specs = [("x", x, None, act), ("conv_w", conv_w, f32, (2, Di, 3)), ("conv_b", conv_b, f32, (2, Di)),
             ("delta", delta, io, act), ("z", z, io, act), ("B", B, io, bc), ("C", C, io, bc),
             ("A", A, f32, (2, Di, N)), ("D", D, f32, (2, Di)), ("delta_bias", delta_bias, f32, (2, Di)),
             ("dout", dout, io, act)]
    if out is not None:
        specs += [("out['dx']", out["dx"], io, act), ("out['dconv_w']", out["dconv_w"], f32, (2, Di, 3)),
                  ("out['dconv_b']", out["dconv_b"], f32, (2, Di)), ("out['ddelta']", out["ddelta"], io, act),
                  ("out['dz']", out["dz"], io, act), ("out['dB']", out["dB"], f32, bc),
                  ("out['dC']", out["dC"], f32, bc), ("out['dA']", out["dA"], f32, (2, Di, N)),
                  ("out['dD']", out["dD"], f32, (2, Di)), ("out['ddelta_bias']", out["ddelta_bias"], f32, (2, Di))]
    ptrs = _ptrs("vim_scan_bidir_conv_bwd", x, specs)
    ws, ws_bytes = _workspace(vim_scan_conv_bwd_workspace_bytes(batch, L, Di, N, dt, bc_dir_stride > 0), workspace,
                              dev)
    if ckpt is not None:
        (pk,) = _ptrs("vim_scan_bidir_conv_bwd", x, [("ckpt", ckpt, f32, ckpt_shape(batch, L, Di, N))])
        st = lib.vim_scan_bidir_conv_bwd_ckpt(
            *ptrs[:7], int(bc_dir_stride), *ptrs[7:10], pk, *ptrs[10:], batch, L, Di, N, dt,
            VIM_FLAG_ZOH_EXACT if zoh else 0, None if ws is None else ws.data_ptr(), ws_bytes, _stream(stream))
    else:
        st = lib.vim_scan_bidir_conv_bwd_ex(
            *ptrs[:7], int(bc_dir_stride), *ptrs[7:], batch, L, Di, N, dt, VIM_FLAG_ZOH_EXACT if zoh else 0,
            None if ws is None else ws.data_ptr(), ws_bytes, _stream(stream))
    if st != VIM_OK:
        raise VimScanError(st, "vim_scan_bidir_conv_bwd")
    return out


def vmamba_cross_scan4_bwd(u, delta, z, B, C, A, D, delta_bias, dout, *, workspace=None, stream=None, out=None,
                           zoh=False, ckpt=None):
    """Derivatives of vmamba_cross_scan4 (first-order Bbar, or with ``zoh`` the exact
    zero-order hold) for a loss whose derivative
    with respect to y is ``dout``; see include/vimscan.h.  Returns a dict: du, ddelta, dz
    (None without z) in the input dtype; dB, dC [4, batch, H*W, N], dA [4, C, N], dD and
    ddelta_bias [4, C] in fp32.  ``out`` may hold those tensors from an earlier call.
    ``ckpt``: the checkpoints vmamba_cross_scan4(ckpt=...) wrote for the same inputs
    (vmamba_cross_scan4_bwd_ckpt).
    """
    batch, H, W, Ch = u.shape
    N = B.shape[-1]
    dev = u.device
    act = (batch, H, W, Ch)
    bc = (4, batch, H * W, N)
    if out is not None:
        if z is not None and out["dz"] is None:
            raise ValueError("vmamba_cross_scan4_bwd: out['dz'] is needed when z is given")
    elif isinstance(u, torch.Tensor) and u.is_cuda:
        e32 = lambda *shape: torch.empty(shape, dtype=torch.float32, device=dev)
        out = dict(du=torch.empty_like(u), ddelta=torch.empty_like(u), dz=torch.empty_like(u) if z is not None else None,
                   dB=e32(*B.shape), dC=e32(*C.shape), dA=e32(4, Ch, N), dD=e32(4, Ch), ddelta_bias=e32(4, Ch))
    f32, io = torch.float32, u.dtype
    ptrs = _ptrs("vmamba_cross_scan4_bwd", u, [
        ("u", u, None, act), ("delta", delta, io, act), ("z", z, io, act), ("B", B, io, bc), ("C", C, io, bc),
        ("A", A, f32, (4, Ch, N)), ("D", D, f32, (4, Ch)), ("delta_bias", delta_bias, f32, (4, Ch)),
        ("dout", dout, io, act)] + _out_specs(out, io, act, bc, (4, Ch, N), (4, Ch)))
    ws, ws_bytes = _workspace(int(lib.vmamba_cross_scan4_bwd_workspace_bytes(batch, H, W, Ch, N)), workspace, dev)
    if ckpt is not None:
        (pk,) = _ptrs("vmamba_cross_scan4_bwd", u, [("ckpt", ckpt, f32, cross_ckpt_shape(batch, H, W, Ch, N))])
        st = lib.vmamba_cross_scan4_bwd_ckpt(
            *ptrs[:8], pk, *ptrs[8:], batch, H, W, Ch, N, _dtype_code(u), VIM_FLAG_ZOH_EXACT if zoh else 0,
            None if ws is None else ws.data_ptr(), ws_bytes, _stream(stream))
    else:
        fn = lib.vmamba_cross_scan4_bwd_ex if zoh else lib.vmamba_cross_scan4_bwd
        flags = (VIM_FLAG_ZOH_EXACT,) if zoh else ()
        st = fn(
            *ptrs,
            batch, H, W, Ch, N, _dtype_code(u), *flags, None if ws is None else ws.data_ptr(), ws_bytes,
            _stream(stream))
    if st != VIM_OK:
        raise VimScanError(st, "vmamba_cross_scan4_bwd")
    return out


def vim_block_workspace_bytes(batch, L, d_inner, d_state):
    return int(lib.vim_block_workspace_bytes(batch, L, d_inner, d_state))


def vim_block_scan(x, Wx, Wdt, dt_bias, A, D, z, *, conv_w=None, conv_b=None, y=None, workspace=None,
                   stream=None, events=None):
    """The Vim block's two S6 modules from their common input x with their own
    projections (x_proj on the tensor cores, dt_proj inside the scan) and optionally
    the convolution front; see include/vimscan.h.  bf16 x, z, Wx [2, d_inner, 2N+1];
    fp32 Wdt, dt_bias, D [2, d_inner], A [2, d_inner, N].  Returns y [batch, L, d_inner].
    """
    batch, L, Di = x.shape
    N = A.shape[-1]
    act = (batch, L, Di)
    if y is None and isinstance(x, torch.Tensor) and x.is_cuda:
        y = torch.empty_like(x)
    f32, io = torch.float32, x.dtype
    ptrs = _ptrs("vim_block_scan", x, [
        ("x", x, None, act), ("conv_w", conv_w, f32, (2, Di, 3)), ("conv_b", conv_b, f32, (2, Di)),
        ("Wx", Wx, io, (2, Di, 2 * N + 1)), ("Wdt", Wdt, f32, (2, Di)), ("dt_bias", dt_bias, f32, (2, Di)),
        ("A", A, f32, (2, Di, N)), ("D", D, f32, (2, Di)), ("z", z, io, act), ("y", y, io, act)])
    ws, ws_bytes = _workspace(vim_block_workspace_bytes(batch, L, Di, N), workspace, x.device)
    st = lib.vim_block_scan(
        *ptrs,
        batch, L, Di, N, _dtype_code(x), None if ws is None else ws.data_ptr(), ws_bytes, _stream(stream),
        None if events is None else _events(events))
    if st != VIM_OK:
        raise VimScanError(st, "vim_block_scan")
    return y


def vim_block_bwd_workspace_bytes(batch, L, d_inner, d_state):
    return int(lib.vim_block_bwd_workspace_bytes(batch, L, d_inner, d_state))


def vim_block_scan_bwd(x, Wx, Wdt, dt_bias, A, D, z, dout, *, conv_w=None, conv_b=None, workspace=None, stream=None,
                       out=None):
    """Derivatives of vim_block_scan for a loss whose derivative with respect to y is
    ``dout``; see include/vimscan.h.  bf16 x, z, dout, Wx.

    Returns a dict: dx, dz (None without z) in bf16; dWx [2, d_inner, 2N+1], dWdt,
    ddt_bias, dD [2, d_inner], dA [2, d_inner, N] fp32; dconv_w [2, d_inner, 3] and
    dconv_b [2, d_inner] fp32 with the convolution front (else None).  ``out`` may hold
    those tensors from an earlier call.
    """
    batch, L, Di = x.shape
    N = A.shape[-1]
    NO = 2 * N + 1
    dev = x.device
    act = (batch, L, Di)
    conv = conv_w is not None
    if out is not None:
        if (z is not None) != (out["dz"] is not None) or conv != (out["dconv_w"] is not None):
            raise ValueError("vim_block_scan_bwd: out['dz'] and out['dconv_w'] must match z and conv_w")
    elif isinstance(x, torch.Tensor) and x.is_cuda:
        e32 = lambda *shape: torch.empty(shape, dtype=torch.float32, device=dev)
        out = dict(dx=torch.empty_like(x), dz=torch.empty_like(x) if z is not None else None, dWx=e32(2, Di, NO),
                   dWdt=e32(2, Di), ddt_bias=e32(2, Di), dA=e32(2, Di, N), dD=e32(2, Di),
                   dconv_w=e32(2, Di, 3) if conv else None, dconv_b=e32(2, Di) if conv else None)
    f32, io = torch.float32, x.dtype
    specs = [("x", x, None, act), ("conv_w", conv_w, f32, (2, Di, 3)), ("conv_b", conv_b, f32, (2, Di)),
             ("Wx", Wx, io, (2, Di, NO)), ("Wdt", Wdt, f32, (2, Di)), ("dt_bias", dt_bias, f32, (2, Di)),
             ("A", A, f32, (2, Di, N)), ("D", D, f32, (2, Di)), ("z", z, io, act), ("dout", dout, io, act)]
    if out is not None:
        specs += [("out['dx']", out["dx"], io, act), ("out['dconv_w']", out["dconv_w"], f32, (2, Di, 3)),
                  ("out['dconv_b']", out["dconv_b"], f32, (2, Di)), ("out['dWx']", out["dWx"], f32, (2, Di, NO)),
                  ("out['dWdt']", out["dWdt"], f32, (2, Di)), ("out['ddt_bias']", out["ddt_bias"], f32, (2, Di)),
                  ("out['dA']", out["dA"], f32, (2, Di, N)), ("out['dD']", out["dD"], f32, (2, Di)),
                  ("out['dz']", out["dz"], io, act)]
    ptrs = _ptrs("vim_block_scan_bwd", x, specs)
    ws, ws_bytes = _workspace(vim_block_bwd_workspace_bytes(batch, L, Di, N), workspace, dev)
    st = lib.vim_block_scan_bwd(*ptrs, batch, L, Di, N, _dtype_code(x), None if ws is None else ws.data_ptr(),
                                ws_bytes, _stream(stream))
    if st != VIM_OK:
        raise VimScanError(st, "vim_block_scan_bwd")
    return out


def vim_scan_bidir_noalloc(u, delta, z, B, C, A, D, delta_bias, *, y=None, bc_dir_stride=0, stream=None):
    """vim_scan_bidir without a workspace, for callers that cannot allocate device memory.

    The chunk carries live in a fixed buffer inside the library
    (VIM_NOALLOC_SCRATCH_BYTES), shared by every call: calls must not overlap on the GPU.
    Problems needing more scratch than that raise VimScanError (VIM_ERR_WORKSPACE).
    ``y`` must be given by callers that cannot allocate; otherwise it is allocated here.
    """
    batch, L, Di = u.shape
    N = B.shape[-1]
    dt = _dtype_code(u)
    act = (batch, L, Di)
    bc = _bc_rule(batch, L, N, bc_dir_stride)
    if y is None and isinstance(u, torch.Tensor) and u.is_cuda:
        y = torch.empty_like(u)
    f32, io = torch.float32, u.dtype
    ptrs = _ptrs("vim_scan_bidir_noalloc", u, [
        ("u", u, None, act), ("delta", delta, io, act), ("z", z, io, act), ("B", B, io, bc), ("C", C, io, bc),
        ("A", A, f32, (2, Di, N)), ("D", D, f32, (2, Di)), ("delta_bias", delta_bias, f32, (2, Di)),
        ("y", y, io, act)])
    st = lib.vim_scan_bidir_noalloc(
        *ptrs[:5], int(bc_dir_stride), *ptrs[5:],
        batch, L, Di, N, dt, _stream(stream))
    if st != VIM_OK:
        raise VimScanError(st, "vim_scan_bidir_noalloc")
    return y


def cross_ckpt_shape(batch, H, W, channels, d_state):
    """Shape of the cross-scan's checkpoints (vmamba_cross_scan4(ckpt=...),
    vmamba_cross_scan4_bwd(ckpt=...)): [2 pairs, batch, ceil(H*W / 32), 2, d_state, C]."""
    return (2,) + ckpt_shape(batch, H * W, channels, d_state)


def vmamba_cross_scan4(u, delta, z, B, C, A, D, delta_bias, *, y=None, workspace=None, stream=None,
                       events=None, zoh=False, ckpt=None):
    """VMamba four-direction cross-scan with CS-Merge; see include/vimscan.h.

    u, delta, z: [batch, H, W, C]; B, C: [4, batch, H*W, d_state] by grid position;
    A: [4, C, d_state] fp32; D, delta_bias: [4, C] fp32.  Returns y [batch, H, W, C].
    zoh=True takes the exact zero-order-hold Bbar (VIM_FLAG_ZOH_EXACT).  ``ckpt``, an fp32
    tensor of cross_ckpt_shape(...), receives the states vmamba_cross_scan4_bwd(ckpt=...)
    takes (vmamba_cross_scan4_ckpt).
    """
    batch, H, W, Ch = u.shape
    N = B.shape[-1]
    dt = _dtype_code(u)
    act = (batch, H, W, Ch)
    bc = (4, batch, H * W, N)
    if y is None:
        y = torch.empty_like(u)
    f32, io = torch.float32, u.dtype
    args = tuple(_ptrs("vmamba_cross_scan4", u, [
        ("u", u, None, act), ("delta", delta, io, act), ("z", z, io, act), ("B", B, io, bc), ("C", C, io, bc),
        ("A", A, f32, (4, Ch, N)), ("D", D, f32, (4, Ch)), ("delta_bias", delta_bias, f32, (4, Ch)),
        ("y", y, io, act)])) + (batch, H, W, Ch, N, dt)
    ws, ws_bytes = _workspace(vim_scan_workspace_bytes(1, batch, H, W, Ch, N), workspace, u.device)
    tail = (None if ws is None else ws.data_ptr(), ws_bytes, _stream(stream))
    ev = None if events is None else _events(events)
    if ckpt is not None:
        (pk,) = _ptrs("vmamba_cross_scan4", u, [("ckpt", ckpt, f32, cross_ckpt_shape(batch, H, W, Ch, N))])
        st = lib.vmamba_cross_scan4_ckpt(*args[:9], pk, *args[9:], VIM_FLAG_ZOH_EXACT if zoh else 0, *tail, ev)
    elif zoh:
        st = lib.vmamba_cross_scan4_ex(*args, VIM_FLAG_ZOH_EXACT, *tail, ev)
    elif ev is None:
        st = lib.vmamba_cross_scan4(*args, *tail)
    else:
        st = lib.vmamba_cross_scan4_events(*args, *tail, ev)
    if st != VIM_OK:
        raise VimScanError(st, "vmamba_cross_scan4")
    return y


def cross_merge4(ys, z, H, W, *, y=None, stream=None):
    """CS-Merge alone: ys [4, batch, H*W, C] in scan order -> y [batch, H, W, C]."""
    _, batch, L, Ch = ys.shape
    if ys.shape[0] != 4 or L != H * W:
        raise ValueError("ys must be [4, batch, H*W, C]")
    act = (batch, H, W, Ch)
    dt = _dtype_code(ys)
    if y is None and isinstance(ys, torch.Tensor) and ys.is_cuda:
        y = torch.empty((batch, H, W, Ch), dtype=ys.dtype, device=ys.device)
    pys, pz, py = _ptrs("cross_merge4", ys, [("ys", ys, None, tuple(ys.shape)), ("z", z, ys.dtype, act),
                                             ("y", y, ys.dtype, act)])
    st = lib.cross_merge4(pys, pz, py, batch, H, W, Ch, dt, _stream(stream))
    if st != VIM_OK:
        raise VimScanError(st, "cross_merge4")
    return y


def vim_scan_host_workspace_bytes(batch, L, d_inner, d_state, dtype_code, slices, two_bc):
    return int(lib.vim_scan_host_workspace_bytes(batch, L, d_inner, d_state, dtype_code, slices, int(bool(two_bc))))


_copy_streams = {}


def _host_streams(device):
    """Two non-blocking streams per device for the host entry's uploads and downloads."""
    idx = device.index if device.index is not None else torch.cuda.current_device()
    if idx not in _copy_streams:
        _copy_streams[idx] = (torch.cuda.Stream(idx), torch.cuda.Stream(idx))
    return _copy_streams[idx]


def vim_scan_bidir_host(u, delta, z, B, C, A, D, delta_bias, *, y=None, bc_dir_stride=0, slices=4,
                        workspace=None, stream=None, upload=None, download=None, zoh=False):
    """vim_scan_bidir for activations in host memory; see include/vimscan.h.

    u, delta, z, B, C: CPU tensors shaped as for vim_scan_bidir (pinned memory lets the
    copies overlap the scan); A, D, delta_bias: CUDA tensors on the current device.
    Returns y, a CPU tensor (pinned when allocated here), complete once ``stream``
    (default: the current stream) has reached the end of the call.
    """
    if not all(isinstance(t, torch.Tensor) for t in (u, delta, B, C)):
        raise TypeError("vim_scan_bidir_host: u, delta, B and C must be tensors")
    batch, L, Di = u.shape
    N = B.shape[-1]
    dt = _dtype_code(u)
    act = (batch, L, Di)
    bc = _bc_rule(batch, L, N, bc_dir_stride)
    if y is None:
        y = torch.empty(act, dtype=u.dtype, pin_memory=True)
    for name, t, rule in (("u", u, act), ("delta", delta, act), ("z", z, act), ("B", B, bc), ("C", C, bc),
                          ("y", y, act)):
        if t is None:
            continue
        if not isinstance(t, torch.Tensor) or t.device.type != "cpu":
            raise TypeError(f"vim_scan_bidir_host: {name} must be a CPU tensor")
        if t.dtype != u.dtype:
            raise TypeError(f"vim_scan_bidir_host: {name} must be {u.dtype}, got {t.dtype}")
        if not t.is_contiguous():
            raise ValueError(f"vim_scan_bidir_host: {name} must be contiguous")
        if rule[0] == "numel":
            if t.numel() < rule[1] or t.dim() == 0 or t.shape[-1] != rule[2]:
                raise ValueError(f"vim_scan_bidir_host: {name} has shape {tuple(t.shape)}; it needs at least "
                                 f"{rule[1]} elements with last dimension {rule[2]}")
        elif t.shape != rule:
            raise ValueError(f"vim_scan_bidir_host: {name} has shape {tuple(t.shape)}, expected {rule}")
    f32 = torch.float32
    pA, pD, pbias = _ptrs("vim_scan_bidir_host", A, [("A", A, f32, (2, Di, N)), ("D", D, f32, (2, Di)),
                                                     ("delta_bias", delta_bias, f32, (2, Di))])
    dev = A.device
    nbytes = vim_scan_host_workspace_bytes(batch, L, Di, N, dt, slices, bc_dir_stride > 0)
    ws, ws_bytes = _workspace(nbytes, workspace, dev)
    if upload is None or download is None:
        up, down = _host_streams(dev)
        upload = upload or up
        download = download or down
    st = lib.vim_scan_bidir_host(
        u.data_ptr(), delta.data_ptr(), None if z is None else z.data_ptr(), B.data_ptr(), C.data_ptr(),
        int(bc_dir_stride), pA, pD, pbias, y.data_ptr(), batch, L, Di, N, dt,
        VIM_FLAG_ZOH_EXACT if zoh else 0, int(slices), None if ws is None else ws.data_ptr(), ws_bytes,
        _stream(stream), upload.cuda_stream, download.cuda_stream)
    if st != VIM_OK:
        raise VimScanError(st, "vim_scan_bidir_host")
    return y
