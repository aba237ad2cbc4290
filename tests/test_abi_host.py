"""The C ABI without a GPU: the library loads, exports every declared symbol, and
rejects bad arguments on the host before anything is launched.

Every call below fails a host-side check (or is a size-0 no-op), so none of them
reaches a kernel launch; that keeps these tests safe on a machine with a GPU too.
"""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "vimscan.h")


@pytest.fixture(scope="module")
def vs():
    from vision_mamba_selective_b200 import build

    build.build()
    from vision_mamba_selective_b200 import vimscan

    return vimscan


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^\s*(?:vim_status|size_t|const char \*)\s*\*?\s*(\w+)\s*\(", text, flags=re.M)


def test_header_declares_the_boundary():
    names = declared_functions()
    assert set(names) == {"vim_scan_bidir", "vmamba_cross_scan4", "cross_merge4",
                          "vim_scan_bidir_events", "vmamba_cross_scan4_events", "vim_scan_bidir_noalloc", "vim_scan_bidir_conv", "vim_scan_bidir_conv_events",
                          "vim_scan_bidir_ex", "vmamba_cross_scan4_ex",
                          "vim_scan_bidir_bwd", "vim_scan_bwd_workspace_bytes", "vim_scan_bidir_bwd_events",
                          "vim_scan_bidir_bwd_ex",
                          "vim_block_scan", "vim_block_workspace_bytes",
                          "vmamba_cross_scan4_bwd", "vmamba_cross_scan4_bwd_workspace_bytes",
                          "vmamba_cross_scan4_bwd_ex",
                          "vim_scan_bidir_host", "vim_scan_host_workspace_bytes",
                          "vim_scan_bidir_conv_bwd", "vim_scan_bidir_conv_bwd_ex", "vim_scan_conv_bwd_workspace_bytes",
                          "vim_block_scan_bwd", "vim_block_bwd_workspace_bytes",
                          "vim_scan_bidir_ckpt", "vim_scan_bidir_bwd_ckpt", "vim_scan_ckpt_bytes",
                          "vim_scan_bidir_conv_ckpt", "vim_scan_bidir_conv_bwd_ckpt",
                          "vmamba_cross_scan4_ckpt", "vmamba_cross_scan4_bwd_ckpt", "vmamba_cross_ckpt_bytes",
                          "vim_scan_workspace_bytes", "vim_status_string"}, names


def test_header_compiles_as_c():
    subprocess.run(["gcc", "-fsyntax-only", "-x", "c", "-std=c99", "-I/usr/local/cuda/include", HEADER],
                   check=True)


def test_exports_every_symbol(vs):
    out = subprocess.run(["nm", "-D", "--defined-only", vs.LIB_PATH], check=True,
                         capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(vs.lib, name)


def test_status_strings(vs):
    for code in range(6):
        s = vs.status_string(code)
        assert isinstance(s, str) and s
    assert vs.status_string(0) == "ok"
    assert "unknown" in vs.status_string(99)


def test_workspace_bytes(vs):
    assert vs.vim_scan_workspace_bytes(0, 64, 197, 0, 768, 16) == 0          # one chunk
    n = vs.vim_scan_workspace_bytes(0, 8, 4097, 0, 384, 16)
    G = (4097 + 127) // 128
    assert n >= 8 * G * 2 * 384 * 17 * 4 and n % 256 == 0
    m = vs.vim_scan_workspace_bytes(1, 16, 64, 64, 192, 16)
    assert m >= 16 * 4096 * 192 * 4 + 16 * 32 * 2 * 192 * 17 * 4
    assert vs.vim_scan_workspace_bytes(0, 1, 100, 0, 8, 3) == 0               # unsupported N
    assert vs.vim_scan_workspace_bytes(7, 1, 100, 0, 8, 16) == 0              # unknown kind


FAKE = 0x7f0000000000   # 256-byte aligned, never dereferenced: every call fails a check first


def bidir(vs, **kw):
    a = dict(u=FAKE, delta=FAKE, z=FAKE, B=FAKE, C=FAKE, stride=0, A=FAKE, D=FAKE, bias=FAKE, y=FAKE,
             batch=2, L=33, Di=64, N=16, dt=vs.VIM_BF16, ws=None, ws_bytes=0)
    a.update(kw)
    return vs.lib.vim_scan_bidir(a["u"], a["delta"], a["z"], a["B"], a["C"], a["stride"], a["A"],
                                 a["D"], a["bias"], a["y"], a["batch"], a["L"], a["Di"], a["N"],
                                 a["dt"], a["ws"], a["ws_bytes"], None)


def test_bidir_rejects(vs):
    assert bidir(vs, u=None) == vs.VIM_ERR_INVALID_ARG
    assert bidir(vs, y=None) == vs.VIM_ERR_INVALID_ARG
    assert bidir(vs, A=None) == vs.VIM_ERR_INVALID_ARG
    assert bidir(vs, u=FAKE + 8) == vs.VIM_ERR_INVALID_ARG            # not 16-byte aligned
    assert bidir(vs, z=FAKE + 2) == vs.VIM_ERR_INVALID_ARG
    assert bidir(vs, B=FAKE + 1) == vs.VIM_ERR_INVALID_ARG            # not element aligned
    assert bidir(vs, D=FAKE + 2) == vs.VIM_ERR_INVALID_ARG
    assert bidir(vs, batch=-1) == vs.VIM_ERR_INVALID_ARG
    assert bidir(vs, L=-5) == vs.VIM_ERR_INVALID_ARG
    assert bidir(vs, stride=-1) == vs.VIM_ERR_INVALID_ARG
    assert bidir(vs, dt=7) == vs.VIM_ERR_INVALID_ARG
    assert bidir(vs, N=3) == vs.VIM_ERR_UNSUPPORTED
    assert bidir(vs, N=32) == vs.VIM_ERR_UNSUPPORTED
    assert bidir(vs, Di=12) == vs.VIM_ERR_UNSUPPORTED                 # bf16 needs multiples of 8
    assert bidir(vs, Di=6, dt=vs.VIM_F32) == vs.VIM_ERR_UNSUPPORTED   # fp32 needs multiples of 4
    # long sequences need the caller's workspace
    assert bidir(vs, L=4097, ws=None) == vs.VIM_ERR_WORKSPACE
    assert bidir(vs, L=4097, ws=FAKE, ws_bytes=16) == vs.VIM_ERR_WORKSPACE
    assert bidir(vs, L=4097, ws=FAKE + 16, ws_bytes=1 << 40) == vs.VIM_ERR_WORKSPACE


def host(vs, **kw):
    """vim_scan_bidir_host on fake addresses; every case below fails a host check (or is
    an empty problem), before any CUDA call."""
    a = dict(u=FAKE, delta=FAKE, z=FAKE, B=FAKE, C=FAKE, stride=0, A=FAKE, D=FAKE, bias=FAKE, y=FAKE,
             batch=8, L=4097, Di=384, N=16, dt=vs.VIM_BF16, flags=0, slices=8, ws=FAKE, ws_bytes=1 << 40)
    a.update(kw)
    return vs.lib.vim_scan_bidir_host(a["u"], a["delta"], a["z"], a["B"], a["C"], a["stride"], a["A"], a["D"],
                                      a["bias"], a["y"], a["batch"], a["L"], a["Di"], a["N"], a["dt"], a["flags"],
                                      a["slices"], a["ws"], a["ws_bytes"], None, None, None)


def test_host_entry_rejects(vs):
    assert host(vs, u=None) == vs.VIM_ERR_INVALID_ARG
    assert host(vs, y=None) == vs.VIM_ERR_INVALID_ARG
    assert host(vs, A=None) == vs.VIM_ERR_INVALID_ARG
    assert host(vs, D=FAKE + 2) == vs.VIM_ERR_INVALID_ARG             # parameters are fp32 on the device
    assert host(vs, slices=0) == vs.VIM_ERR_INVALID_ARG
    assert host(vs, stride=-1) == vs.VIM_ERR_INVALID_ARG
    assert host(vs, flags=4) == vs.VIM_ERR_INVALID_ARG
    assert host(vs, N=3) == vs.VIM_ERR_UNSUPPORTED
    assert host(vs, Di=12) == vs.VIM_ERR_UNSUPPORTED
    assert host(vs, ws=None) == vs.VIM_ERR_WORKSPACE
    assert host(vs, ws_bytes=1024) == vs.VIM_ERR_WORKSPACE
    assert host(vs, ws=FAKE + 16) == vs.VIM_ERR_WORKSPACE
    assert host(vs, batch=0, ws=None) == vs.VIM_OK                    # empty: nothing to do
    assert host(vs, L=0, u=None, ws=None) == vs.VIM_OK


def conv_bwd(vs, **kw):
    """vim_scan_bidir_conv_bwd_ex on fake device addresses; every case fails a host check."""
    a = dict(x=FAKE, cw=FAKE, cb=FAKE, delta=FAKE, z=FAKE, B=FAKE, C=FAKE, stride=0, A=FAKE, D=FAKE, bias=FAKE,
             dout=FAKE, dx=FAKE, dcw=FAKE, dcb=FAKE, ddelta=FAKE, dz=FAKE, dB=FAKE, dC=FAKE, dA=FAKE, dD=FAKE,
             dbias=FAKE, batch=2, L=100, Di=64, N=16, dt=vs.VIM_BF16, flags=0, ws=FAKE, ws_bytes=1 << 40)
    a.update(kw)
    return vs.lib.vim_scan_bidir_conv_bwd_ex(
        a["x"], a["cw"], a["cb"], a["delta"], a["z"], a["B"], a["C"], a["stride"], a["A"], a["D"], a["bias"],
        a["dout"], a["dx"], a["dcw"], a["dcb"], a["ddelta"], a["dz"], a["dB"], a["dC"], a["dA"], a["dD"], a["dbias"],
        a["batch"], a["L"], a["Di"], a["N"], a["dt"], a["flags"], a["ws"], a["ws_bytes"], None)


def test_conv_bwd_rejects(vs):
    assert conv_bwd(vs, x=None) == vs.VIM_ERR_INVALID_ARG
    assert conv_bwd(vs, cw=None) == vs.VIM_ERR_INVALID_ARG
    assert conv_bwd(vs, dcb=None) == vs.VIM_ERR_INVALID_ARG
    assert conv_bwd(vs, dx=None) == vs.VIM_ERR_INVALID_ARG
    assert conv_bwd(vs, z=None) == vs.VIM_ERR_INVALID_ARG                 # dz without z
    assert conv_bwd(vs, cw=FAKE + 2) == vs.VIM_ERR_INVALID_ARG
    assert conv_bwd(vs, x=FAKE + 8) == vs.VIM_ERR_INVALID_ARG             # not 16-byte aligned
    assert conv_bwd(vs, flags=2) == vs.VIM_ERR_INVALID_ARG
    assert conv_bwd(vs, stride=-1) == vs.VIM_ERR_INVALID_ARG
    assert conv_bwd(vs, N=3) == vs.VIM_ERR_UNSUPPORTED
    assert conv_bwd(vs, ws=None) == vs.VIM_ERR_WORKSPACE
    assert conv_bwd(vs, ws_bytes=4096) == vs.VIM_ERR_WORKSPACE
    assert conv_bwd(vs, ws=FAKE + 16) == vs.VIM_ERR_WORKSPACE
    f = vs.vim_scan_conv_bwd_workspace_bytes
    n = f(8, 4097, 384, 16, vs.VIM_BF16, False)
    assert n % 256 == 0 and n > vs.vim_scan_bwd_workspace_bytes(8, 4097, 384, 16, False) + 4 * 8 * 4097 * 384 * 4
    assert f(8, 4097, 384, 16, vs.VIM_BF16, True) > n
    assert f(0, 4097, 384, 16, vs.VIM_BF16, False) == 0 and f(8, 4097, 384, 5, vs.VIM_BF16, False) == 0


def test_block_bwd_rejects(vs):
    f = vs.lib.vim_block_scan_bwd

    def call(**kw):
        a = dict(x=FAKE, cw=FAKE, cb=FAKE, Wx=FAKE, Wdt=FAKE, bias=FAKE, A=FAKE, D=FAKE, z=FAKE, dout=FAKE, dx=FAKE,
                 dcw=FAKE, dcb=FAKE, dWx=FAKE, dWdt=FAKE, dbias=FAKE, dA=FAKE, dD=FAKE, dz=FAKE, batch=2, L=100, Di=64,
                 N=16, dt=vs.VIM_BF16, ws=FAKE, ws_bytes=1 << 40)
        a.update(kw)
        return f(a["x"], a["cw"], a["cb"], a["Wx"], a["Wdt"], a["bias"], a["A"], a["D"], a["z"], a["dout"], a["dx"],
                 a["dcw"], a["dcb"], a["dWx"], a["dWdt"], a["dbias"], a["dA"], a["dD"], a["dz"], a["batch"], a["L"],
                 a["Di"], a["N"], a["dt"], a["ws"], a["ws_bytes"], None)

    assert call(dt=vs.VIM_F32) == vs.VIM_ERR_UNSUPPORTED
    assert call(cw=None) == vs.VIM_ERR_INVALID_ARG                      # one of the front's two
    assert call(dcb=None) == vs.VIM_ERR_INVALID_ARG                     # front given, its derivative not
    assert call(z=None) == vs.VIM_ERR_INVALID_ARG                       # dz without z
    assert call(Wx=FAKE + 1) == vs.VIM_ERR_INVALID_ARG
    assert call(x=FAKE + 8) == vs.VIM_ERR_INVALID_ARG
    assert call(dWx=None) == vs.VIM_ERR_INVALID_ARG
    assert call(N=3) == vs.VIM_ERR_UNSUPPORTED
    assert call(ws=None) == vs.VIM_ERR_WORKSPACE
    assert call(ws_bytes=1024) == vs.VIM_ERR_WORKSPACE
    n = vs.vim_block_bwd_workspace_bytes(8, 4097, 384, 16)
    assert n % 256 == 0 and n > vs.vim_scan_bwd_workspace_bytes(8, 4097, 384, 16, True)
    assert vs.vim_block_bwd_workspace_bytes(0, 4097, 384, 16) == 0


def test_host_workspace_bytes(vs):
    f = vs.vim_scan_host_workspace_bytes
    one = f(8, 4097, 384, 16, vs.VIM_BF16, 8, False)
    act = 4097 * 384 * 2                                  # one batch item of u (bf16)
    assert one % 256 == 0 and one >= 2 * (4 * act + 2 * 4097 * 16 * 2) + vs.vim_scan_workspace_bytes(0, 1, 4097, 0, 384, 16)
    assert f(8, 4097, 384, 16, vs.VIM_BF16, 8, True) > one            # two copies of B and C
    assert f(8, 4097, 384, 16, vs.VIM_BF16, 64, False) == one         # at most one piece per batch item
    assert f(8, 4097, 384, 16, vs.VIM_BF16, 2, False) > one           # larger pieces
    assert f(8, 4097, 384, 16, vs.VIM_BF16, 0, False) == 0
    assert f(0, 4097, 384, 16, vs.VIM_BF16, 8, False) == 0
    assert f(8, 4097, 384, 3, vs.VIM_BF16, 8, False) == 0


def bwd(vs, **kw):
    """vim_scan_bidir_bwd on fake device addresses; every case below fails a host check."""
    a = dict(u=FAKE, delta=FAKE, z=FAKE, B=FAKE, C=FAKE, stride=0, A=FAKE, D=FAKE, bias=FAKE, dout=FAKE,
             du=FAKE, ddelta=FAKE, dz=FAKE, dB=FAKE, dC=FAKE, dA=FAKE, dD=FAKE, dbias=FAKE,
             batch=2, L=100, Di=64, N=16, dt=vs.VIM_BF16, ws=FAKE, ws_bytes=1 << 40)
    a.update(kw)
    return vs.lib.vim_scan_bidir_bwd(a["u"], a["delta"], a["z"], a["B"], a["C"], a["stride"], a["A"], a["D"],
                                     a["bias"], a["dout"], a["du"], a["ddelta"], a["dz"], a["dB"], a["dC"],
                                     a["dA"], a["dD"], a["dbias"], a["batch"], a["L"], a["Di"], a["N"],
                                     a["dt"], a["ws"], a["ws_bytes"], None)


def bwd_ex(vs, flags, **kw):
    """vim_scan_bidir_bwd_ex on fake device addresses (each case fails a host check)."""
    a = dict(u=FAKE, delta=FAKE, z=FAKE, B=FAKE, C=FAKE, stride=0, A=FAKE, D=FAKE, bias=FAKE, dout=FAKE,
             du=FAKE, ddelta=FAKE, dz=FAKE, dB=FAKE, dC=FAKE, dA=FAKE, dD=FAKE, dbias=FAKE,
             batch=2, L=100, Di=64, N=16, dt=vs.VIM_BF16, ws=FAKE, ws_bytes=1 << 40)
    a.update(kw)
    return vs.lib.vim_scan_bidir_bwd_ex(a["u"], a["delta"], a["z"], a["B"], a["C"], a["stride"], a["A"], a["D"],
                                        a["bias"], a["dout"], a["du"], a["ddelta"], a["dz"], a["dB"], a["dC"],
                                        a["dA"], a["dD"], a["dbias"], a["batch"], a["L"], a["Di"], a["N"],
                                        a["dt"], flags, a["ws"], a["ws_bytes"], None, None)


def bwd_ckpt(vs, flags, **kw):
    """vim_scan_bidir_bwd_ckpt on fake device addresses (each case fails a host check)."""
    a = dict(u=FAKE, delta=FAKE, z=FAKE, B=FAKE, C=FAKE, stride=0, A=FAKE, D=FAKE, bias=FAKE, ckpt=FAKE,
             dout=FAKE, du=FAKE, ddelta=FAKE, dz=FAKE, dB=FAKE, dC=FAKE, dA=FAKE, dD=FAKE, dbias=FAKE,
             batch=2, L=100, Di=64, N=16, dt=vs.VIM_BF16, ws=FAKE, ws_bytes=1 << 40)
    a.update(kw)
    return vs.lib.vim_scan_bidir_bwd_ckpt(a["u"], a["delta"], a["z"], a["B"], a["C"], a["stride"], a["A"],
                                          a["D"], a["bias"], a["ckpt"], a["dout"], a["du"], a["ddelta"], a["dz"],
                                          a["dB"], a["dC"], a["dA"], a["dD"], a["dbias"], a["batch"], a["L"],
                                          a["Di"], a["N"], a["dt"], flags, a["ws"], a["ws_bytes"], None, None)


def fwd_ckpt(vs, flags, **kw):
    """vim_scan_bidir_ckpt on fake device addresses (each case fails a host check)."""
    a = dict(u=FAKE, delta=FAKE, z=FAKE, B=FAKE, C=FAKE, stride=0, A=FAKE, D=FAKE, bias=FAKE, y=FAKE, ckpt=FAKE,
             batch=2, L=100, Di=64, N=16, dt=vs.VIM_BF16, ws=FAKE, ws_bytes=1 << 40)
    a.update(kw)
    return vs.lib.vim_scan_bidir_ckpt(a["u"], a["delta"], a["z"], a["B"], a["C"], a["stride"], a["A"], a["D"],
                                      a["bias"], a["y"], a["ckpt"], a["batch"], a["L"], a["Di"], a["N"], a["dt"],
                                      flags, a["ws"], a["ws_bytes"], None, None)


def test_ckpt_pair_rejects(vs):
    # the checkpoints are required, 8-byte aligned; the rest is checked as without them
    assert fwd_ckpt(vs, 0, ckpt=None) == vs.VIM_ERR_INVALID_ARG
    assert fwd_ckpt(vs, 0, ckpt=FAKE + 4) == vs.VIM_ERR_INVALID_ARG
    assert fwd_ckpt(vs, 2) == vs.VIM_ERR_INVALID_ARG                  # unknown flag bit
    assert fwd_ckpt(vs, 0, N=3) == vs.VIM_ERR_UNSUPPORTED
    assert fwd_ckpt(vs, vs.VIM_FLAG_ZOH_EXACT, ws=None) == vs.VIM_ERR_WORKSPACE
    assert bwd_ckpt(vs, 0, ckpt=None) == vs.VIM_ERR_INVALID_ARG
    assert bwd_ckpt(vs, 0, ckpt=FAKE + 4) == vs.VIM_ERR_INVALID_ARG
    assert bwd_ckpt(vs, 2) == vs.VIM_ERR_INVALID_ARG
    assert bwd_ckpt(vs, 0, dz=None) == vs.VIM_ERR_INVALID_ARG
    assert bwd_ckpt(vs, vs.VIM_FLAG_ZOH_EXACT, ws=None) == vs.VIM_ERR_WORKSPACE
    # [batch][ceil(L / 32)][2][d_state][d_inner] fp32
    assert vs.lib.vim_scan_ckpt_bytes(2, 100, 64, 16) == 2 * 4 * 2 * 64 * 16 * 4
    assert vs.lib.vim_scan_ckpt_bytes(8, 4097, 384, 16) == 8 * 129 * 2 * 384 * 16 * 4
    assert vs.lib.vim_scan_ckpt_bytes(0, 100, 64, 16) == 0
    assert vs.lib.vim_scan_ckpt_bytes(2, 100, 64, 3) == 0
    assert vs.ckpt_shape(2, 100, 64, 16) == (2, 4, 2, 16, 64)


def test_conv_ckpt_pair_rejects(vs):
    lib, F = vs.lib, FAKE
    fwd = lambda ckpt=F, cw=F, ws=F: lib.vim_scan_bidir_conv_ckpt(F, cw, F, F, F, F, F, 0, F, F, F, F, ckpt, 2, 100,
                                                                   64, 16, vs.VIM_BF16, 0, ws, 1 << 40, None, None)
    assert fwd(ckpt=None) == vs.VIM_ERR_INVALID_ARG
    assert fwd(cw=None) == vs.VIM_ERR_INVALID_ARG          # the front is required
    assert fwd(ckpt=F + 4) == vs.VIM_ERR_INVALID_ARG
    assert fwd(ws=None) == vs.VIM_ERR_WORKSPACE
    bwd = lambda ckpt=F, ws=F: lib.vim_scan_bidir_conv_bwd_ckpt(F, F, F, F, F, F, F, 0, F, F, F, ckpt, F, F, F, F, F,
                                                                F, F, F, F, F, F, 2, 100, 64, 16, vs.VIM_BF16, 0,
                                                                ws, 1 << 40, None)
    assert bwd(ckpt=None) == vs.VIM_ERR_INVALID_ARG
    assert bwd(ckpt=F + 4) == vs.VIM_ERR_INVALID_ARG
    assert bwd(ws=None) == vs.VIM_ERR_WORKSPACE


def test_cross_ckpt_pair_rejects(vs):
    lib, F = vs.lib, FAKE
    fwd = lambda ckpt=F, ws=F: lib.vmamba_cross_scan4_ckpt(F, F, F, F, F, F, F, F, F, ckpt, 2, 8, 8, 64, 16,
                                                            vs.VIM_BF16, 0, ws, 1 << 40, None, None)
    assert fwd(ckpt=None) == vs.VIM_ERR_INVALID_ARG
    assert fwd(ckpt=F + 4) == vs.VIM_ERR_INVALID_ARG
    assert fwd(ws=None) == vs.VIM_ERR_WORKSPACE
    bwd = lambda ckpt=F, ws=F: lib.vmamba_cross_scan4_bwd_ckpt(F, F, F, F, F, F, F, F, ckpt, F, F, F, F, F, F, F, F,
                                                                F, 2, 8, 8, 64, 16, vs.VIM_BF16, 0, ws, 1 << 40, None)
    assert bwd(ckpt=None) == vs.VIM_ERR_INVALID_ARG
    assert bwd(ckpt=F + 4) == vs.VIM_ERR_INVALID_ARG
    assert bwd(ws=None) == vs.VIM_ERR_WORKSPACE
    assert lib.vmamba_cross_ckpt_bytes(2, 8, 8, 64, 16) == 2 * 2 * 2 * 2 * 16 * 64 * 4
    assert lib.vmamba_cross_ckpt_bytes(0, 8, 8, 64, 16) == 0
    assert vs.cross_ckpt_shape(2, 8, 8, 64, 16) == (2, 2, 2, 2, 16, 64)


def test_bwd_ex_rejects(vs):
    assert bwd_ex(vs, 2) == vs.VIM_ERR_INVALID_ARG                  # unknown flag bit
    assert bwd_ex(vs, vs.VIM_FLAG_ZOH_EXACT | 4) == vs.VIM_ERR_INVALID_ARG
    assert bwd_ex(vs, vs.VIM_FLAG_ZOH_EXACT, N=3) == vs.VIM_ERR_UNSUPPORTED
    assert bwd_ex(vs, vs.VIM_FLAG_ZOH_EXACT, dz=None) == vs.VIM_ERR_INVALID_ARG
    assert bwd_ex(vs, vs.VIM_FLAG_ZOH_EXACT, ws=None) == vs.VIM_ERR_WORKSPACE


def test_bwd_rejects(vs):
    assert bwd(vs, dz=None) == vs.VIM_ERR_INVALID_ARG              # z given, dz missing
    assert bwd(vs, z=None) == vs.VIM_ERR_INVALID_ARG               # dz given, z missing
    assert bwd(vs, A=None) == vs.VIM_ERR_INVALID_ARG
    assert bwd(vs, dA=FAKE + 2) == vs.VIM_ERR_INVALID_ARG
    assert bwd(vs, u=FAKE + 8) == vs.VIM_ERR_INVALID_ARG
    assert bwd(vs, dout=None) == vs.VIM_ERR_INVALID_ARG
    assert bwd(vs, dB=FAKE + 2) == vs.VIM_ERR_INVALID_ARG
    assert bwd(vs, stride=-3) == vs.VIM_ERR_INVALID_ARG
    assert bwd(vs, N=3) == vs.VIM_ERR_UNSUPPORTED
    assert bwd(vs, Di=12) == vs.VIM_ERR_UNSUPPORTED
    assert bwd(vs, ws=None) == vs.VIM_ERR_WORKSPACE
    assert bwd(vs, ws_bytes=64) == vs.VIM_ERR_WORKSPACE
    assert bwd(vs, ws=FAKE + 16) == vs.VIM_ERR_WORKSPACE
    # the workspace grows with the sequence and with separate B/C
    small = vs.vim_scan_bwd_workspace_bytes(2, 100, 64, 16, False)
    assert 0 < small < vs.vim_scan_bwd_workspace_bytes(2, 1000, 64, 16, False)
    assert small < vs.vim_scan_bwd_workspace_bytes(2, 100, 64, 16, True)
    assert vs.vim_scan_bwd_workspace_bytes(0, 100, 64, 16, False) == 0


def test_cross_bwd_and_block_reject(vs):
    lib = vs.lib
    F = FAKE
    # cross-scan derivative: z without dz, unsupported d_state, missing workspace
    args = [F] * 17 + [2, 8, 8, 64, 16, vs.VIM_BF16, F, 1 << 40, None]
    def xb(**kw):
        a = list(args)
        for i, v in kw.items():
            a[int(i[1:])] = v
        return lib.vmamba_cross_scan4_bwd(*a)
    assert xb(a11=None) == vs.VIM_ERR_INVALID_ARG             # dz missing while z is given
    assert xb(a5=None) == vs.VIM_ERR_INVALID_ARG              # A
    assert xb(a0=F + 8) == vs.VIM_ERR_INVALID_ARG             # u not 16-byte aligned
    assert xb(a21=3) == vs.VIM_ERR_UNSUPPORTED                # d_state
    assert xb(a23=None) == vs.VIM_ERR_WORKSPACE
    assert xb(a23=F + 16) == vs.VIM_ERR_WORKSPACE
    assert vs.lib.vmamba_cross_scan4_bwd_workspace_bytes(2, 8, 8, 64, 16) > 0
    # the options entry: an unknown flag bit is refused; the exact hold's flag passes the
    # flag check and stops at the missing workspace (no call here reaches a launch)
    ex = lambda flags, ws: lib.vmamba_cross_scan4_bwd_ex(*(args[:23] + [flags, ws] + args[24:]))
    assert ex(2, F) == vs.VIM_ERR_INVALID_ARG
    assert ex(vs.VIM_FLAG_ZOH_EXACT, None) == vs.VIM_ERR_WORKSPACE
    # block scan: fp32 unsupported, half a convolution front, missing weights
    def blk(**kw):
        a = dict(x=F, cw=F, cb=F, Wx=F, Wdt=F, db=F, A=F, D=F, z=F, y=F, b=2, L=100, Di=64, N=16,
                 dt=vs.VIM_BF16, ws=F, wsb=1 << 40)
        a.update(kw)
        return lib.vim_block_scan(a["x"], a["cw"], a["cb"], a["Wx"], a["Wdt"], a["db"], a["A"], a["D"], a["z"],
                                  a["y"], a["b"], a["L"], a["Di"], a["N"], a["dt"], a["ws"], a["wsb"], None, None)
    assert blk(dt=vs.VIM_F32) == vs.VIM_ERR_UNSUPPORTED
    assert blk(cb=None) == vs.VIM_ERR_INVALID_ARG
    assert blk(Wx=None) == vs.VIM_ERR_INVALID_ARG
    assert blk(x=F + 8) == vs.VIM_ERR_INVALID_ARG
    assert blk(Di=3000) == vs.VIM_ERR_UNSUPPORTED             # Wx^T would not fit in shared memory
    assert blk(ws=None) == vs.VIM_ERR_WORKSPACE
    # the workspace holds B, C (bf16), s (fp32) and, with the front, both pathways' u (bf16)
    M, N, Di = 2 * 100, 16, 64
    need = vs.vim_block_workspace_bytes(2, 100, Di, N)
    assert need >= 2 * (2 * M * N * 2) + 2 * M * 4 + 2 * M * Di * 2
    assert blk(wsb=need - 1) == vs.VIM_ERR_WORKSPACE          # with the front: one byte short


def test_size_zero_is_a_noop(vs):
    # nothing is read or launched, so even null pointers are fine
    assert bidir(vs, batch=0, u=None, y=None) == vs.VIM_OK
    assert bidir(vs, L=0, u=None) == vs.VIM_OK
    assert bidir(vs, Di=0, u=None) == vs.VIM_OK
    assert vs.lib.cross_merge4(None, None, None, 0, 4, 4, 8, vs.VIM_BF16, None) == vs.VIM_OK


def test_cross4_rejects(vs):
    f = vs.lib.vmamba_cross_scan4

    def call(**kw):
        a = dict(u=FAKE, delta=FAKE, z=None, B=FAKE, C=FAKE, A=FAKE, D=FAKE, bias=FAKE, y=FAKE,
                 batch=2, H=8, W=8, ch=64, N=16, dt=vs.VIM_BF16, ws=None, ws_bytes=0)
        a.update(kw)
        return f(a["u"], a["delta"], a["z"], a["B"], a["C"], a["A"], a["D"], a["bias"], a["y"],
                 a["batch"], a["H"], a["W"], a["ch"], a["N"], a["dt"], a["ws"], a["ws_bytes"], None)

    assert call(u=None) == vs.VIM_ERR_INVALID_ARG
    assert call(H=-1) == vs.VIM_ERR_INVALID_ARG
    assert call(N=5) == vs.VIM_ERR_UNSUPPORTED
    assert call() == vs.VIM_ERR_WORKSPACE            # the merge always needs the fp32 partial
    assert call(ws=FAKE + 128, ws_bytes=1 << 40) == vs.VIM_ERR_WORKSPACE
    assert call(H=0) == vs.VIM_OK


def test_merge_rejects(vs):
    f = vs.lib.cross_merge4
    assert f(None, None, FAKE, 1, 4, 4, 8, vs.VIM_BF16, None) == vs.VIM_ERR_INVALID_ARG
    assert f(FAKE, None, None, 1, 4, 4, 8, vs.VIM_BF16, None) == vs.VIM_ERR_INVALID_ARG
    assert f(FAKE + 4, None, FAKE, 1, 4, 4, 8, vs.VIM_BF16, None) == vs.VIM_ERR_INVALID_ARG
    assert f(FAKE, None, FAKE, 1, 4, 4, 6, vs.VIM_BF16, None) == vs.VIM_ERR_UNSUPPORTED
    assert f(FAKE, None, FAKE, -1, 4, 4, 8, vs.VIM_BF16, None) == vs.VIM_ERR_INVALID_ARG


def test_binding_refuses_cpu_tensors(vs):
    import torch

    x = torch.zeros(1, 4, 8)
    with pytest.raises(TypeError):
        vs.vim_scan_bidir(x, x, x, torch.zeros(1, 4, 2), torch.zeros(1, 4, 2), torch.zeros(2, 8, 2),
                          torch.zeros(2, 8), torch.zeros(2, 8), y=torch.zeros(1, 4, 8))
