"""B200-native selective scan (S6) for Vision Mamba and VMamba.

The compute lives in ``libvimscan.so`` (hand-written sm_100a CUDA behind a C ABI,
declared in ``include/vimscan.h``); ``vision_mamba_selective_b200.vimscan`` is the thin
ctypes binding with the same names.  Importing the package itself loads nothing, so
that the seeded input generators (``workloads``) can be used on machines without a
GPU; the first use of a scan entry point loads the library and fails loudly if it is
missing.
"""

__all__ = ["vim_scan_bidir", "vmamba_cross_scan4", "cross_merge4", "vim_scan_workspace_bytes",
           "vim_scan_bidir_conv", "vim_scan_bidir_bwd", "vim_scan_bwd_workspace_bytes", "vim_block_scan",
           "vim_block_workspace_bytes", "vim_scan_bidir_noalloc"]


def __getattr__(name):
    if name in __all__:
        from . import vimscan

        return getattr(vimscan, name)
    raise AttributeError(name)
