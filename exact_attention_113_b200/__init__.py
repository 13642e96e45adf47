"""B200-native exact attention forward (sm_100a: tcgen05 / TMEM / TMA).

The compute path is libfa.so (C ABI in include/fa.h); this package holds its
sources (csrc/), its build step (build.py), the ctypes binding (binding.py)
and the seeded input generator (inputs.py).
"""
from .binding import (FA_BF16, FA_F16, FaError, choose_splits, fa_bwd, fa_bwd_ex,
                      fa_bwd_workspace_bytes,
                      fa_fwd, fa_fwd_ex, fa_fwd_fp8, fa_fwd_fp8_ex, fa_fwd_fp8_splitkv,
                      fa_fwd_host, fa_fwd_host_workspace_bytes,
                      fa_fwd_splitkv, fa_fwd_splitkv_static, fa_get_device_status,
                      fa_selftest_wait_timeout, fa_splitkv_workspace_bytes, fa_version,
                      flash_bwd, flash_fwd, flash_fwd_fp8, flash_fwd_host, load,
                      selftest_wait_timeout, status_string)

__all__ = ["FA_BF16", "FA_F16", "FaError", "choose_splits", "fa_bwd", "fa_bwd_ex",
           "fa_bwd_workspace_bytes",
           "fa_fwd", "fa_fwd_ex", "fa_fwd_fp8", "fa_fwd_fp8_ex", "fa_fwd_fp8_splitkv",
           "fa_fwd_host", "fa_fwd_host_workspace_bytes",
           "fa_fwd_splitkv", "fa_fwd_splitkv_static", "fa_get_device_status",
           "fa_selftest_wait_timeout", "fa_splitkv_workspace_bytes", "fa_version", "flash_bwd",
           "flash_fwd", "flash_fwd_fp8", "flash_fwd_host", "load", "selftest_wait_timeout",
           "status_string"]
