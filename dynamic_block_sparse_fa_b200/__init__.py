"""BLASST attention forward for NVIDIA B200 (sm_100a).

The kernels live in libblasst.so (C ABI: include/blasst.h); this package is
its Python binding.  Importing it loads the library and fails if it has not
been built (``python dynamic_block_sparse_fa_b200/build.py``).
"""
from .blasst import (BlasstError, Stats, blasst_calibrate,
                     blasst_check_device_error, blasst_decode,
                     blasst_decode_batched, blasst_decode_noalloc,
                     blasst_decode_paged,
                     blasst_decode_group_splits,
                     blasst_decode_splits, blasst_decode_wide,
                     blasst_decode_wide_splits, blasst_decode_window,
                     blasst_decode_workspace_size,
                     blasst_fit_a, blasst_last_error, blasst_mla_decode,
                     blasst_mla_decode_splits,
                     blasst_mla_decode_workspace_size, blasst_prefill,
                     blasst_prefill_backward,
                     blasst_prefill_backward_workspace_size,
                     blasst_prefill_window,
                     blasst_selftest_wait_timeout, blasst_skip_stats_reset,
                     blasst_strerror, blasst_version)

__all__ = ["BlasstError", "Stats", "blasst_calibrate",
           "blasst_check_device_error", "blasst_decode",
           "blasst_decode_batched", "blasst_decode_noalloc",
           "blasst_decode_paged",
           "blasst_decode_group_splits",
           "blasst_decode_splits", "blasst_decode_wide",
           "blasst_decode_wide_splits", "blasst_decode_window",
           "blasst_decode_workspace_size", "blasst_fit_a", "blasst_last_error",
           "blasst_mla_decode", "blasst_mla_decode_splits",
           "blasst_mla_decode_workspace_size",
           "blasst_prefill", "blasst_prefill_backward",
           "blasst_prefill_backward_workspace_size", "blasst_prefill_window",
           "blasst_selftest_wait_timeout",
           "blasst_skip_stats_reset", "blasst_strerror",
           "blasst_version"]
