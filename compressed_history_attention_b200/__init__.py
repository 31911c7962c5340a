"""NanoKV compressed-history attention for B200 (sm_100a).

The work runs in libnanokv.so (hand-written CUDA kernels behind a C ABI, see
include/nanokv.h); this package is its thin Python binding plus the build
script and the arithmetic accounting used by the benchmark.
"""
from ._lib import (  # noqa: F401
    Codec, Hist, NanoKVError, alloc_hist, lib, nanokv_attend, nanokv_attend_workspace,
    nanokv_attend_static, nanokv_check, nanokv_encode, nanokv_lse_merge, nanokv_set_kernel_path,
    nanokv_timing_enable,
    nanokv_timing_read, nanokv_version, nanokv_selftest_wait, nanokv_attend_full_tokens,
    nanokv_attend_routed, nanokv_attend_routed_workspace, Lowdim, nanokv_lowdim_prepare,
    nanokv_lowdim_analytic, nanokv_calibrate, nanokv_attend_partial,
)
