"""MoE expert-parallel dispatch / combine on one B200 (sm_100a).

Hand-written CUDA kernels behind a C ABI (include/ep.h, libep_b200.so);
this package is the thin Python binding.  See ``ep.py``.
"""

from .ep import (EP_DEVERR_BAD_TOPK_IDX, EP_DEVERR_CAPACITY, EP_DEVERR_TIMEOUT, EP_X_BF16,
                 EP_X_BF16_TO_FP8, EP_X_BF16_TO_NVFP4, EP_X_FP8, EPError, EPHandle, combine,
                 combine_backward, combine_fp8, dispatch, dispatch_mn_scales, dispatch_with_handle,
                 get_layout, get_num_sms, lib, library_path, max_recv_rows, set_num_sms, sm_budget)
from . import mgpu

__all__ = ["mgpu", "EPHandle", "EPError", "get_layout", "dispatch", "dispatch_with_handle", "combine",
           "combine_backward", "combine_fp8", "dispatch_mn_scales",
           "max_recv_rows", "set_num_sms", "get_num_sms", "sm_budget", "lib", "library_path", "EP_X_BF16", "EP_X_FP8", "EP_X_BF16_TO_FP8",
           "EP_X_BF16_TO_NVFP4", "EP_DEVERR_BAD_TOPK_IDX", "EP_DEVERR_CAPACITY", "EP_DEVERR_TIMEOUT"]
