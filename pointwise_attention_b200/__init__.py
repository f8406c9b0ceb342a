"""HSTU causal pointwise aggregated attention for NVIDIA B200 (sm_100a).

The computation lives in ``libhstu.so`` (CUDA kernels behind the C ABI of
``include/hstu.h``); this package is its thin Python binding.  Build the
library with ``python -m pointwise_attention_b200.build``.
"""
from ._binding import (EXPORTED, HSTUError, hstu_attn_bwd, hstu_attn_check, hstu_attn_fwd,
                       hstu_cand_fwd,
                       hstu_attn_workspace_size, hstu_out_fwd, hstu_problem_t,
                       hstu_selftest_wait_timeout, hstu_time_bucket_thresholds, hstu_uvqk_fwd,
                       load_library, make_problem, new_workspace, status_string)

__all__ = ["EXPORTED", "HSTUError", "hstu_attn_bwd", "hstu_attn_check", "hstu_attn_fwd",
           "hstu_cand_fwd",
           "hstu_attn_workspace_size", "hstu_out_fwd", "hstu_problem_t",
           "hstu_selftest_wait_timeout", "hstu_time_bucket_thresholds", "hstu_uvqk_fwd",
           "load_library", "make_problem", "new_workspace", "status_string"]
