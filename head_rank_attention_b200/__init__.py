"""B200-native (sm_100a) decode and prefill over a compressed latent KV cache.

MLA (one branch) and MLRA (2 or 4 branches) decode, and causal multi-token prefill in the
expanded form, behind the C ABI of libhra.so
(include/hra.h); this package is the thin Python binding of that ABI, plus the shard
layout and all-reduce of tensor parallelism by branch (``tp``).  PyTorch only supplies
device memory, streams and the process group.  Build the library with
``python -m head_rank_attention_b200.build``.
"""
from ._binding import (EXPORTS, HRA_BF16, HRA_F32, HRA_INT8, HraDecodeParams, HraError, HraPrefillParams, LIB_PATH,
                       alloc_prefill_workspace, alloc_workspace, check_device_status, check_prefill_status,
                       combine_partials,
                       last_error, load_library, make_params, make_prefill_params, mla_decode, mlra_decode,
                       mlra_decode_static, mlra_prefill, prefill_workspace_size,
                       selftest_wait_timeout, version, workspace_size)
from . import cp, tp

__all__ = ["EXPORTS", "HRA_BF16", "HRA_F32", "HRA_INT8", "HraDecodeParams", "HraError", "HraPrefillParams",
           "LIB_PATH", "alloc_prefill_workspace", "alloc_workspace", "check_device_status", "check_prefill_status",
           "combine_partials", "cp",
           "last_error", "load_library", "make_params", "make_prefill_params", "mla_decode", "mlra_decode",
           "mlra_decode_static", "mlra_prefill", "prefill_workspace_size",
           "selftest_wait_timeout", "tp", "version", "workspace_size"]
