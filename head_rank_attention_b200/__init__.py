"""B200-native (sm_100a) single-token decode over a compressed latent KV cache.

MLA (one branch) and MLRA (2 or 4 branches) decode behind the C ABI of libhra.so
(include/hra.h); this package is the thin Python binding of that ABI, plus the shard
layout and all-reduce of tensor parallelism by branch (``tp``).  PyTorch only supplies
device memory, streams and the process group.  Build the library with
``python -m head_rank_attention_b200.build``.
"""
from ._binding import (EXPORTS, HRA_BF16, HRA_F32, HraDecodeParams, HraError, LIB_PATH, alloc_workspace,
                       check_device_status, last_error, load_library, make_params, mla_decode, mlra_decode,
                       mlra_decode_static,
                       selftest_wait_timeout, version, workspace_size)
from . import tp

__all__ = ["EXPORTS", "HRA_BF16", "HRA_F32", "HraDecodeParams", "HraError", "LIB_PATH", "alloc_workspace",
           "check_device_status", "last_error", "load_library", "make_params", "mla_decode", "mlra_decode",
           "mlra_decode_static",
           "selftest_wait_timeout", "tp", "version", "workspace_size"]
