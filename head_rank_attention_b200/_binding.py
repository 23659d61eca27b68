"""ctypes binding of libhra.so (include/hra.h).  Argument marshalling only: every step of
the decode runs in the library's CUDA kernels.  There is no fallback: if the library is
missing or fails to load, importing a call raises.
"""
from __future__ import annotations

import ctypes
import math
import pathlib
from typing import Optional

LIB_PATH = pathlib.Path(__file__).resolve().with_name("libhra.so")

HRA_OK = 0
HRA_ERR_INVALID_ARG = -1
HRA_ERR_UNSUPPORTED = -2
HRA_ERR_WORKSPACE = -3
HRA_ERR_CUDA = -4
HRA_ERR_DEVICE_TIMEOUT = -5
HRA_BF16 = 0
HRA_F32 = 1
HRA_INT8 = 2

STATUS_NAMES = {0: "HRA_OK", -1: "HRA_ERR_INVALID_ARG", -2: "HRA_ERR_UNSUPPORTED", -3: "HRA_ERR_WORKSPACE",
                -4: "HRA_ERR_CUDA", -5: "HRA_ERR_DEVICE_TIMEOUT"}

# Symbols declared in include/hra.h.
EXPORTS = ("hra_workspace_size", "mlra_decode", "mla_decode", "mlra_decode_static", "hra_check_device_status",
           "hra_selftest_wait_timeout", "hra_last_error", "hra_version", "hra_prefill_workspace_size", "mlra_prefill",
           "hra_check_prefill_status", "hra_combine_partials")


class HraError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class HraDecodeParams(ctypes.Structure):
    """Mirror of hra_decode_params (field order and C types as in include/hra.h)."""
    _fields_ = [
        ("batch", ctypes.c_int), ("num_heads", ctypes.c_int), ("n_branch", ctypes.c_int),
        ("d_c", ctypes.c_int), ("d_rope", ctypes.c_int), ("d_nope", ctypes.c_int), ("d_v", ctypes.c_int),
        ("q", ctypes.c_void_p), ("ckv", ctypes.c_void_p), ("krope", ctypes.c_void_p),
        ("ckv_stride", ctypes.c_int64), ("krope_stride", ctypes.c_int64), ("cache_rows", ctypes.c_int64),
        ("seq_lens", ctypes.c_void_p), ("block_table", ctypes.c_void_p),
        ("max_pages", ctypes.c_int32), ("page_size", ctypes.c_int32), ("seq_stride", ctypes.c_int64),
        ("w_uk", ctypes.c_void_p), ("w_uv", ctypes.c_void_p),
        ("alpha_q", ctypes.c_float), ("alpha_kv", ctypes.c_float), ("branch_scale", ctypes.c_float),
        ("softmax_scale", ctypes.c_float), ("rope_theta", ctypes.c_float),
        ("out", ctypes.c_void_p), ("out_dtype", ctypes.c_int),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("num_splits", ctypes.c_int), ("wait_limit", ctypes.c_int),
        ("stage_events", ctypes.c_void_p),
        ("out_accumulate", ctypes.c_int), ("n_out_peers", ctypes.c_int), ("out_peers", ctypes.c_void_p),
        ("cache_dtype", ctypes.c_int), ("ckv_scale", ctypes.c_void_p), ("ckv_scale_stride", ctypes.c_int64),
        ("q_positions", ctypes.c_void_p), ("part_o", ctypes.c_void_p), ("part_lse", ctypes.c_void_p),
    ]


class HraPrefillParams(ctypes.Structure):
    """Mirror of hra_prefill_params (field order and C types as in include/hra.h)."""
    _fields_ = [
        ("num_heads", ctypes.c_int), ("n_branch", ctypes.c_int),
        ("d_c", ctypes.c_int), ("d_rope", ctypes.c_int), ("d_nope", ctypes.c_int), ("d_v", ctypes.c_int),
        ("seq_len", ctypes.c_int), ("n_query", ctypes.c_int),
        ("q", ctypes.c_void_p), ("ckv", ctypes.c_void_p), ("krope", ctypes.c_void_p),
        ("ckv_stride", ctypes.c_int64), ("krope_stride", ctypes.c_int64),
        ("w_uk", ctypes.c_void_p), ("w_uv", ctypes.c_void_p),
        ("alpha_q", ctypes.c_float), ("alpha_kv", ctypes.c_float), ("branch_scale", ctypes.c_float),
        ("softmax_scale", ctypes.c_float), ("rope_theta", ctypes.c_float),
        ("out", ctypes.c_void_p), ("out_dtype", ctypes.c_int),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("wait_limit", ctypes.c_int),
    ]


_lib: Optional[ctypes.CDLL] = None


def load_library() -> ctypes.CDLL:
    """Load libhra.so from the package directory (raises if it is not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not LIB_PATH.exists():
        raise ImportError(f"{LIB_PATH} is not built; run `python -m head_rank_attention_b200.build`")
    lib = ctypes.CDLL(str(LIB_PATH))
    P = ctypes.POINTER(HraDecodeParams)
    lib.hra_workspace_size.argtypes = [P]
    lib.hra_workspace_size.restype = ctypes.c_size_t
    for name in ("mlra_decode", "mla_decode", "mlra_decode_static", "hra_check_device_status"):
        getattr(lib, name).argtypes = [P, ctypes.c_void_p]
        getattr(lib, name).restype = ctypes.c_int
    PP = ctypes.POINTER(HraPrefillParams)
    lib.hra_prefill_workspace_size.argtypes = [PP]
    lib.hra_prefill_workspace_size.restype = ctypes.c_size_t
    for name in ("mlra_prefill", "hra_check_prefill_status"):
        getattr(lib, name).argtypes = [PP, ctypes.c_void_p]
        getattr(lib, name).restype = ctypes.c_int
    lib.hra_combine_partials.argtypes = [P, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    lib.hra_combine_partials.restype = ctypes.c_int
    lib.hra_selftest_wait_timeout.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
    lib.hra_selftest_wait_timeout.restype = ctypes.c_int
    lib.hra_last_error.argtypes = []
    lib.hra_last_error.restype = ctypes.c_char_p
    lib.hra_version.argtypes = []
    lib.hra_version.restype = ctypes.c_char_p
    _lib = lib
    return lib


def last_error() -> str:
    return load_library().hra_last_error().decode()


def version() -> str:
    return load_library().hra_version().decode()


def _check(status: int) -> None:
    if status != HRA_OK:
        raise HraError(status, last_error())


def _stream_handle(stream) -> int:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def _ptr(t) -> int:
    return 0 if t is None else int(t.data_ptr())


def make_params(q, ckv, krope, seq_lens, w_uk, w_uv, out, workspace=None, *, n_branch: int,
                alpha_q: float = 1.0, alpha_kv: float = 1.0, branch_scale: Optional[float] = None,
                softmax_scale: float = 0.0, rope_theta: float = 10000.0, block_table=None,
                page_size: int = 0, seq_stride: int = 0, cache_rows: Optional[int] = None,
                num_splits: int = 0, wait_limit: int = 0, out_accumulate: bool = False,
                out_peers=None, ckv_scale=None, q_positions=None, part_o=None,
                part_lse=None) -> HraDecodeParams:
    """Fill hra_decode_params from torch tensors (shapes/dtypes as documented in hra.h).

    ckv / krope are 2-D row views of the cache (e.g. cache[:, :512], cache[:, 512:]);
    their row strides become ckv_stride / krope_stride.  An int8 ckv selects the quantised
    cache: ckv_scale is then the fp32 [rows, d_c / 128] view of its block scales.  out_peers: device addresses (ints)
    or tensors of other ranks' out buffers for out_accumulate (the array is kept alive on
    the returned object).  q_positions (int32 [B]), part_o (fp32 [B, h, d_c]) and part_lse
    (fp32 [B, h, d_c / 128]) make the call the decode of one token range of longer
    sequences (see hra.h); out may then be None.
    """
    import torch
    p = HraDecodeParams()
    p.batch, p.num_heads = int(q.shape[0]), int(q.shape[1])
    p.n_branch = int(n_branch)
    p.d_c, p.d_rope, p.d_nope, p.d_v = int(ckv.shape[1]), int(krope.shape[1]), int(q.shape[2]) - int(krope.shape[1]), int(w_uv.shape[2])
    p.q, p.ckv, p.krope = _ptr(q), _ptr(ckv), _ptr(krope)
    p.ckv_stride, p.krope_stride = int(ckv.stride(0)), int(krope.stride(0))
    if ckv.dtype == torch.int8:
        if ckv_scale is None:
            raise ValueError("an int8 cache needs ckv_scale")
        p.cache_dtype = HRA_INT8
        p.ckv_scale, p.ckv_scale_stride = _ptr(ckv_scale), int(ckv_scale.stride(0))
    p.cache_rows = int(ckv.shape[0]) if cache_rows is None else int(cache_rows)
    p.seq_lens = _ptr(seq_lens)
    p.block_table = _ptr(block_table)
    p.max_pages = int(block_table.shape[1]) if block_table is not None else 0
    p.page_size = int(page_size)
    p.seq_stride = int(seq_stride)
    p.w_uk, p.w_uv = _ptr(w_uk), _ptr(w_uv)
    p.alpha_q, p.alpha_kv = float(alpha_q), float(alpha_kv)
    p.branch_scale = float(1.0 / math.sqrt(n_branch) if branch_scale is None else branch_scale)
    p.softmax_scale, p.rope_theta = float(softmax_scale), float(rope_theta)
    p.out = _ptr(out)
    p.out_dtype = HRA_F32 if out is not None and out.dtype == torch.float32 else HRA_BF16
    p.workspace = _ptr(workspace)
    p.workspace_bytes = 0 if workspace is None else int(workspace.numel() * workspace.element_size())
    p.num_splits, p.wait_limit = int(num_splits), int(wait_limit)
    p.out_accumulate = int(bool(out_accumulate))
    peers = [x if isinstance(x, int) else _ptr(x) for x in (out_peers or [])]
    p._out_peers = (ctypes.c_void_p * max(1, len(peers)))(*peers)
    p.out_peers = ctypes.cast(p._out_peers, ctypes.c_void_p).value if peers else None
    p.n_out_peers = len(peers)
    p.q_positions, p.part_o, p.part_lse = _ptr(q_positions), _ptr(part_o), _ptr(part_lse)
    return p


def workspace_size(p: HraDecodeParams) -> int:
    n = load_library().hra_workspace_size(ctypes.byref(p))
    if n == 0:
        raise HraError(HRA_ERR_INVALID_ARG, last_error())
    return int(n)


def mlra_decode(p: HraDecodeParams, stream=None) -> None:
    _check(load_library().mlra_decode(ctypes.byref(p), ctypes.c_void_p(_stream_handle(stream))))


def mla_decode(p: HraDecodeParams, stream=None) -> None:
    _check(load_library().mla_decode(ctypes.byref(p), ctypes.c_void_p(_stream_handle(stream))))


def mlra_decode_static(p: HraDecodeParams, stream=None) -> None:
    """Decode without a workspace (scratch from the library's 32 MiB static device array):
    for callers that cannot allocate device memory.  p.workspace is ignored."""
    _check(load_library().mlra_decode_static(ctypes.byref(p), ctypes.c_void_p(_stream_handle(stream))))


def combine_partials(p: HraDecodeParams, parts_o, parts_lse, stream=None) -> None:
    """Merge the gathered token-range states parts_o (fp32 [n, B, h, d_c]) and parts_lse
    (fp32 [n, B, h, d_c / 128]) and finish the decode into p.out (hra_combine_partials)."""
    _check(load_library().hra_combine_partials(ctypes.byref(p), int(parts_o.shape[0]), ctypes.c_void_p(_ptr(parts_o)),
                                               ctypes.c_void_p(_ptr(parts_lse)),
                                               ctypes.c_void_p(_stream_handle(stream))))


def check_device_status(p: HraDecodeParams, stream=None) -> None:
    _check(load_library().hra_check_device_status(ctypes.byref(p), ctypes.c_void_p(_stream_handle(stream))))


def selftest_wait_timeout(workspace, limit_us: int, stream=None) -> None:
    _check(load_library().hra_selftest_wait_timeout(ctypes.c_void_p(_ptr(workspace)), int(limit_us),
                                                    ctypes.c_void_p(_stream_handle(stream))))


def alloc_workspace(p: HraDecodeParams, device=None):
    """Allocate a workspace for p with torch (256-byte aligned) and attach it to p."""
    import torch
    n = workspace_size(p)
    ws = torch.empty(n + 256, dtype=torch.uint8, device=device or "cuda")
    off = (-ws.data_ptr()) % 256
    ws = ws[off:off + n]
    p.workspace, p.workspace_bytes = ws.data_ptr(), n
    return ws


def make_prefill_params(q, ckv, krope, w_uk, w_uv, out, *, n_branch: int, alpha_q: float = 1.0,
                        alpha_kv: float = 1.0, branch_scale: Optional[float] = None, softmax_scale: float = 0.0,
                        rope_theta: float = 10000.0, wait_limit: int = 0) -> HraPrefillParams:
    """Fill hra_prefill_params from torch tensors: q [n, h, 192] bf16, ckv / krope 2-D row
    views of the sequence's L cached rows, out [n, h, 128] (bf16 or fp32)."""
    import torch
    p = HraPrefillParams()
    p.num_heads, p.n_branch = int(q.shape[1]), int(n_branch)
    p.d_c, p.d_rope, p.d_nope, p.d_v = int(ckv.shape[1]), int(krope.shape[1]), int(q.shape[2]) - int(krope.shape[1]), int(w_uv.shape[2])
    p.seq_len, p.n_query = int(ckv.shape[0]), int(q.shape[0])
    p.q, p.ckv, p.krope = _ptr(q), _ptr(ckv), _ptr(krope)
    p.ckv_stride, p.krope_stride = int(ckv.stride(0)), int(krope.stride(0))
    p.w_uk, p.w_uv = _ptr(w_uk), _ptr(w_uv)
    p.alpha_q, p.alpha_kv = float(alpha_q), float(alpha_kv)
    p.branch_scale = float(1.0 / math.sqrt(n_branch) if branch_scale is None else branch_scale)
    p.softmax_scale, p.rope_theta = float(softmax_scale), float(rope_theta)
    p.out = _ptr(out)
    p.out_dtype = HRA_F32 if out is not None and out.dtype == torch.float32 else HRA_BF16
    p.wait_limit = int(wait_limit)
    return p


def prefill_workspace_size(p: HraPrefillParams) -> int:
    n = load_library().hra_prefill_workspace_size(ctypes.byref(p))
    if n == 0:
        raise HraError(HRA_ERR_INVALID_ARG, last_error())
    return int(n)


def alloc_prefill_workspace(p: HraPrefillParams, device=None):
    """Allocate a prefill workspace with torch (256-byte aligned) and attach it to p."""
    import torch
    n = prefill_workspace_size(p)
    ws = torch.empty(n + 256, dtype=torch.uint8, device=device or "cuda")
    off = (-ws.data_ptr()) % 256
    ws = ws[off:off + n]
    p.workspace, p.workspace_bytes = ws.data_ptr(), n
    return ws


def mlra_prefill(p: HraPrefillParams, stream=None) -> None:
    _check(load_library().mlra_prefill(ctypes.byref(p), ctypes.c_void_p(_stream_handle(stream))))


def check_prefill_status(p: HraPrefillParams, stream=None) -> None:
    _check(load_library().hra_check_prefill_status(ctypes.byref(p), ctypes.c_void_p(_stream_handle(stream))))
