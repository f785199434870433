"""ctypes binding of libfp2.so (include/fp2.h).  Argument marshalling only.

Every step of the attention path runs inside the CUDA library; PyTorch is used
here only to hand device pointers and the current stream to it.  Loading fails
loudly when the library has not been built.
"""

from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
# FP2_LIBRARY selects another build of the same library for this process (the tests use it to
# run with libfp2_checked.so); by default libfp2.so next to this file.
LIB_PATH = os.environ.get("FP2_LIBRARY") or os.path.join(_HERE, "libfp2.so")
CHECKED_LIB_PATH = os.path.join(_HERE, "libfp2_checked.so")

FP2_OK, FP2_ERR_INVALID_ARG, FP2_ERR_UNSUPPORTED, FP2_ERR_WORKSPACE_TOO_SMALL = 0, 1, 2, 3
FP2_ERR_CUDA, FP2_ERR_DEVICE_BOUNDS, FP2_ERR_TIMEOUT, FP2_ERR_CHECK_FAILED = 4, 5, 6, 7
FP2_F32, FP2_BF16, FP2_E4M3 = 0, 1, 2
FP2_DEV_PAGE_OOB, FP2_DEV_INDEX_OOB, FP2_DEV_CAPACITY, FP2_DEV_TIMEOUT, FP2_DEV_CHECK = 0x1, 0x2, 0x4, 0x8, 0x10
FP2_BUILD_CHECKED = 0x1
FP2_MAX_SEQS, FP2_MAX_BLOCKS = 512, 4096

STATUS_NAMES = {0: "FP2_OK", 1: "FP2_ERR_INVALID_ARG", 2: "FP2_ERR_UNSUPPORTED", 3: "FP2_ERR_WORKSPACE_TOO_SMALL",
                4: "FP2_ERR_CUDA", 5: "FP2_ERR_DEVICE_BOUNDS", 6: "FP2_ERR_TIMEOUT", 7: "FP2_ERR_CHECK_FAILED"}

EXPORTED = ("fp2_workspace_query", "fp2_workspace_size", "fp2_pool", "fp2_discover", "fp2_attend", "fp2_prefill",
            "fp2_get_device_status", "fp2_last_error", "fp2_version", "fp2_discover_static", "fp2_debug_set",
            "fp2_build_flags")
FP2_DEBUG_WAIT_LIMIT_NS, FP2_DEBUG_WITHHOLD_K_TILE, FP2_DEBUG_MISCOUNT_LOAD = 1, 2, 3
FP2_STATIC_SCRATCH_BYTES = 8 << 20


class fp2_problem(ctypes.Structure):
    _fields_ = [
        ("num_seqs", ctypes.c_int32),
        ("cu_seqlens_q_host", ctypes.POINTER(ctypes.c_int32)),
        ("cu_seqlens_k_host", ctypes.POINTER(ctypes.c_int32)),
        ("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("dtype", ctypes.c_int),
        ("q_descale", ctypes.c_float), ("k_descale", ctypes.c_float), ("v_descale", ctypes.c_float),
        ("softmax_scale", ctypes.c_float),
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("q_stride_tok", ctypes.c_int64), ("kv_stride_tok", ctypes.c_int64),
        ("page_table", ctypes.c_void_p),
        ("page_size", ctypes.c_int32), ("max_pages_per_seq", ctypes.c_int32), ("num_pages", ctypes.c_int32),
        ("kv_prefix_pooled", ctypes.c_int32),
    ]


class fp2_sparse_params(ctypes.Structure):
    _fields_ = [
        ("block_size", ctypes.c_int32), ("alpha", ctypes.c_float), ("sink_blocks", ctypes.c_int32),
        ("window_blocks", ctypes.c_int32), ("last_n_blocks", ctypes.c_int32), ("min_sparse_len", ctypes.c_int32),
        ("mean_correction", ctypes.c_int32), ("kv_splits", ctypes.c_int32),
    ]


class fp2_pooled(ctypes.Structure):
    _fields_ = [("qbar", ctypes.c_void_p), ("kbar", ctypes.c_void_p), ("vbar", ctypes.c_void_p),
                ("kbar_mma", ctypes.c_void_p), ("vbar_mma", ctypes.c_void_p), ("v16", ctypes.c_void_p)]


class fp2_index(ctypes.Structure):
    _fields_ = [("row_ptr", ctypes.c_void_p), ("col_idx", ctypes.c_void_p), ("col_capacity", ctypes.c_int64)]


class fp2_workspace(ctypes.Structure):
    _fields_ = [
        ("total_tokens", ctypes.c_int64), ("total_kv_tokens", ctypes.c_int64), ("total_q_blocks", ctypes.c_int64),
        ("total_kv_blocks", ctypes.c_int64), ("index_rows", ctypes.c_int64), ("col_capacity", ctypes.c_int64),
        ("qbar_bytes", ctypes.c_size_t), ("kbar_bytes", ctypes.c_size_t), ("vbar_bytes", ctypes.c_size_t),
        ("kbar_mma_bytes", ctypes.c_size_t), ("vbar_mma_bytes", ctypes.c_size_t),
        ("row_ptr_bytes", ctypes.c_size_t), ("col_idx_bytes", ctypes.c_size_t),
        ("discover_scratch_bytes", ctypes.c_size_t), ("scratch_bytes", ctypes.c_size_t),
        ("prefill_scratch_bytes", ctypes.c_size_t), ("v16_bytes", ctypes.c_size_t),
    ]


class FP2Error(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libfp2.so (once).  Raises when it is missing: there is no fallback path."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise FileNotFoundError(f"{path} is missing: build it with block_sparse_long_pooled_b200.build.build()")
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER
    vp, sz = ctypes.c_void_p, ctypes.c_size_t
    lib.fp2_workspace_query.argtypes = [P(fp2_problem), P(fp2_sparse_params), P(fp2_workspace)]
    lib.fp2_workspace_size.argtypes = [P(fp2_problem), P(fp2_sparse_params), P(sz), P(sz), P(sz)]
    lib.fp2_pool.argtypes = [P(fp2_problem), P(fp2_sparse_params), P(fp2_pooled), vp, sz, vp]
    lib.fp2_discover.argtypes = [P(fp2_problem), P(fp2_sparse_params), P(fp2_pooled), P(fp2_index), vp, sz, vp]
    lib.fp2_attend.argtypes = [P(fp2_problem), P(fp2_sparse_params), P(fp2_pooled), P(fp2_index), vp, vp, vp, sz, vp]
    lib.fp2_prefill.argtypes = [P(fp2_problem), P(fp2_sparse_params), vp, vp, vp, sz, vp]
    lib.fp2_get_device_status.argtypes = [vp, P(ctypes.c_uint32)]
    lib.fp2_discover_static.argtypes = [P(fp2_problem), P(fp2_sparse_params), P(fp2_pooled), P(fp2_index), vp, vp]
    for name in ("fp2_workspace_query", "fp2_workspace_size", "fp2_pool", "fp2_discover", "fp2_attend", "fp2_prefill",
                 "fp2_get_device_status", "fp2_discover_static"):
        getattr(lib, name).restype = ctypes.c_int
    lib.fp2_debug_set.argtypes = [ctypes.c_int32, ctypes.c_int64]
    lib.fp2_debug_set.restype = ctypes.c_int
    lib.fp2_last_error.argtypes = []
    lib.fp2_last_error.restype = ctypes.c_char_p
    lib.fp2_version.argtypes = []
    lib.fp2_version.restype = ctypes.c_int32
    lib.fp2_build_flags.argtypes = []
    lib.fp2_build_flags.restype = ctypes.c_uint32
    _lib = lib
    return lib


def _check(status: int):
    if status != FP2_OK:
        raise FP2Error(status, load_library().fp2_last_error().decode())


def _ptr(t) -> Optional[int]:
    return None if t is None else int(t.data_ptr())


def _stream_handle(stream) -> Optional[int]:
    if stream is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream)
    return int(stream) if isinstance(stream, int) else int(stream.cuda_stream)


# ------------------------------------------------------------------ problem description

@dataclasses.dataclass
class Problem:
    """An fp2_problem plus the host arrays and tensors it points into (kept alive here)."""
    struct: fp2_problem
    cu_seqlens: np.ndarray
    keep: tuple
    cu_seqlens_k: Optional[np.ndarray] = None


def _dtype_code(t) -> int:
    import torch
    return {torch.float32: FP2_F32, torch.bfloat16: FP2_BF16, torch.float8_e4m3fn: FP2_E4M3,
            torch.uint8: FP2_E4M3}[t.dtype]


def make_problem(q, k, v, cu_seqlens, num_kv_heads: int, q_descale: float = 1.0, k_descale: float = 1.0,
                 v_descale: float = 1.0, softmax_scale: float = 0.0, page_table=None,
                 num_pages: int = 0, cu_seqlens_k=None, kv_prefix_pooled: bool = False) -> Problem:
    """q: [T, Hq, d]; k, v: [Tk, Hkv, d] or a paged cache [P, page_size, Hkv, d] with page_table
    [num_seqs, max_pages] (int32, device).  cu_seqlens: host int sequence [num_seqs + 1] of query
    offsets; cu_seqlens_k: key offsets when the queries are chunks at the end of their sequences
    (chunked prefill), else None.  kv_prefix_pooled: the pooled prefix K/V blocks are already in
    the pooled buffers (see include/fp2.h)."""
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
    cuk = None if cu_seqlens_k is None else np.ascontiguousarray(np.asarray(cu_seqlens_k, dtype=np.int32))
    s = fp2_problem()
    s.num_seqs = len(cu) - 1
    s.cu_seqlens_q_host = cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    s.cu_seqlens_k_host = s.cu_seqlens_q_host if cuk is None else cuk.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    s.kv_prefix_pooled = 1 if kv_prefix_pooled else 0
    s.num_q_heads = q.shape[1]
    s.num_kv_heads = num_kv_heads
    s.head_dim = q.shape[2]
    s.dtype = _dtype_code(q)
    s.q_descale, s.k_descale, s.v_descale = q_descale, k_descale, v_descale
    s.softmax_scale = softmax_scale
    s.q, s.k, s.v = _ptr(q), _ptr(k), _ptr(v)
    s.q_stride_tok = q.stride(0)
    if page_table is not None:
        s.kv_stride_tok = k.stride(1)
        s.page_table = _ptr(page_table)
        s.page_size = k.shape[1]
        s.max_pages_per_seq = page_table.shape[1]
        s.num_pages = num_pages or k.shape[0]
    else:
        s.kv_stride_tok = k.stride(0)
        s.page_table = None
    return Problem(struct=s, cu_seqlens=cu, keep=(q, k, v, page_table), cu_seqlens_k=cuk)


def make_params(block_size: int, alpha: float = 0.1, sink_blocks: int = 2, window_blocks: int = 4,
                last_n_blocks: int = 0, min_sparse_len: int = 0, mean_correction: bool = True,
                kv_splits: int = 0) -> fp2_sparse_params:
    return fp2_sparse_params(block_size, alpha, sink_blocks, window_blocks, last_n_blocks, min_sparse_len,
                             1 if mean_correction else 0, kv_splits)


# ------------------------------------------------------------------ the C entry points

def fp2_workspace_query(problem: Problem, params: fp2_sparse_params) -> fp2_workspace:
    ws = fp2_workspace()
    _check(load_library().fp2_workspace_query(ctypes.byref(problem.struct), ctypes.byref(params), ctypes.byref(ws)))
    return ws


def fp2_workspace_size(problem: Problem, params: fp2_sparse_params) -> tuple:
    """(pooled_bytes, index_bytes, scratch_bytes): the totals for carving the pooled buffers and the
    index from one allocation each (256-byte aligned offsets), and the scratch size."""
    pooled, index, scratch = ctypes.c_size_t(0), ctypes.c_size_t(0), ctypes.c_size_t(0)
    _check(load_library().fp2_workspace_size(ctypes.byref(problem.struct), ctypes.byref(params), ctypes.byref(pooled),
                                             ctypes.byref(index), ctypes.byref(scratch)))
    return pooled.value, index.value, scratch.value


def fp2_pool(problem: Problem, params, pooled: fp2_pooled, scratch, stream=None):
    _check(load_library().fp2_pool(ctypes.byref(problem.struct), ctypes.byref(params), ctypes.byref(pooled),
                                   _ptr(scratch), scratch.numel() * scratch.element_size(), _stream_handle(stream)))


def fp2_discover(problem: Problem, params, pooled: fp2_pooled, index: fp2_index, scratch, stream=None):
    _check(load_library().fp2_discover(ctypes.byref(problem.struct), ctypes.byref(params), ctypes.byref(pooled),
                                       ctypes.byref(index), _ptr(scratch), scratch.numel() * scratch.element_size(),
                                       _stream_handle(stream)))


def fp2_attend(problem: Problem, params, pooled: fp2_pooled, index: fp2_index, out, lse, scratch, stream=None):
    _check(load_library().fp2_attend(ctypes.byref(problem.struct), ctypes.byref(params), ctypes.byref(pooled),
                                     ctypes.byref(index), _ptr(out), _ptr(lse), _ptr(scratch),
                                     scratch.numel() * scratch.element_size(), _stream_handle(stream)))


def fp2_prefill(problem: Problem, params, out, lse, scratch, stream=None):
    _check(load_library().fp2_prefill(ctypes.byref(problem.struct), ctypes.byref(params), _ptr(out), _ptr(lse),
                                      _ptr(scratch), scratch.numel() * scratch.element_size(),
                                      _stream_handle(stream)))


def fp2_discover_static(problem: Problem, params, pooled: fp2_pooled, index: fp2_index, status_dev=None,
                        stream=None):
    """fp2_discover without a scratch argument, for callers that cannot allocate device memory where
    they run discovery.  The library keeps the scratch in its own static device buffer (shared by all
    calls on a GPU: do not overlap calls).  status_dev: optional int32/uint32 device tensor of >= 1
    element that receives the call's FP2_DEV_* status word."""
    _check(load_library().fp2_discover_static(ctypes.byref(problem.struct), ctypes.byref(params),
                                              ctypes.byref(pooled), ctypes.byref(index), _ptr(status_dev),
                                              _stream_handle(stream)))


def fp2_get_device_status(scratch) -> tuple:
    """(status code, raw FP2_DEV_* bits); call after synchronising the stream."""
    bits = ctypes.c_uint32(0)
    st = load_library().fp2_get_device_status(_ptr(scratch), ctypes.byref(bits))
    return st, int(bits.value)


def fp2_debug_set(key: int, value: int):
    """Testing hook (process-wide): FP2_DEBUG_WAIT_LIMIT_NS, FP2_DEBUG_WITHHOLD_K_TILE or
    FP2_DEBUG_MISCOUNT_LOAD (checked builds)."""
    _check(load_library().fp2_debug_set(int(key), int(value)))


def fp2_last_error() -> str:
    return load_library().fp2_last_error().decode()


def fp2_version() -> int:
    return int(load_library().fp2_version())


def fp2_build_flags() -> int:
    """FP2_BUILD_* bits of the loaded library (FP2_BUILD_CHECKED for libfp2_checked.so)."""
    return int(load_library().fp2_build_flags())


# ------------------------------------------------------------------ buffer helpers (torch allocations)

def alloc_pooled(ws: fp2_workspace, problem: Problem, device):
    """Device buffers for fp2_pooled, as torch tensors; returns (struct, dict of tensors)."""
    import torch
    s = problem.struct
    nq, nk, Hq, Hkv, D = ws.total_q_blocks, ws.total_kv_blocks, s.num_q_heads, s.num_kv_heads, s.head_dim
    mma_dtype = {FP2_F32: torch.float32, FP2_BF16: torch.bfloat16, FP2_E4M3: torch.uint8}[s.dtype]
    # the V side of the PV product is f16 for E4M3 inputs (pooled vbar and the copy of V)
    v_dtype = torch.float16 if s.dtype == FP2_E4M3 else mma_dtype
    t = {
        "qbar": torch.empty((nq, Hq, D), dtype=torch.float32, device=device),
        "kbar": torch.empty((nk, Hkv, D), dtype=torch.float32, device=device),
        "vbar": torch.empty((nk, Hkv, D), dtype=torch.float32, device=device),
        "kbar_mma": torch.empty((nk, Hkv, D), dtype=mma_dtype, device=device),
        "vbar_mma": torch.empty((nk, Hkv, D), dtype=v_dtype, device=device),
    }
    if s.dtype == FP2_E4M3:
        t["v16"] = torch.empty((ws.total_kv_tokens, Hkv, D), dtype=torch.float16, device=device)
    return pooled_struct(t), t


def pooled_struct(t: dict) -> fp2_pooled:
    """fp2_pooled from a dict of tensors (qbar, kbar, vbar, kbar_mma, vbar_mma and, for E4M3, v16)."""
    return fp2_pooled(*(_ptr(t.get(k)) for k in ("qbar", "kbar", "vbar", "kbar_mma", "vbar_mma", "v16")))


def index_struct(row_ptr, col_idx) -> fp2_index:
    return fp2_index(_ptr(row_ptr), _ptr(col_idx), int(col_idx.numel()))


def alloc_index(ws: fp2_workspace, device):
    import torch
    row_ptr = torch.empty(ws.index_rows + 1, dtype=torch.int32, device=device)
    col_idx = torch.empty(max(1, ws.col_capacity), dtype=torch.int32, device=device)
    return index_struct(row_ptr, col_idx), {"row_ptr": row_ptr, "col_idx": col_idx}


def alloc_scratch(nbytes: int, device):
    import torch
    return torch.empty(max(256, (nbytes + 255) // 256 * 256), dtype=torch.uint8, device=device)


def out_dtype(problem: Problem):
    import torch
    return torch.float32 if problem.struct.dtype == FP2_F32 else torch.bfloat16
