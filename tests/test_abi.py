"""The C ABI library without a GPU: it loads, exports what include/fp2.h declares, and its
host-side validation and workspace sizing behave (no CUDA call is made by these paths)."""

import ctypes
import os
import re
import subprocess

import numpy as np
import pytest
import torch

from block_sparse_long_pooled_b200 import build as B
from block_sparse_long_pooled_b200 import fp2

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def _built():
    B.build()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "fp2.h")).read()
    return sorted(set(re.findall(r"FP2_API\s+[\w\s\*]+?\b(fp2_\w+)\s*\(", text)))


def test_exports_every_declared_symbol():
    decl = declared_functions()
    assert decl == sorted(fp2.EXPORTED)
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB], capture_output=True, text=True, check=True).stdout
    exported = sorted(l.split()[-1] for l in out.splitlines() if " T " in l)
    assert exported == decl
    lib = fp2.load_library()
    for name in decl:
        assert hasattr(lib, name)
    assert fp2.fp2_version() == 10000


def test_checked_build_exports_the_same_symbols_and_says_so():
    # libfp2_checked.so: the same sources with FP2_CHECKED=1 (device-side hand-off and bounds checks)
    B.build(checked=True)
    decl = declared_functions()
    out = subprocess.run(["nm", "-D", "--defined-only", B.CHECKED_LIB], capture_output=True, text=True,
                         check=True).stdout
    assert sorted(l.split()[-1] for l in out.splitlines() if " T " in l) == decl
    import ctypes
    checked = ctypes.CDLL(B.CHECKED_LIB)
    checked.fp2_build_flags.restype = ctypes.c_uint32
    assert checked.fp2_build_flags() == fp2.FP2_BUILD_CHECKED
    if os.environ.get("FP2_LIBRARY") is None:
        assert fp2.fp2_build_flags() == 0          # the default library has no checks compiled in
    # the status word's check bit maps to its own error code
    assert fp2.STATUS_NAMES[fp2.FP2_ERR_CHECK_FAILED] == "FP2_ERR_CHECK_FAILED"
    assert fp2.FP2_DEV_CHECK not in (fp2.FP2_DEV_PAGE_OOB, fp2.FP2_DEV_INDEX_OOB, fp2.FP2_DEV_CAPACITY,
                                     fp2.FP2_DEV_TIMEOUT)


def _problem(seqlens=(1000, 333), Hq=8, Hkv=2, d=128, dtype=torch.bfloat16, paged=False, page_size=64):
    T = sum(seqlens)
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    q = torch.empty((T, Hq, d), dtype=dtype)
    if paged:
        npages = sum(-(-L // page_size) for L in seqlens)
        k = torch.empty((npages, page_size, Hkv, d), dtype=dtype)
        v = torch.empty_like(k)
        pt = torch.zeros((len(seqlens), max(-(-L // page_size) for L in seqlens)), dtype=torch.int32)
        return fp2.make_problem(q, k, v, cu, Hkv, page_table=pt)
    k = torch.empty((T, Hkv, d), dtype=dtype)
    v = torch.empty_like(k)
    return fp2.make_problem(q, k, v, cu, Hkv)


def test_workspace_sizes():
    prob = _problem()
    ws = fp2.fp2_workspace_query(prob, fp2.make_params(128))
    N = [8, 3]
    assert ws.total_tokens == 1333 and ws.total_q_blocks == 11 and ws.total_kv_blocks == 11 and ws.index_rows == 22
    assert ws.col_capacity == sum(2 * n * (n + 1) // 2 for n in N)
    assert ws.qbar_bytes == 11 * 8 * 128 * 4 and ws.kbar_mma_bytes == 11 * 2 * 128 * 2
    assert ws.row_ptr_bytes == 23 * 4 and ws.col_idx_bytes == ws.col_capacity * 4
    assert ws.prefill_scratch_bytes > ws.scratch_bytes > 0
    assert ws.scratch_bytes % 256 == 0 and ws.prefill_scratch_bytes % 256 == 0


@pytest.mark.parametrize("kw,params,code", [
    (dict(d=96), {}, fp2.FP2_ERR_UNSUPPORTED),
    (dict(Hq=6, Hkv=4), {}, fp2.FP2_ERR_INVALID_ARG),
    (dict(dtype=torch.float32), {}, fp2.FP2_ERR_UNSUPPORTED),       # f32 needs d = 64
    (dict(dtype=torch.float8_e4m3fn, d=64), {}, fp2.FP2_ERR_UNSUPPORTED),
    ({}, dict(block_size=32), fp2.FP2_ERR_UNSUPPORTED),
    ({}, dict(alpha=1.5), fp2.FP2_ERR_INVALID_ARG),
    ({}, dict(sink_blocks=-1), fp2.FP2_ERR_INVALID_ARG),
    (dict(seqlens=(4096 * 128 + 1,)), {}, fp2.FP2_ERR_UNSUPPORTED),
    (dict(paged=True, page_size=24), {}, fp2.FP2_ERR_UNSUPPORTED),
    ({}, dict(kv_splits=65), fp2.FP2_ERR_INVALID_ARG),
    ({}, dict(kv_splits=-4097), fp2.FP2_ERR_INVALID_ARG),
])
def test_validation_errors(kw, params, code):
    prob = _problem(**kw)
    p = dict(block_size=128)
    p.update(params)
    with pytest.raises(fp2.FP2Error) as e:
        fp2.fp2_workspace_query(prob, fp2.make_params(**p))
    assert e.value.status == code
    assert fp2.fp2_last_error() != ""


def test_workspace_size_totals():
    prob = _problem(paged=True)
    params = fp2.make_params(128)
    ws = fp2.fp2_workspace_query(prob, params)
    pooled, index, scratch = fp2.fp2_workspace_size(prob, params)
    up = lambda x: (x + 255) // 256 * 256
    assert pooled == sum(up(b) for b in (ws.qbar_bytes, ws.kbar_bytes, ws.vbar_bytes, ws.kbar_mma_bytes,
                                         ws.vbar_mma_bytes))
    assert index == up(ws.row_ptr_bytes) + up(ws.col_idx_bytes)
    assert scratch == ws.scratch_bytes
    assert ws.v16_bytes == 0


def test_e4m3_v_side_sizes():
    """E4M3 inputs: kbar_mma stays e4m3, the V side of the PV product (vbar_mma and the copy of V)
    is f16, and the pooled total includes the copy."""
    prob = _problem(dtype=torch.float8_e4m3fn, paged=True)
    params = fp2.make_params(128)
    ws = fp2.fp2_workspace_query(prob, params)
    assert ws.kbar_mma_bytes == 11 * 2 * 128 * 1 and ws.vbar_mma_bytes == 11 * 2 * 128 * 2
    assert ws.v16_bytes == 1333 * 2 * 128 * 2
    pooled, _, _ = fp2.fp2_workspace_size(prob, params)
    up = lambda x: (x + 255) // 256 * 256
    assert pooled == sum(up(b) for b in (ws.qbar_bytes, ws.kbar_bytes, ws.vbar_bytes, ws.kbar_mma_bytes,
                                         ws.vbar_mma_bytes, ws.v16_bytes))
    assert ws.prefill_scratch_bytes >= ws.scratch_bytes + ws.v16_bytes
    # every output is optional; validation is the same as fp2_workspace_query's
    lib = fp2.load_library()
    assert lib.fp2_workspace_size(ctypes.byref(prob.struct), ctypes.byref(params), None, None, None) == fp2.FP2_OK
    bad = fp2.make_params(128, alpha=2.0)
    with pytest.raises(fp2.FP2Error) as e:
        fp2.fp2_workspace_size(prob, bad)
    assert e.value.status == fp2.FP2_ERR_INVALID_ARG


def test_split_modes_size_their_partials():
    # 22 index rows x 2 parts = 44 row CTAs: few, so kv_splits = 0 splits every row uniformly into
    # min(8, ceil(296 / 44)) = 7 ranges
    prob = _problem()
    one = fp2.fp2_workspace_query(prob, fp2.make_params(128, kv_splits=1))
    auto = fp2.fp2_workspace_query(prob, fp2.make_params(128, kv_splits=0))
    uni = fp2.fp2_workspace_query(prob, fp2.make_params(128, kv_splits=3))
    T, Hq, d = 1333, 8, 128
    assert uni.scratch_bytes - one.scratch_bytes >= 3 * T * Hq * d * 4
    assert auto.scratch_bytes - one.scratch_bytes >= 7 * T * Hq * d * 4
    # adaptive (kv_splits < 0): at most 64 ranges per row part (44 row parts here), slots of
    # 2 x 128 packed rows x d fp32 each; many rows switch the automatic mode to adaptive as well
    ada = fp2.fp2_workspace_query(prob, fp2.make_params(128, kv_splits=-5))
    assert ada.scratch_bytes - one.scratch_bytes >= min(768, 44 * 64) * 256 * d * 4
    many = _problem(seqlens=(40000,))  # 313 blocks x 2 KV heads x 2 parts = 1252 row CTAs
    m1 = fp2.fp2_workspace_query(many, fp2.make_params(128, kv_splits=1))
    m0 = fp2.fp2_workspace_query(many, fp2.make_params(128, kv_splits=0))
    assert m0.scratch_bytes - m1.scratch_bytes >= 768 * 256 * d * 4
    assert m0.discover_scratch_bytes == m1.discover_scratch_bytes
    # launches of 16 waves of 148 SMs or more are left whole in the automatic mode
    huge = _problem(seqlens=(131072,), Hq=32, Hkv=8)  # 1024 blocks x 8 KV heads x 2 parts
    h1 = fp2.fp2_workspace_query(huge, fp2.make_params(128, kv_splits=1))
    h0 = fp2.fp2_workspace_query(huge, fp2.make_params(128, kv_splits=0))
    hf = fp2.fp2_workspace_query(huge, fp2.make_params(128, kv_splits=-64))
    assert h0.scratch_bytes == h1.scratch_bytes < hf.scratch_bytes


def test_chunked_prefill_sizes_and_rules():
    # queries: chunks of 1000 and 333 tokens; keys: 1000 + 256 and 333 + 512 (prefixes of 2 and 4 blocks)
    T, Tk, Hq, Hkv, d = 1333, 2101, 8, 2, 128
    q = torch.empty((T, Hq, d), dtype=torch.bfloat16)
    k = torch.empty((Tk, Hkv, d), dtype=torch.bfloat16)
    prob = fp2.make_problem(q, k, k, [0, 1000, 1333], Hkv, cu_seqlens_k=[0, 1256, 2101])
    ws = fp2.fp2_workspace_query(prob, fp2.make_params(128))
    assert ws.total_kv_tokens == Tk and ws.total_q_blocks == 8 + 3 and ws.total_kv_blocks == 10 + 7
    assert ws.col_capacity == 2 * (sum(2 + i + 1 for i in range(8)) + sum(4 + i + 1 for i in range(3)))
    assert ws.kbar_bytes == 17 * Hkv * d * 4 and ws.qbar_bytes == 11 * Hq * d * 4
    for cuk, code in (([0, 1200, 2045], fp2.FP2_ERR_UNSUPPORTED),      # prefix 200 not a multiple of 128
                      ([0, 900, 1745], fp2.FP2_ERR_INVALID_ARG)):      # kv_len < q_len
        bad = fp2.make_problem(q, k, k, [0, 1000, 1333], Hkv, cu_seqlens_k=cuk)
        with pytest.raises(fp2.FP2Error) as e:
            fp2.fp2_workspace_query(bad, fp2.make_params(128))
        assert e.value.status == code


def test_scratch_too_small_rejected_before_launch():
    prob = _problem()
    params = fp2.make_params(128)
    ws = fp2.fp2_workspace_query(prob, params)
    raw = torch.empty(ws.scratch_bytes + 256, dtype=torch.uint8)
    off = (-raw.data_ptr()) % 256
    scratch = raw[off: off + ws.scratch_bytes - 256]
    pooled, _ = fp2.alloc_pooled(ws, prob, "cpu")
    with pytest.raises(fp2.FP2Error) as e:
        fp2.fp2_pool(prob, params, pooled, scratch, stream=0)
    assert e.value.status == fp2.FP2_ERR_WORKSPACE_TOO_SMALL


def test_library_missing_fails_loudly(tmp_path):
    with pytest.raises(FileNotFoundError):
        fp2.load_library.__wrapped__(str(tmp_path / "nope.so")) if hasattr(fp2.load_library, "__wrapped__") \
            else _load_fresh(str(tmp_path / "nope.so"))


def _load_fresh(path):
    saved = fp2._lib
    fp2._lib = None
    try:
        return fp2.load_library(path)
    finally:
        fp2._lib = saved


def test_debug_hooks_validate_and_reset():
    with pytest.raises(fp2.FP2Error):
        fp2.fp2_debug_set(99, 0)
    with pytest.raises(fp2.FP2Error):
        fp2.fp2_debug_set(fp2.FP2_DEBUG_WAIT_LIMIT_NS, 10)           # below 0.1 ms
    with pytest.raises(fp2.FP2Error):
        fp2.fp2_debug_set(fp2.FP2_DEBUG_WITHHOLD_K_TILE, -2)
    fp2.fp2_debug_set(fp2.FP2_DEBUG_WAIT_LIMIT_NS, 2_000_000)
    fp2.fp2_debug_set(fp2.FP2_DEBUG_WAIT_LIMIT_NS, 0)
    fp2.fp2_debug_set(fp2.FP2_DEBUG_WITHHOLD_K_TILE, 3)
    fp2.fp2_debug_set(fp2.FP2_DEBUG_WITHHOLD_K_TILE, -1)
    with pytest.raises(fp2.FP2Error):
        fp2.fp2_debug_set(fp2.FP2_DEBUG_MISCOUNT_LOAD, -2)
    with pytest.raises(fp2.FP2Error):
        fp2.fp2_debug_set(fp2.FP2_DEBUG_MISCOUNT_LOAD, 2 * fp2.FP2_MAX_BLOCKS + 1)
    fp2.fp2_debug_set(fp2.FP2_DEBUG_MISCOUNT_LOAD, 2)
    fp2.fp2_debug_set(fp2.FP2_DEBUG_MISCOUNT_LOAD, -1)


def test_sequence_count_limit():
    ok = _problem(seqlens=(3,) * fp2.FP2_MAX_SEQS, Hq=4, Hkv=2)
    ws = fp2.fp2_workspace_query(ok, fp2.make_params(64))
    assert ws.index_rows == fp2.FP2_MAX_SEQS * 2
    too_many = _problem(seqlens=(3,) * (fp2.FP2_MAX_SEQS + 1), Hq=4, Hkv=2)
    with pytest.raises(fp2.FP2Error) as e:
        fp2.fp2_workspace_query(too_many, fp2.make_params(64))
    assert e.value.status == fp2.FP2_ERR_UNSUPPORTED
