"""fp2_discover_static: discovery for callers that cannot allocate device memory.

Some callers of this library run discovery where no allocation is allowed -- a serving
runtime that has handed all device memory to its KV cache at start-up, or a C host with no
device allocator -- so the library offers a variant of fp2_discover whose scratch lives in a
static device buffer instead of a caller-provided one.  These tests call it through the C ABI
twice in a row, on two different problems (the second smaller than the first, so stale
contents of the shared buffer would show), and require the same CSR index as fp2_discover
with caller scratch.  The index is integer output, so the comparison is exact.
"""

import numpy as np
import pytest

from synth import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from block_sparse_long_pooled_b200 import build
    build.build()


def _index_both_ways(w):
    import torch
    from block_sparse_long_pooled_b200 import fp2
    from tests import harness as Hn
    inp = W.generate(w)
    dev = Hn.to_device(inp)
    prob = Hn.make_gpu_problem(inp, dev)
    params = Hn.gpu_params(w)
    ws = fp2.fp2_workspace_query(prob, params)
    assert ws.discover_scratch_bytes <= fp2.FP2_STATIC_SCRATCH_BYTES
    pst, _ = fp2.alloc_pooled(ws, prob, "cuda")
    scratch = fp2.alloc_scratch(ws.scratch_bytes, "cuda")
    fp2.fp2_pool(prob, params, pst, scratch)
    ref_st, ref = fp2.alloc_index(ws, "cuda")
    fp2.fp2_discover(prob, params, pst, ref_st, scratch)
    new_st, new = fp2.alloc_index(ws, "cuda")
    new["row_ptr"].fill_(-7)
    new["col_idx"].fill_(-7)
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    fp2.fp2_discover_static(prob, params, pst, new_st, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    rp_ref, rp_new = ref["row_ptr"].cpu().numpy(), new["row_ptr"].cpu().numpy()
    assert np.array_equal(rp_ref, rp_new)
    nnz = int(rp_ref[-1])
    assert np.array_equal(ref["col_idx"][:nnz].cpu().numpy(), new["col_idx"][:nnz].cpu().numpy())
    return nnz


def test_static_discovery_matches_caller_scratch_twice():
    big = W.Workload(name="noalloc_a", seqlens=(6000, 2500), num_q_heads=16, num_kv_heads=4, head_dim=128,
                     block_size=128, dtype="bf16", sink_blocks=2, window_blocks=4, alpha=0.1, seed=11)
    small = W.Workload(name="noalloc_b", seqlens=(1500,), num_q_heads=8, num_kv_heads=1, head_dim=64,
                       block_size=64, dtype="bf16", sink_blocks=1, window_blocks=2, alpha=0.3, seed=12,
                       paged=True, page_size=16)
    n1 = _index_both_ways(big)
    n2 = _index_both_ways(small)
    assert n1 > 0 and n2 > 0


def test_static_discovery_rejects_oversized_problem():
    import torch
    from block_sparse_long_pooled_b200 import fp2
    # one 262144-token sequence, block 64 (4096 blocks), 8 KV heads: the kept-bit rows alone need
    # 32768 rows x 128 words x 4 B = 16 MiB of scratch, twice the static buffer.  Validation fails
    # on the host, so nothing is launched and the placeholder pointers are never dereferenced.
    cu = np.array([0, 4096 * 64], dtype=np.int32)
    q = torch.empty((1, 8, 64), dtype=torch.bfloat16, device="cuda")
    prob = fp2.make_problem(q, q, q, cu, 8)
    params = fp2.make_params(64)
    ws = fp2.fp2_workspace_query(prob, params)
    assert ws.discover_scratch_bytes > fp2.FP2_STATIC_SCRATCH_BYTES
    pst = fp2.fp2_pooled(q.data_ptr(), q.data_ptr(), q.data_ptr(), q.data_ptr(), q.data_ptr())
    ix = fp2.fp2_index(q.data_ptr(), q.data_ptr(), 1)
    with pytest.raises(fp2.FP2Error) as e:
        fp2.fp2_discover_static(prob, params, pst, ix)
    assert e.value.status == fp2.FP2_ERR_UNSUPPORTED and "static buffer" in str(e.value)


def test_static_discovery_reports_device_status_to_caller():
    """A device-side condition seen during the call (here: more kept blocks than col_capacity)
    reaches the caller's status_dev word.  scan_kernel raises FP2_DEV_CAPACITY and scatter_kernel
    writes no row that would end past the capacity, so nothing is written out of bounds."""
    import torch
    from block_sparse_long_pooled_b200 import fp2
    from tests import harness as Hn
    w = W.Workload(name="noalloc_cap", seqlens=(1200,), num_q_heads=8, num_kv_heads=2, head_dim=128,
                   block_size=128, dtype="bf16", sink_blocks=1, window_blocks=2, alpha=0.1, seed=13)
    inp = W.generate(w)
    dev = Hn.to_device(inp)
    prob = Hn.make_gpu_problem(inp, dev)
    params = Hn.gpu_params(w)
    ws = fp2.fp2_workspace_query(prob, params)
    pst, _ = fp2.alloc_pooled(ws, prob, "cuda")
    scratch = fp2.alloc_scratch(ws.scratch_bytes, "cuda")
    fp2.fp2_pool(prob, params, pst, scratch)
    rp = torch.zeros(ws.index_rows + 1, dtype=torch.int32, device="cuda")
    ci = torch.full((4,), -7, dtype=torch.int32, device="cuda")
    ix = fp2.fp2_index(rp.data_ptr(), ci.data_ptr(), 1)       # room for one column only
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    fp2.fp2_discover_static(prob, params, pst, ix, status)
    torch.cuda.synchronize()
    assert int(status.item()) & fp2.FP2_DEV_CAPACITY
    assert int(rp[-1].item()) > 1                               # the true count is still reported
    assert torch.all(ci[1:] == -7)                              # nothing written past the capacity
    # a clean call afterwards starts from a cleared status word
    ref_st, ref = fp2.alloc_index(ws, "cuda")
    fp2.fp2_discover_static(prob, params, pst, ref_st, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
