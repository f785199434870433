"""The attention kernel's bounded waits, exercised on the GPU without a fault.

A testing hook makes the producer of every attention CTA skip the K load of its first key tile, so
the barrier that load would complete never does.  With the wait limit lowered to 2 ms, the MMA
warp's wait runs out, every role of the CTA gives up and drains through its bounded paths, and the
call reports FP2_DEV_TIMEOUT through the status word.  A clean call on the same scratch right after
returns OK and matches the oracle: the context and the library are unaffected.
"""

import numpy as np
import pytest

from synth import workloads as W
from tests import harness as Hn

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from block_sparse_long_pooled_b200 import build
    build.build()


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_attention_wait_timeout_is_reported_and_recoverable(dtype):
    import torch
    from block_sparse_long_pooled_b200 import fp2
    w = W.Workload(name=f"timeout_{dtype}", seqlens=(700,), num_q_heads=8, num_kv_heads=2, head_dim=128,
                   block_size=128, dtype=dtype, sink_blocks=1, window_blocks=2, alpha=0.1, seed=31)
    inp = W.generate(w)
    ora = Hn.oracle_discovery(inp)
    dev = Hn.to_device(inp)
    prob = Hn.make_gpu_problem(inp, dev)
    params = Hn.gpu_params(w, kv_splits=1)
    ws = fp2.fp2_workspace_query(prob, params)
    pst, _ = fp2.alloc_pooled(ws, prob, "cuda")
    ist, _ = fp2.alloc_index(ws, "cuda")
    scratch = fp2.alloc_scratch(ws.scratch_bytes, "cuda")
    fp2.fp2_pool(prob, params, pst, scratch)
    fp2.fp2_discover(prob, params, pst, ist, scratch)
    torch.cuda.synchronize()
    assert fp2.fp2_get_device_status(scratch) == (0, 0)
    out = torch.zeros(inp.q.shape, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((w.num_q_heads, w.total_tokens), dtype=torch.float32, device="cuda")
    try:
        fp2.fp2_debug_set(fp2.FP2_DEBUG_WAIT_LIMIT_NS, 2_000_000)
        fp2.fp2_debug_set(fp2.FP2_DEBUG_WITHHOLD_K_TILE, 0)
        fp2.fp2_attend(prob, params, pst, ist, out, lse, scratch)
        torch.cuda.synchronize()
    finally:
        fp2.fp2_debug_set(fp2.FP2_DEBUG_WITHHOLD_K_TILE, -1)
        fp2.fp2_debug_set(fp2.FP2_DEBUG_WAIT_LIMIT_NS, 0)
    st, bits = fp2.fp2_get_device_status(scratch)
    assert st == fp2.FP2_ERR_TIMEOUT and bits & fp2.FP2_DEV_TIMEOUT, (st, bits)
    # the same scratch, a clean call: OK and the oracle's output
    fp2.fp2_attend(prob, params, pst, ist, out, lse, scratch)
    torch.cuda.synchronize()
    assert fp2.fp2_get_device_status(scratch) == (0, 0)

    class R:
        pass
    run = R()
    run.out, run.lse = out, lse
    Hn.compare_attention_full(run, inp, ora)
