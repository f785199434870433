"""GPU parity for chunked prefill (queries = the last q_len tokens of each sequence, q_len <= kv_len).

The paper page's Table 6 serves long prompts in chunks and re-runs discovery per chunk.  Each case
draws whole sequences, keeps the last q_len query rows of each as the chunk, and compares the
library (pool, discover, attend through the C ABI) with the fp64 oracle's chunked prefill: pooled
means, the kept-block index (exact except borderline blocks), and every output row, both on the
oracle's index and on the library's own.  A second test pools a chunk's prefix blocks in an
earlier call and reuses them (kv_prefix_pooled).
"""

import math

import numpy as np
import pytest
import torch

from oracle import fp2_oracle as O
from synth import workloads as W
from tests import harness as Hn

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from block_sparse_long_pooled_b200 import build
    build.build()


def chunk_case(name, seqlens_k, q_lens, kv_splits=0, **kw):
    base = dict(num_q_heads=8, num_kv_heads=2, head_dim=128, block_size=128, dtype="bf16", sink_blocks=1,
                window_blocks=2, alpha=0.1, seed=17)
    base.update(kw)
    return W.Workload(name=name, seqlens=tuple(seqlens_k), **base), list(q_lens), kv_splits


CASES = [
    chunk_case("chunk_bf16_single", (1500,), (476,)),
    chunk_case("chunk_bf16_varlen", (1280, 700, 2000), (256, 700, 720)),
    chunk_case("chunk_bf16_paged64", (1800, 900), (520, 388), paged=True, page_size=64, num_q_heads=16),
    chunk_case("chunk_e4m3", (2100,), (564,), dtype="e4m3"),
    chunk_case("chunk_bf16_d64_b64", (1000,), (296,), head_dim=64, block_size=64, num_q_heads=4,
               last_n_blocks=1, sink_blocks=2, window_blocks=3),
    # adaptive KV splits (ranges of at most 2 or 3 key tiles) over prefixes, paged, FP8
    chunk_case("chunk_bf16_varlen_adaptive", (1280, 700, 2000), (256, 700, 720), kv_splits=-2),
    chunk_case("chunk_e4m3_paged_adaptive", (2100, 1500), (564, 220), kv_splits=-3, dtype="e4m3", paged=True,
               page_size=64),
    # a short chunk after a long prefix (304 prefix + 9 query blocks, 3 key chunks of 128): discovery splits each
    # tile's key chunks over several CTAs (partial row maxima, then thresholds)
    chunk_case("chunk_bf16_long_prefix", (40000,), (1088,)),
]


def split_queries(inp, q_lens):
    """Query rows of each sequence's chunk, packed; returns (q chunk tensor, cu_q, cu_k)."""
    cu_k = inp.cu_seqlens
    rows = np.concatenate([np.arange(cu_k[r + 1] - ql, cu_k[r + 1]) for r, ql in enumerate(q_lens)])
    cu_q = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    return inp.q[torch.from_numpy(rows)], cu_q, cu_k, rows


def oracle_chunked(inp, w, qc, cu_q, cu_k):
    p = Hn.oracle_params(w)
    qd = qc.to(torch.float64).numpy() * inp.q_descale
    if inp.page_table is not None:
        kc = inp.k_cache.to(torch.float64).numpy() * inp.k_descale
        vc = inp.v_cache.to(torch.float64).numpy() * inp.v_descale
        return O.prefill(qd, None, None, cu_q, w.num_kv_heads, p, k_cache=kc, v_cache=vc,
                         page_table=inp.page_table, cu_seqlens_k=cu_k)
    return O.prefill(qd, inp.dequant("k"), inp.dequant("v"), cu_q, w.num_kv_heads, p, cu_seqlens_k=cu_k)


def gpu_problem(inp, w, qc, cu_q, cu_k, kv_prefix_pooled=False):
    from block_sparse_long_pooled_b200 import fp2
    dev = {"q": qc.cuda()}
    if inp.page_table is not None:
        dev["k"], dev["v"] = inp.k_cache.cuda(), inp.v_cache.cuda()
        dev["pt"] = torch.from_numpy(inp.page_table).cuda()
        prob = fp2.make_problem(dev["q"], dev["k"], dev["v"], cu_q, w.num_kv_heads, inp.q_descale, inp.k_descale,
                                inp.v_descale, page_table=dev["pt"], cu_seqlens_k=cu_k,
                                kv_prefix_pooled=kv_prefix_pooled)
    else:
        dev["k"], dev["v"] = inp.k.cuda(), inp.v.cuda()
        prob = fp2.make_problem(dev["q"], dev["k"], dev["v"], cu_q, w.num_kv_heads, inp.q_descale, inp.k_descale,
                                inp.v_descale, cu_seqlens_k=cu_k, kv_prefix_pooled=kv_prefix_pooled)
    return prob, dev


def gpu_kept_chunked(rp, ci, q_lens, k_lens, B, Hkv):
    out, row = [], 0
    for Lq, Lk in zip(q_lens, k_lens):
        N, Nk = -(-Lq // B), -(-Lk // B)
        kept = np.zeros((Hkv, N, Nk), dtype=bool)
        for i in range(N):
            for g in range(Hkv):
                cols = ci[rp[row]:rp[row + 1]]
                assert np.all(np.diff(cols) > 0)
                kept[g, i, cols] = True
                row += 1
        out.append(kept)
    return out


@pytest.mark.parametrize("case", CASES, ids=[c[0].name for c in CASES])
def test_chunked_parity(case):
    from block_sparse_long_pooled_b200 import fp2
    w, q_lens, kv_splits = case
    inp = W.generate(w)
    qc, cu_q, cu_k, _ = split_queries(inp, q_lens)
    ref = oracle_chunked(inp, w, qc, cu_q, cu_k)
    prob, dev = gpu_problem(inp, w, qc, cu_q, cu_k)
    params = Hn.gpu_params(w, kv_splits=kv_splits)
    ws = fp2.fp2_workspace_query(prob, params)
    pst, pooled = fp2.alloc_pooled(ws, prob, "cuda")
    ist, index = fp2.alloc_index(ws, "cuda")
    scratch = fp2.alloc_scratch(ws.scratch_bytes, "cuda")
    fp2.fp2_pool(prob, params, pst, scratch)
    fp2.fp2_discover(prob, params, pst, ist, scratch)
    torch.cuda.synchronize()
    assert fp2.fp2_get_device_status(scratch) == (0, 0)
    # pooled means
    for name, refs in (("qbar", ref["qbar"]), ("kbar", ref["kbar"]), ("vbar", ref["vbar"])):
        g = pooled[name].double().cpu().numpy()
        o = np.concatenate(refs)
        assert np.abs(g - o).max() <= 2e-5 * max(1.0, np.abs(o).max()), name
    # index: exact except borderline blocks
    k_lens = [int(cu_k[r + 1] - cu_k[r]) for r in range(len(q_lens))]
    gk = gpu_kept_chunked(index["row_ptr"].cpu().numpy(), index["col_idx"].cpu().numpy(), q_lens, k_lens,
                          w.block_size, w.num_kv_heads)
    mism = 0
    for a_, o_, b_ in zip(gk, ref["kept"], ref["borderline"]):
        assert a_.shape == o_.shape
        assert not np.any((a_ != o_) & ~b_)
        mism += int((a_ != o_).sum())
    # attention on the oracle's index, then on the library's own
    out = torch.empty(qc.shape, dtype=fp2.out_dtype(prob), device="cuda")
    lse = torch.empty((w.num_q_heads, qc.shape[0]), dtype=torch.float32, device="cuda")
    rp = torch.from_numpy(ref["row_ptr"].astype(np.int32)).cuda()
    ci = torch.from_numpy(ref["col_idx"].astype(np.int32)).cuda()
    fp2.fp2_attend(prob, params, pst, fp2.index_struct(rp, ci), out, lse, scratch)
    torch.cuda.synchronize()
    assert fp2.fp2_get_device_status(scratch) == (0, 0)
    Hn.check_tol(out.double().cpu().numpy(), ref["O"], w.dtype)
    assert np.abs(lse.double().cpu().numpy() - ref["LSE"]).max() < Hn.LSE_TOL[w.dtype]
    if mism == 0:
        fp2.fp2_attend(prob, params, pst, ist, out, None, scratch)
        torch.cuda.synchronize()
        Hn.check_tol(out.double().cpu().numpy(), ref["O"], w.dtype)


def test_prefix_pooled_in_an_earlier_call_is_reused():
    """Chunk 1 (the first 1024 tokens) pools key blocks 0-7; chunk 2 (tokens 1024-1499) reuses them."""
    from block_sparse_long_pooled_b200 import fp2
    w = W.Workload(name="chunk_reuse", seqlens=(1500,), num_q_heads=8, num_kv_heads=2, head_dim=128,
                   block_size=128, dtype="bf16", sink_blocks=1, window_blocks=2, alpha=0.1, seed=23)
    inp = W.generate(w)
    params = Hn.gpu_params(w)
    k, v = inp.k.cuda(), inp.v.cuda()
    q1 = inp.q[:1024].cuda()
    q2 = inp.q[1024:].cuda()
    p1 = fp2.make_problem(q1, k, v, [0, 1024], 2, cu_seqlens_k=[0, 1024])
    p2 = fp2.make_problem(q2, k, v, [0, 476], 2, cu_seqlens_k=[0, 1500])
    p2_reuse = fp2.make_problem(q2, k, v, [0, 476], 2, cu_seqlens_k=[0, 1500], kv_prefix_pooled=True)
    ws2 = fp2.fp2_workspace_query(p2, params)
    ws1 = fp2.fp2_workspace_query(p1, params)
    # shared kbar/vbar buffers sized for chunk 2; qbar sized for the larger chunk
    _, pooled = fp2.alloc_pooled(ws2, p2, "cuda")
    pooled["qbar"] = torch.empty((ws1.total_q_blocks, 8, 128), dtype=torch.float32, device="cuda")
    pst = fp2.pooled_struct(pooled)
    scratch = fp2.alloc_scratch(max(ws1.prefill_scratch_bytes, ws2.prefill_scratch_bytes), "cuda")
    kv_names = ("kbar", "vbar", "kbar_mma", "vbar_mma")

    def chunk2(prob):
        fp2.fp2_pool(prob, params, pst, scratch)
        ist, _ = fp2.alloc_index(ws2, "cuda")
        fp2.fp2_discover(prob, params, pst, ist, scratch)
        out = torch.empty(q2.shape, dtype=torch.bfloat16, device="cuda")
        fp2.fp2_attend(prob, params, pst, ist, out, None, scratch)
        torch.cuda.synchronize()
        assert fp2.fp2_get_device_status(scratch) == (0, 0)
        return out

    for n in kv_names:
        pooled[n].zero_()
    fresh = chunk2(p2)                      # pools all 12 key blocks
    for n in kv_names:
        pooled[n].zero_()
    fp2.fp2_pool(p1, params, pst, scratch)  # chunk 1 pools key blocks 0-7
    reused = chunk2(p2_reuse)               # pools blocks 8-11 only
    assert torch.equal(fresh, reused)
    # with kv_prefix_pooled the prefix rows are left alone
    pooled["kbar"][:8].fill_(7.0)
    fp2.fp2_pool(p2_reuse, params, pst, scratch)
    torch.cuda.synchronize()
    assert bool((pooled["kbar"][:8] == 7.0).all()) and not bool((pooled["kbar"][8:] == 7.0).any())


def test_prefix_pooled_reuse_e4m3_keeps_the_v_copy():
    """E4M3 chunked prefill with kv_prefix_pooled: the prefix rows of the f16 copy of V (read by the
    PV product) come from the earlier chunk's fp2_pool, like kbar/vbar, and the result equals a
    fresh pooling of the whole key range; paged K/V, 64-token pages."""
    from block_sparse_long_pooled_b200 import fp2
    w = W.Workload(name="chunk_reuse_e4m3", seqlens=(1500,), num_q_heads=8, num_kv_heads=2, head_dim=128,
                   block_size=128, dtype="e4m3", sink_blocks=1, window_blocks=2, alpha=0.1, seed=29,
                   paged=True, page_size=64)
    inp = W.generate(w)
    params = Hn.gpu_params(w)
    dev = Hn.to_device(inp)
    kc, vc, pt = dev["k_cache"], dev["v_cache"], dev["page_table"]
    q1, q2 = dev["q"][:1024], dev["q"][1024:]
    ds = (inp.q_descale, inp.k_descale, inp.v_descale)
    p1 = fp2.make_problem(q1, kc, vc, [0, 1024], 2, *ds, page_table=pt, cu_seqlens_k=[0, 1024])
    p2 = fp2.make_problem(q2, kc, vc, [0, 476], 2, *ds, page_table=pt, cu_seqlens_k=[0, 1500])
    p2_reuse = fp2.make_problem(q2, kc, vc, [0, 476], 2, *ds, page_table=pt, cu_seqlens_k=[0, 1500],
                                kv_prefix_pooled=True)
    ws1, ws2 = fp2.fp2_workspace_query(p1, params), fp2.fp2_workspace_query(p2, params)
    _, pooled = fp2.alloc_pooled(ws2, p2, "cuda")
    pooled["qbar"] = torch.empty((ws1.total_q_blocks, 8, 128), dtype=torch.float32, device="cuda")
    pst = fp2.pooled_struct(pooled)
    scratch = fp2.alloc_scratch(max(ws1.prefill_scratch_bytes, ws2.prefill_scratch_bytes), "cuda")

    def chunk2(prob):
        fp2.fp2_pool(prob, params, pst, scratch)
        ist, _ = fp2.alloc_index(ws2, "cuda")
        fp2.fp2_discover(prob, params, pst, ist, scratch)
        out = torch.empty(q2.shape, dtype=torch.bfloat16, device="cuda")
        fp2.fp2_attend(prob, params, pst, ist, out, None, scratch)
        torch.cuda.synchronize()
        assert fp2.fp2_get_device_status(scratch) == (0, 0)
        return out

    for n in ("kbar", "vbar", "kbar_mma", "vbar_mma", "v16"):
        pooled[n].zero_()
    fresh = chunk2(p2)
    for n in ("kbar", "vbar", "kbar_mma", "vbar_mma", "v16"):
        pooled[n].zero_()
    fp2.fp2_pool(p1, params, pst, scratch)   # chunk 1 pools key blocks 0-7 and V rows 0-1023
    reused = chunk2(p2_reuse)                # pools key blocks 8-11 and V rows 1024-1499 only
    assert torch.equal(fresh, reused)
    assert torch.equal(pooled["v16"].cpu(), inp.v.to(torch.float16))
