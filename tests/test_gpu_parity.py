"""GPU parity: the CUDA library (through its C ABI) against the fp64 oracle.

Small cases compare every output element and span several tiles with ragged
tails, every supported (dtype, head_dim, block) kernel, GQA groups 1/2/4/8,
contiguous and paged K/V (page sizes 16/64/128), varlen batches with a dense
cutoff, alpha = 0, last-n rows, mean correction off, an external index, and
device-side bounds checks.  The five workloads at full size compare the whole
block index and every element of selected whole (KV group, query block) pairs
of the output and the LSE.
"""

import math

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


def small(name, **kw):
    base = dict(seqlens=(1000, 333), num_q_heads=8, num_kv_heads=2, head_dim=128, block_size=128, dtype="bf16",
                sink_blocks=1, window_blocks=1, alpha=0.1, seed=7)
    base.update(kw)
    return W.Workload(name=name, **base)


SMALL = [
    small("bf16_g4_d128_b128", seqlens=(1000, 333)),
    small("bf16_g8_d128_b128_paged64", num_q_heads=16, num_kv_heads=2, seqlens=(700, 1500), paged=True, page_size=64),
    small("bf16_g1_d64_b64", num_q_heads=2, num_kv_heads=2, head_dim=64, block_size=64, seqlens=(1300,)),
    small("bf16_g2_d64_b64_paged16", num_q_heads=4, num_kv_heads=2, head_dim=64, block_size=64, seqlens=(500, 777),
          paged=True, page_size=16),
    small("bf16_g4_d64_b128", head_dim=64, seqlens=(900,)),
    small("bf16_g4_d128_b64", block_size=64, seqlens=(1100,)),
    small("e4m3_g4_d128_b128_paged128", dtype="e4m3", seqlens=(2000, 900), paged=True, page_size=128),
    small("e4m3_g4_d128_b64", dtype="e4m3", block_size=64, seqlens=(1234,)),
    small("f32_g1_d64_b64", dtype="f32", num_q_heads=1, num_kv_heads=1, head_dim=64, block_size=64, seqlens=(1024,)),
    small("f32_g2_d64_b128", dtype="f32", num_q_heads=4, num_kv_heads=2, head_dim=64, seqlens=(640, 260)),
    small("bf16_dense_alpha0", alpha=0.0),
    small("bf16_no_correction", mean_correction=False, seqlens=(1500,)),
    small("bf16_min_sparse_last_n", seqlens=(300, 1700), min_sparse_len=512, last_n_blocks=2),
    small("bf16_tiny_and_empty_seqs", seqlens=(0, 1, 5, 130, 0, 257)),
    small("bf16_sink2_window4", sink_blocks=2, window_blocks=4, seqlens=(2500,)),
]


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_small_full_parity(w):
    inp = W.generate(w)
    ora = Hn.oracle_discovery(inp)
    # attention on the oracle's own mask (external index) ...
    rp, ci = Hn.oracle_csr(ora)
    run = Hn.run_gpu(inp, external_index=(rp, ci))
    Hn.compare_pooled(run, inp, ora)
    stats = Hn.compare_index(run, inp, ora)
    Hn.compare_attention_full(run, inp, ora)
    # ... and end to end on the library's own mask
    run2 = Hn.run_gpu(inp)
    if stats["borderline_mismatches"] == 0:
        Hn.compare_attention_full(run2, inp, ora)


SPLIT_CASES = [
    (small("split_bf16_g4", seqlens=(1500, 600)), 2),
    (small("split_bf16_g8_paged", num_q_heads=16, num_kv_heads=2, seqlens=(2000,), paged=True, page_size=64), 3),
    (small("split_e4m3", dtype="e4m3", seqlens=(1800,)), 5),
    (small("split_f32_d64_b64", dtype="f32", num_q_heads=2, num_kv_heads=2, head_dim=64, block_size=64,
           seqlens=(1100,)), 4),
    # few rows (one KV head, 2048 tokens): the automatic rule splits every row
    (small("split_auto_few_rows", num_q_heads=4, num_kv_heads=1, seqlens=(2048,), sink_blocks=2, window_blocks=4), 0),
]


@pytest.mark.parametrize("case", SPLIT_CASES, ids=[c[0].name for c in SPLIT_CASES])
def test_kv_splits_match_oracle(case):
    """Count-balanced KV splits (per-range partials merged by LSE) give the oracle's output."""
    from block_sparse_long_pooled_b200 import fp2
    w, splits = case
    inp = W.generate(w)
    ora = Hn.oracle_discovery(inp)
    rp, ci = Hn.oracle_csr(ora)
    run = Hn.run_gpu(inp, external_index=(rp, ci), kv_splits=splits)
    Hn.compare_attention_full(run, inp, ora)
    if splits == 0:
        ws = fp2.fp2_workspace_query(run.problem, run.params)
        one = fp2.fp2_workspace_query(run.problem, Hn.gpu_params(w, kv_splits=1))
        assert ws.scratch_bytes > one.scratch_bytes          # partial buffers were sized: it did split


# Adaptive splits: kv_splits < 0 cuts rows with more key tiles than -kv_splits into ranges of at
# most that many tiles (planned on the device; the last range of a row part to finish merges them).
# The G = 8 paged case needs more ranges than the 768 a call holds, so its later rows stay whole.
ADAPTIVE = [
    (small("adapt_bf16_g4", seqlens=(1500, 600), sink_blocks=2, window_blocks=4), -3),
    (small("adapt_bf16_g8_paged", num_q_heads=16, num_kv_heads=2, seqlens=(2000, 1900), paged=True, page_size=64), -1),
    (small("adapt_e4m3", dtype="e4m3", seqlens=(1800, 700)), -4),
    (small("adapt_f32_d64_b64", dtype="f32", num_q_heads=4, num_kv_heads=2, head_dim=64, block_size=64,
           seqlens=(1100,)), -5),
    (small("adapt_bf16_g1_d64_b64", num_q_heads=2, num_kv_heads=2, head_dim=64, block_size=64,
           seqlens=(2100, 50)), -7),
]


@pytest.mark.parametrize("case", ADAPTIVE, ids=lambda c: c[0].name)
def test_adaptive_splits_match_oracle(case):
    w, splits = case
    inp = W.generate(w)
    ora = Hn.oracle_discovery(inp)
    rp, ci = Hn.oracle_csr(ora)
    run = Hn.run_gpu(inp, external_index=(rp, ci), kv_splits=splits)
    Hn.compare_attention_full(run, inp, ora)


def test_prefill_single_call_with_adaptive_splits():
    """fp2_prefill (pool, discover and attend in one call, index and pooled buffers carved from its
    scratch) with ranges of at most two key tiles, against the oracle, output and LSE."""
    import torch
    from block_sparse_long_pooled_b200 import fp2
    w = small("prefill_adaptive", seqlens=(1700, 900), sink_blocks=2, window_blocks=4)
    inp = W.generate(w)
    ora = Hn.oracle_discovery(inp)
    dev = Hn.to_device(inp)
    prob = Hn.make_gpu_problem(inp, dev)
    params = Hn.gpu_params(w, kv_splits=-2)
    ws = fp2.fp2_workspace_query(prob, params)
    scratch = fp2.alloc_scratch(ws.prefill_scratch_bytes, "cuda")
    out = torch.empty(inp.q.shape, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((w.num_q_heads, w.total_tokens), dtype=torch.float32, device="cuda")
    fp2.fp2_prefill(prob, params, out, lse, scratch)
    torch.cuda.synchronize()
    assert fp2.fp2_get_device_status(scratch) == (0, 0)

    class R:
        pass
    run = R()
    run.out, run.lse = out, lse
    Hn.compare_attention_full(run, inp, ora)


def test_adaptive_splits_automatic_on_a_mixed_batch():
    """kv_splits = 0 with many rows (1220 row CTAs, under 16 waves): one 16K sequence among sixty
    300-token ones; its long rows are cut into ranges (range size = the launch's tile work over
    4 x SMs), the rest stay whole."""
    w = small("adapt_auto_mixed", seqlens=(300,) * 60 + (16000,), sink_blocks=2, window_blocks=4)
    inp = W.generate(w)
    ora = Hn.oracle_discovery(inp)
    rp, ci = Hn.oracle_csr(ora)
    run = Hn.run_gpu(inp, external_index=(rp, ci), kv_splits=0)
    pairs = Hn.select_pairs(inp, ora, n_random=1)
    Hn.compare_attention_pairs(run, inp, Hn.oracle_pairs(inp, ora, pairs))


def test_continuous_batch_of_301_requests():
    """A continuous batch above the former 128-request limit: 300 short requests of 1 to 600 tokens
    and one 20K-token request, paged; the whole index and whole pairs of every request's first and
    last blocks (and the long request's needle and heaviest rows) against the oracle."""
    rng = np.random.default_rng(5)
    lens = tuple(int(x) for x in rng.integers(1, 601, size=300)) + (20000,)
    w = small("batch301_paged", seqlens=lens, num_q_heads=8, num_kv_heads=2, paged=True, page_size=64,
              sink_blocks=2, window_blocks=4, min_sparse_len=256)
    inp = W.generate(w)
    ora = Hn.oracle_discovery(inp)
    rp, ci = Hn.oracle_csr(ora)
    run = Hn.run_gpu(inp, external_index=(rp, ci))
    Hn.compare_pooled(run, inp, ora)
    stats = Hn.compare_index(run, inp, ora)
    pairs = Hn.select_pairs(inp, ora, n_random=0)
    Hn.compare_attention_pairs(run, inp, Hn.oracle_pairs(inp, ora, pairs))
    if stats["borderline_mismatches"] == 0:
        run2 = Hn.run_gpu(inp)
        Hn.compare_attention_pairs(run2, inp, Hn.oracle_pairs(inp, ora, pairs))


def test_tiny_workload_end_to_end():
    """The 1K fp32 workload with its four planted needle blocks, through fp2_prefill."""
    import torch
    from block_sparse_long_pooled_b200 import fp2
    w = W.WORKLOADS["tiny_1k_f32"]
    inp = W.generate(w)
    ora = Hn.oracle_discovery(inp)
    dev = Hn.to_device(inp)
    prob = Hn.make_gpu_problem(inp, dev)
    params = Hn.gpu_params(w)
    ws = fp2.fp2_workspace_query(prob, params)
    scratch = fp2.alloc_scratch(ws.prefill_scratch_bytes, "cuda")
    out = torch.empty(inp.q.shape, dtype=torch.float32, device="cuda")
    lse = torch.empty((w.num_q_heads, w.total_tokens), dtype=torch.float32, device="cuda")
    fp2.fp2_prefill(prob, params, out, lse, scratch)
    torch.cuda.synchronize()
    assert fp2.fp2_get_device_status(scratch) == (0, 0)
    # needle blocks are kept for the needle query rows' blocks
    assert all(ora[0].kept[0, i, j] for j in inp.needle_key_blocks[0] for i in range(j, 16))

    class R:
        pass
    run = R()
    run.out, run.lse = out, lse
    Hn.compare_attention_full(run, inp, ora)


# The five workloads, plus the served configuration's last-n-blocks 8 on the 64K FP8 layer.
FULL = ["llama8b_32k_bf16", "llama8b_128k_bf16", "llama8b_128k_e4m3", "qwen30b_64k_paged_bf16",
        "varlen6_paged_e4m3", "qwen4b_64k_e4m3_lastn8"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_workloads(name):
    """A full-size workload: the pooled means, the whole index, and whole (KV group, query block)
    pairs of the output and LSE (every head of the group, every token of the block; needle blocks,
    the last blocks, the heaviest rows and the dense-cutoff requests among them), first attending on
    the oracle's index, then, when no borderline block differs, on the library's own index."""
    import torch
    w = W.WORKLOADS[name]
    inp = W.generate(w)
    ora = Hn.oracle_discovery(inp)
    rp, ci = Hn.oracle_csr(ora)
    run = Hn.run_gpu(inp, external_index=(rp, ci), lse=True)
    Hn.compare_pooled(run, inp, ora)
    stats = Hn.compare_index(run, inp, ora)
    pairs = Hn.select_pairs(inp, ora)
    assert len(pairs) >= 32
    ref = Hn.oracle_pairs(inp, ora, pairs)
    r1 = Hn.compare_attention_pairs(run, inp, ref)
    print(f"{name}: density {stats['density']*100:.2f}%  borderline {stats['borderline_blocks']} "
          f"mismatched {stats['borderline_mismatches']}  pairs {len(pairs)} rows {r1['rows']} "
          f"max-abs {r1['max_abs']:.2e} rel-L2 {r1['rel_l2']:.2e} lse {r1['lse_max_abs']:.2e}")
    if name == "llama8b_128k_bf16":
        assert 0.04 <= stats["density"] <= 0.06
    if w.min_sparse_len > 0:
        dense_pairs = [p for p in pairs if w.seqlens[p[0]] < w.min_sparse_len]
        assert len(dense_pairs) >= 2 * w.num_kv_heads
    del run
    torch.cuda.empty_cache()
    if stats["borderline_mismatches"] == 0:
        run2 = Hn.run_gpu(inp, lse=True)
        r2 = Hn.compare_attention_pairs(run2, inp, ref)
        print(f"{name} (own index): max-abs {r2['max_abs']:.2e} rel-L2 {r2['rel_l2']:.2e} "
              f"lse {r2['lse_max_abs']:.2e}")


# More than 1024 key blocks: discovery streams 11 to 32 key chunks of 128 blocks through each
# CTA, twice (row maxima, then the threshold test); the last case is the largest sequence the ABI
# accepts (FP2_MAX_BLOCKS = 4096).
LONG = [
    small("long_g4_tile24", num_q_heads=4, num_kv_heads=1, head_dim=64, block_size=64, seqlens=(1400 * 64 - 17,),
          sink_blocks=2, window_blocks=4),
    small("long_g8_tile16", num_q_heads=8, num_kv_heads=1, head_dim=64, block_size=64, seqlens=(2100 * 64 + 5,),
          sink_blocks=2, window_blocks=4),
    small("long_g4_max_blocks", num_q_heads=4, num_kv_heads=1, head_dim=64, block_size=64, seqlens=(4096 * 64,),
          sink_blocks=2, window_blocks=4),
]


@pytest.mark.parametrize("w", LONG, ids=lambda w: w.name)
def test_long_sequences(w):
    inp = W.generate(w)
    ora = Hn.oracle_discovery(inp, head_chunk=4)
    rp, ci = Hn.oracle_csr(ora)
    run = Hn.run_gpu(inp, external_index=(rp, ci), lse=True)
    Hn.compare_pooled(run, inp, ora)
    stats = Hn.compare_index(run, inp, ora)
    print(f"{w.name}: density {stats['density']*100:.2f}%  borderline {stats['borderline_blocks']} "
          f"mismatched {stats['borderline_mismatches']}")
    Hn.compare_attention_pairs(run, inp, Hn.oracle_pairs(inp, ora, Hn.select_pairs(inp, ora)))


def test_page_table_out_of_range_is_reported_not_faulted():
    """A corrupt page id is clamped on the device and reported through the status word."""
    import torch
    from block_sparse_long_pooled_b200 import fp2
    w = small("paged_corrupt", paged=True, page_size=64, seqlens=(600,))
    inp = W.generate(w)
    dev = Hn.to_device(inp)
    dev["page_table"][0, 3] = 10 ** 6
    prob = Hn.make_gpu_problem(inp, dev)
    params = Hn.gpu_params(w)
    ws = fp2.fp2_workspace_query(prob, params)
    scratch = fp2.alloc_scratch(ws.prefill_scratch_bytes, "cuda")
    out = torch.empty(inp.q.shape, dtype=torch.bfloat16, device="cuda")
    fp2.fp2_prefill(prob, params, out, None, scratch)
    torch.cuda.synchronize()
    st, bits = fp2.fp2_get_device_status(scratch)
    assert st == fp2.FP2_ERR_DEVICE_BOUNDS and bits & fp2.FP2_DEV_PAGE_OOB
    # the context is still healthy: a clean call succeeds afterwards
    dev["page_table"][0, 3] = int(inp.page_table[0, 3])
    fp2.fp2_prefill(prob, params, out, None, scratch)
    torch.cuda.synchronize()
    assert fp2.fp2_get_device_status(scratch) == (0, 0)


def test_external_index_without_diagonal_is_reported():
    import torch
    from block_sparse_long_pooled_b200 import fp2
    w = small("bad_index", seqlens=(512,))
    inp = W.generate(w)
    N = 4
    rows = N * w.num_kv_heads
    # every row keeps only block 0: rows i > 0 miss their diagonal block
    rp = np.arange(rows + 1, dtype=np.int32)
    ci = np.zeros(rows, dtype=np.int32)
    dev = Hn.to_device(inp)
    prob = Hn.make_gpu_problem(inp, dev)
    params = Hn.gpu_params(w)
    ws = fp2.fp2_workspace_query(prob, params)
    pst, _ = fp2.alloc_pooled(ws, prob, "cuda")
    scratch = fp2.alloc_scratch(ws.scratch_bytes, "cuda")
    fp2.fp2_pool(prob, params, pst, scratch)
    ix = fp2.index_struct(torch.from_numpy(rp).cuda(), torch.from_numpy(ci).cuda())
    out = torch.empty(inp.q.shape, dtype=torch.bfloat16, device="cuda")
    fp2.fp2_attend(prob, params, pst, ix, out, None, scratch)
    torch.cuda.synchronize()
    st, bits = fp2.fp2_get_device_status(scratch)
    assert st == fp2.FP2_ERR_DEVICE_BOUNDS and bits & fp2.FP2_DEV_INDEX_OOB


def test_host_validation_launches_nothing():
    import torch
    from block_sparse_long_pooled_b200 import fp2
    w = small("val", seqlens=(256,))
    inp = W.generate(w)
    dev = Hn.to_device(inp)
    prob = Hn.make_gpu_problem(inp, dev)
    params = Hn.gpu_params(w)
    ws = fp2.fp2_workspace_query(prob, params)
    scratch = fp2.alloc_scratch(ws.prefill_scratch_bytes, "cuda")
    out = torch.empty(inp.q.shape, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fp2.FP2Error) as e:
        fp2.fp2_prefill(prob, params, out, None, scratch[: ws.prefill_scratch_bytes - 256])
    assert e.value.status == fp2.FP2_ERR_WORKSPACE_TOO_SMALL
