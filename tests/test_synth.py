"""The seeded input generators: determinism, shapes, needle structure and FP8 quantisation."""

import math

import numpy as np
import torch

from synth import workloads as W


def _small(**kw):
    base = W.WORKLOADS["llama8b_32k_bf16"].replace(seqlens=(700, 300), num_q_heads=4, num_kv_heads=2,
                                                     head_dim=64, block_size=64)
    return base.replace(**kw)


def test_deterministic_and_shapes():
    w = _small()
    a, b = W.generate(w), W.generate(w)
    assert a.q.shape == (1000, 4, 64) and a.k.shape == (1000, 2, 64) and a.q.dtype == torch.bfloat16
    assert torch.equal(a.q, b.q) and torch.equal(a.k, b.k) and torch.equal(a.v, b.v)
    c = W.generate(w.replace(seed=99))
    assert not torch.equal(a.q, c.q)
    assert list(a.cu_seqlens) == [0, 700, 1000]


def test_needles_planted():
    w = _small()
    inp = W.generate(w)
    d = w.head_dim
    for r, blocks in enumerate(inp.needle_key_blocks):
        assert len(blocks) == 1 and 0 not in blocks
        j = blocks[0]
        t0 = int(inp.cu_seqlens[r]) + j * w.block_size
        for g in range(w.num_kv_heads):
            kk = inp.k[t0, g].float()
            assert abs(float(kk.norm()) - 3 * math.sqrt(d)) < 0.05 * 3 * math.sqrt(d)
            assert torch.equal(inp.k[t0, g], inp.k[t0 + 5, g])
    # 10 % of the query rows of every sequence carry the needle direction of their KV head
    q = inp.q.float()
    norms = q.norm(dim=-1)
    frac = float((norms[:700, 0] > 2.5 * math.sqrt(d)).float().mean())
    assert abs(frac - 0.10) < 0.02


def test_fp8_quantisation_per_tensor_absmax():
    w = _small(dtype="e4m3")
    inp = W.generate(w)
    ref = W.generate(w.replace(dtype="bf16"))
    for name in ("q", "k", "v"):
        x8 = getattr(inp, name)
        assert x8.dtype == torch.float8_e4m3fn
        xs = getattr(ref, name).to(torch.float64)
        ds = getattr(inp, name + "_descale")
        assert ds == float(np.float32(float(xs.abs().max()) / 448.0))
        deq = x8.to(torch.float64) * ds
        assert float(x8.to(torch.float32).abs().max()) <= 448.0
        # relative error of round-to-nearest e4m3 (3 mantissa bits) is at most 2^-4 for normal values
        big = xs.abs() > 2 ** -6 * ds
        rel = ((deq - xs).abs() / xs.abs())[big]
        assert float(rel.max()) <= 2 ** -4 + 1e-6


def test_paged_cache_matches_contiguous():
    w = _small(paged=True, page_size=64)
    inp = W.generate(w)
    pt = inp.page_table
    perm = sorted(int(x) for x in pt[pt >= 0])
    assert perm == list(range(inp.k_cache.shape[0]))
    for r, L in enumerate(w.seqlens):
        for t in (0, 63, 64, L - 1):
            page, off = pt[r, t // 64], t % 64
            assert torch.equal(inp.k_cache[page, off], inp.k[int(inp.cu_seqlens[r]) + t])
            assert torch.equal(inp.v_cache[page, off], inp.v[int(inp.cu_seqlens[r]) + t])


def test_workload_table():
    ws = W.WORKLOADS
    assert ws["llama8b_128k_bf16"].dense_equiv_flops() == 4 * 128 * 32 * 131072 * 131073 / 2
    assert abs(ws["llama8b_128k_bf16"].dense_equiv_flops() - 1.407e14) / 1.407e14 < 1e-3
    assert ws["varlen6_paged_e4m3"].total_tokens == 251904
    assert ws["tiny_1k_f32"].iid and ws["tiny_1k_f32"].dtype == "f32"
