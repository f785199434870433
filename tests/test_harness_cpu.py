"""CPU checks of the test harness itself: the per-pair oracle used at full size gives the same
rows as the whole-sequence oracle, and the pair selection covers what it promises."""

import math

import numpy as np

from oracle import fp2_oracle as O
from synth import workloads as W
from tests import harness as Hn


def _whole(inp, ora):
    w = inp.workload
    scale = 1.0 / math.sqrt(w.head_dim)
    outs, lses = [], []
    for r in range(len(w.seqlens)):
        a, b = int(inp.cu_seqlens[r]), int(inp.cu_seqlens[r + 1])
        if b == a:
            continue
        k, v = Hn.seq_kv(inp, r)
        o = ora[r]
        Or, Lr = O.attend(inp.dequant("q", tokens=slice(a, b)), k, v, o.kbar, o.vbar, o.counts, o.kept,
                          w.block_size, scale, w.mean_correction)
        outs.append(Or)
        lses.append(Lr)
    return np.concatenate(outs), np.concatenate(lses, axis=1)


def test_pair_oracle_matches_whole_sequence_oracle():
    for w in (W.Workload(name="pairs_a", seqlens=(700, 0, 1300), num_q_heads=8, num_kv_heads=2, head_dim=64,
                         block_size=64, dtype="bf16", min_sparse_len=800, seed=21),
              W.Workload(name="pairs_b", seqlens=(1500,), num_q_heads=8, num_kv_heads=1, head_dim=64,
                         block_size=128, dtype="e4m3", paged=True, page_size=64, seed=22)):
        inp = W.generate(w)
        ora = Hn.oracle_discovery(inp)
        pairs = Hn.select_pairs(inp, ora, n_random=2)
        O_ref, L_ref, toks, heads = Hn.oracle_pairs(inp, ora, pairs)
        O_all, L_all = _whole(inp, ora)
        assert np.array_equal(O_ref, O_all[toks, heads])
        assert np.array_equal(L_ref, L_all[heads, toks])
        # every row of every selected pair is there, once
        B, G = w.block_size, w.group
        want = sum(G * (min(w.seqlens[r], (i + 1) * B) - i * B) for r, g, i in pairs)
        assert len(toks) == want == len(set(zip(toks.tolist(), heads.tolist())))


def test_pair_selection_covers_last_heavy_needle_and_dense_blocks():
    w = W.Workload(name="pairs_c", seqlens=(1000, 9000), num_q_heads=8, num_kv_heads=2, head_dim=64,
                   block_size=64, dtype="bf16", min_sparse_len=2000, seed=23)
    inp = W.generate(w)
    ora = Hn.oracle_discovery(inp)
    pairs = set(Hn.select_pairs(inp, ora))
    for r, L in enumerate(w.seqlens):
        N = -(-L // w.block_size)
        for i in range(N - 2, N):
            assert all((r, g, i) in pairs for g in range(w.num_kv_heads))
        for j in inp.needle_key_blocks[r]:
            assert any(p[0] == r and p[2] == j for p in pairs)
    assert all(any(p[0] == 0 and p[2] == i for p in pairs) for i in range(-(-1000 // 64)))   # dense request
    heavy = max((int(ora[r].kept[g, i].sum()), r, g, i) for r in range(2) for g in range(2)
                for i in range(ora[r].kept.shape[1]))
    assert heavy[1:] in pairs
