"""Pins of the fp64 oracle against facts fixed by the pages and by mathematics.

Each test checks the oracle against something other than itself: torch's
scaled-dot-product attention, a closed form in which mean correction is exact,
pure-Python brute force on tiny inputs, exact rational arithmetic, invariants of
the max-based threshold rule, and the index-size arithmetic printed in Table 7
of the FlashPrefill V2 paper page.
"""

import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import fp2_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def sdpa_dense(q, k, v, scale, allowed=None):
    """torch's fp64 attention; allowed: optional [Hq, L, L] boolean of visible (t, u) pairs."""
    L, Hq, d = q.shape
    G = Hq // k.shape[1]
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]
    kt = torch.from_numpy(np.repeat(k, G, axis=1)).permute(1, 0, 2)[None]
    vt = torch.from_numpy(np.repeat(v, G, axis=1)).permute(1, 0, 2)[None]
    if allowed is None:
        o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=scale)
    else:
        o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=torch.from_numpy(allowed)[None],
                                                             scale=scale)
    return o[0].permute(1, 0, 2).numpy()


def rand_qkv(rng, L, Hq, Hkv, d):
    return (rng.standard_normal((L, Hq, d)), rng.standard_normal((L, Hkv, d)), rng.standard_normal((L, Hkv, d)))


# ---------------------------------------------------------------- pooling

def test_pool_matches_python_loops():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((13, 2, 3))
    means, counts = O.pool_blocks(x, 4)
    assert list(counts) == [4, 4, 4, 1]
    for i in range(4):
        toks = range(4 * i, min(13, 4 * i + 4))
        for h in range(2):
            for c in range(3):
                acc = 0.0
                for t in toks:
                    acc += x[t, h, c]
                assert abs(means[i, h, c] - acc / len(toks)) < 1e-15


def test_pool_exact_rational_identity():
    """mean = (block sum)/n exactly rounded, checked in rational arithmetic on integer inputs."""
    rng = np.random.default_rng(1)
    x = rng.integers(-1000, 1000, size=(37, 1, 5)).astype(np.float64)
    means, counts = O.pool_blocks(x, 8)
    for i in range(len(counts)):
        for c in range(5):
            s = sum(Fraction(int(v)) for v in x[8 * i: 8 * i + counts[i], 0, c])
            assert means[i, 0, c] == float(s / int(counts[i]))


def test_varlen_pool_concatenates_sequences():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((10 + 7, 1, 2))
    m, c = O.pool_varlen(x, [0, 10, 17], 4)
    m0, c0 = O.pool_blocks(x[:10], 4)
    m1, c1 = O.pool_blocks(x[10:], 4)
    assert np.array_equal(c, np.concatenate([c0, c1])) and list(c) == [4, 4, 2, 4, 3]
    assert np.allclose(m, np.concatenate([m0, m1]), rtol=0, atol=0)


# ---------------------------------------------------------------- selection

def _params(**kw):
    base = dict(block_size=4, alpha=0.1, sink_blocks=1, window_blocks=1, last_n_blocks=0, min_sparse_len=0)
    base.update(kw)
    return O.SparseParams(**base)


def test_select_bruteforce_tiny():
    """Per-element Python loop of the rule on L <= 64, B = 4, d = 4."""
    rng = np.random.default_rng(3)
    for trial in range(6):
        L = int(rng.integers(5, 65))
        Hq, Hkv, d, B = 4, 2, 4, 4
        q, k, _ = rand_qkv(rng, L, Hq, Hkv, d)
        qbar, _ = O.pool_blocks(q, B)
        kbar, _ = O.pool_blocks(k, B)
        p = _params(alpha=float(rng.choice([0.05, 0.3, 0.7])), sink_blocks=int(rng.integers(0, 3)),
                    window_blocks=int(rng.integers(0, 3)), last_n_blocks=int(rng.integers(0, 2)))
        s = O.block_scores(qbar, kbar, 0.5)
        kept, _ = O.select_blocks(s, Hkv, L, p)
        N = qbar.shape[0]
        for g in range(Hkv):
            for i in range(N):
                for j in range(N):
                    want = False
                    if j <= i:
                        if j < p.sink_blocks or j > i - max(1, p.window_blocks) or i >= N - p.last_n_blocks:
                            want = True
                        for h in (2 * g, 2 * g + 1):
                            sc = [sum(qbar[i, h, c] * kbar[jj, g, c] for c in range(d)) * 0.5 for jj in range(i + 1)]
                            if sc[j] >= max(sc) + math.log(p.alpha):
                                want = True
                    assert kept[g, i, j] == want, (trial, g, i, j)


def test_select_invariants():
    rng = np.random.default_rng(4)
    N, Hq, Hkv = 40, 8, 2
    s = rng.standard_normal((Hq, N, N)) * 2
    s[:, ~np.tri(N, dtype=bool)] = -np.inf
    L = N * 16
    causal = np.tri(N, dtype=bool)
    base = _params(block_size=16, sink_blocks=2, window_blocks=3)
    prev = None
    for a in (0.9, 0.5, 0.1, 0.01, 1e-4):
        kept, _ = O.select_blocks(s, Hkv, L, O.SparseParams(**{**base.__dict__, "alpha": a}))
        assert not np.any(kept & ~causal)
        for i in range(N):
            assert kept[:, i, i].all()                          # diagonal
            assert kept[:, i, : min(2, i + 1)].all()            # sinks
            assert kept[:, i, max(0, i - 2): i + 1].all()       # window of 3
        if prev is not None:
            assert np.all(prev <= kept)                          # higher alpha keeps a subset
        prev = kept
    # alpha = 0 keeps every causal block
    kept0, _ = O.select_blocks(s, Hkv, L, O.SparseParams(**{**base.__dict__, "alpha": 0.0}))
    assert np.array_equal(kept0, np.broadcast_to(causal, kept0.shape))
    # alpha = 1 keeps forced blocks plus the per-head argmax only
    kept1, _ = O.select_blocks(s, Hkv, L, O.SparseParams(**{**base.__dict__, "alpha": 1.0}))
    forced = O.forced_blocks(N, L, O.SparseParams(**{**base.__dict__, "alpha": 1.0}))
    for g in range(Hkv):
        want = forced.copy()
        for h in range(g * 4, g * 4 + 4):
            for i in range(N):
                want[i, int(np.argmax(s[h, i, : i + 1]))] = True
        assert np.array_equal(kept1[g], want)


def test_select_union_over_group_equals_per_head_runs():
    """G query heads: the KV-head row is the OR of each head's own G = 1 selection."""
    rng = np.random.default_rng(5)
    N, Hq, Hkv = 24, 6, 2
    s = rng.standard_normal((Hq, N, N))
    s[:, ~np.tri(N, dtype=bool)] = -np.inf
    p = _params(block_size=8, sink_blocks=1, window_blocks=2, alpha=0.2)
    kept, _ = O.select_blocks(s, Hkv, N * 8, p)
    for g in range(Hkv):
        union = np.zeros((N, N), dtype=bool)
        for h in range(3 * g, 3 * g + 3):
            kh, _ = O.select_blocks(s[h:h + 1], 1, N * 8, p)
            union |= kh[0]
        assert np.array_equal(kept[g], union)


def test_select_dense_cutoff_and_last_n():
    rng = np.random.default_rng(6)
    N = 12
    s = rng.standard_normal((2, N, N))
    s[:, ~np.tri(N, dtype=bool)] = -np.inf
    causal = np.tri(N, dtype=bool)
    kept, border = O.select_blocks(s, 1, N * 4, _params(min_sparse_len=N * 4 + 1, alpha=0.9))
    assert np.array_equal(kept[0], causal) and not border.any()
    kept, _ = O.select_blocks(s, 1, N * 4, _params(last_n_blocks=3, alpha=0.99))
    assert kept[0, N - 3:].sum() == causal[N - 3:].sum()


def test_borderline_flags_only_near_threshold():
    s = np.full((1, 3, 3), -np.inf)
    s[0, 2, :] = [0.0, math.log(0.5) + 5e-4, 0.0]
    s[0, 1, :2] = [0.0, 0.0]
    s[0, 0, 0] = 0.0
    p = _params(alpha=0.5, sink_blocks=0, window_blocks=1)
    kept, border = O.select_blocks(s, 1, 12, p)
    assert kept[0, 2, 1] and border[0, 2, 1] and not border[0, 2, 0]


def test_index_memory_matches_table7():
    g = json.load(open(os.path.join(GOLDEN, "table7_index_memory.json")))
    rng = np.random.default_rng(7)
    for L, mask_mb, csr_mb, dens in zip(g["seq_len"], g["dense_mask_MB"], g["csr_MB"], g["density"]):
        nq = L // g["q_tile"]
        nk_mask = L // g["mask_kv_tile"]
        assert g["num_q_heads"] * nq * nk_mask == mask_mb * 2 ** 20          # 1 byte per tile, exact
        nk = L // g["csr_kv_tile"]
        # a kept pattern at the stated density over the causal (Q tile, 64-token KV tile) pairs
        causal = (np.arange(nk)[None, :] * g["csr_kv_tile"]) < ((np.arange(nq)[:, None] + 1) * g["q_tile"])
        kept = np.stack([causal & (rng.random(causal.shape) < dens) for _ in range(g["num_q_heads"])])
        nnz = 0
        for h in range(g["num_q_heads"]):
            row_ptr, col_idx = O.csr_from_kept([kept[h:h + 1]])
            nnz += len(col_idx)
        nbytes = 4 * nnz
        assert abs(nbytes / 1e6 - csr_mb) / csr_mb < 0.15, (L, nbytes)


# ---------------------------------------------------------------- attention

def _run(q, k, v, B, p, Hkv):
    return O.prefill(q, k, v, [0, q.shape[0]], Hkv, p)


@pytest.mark.parametrize("L,B,G", [(37, 8, 1), (64, 16, 2), (50, 4, 4)])
def test_alpha_zero_equals_dense_softmax_attention(L, B, G):
    rng = np.random.default_rng(8)
    Hkv, d = 2, 8
    q, k, v = rand_qkv(rng, L, Hkv * G, Hkv, d)
    r = _run(q, k, v, B, _params(block_size=B, alpha=0.0), Hkv)
    ref = sdpa_dense(q, k, v, 1 / math.sqrt(d))
    assert np.max(np.abs(r["O"] - ref)) < 1e-12
    # LSE is the log of the dense causal softmax normaliser
    z = np.einsum("thd,uhd->htu", q, np.repeat(k, G, axis=1)) / math.sqrt(d)
    z[:, ~np.tri(L, dtype=bool)] = -np.inf
    lse = torch.logsumexp(torch.from_numpy(z), dim=-1).numpy()
    assert np.max(np.abs(r["LSE"] - lse)) < 1e-12


def test_short_sequence_below_min_sparse_len_is_dense():
    rng = np.random.default_rng(9)
    q, k, v = rand_qkv(rng, 40, 2, 1, 8)
    r = _run(q, k, v, 4, _params(alpha=0.9, min_sparse_len=41), 1)
    assert np.max(np.abs(r["O"] - sdpa_dense(q, k, v, 1 / math.sqrt(8)))) < 1e-12


@pytest.mark.parametrize("alpha", [0.05, 0.3, 0.9, 1.0])
def test_mean_correction_exact_when_keys_constant_in_blocks(alpha):
    """Closed form: if every key of block j equals kbar_j, the pruned block's exact contribution
    sum_u e^{q.k_u s} (v_u, 1) equals n_j e^{q.kbar_j s} (vbar_j, 1), so O equals dense attention."""
    rng = np.random.default_rng(10)
    L, B, Hq, Hkv, d = 77, 8, 4, 2, 6
    q, _, v = rand_qkv(rng, L, Hq, Hkv, d)
    N = O.num_blocks(L, B)
    q = q * 2.0
    kb = rng.standard_normal((N, Hkv, d)) * 3.0
    k = np.repeat(kb, B, axis=0)[:L]
    r = _run(q, k, v, B, _params(block_size=B, alpha=alpha, sink_blocks=0, window_blocks=1), Hkv)
    assert sum(x.sum() for x in r["kept"]) < sum(np.tri(N).sum() * Hkv for _ in [0])   # something is pruned
    assert np.max(np.abs(r["O"] - sdpa_dense(q, k, v, 1 / math.sqrt(d)))) < 1e-12
    # ... and without the correction the result differs
    r2 = _run(q, k, v, B, O.SparseParams(**{**_params(block_size=B, alpha=alpha, sink_blocks=0,
                                                      window_blocks=1).__dict__, "mean_correction": False}), Hkv)
    assert np.max(np.abs(r2["O"] - r["O"])) > 1e-3


def test_no_correction_equals_masked_dense():
    rng = np.random.default_rng(11)
    L, B, Hq, Hkv, d = 96, 8, 4, 1, 8
    q, k, v = rand_qkv(rng, L, Hq, Hkv, d)
    q += np.repeat(rng.standard_normal((L // B, Hq, d)) * 2, B, axis=0)
    k += np.repeat(rng.standard_normal((L // B, Hkv, d)) * 2, B, axis=0)
    p = _params(block_size=B, alpha=0.3, sink_blocks=1, window_blocks=2, mean_correction=False)
    r = _run(q, k, v, B, p, Hkv)
    kept = r["kept"][0]
    tok_block = np.arange(L) // B
    allowed = np.zeros((Hq, L, L), dtype=bool)
    for h in range(Hq):
        allowed[h] = kept[h // (Hq // Hkv)][tok_block[:, None], tok_block[None, :]] & np.tri(L, dtype=bool)
    assert (~kept[0] & np.tri(kept.shape[1], dtype=bool)).any()
    assert np.max(np.abs(r["O"] - sdpa_dense(q, k, v, 1 / math.sqrt(d), allowed))) < 1e-12


def test_output_in_convex_hull_of_values_and_means():
    rng = np.random.default_rng(12)
    L, B, d = 80, 8, 5
    q, k, v = rand_qkv(rng, L, 2, 1, d)
    r = _run(q, k, v, B, _params(block_size=B, alpha=0.5, sink_blocks=0, window_blocks=1), 1)
    vbar = r["vbar"][0]
    for t in range(L):
        i = t // B
        pool = np.concatenate([v[: (i + 1) * B, 0], vbar[: i + 1, 0]])
        for h in range(2):
            assert np.all(r["O"][t, h] >= pool.min(axis=0) - 1e-12)
            assert np.all(r["O"][t, h] <= pool.max(axis=0) + 1e-12)


def test_attention_bruteforce_token_loop():
    """Token-by-token pure-Python evaluation of the Figure 4 estimator on a tiny case."""
    rng = np.random.default_rng(13)
    L, B, Hq, Hkv, d = 23, 4, 2, 1, 3
    q, k, v = rand_qkv(rng, L, Hq, Hkv, d)
    p = _params(block_size=B, alpha=0.4, sink_blocks=0, window_blocks=1)
    r = _run(q, k, v, B, p, Hkv)
    kept = r["kept"][0][0]
    sc = 1 / math.sqrt(d)
    for h in range(Hq):
        for t in range(L):
            i = t // B
            terms = []
            for j in range(i + 1):
                toks = list(range(j * B, min(L, (j + 1) * B)))
                if kept[i, j]:
                    for u in toks:
                        if u <= t:
                            terms.append((sum(q[t, h, c] * k[u, 0, c] for c in range(d)) * sc, list(v[u, 0])))
                else:
                    kb = [sum(k[u, 0, c] for u in toks) / len(toks) for c in range(d)]
                    vb = [sum(v[u, 0, c] for u in toks) / len(toks) for c in range(d)]
                    logit = sum(q[t, h, c] * kb[c] for c in range(d)) * sc
                    terms.append((logit + math.log(len(toks)), vb))
            m = max(z for z, _ in terms)
            den = sum(math.exp(z - m) for z, _ in terms)
            for c in range(d):
                num = sum(math.exp(z - m) * vv[c] for z, vv in terms)
                assert abs(r["O"][t, h, c] - num / den) < 1e-12
            assert abs(r["LSE"][h, t] - (m + math.log(den))) < 1e-12


def test_varlen_equals_per_sequence_and_paged_equals_contiguous():
    rng = np.random.default_rng(14)
    lens = [19, 40, 8]
    B, Hq, Hkv, d, ps = 8, 4, 2, 4, 4
    T = sum(lens)
    q, k, v = rand_qkv(rng, T, Hq, Hkv, d)
    cu = np.concatenate([[0], np.cumsum(lens)])
    p = _params(block_size=B, alpha=0.3, sink_blocks=1, window_blocks=1)
    packed = O.prefill(q, k, v, cu, Hkv, p)
    for r in range(3):
        a, b = cu[r], cu[r + 1]
        single = O.prefill(q[a:b], k[a:b], v[a:b], [0, b - a], Hkv, p)
        assert np.max(np.abs(single["O"] - packed["O"][a:b])) == 0.0
    # paged cache with a shuffled page table
    npages = [-(-L // ps) for L in lens]
    perm = rng.permutation(sum(npages))
    pt = np.full((3, max(npages)), -1)
    kc = np.zeros((sum(npages), ps, Hkv, d))
    vc = np.zeros_like(kc)
    off = 0
    for r, L in enumerate(lens):
        for pg in range(npages[r]):
            pid = perm[off + pg]
            pt[r, pg] = pid
            rows = slice(cu[r] + pg * ps, cu[r] + min(L, (pg + 1) * ps))
            n = rows.stop - rows.start
            kc[pid, :n] = k[rows]
            vc[pid, :n] = v[rows]
        off += npages[r]
    paged = O.prefill(q, None, None, cu, Hkv, p, k_cache=kc, v_cache=vc, page_table=pt)
    assert np.max(np.abs(paged["O"] - packed["O"])) == 0.0
    assert np.array_equal(paged["row_ptr"], packed["row_ptr"]) and np.array_equal(paged["col_idx"], packed["col_idx"])


def test_group_of_one_equals_per_head():
    rng = np.random.default_rng(15)
    L, B, d = 48, 8, 4
    q, k, v = rand_qkv(rng, L, 2, 2, d)
    p = _params(block_size=B, alpha=0.3)
    both = _run(q, k, v, B, p, 2)
    for h in range(2):
        one = _run(q[:, h:h + 1], k[:, h:h + 1], v[:, h:h + 1], B, p, 1)
        assert np.max(np.abs(one["O"][:, 0] - both["O"][:, h])) == 0.0


def test_sampled_rows_equal_full_output():
    rng = np.random.default_rng(16)
    L, B, Hq, Hkv, d = 70, 8, 4, 2, 4
    q, k, v = rand_qkv(rng, L, Hq, Hkv, d)
    p = _params(block_size=B, alpha=0.3)
    r = _run(q, k, v, B, p, Hkv)
    rows = np.array([[0, 0], [69, 3], [35, 1], [36, 1], [8, 2]])
    o, lse = O.attend(q, k, v, r["kbar"][0], r["vbar"][0], r["counts"][0], r["kept"][0], B, 0.5, True, rows=rows)
    for n, (t, h) in enumerate(rows):
        assert np.max(np.abs(o[n] - r["O"][t, h])) < 1e-14
        assert abs(lse[n] - r["LSE"][h, t]) < 1e-14


def test_csr_layout_row_order():
    kept0 = np.zeros((2, 2, 2), dtype=bool)
    kept0[0] = [[1, 0], [1, 1]]
    kept0[1] = [[1, 0], [0, 1]]
    kept1 = np.ones((2, 1, 1), dtype=bool)
    row_ptr, col_idx = O.csr_from_kept([kept0, kept1])
    # rows: (blk0,g0) (blk0,g1) (blk1,g0) (blk1,g1) (seq1 blk0,g0) (seq1 blk0,g1)
    assert list(row_ptr) == [0, 1, 2, 4, 5, 6, 7]
    assert list(col_idx) == [0, 0, 0, 1, 1, 0, 0]
    back = O.kept_from_csr(row_ptr, col_idx, [2, 1], 1, 2)
    assert np.array_equal(back[0], kept0) and np.array_equal(back[1], kept1)


# ---------------------------------------------------------------- chunked prefill (q_len < kv_len)

def test_chunk_equals_last_rows_of_whole_sequence():
    """Bottom-right alignment: a chunk's selection and output are the whole sequence's last rows."""
    rng = np.random.default_rng(20)
    L, B, Hq, Hkv, d = 100, 8, 4, 2, 6
    q, k, v = rand_qkv(rng, L, Hq, Hkv, d)
    q += np.repeat(rng.standard_normal((13, Hq, d)) * 2, B, axis=0)[:L]
    k += np.repeat(rng.standard_normal((13, Hkv, d)) * 2, B, axis=0)[:L]
    p = _params(block_size=B, alpha=0.3, sink_blocks=1, window_blocks=2, last_n_blocks=1)
    whole = O.prefill(q, k, v, [0, L], Hkv, p)
    for prefix in (0, 32, 64, 96):
        ch = O.prefill(q[prefix:], k, v, [0, L - prefix], Hkv, p, cu_seqlens_k=[0, L])
        assert np.array_equal(ch["kept"][0], whole["kept"][0][:, prefix // B:, :])
        assert np.max(np.abs(ch["O"] - whole["O"][prefix:])) < 1e-13
        assert np.max(np.abs(ch["LSE"] - whole["LSE"][:, prefix:])) < 1e-13
    assert (~whole["kept"][0] & np.tri(13, dtype=bool)).any()


def test_chunk_alpha_zero_equals_bottom_right_causal_attention():
    rng = np.random.default_rng(21)
    Lk, Lq, B, Hq, Hkv, d = 90, 26, 8, 4, 1, 5
    q, _, _ = rand_qkv(rng, Lq, Hq, Hkv, d)
    _, k, v = rand_qkv(rng, Lk, Hq, Hkv, d)
    r = O.prefill(q, k, v, [0, Lq], Hkv, _params(block_size=B, alpha=0.0), cu_seqlens_k=[0, Lk])
    allowed = np.arange(Lk)[None, :] <= (np.arange(Lq)[:, None] + (Lk - Lq))
    ref = sdpa_dense(q, k, v, 1 / math.sqrt(d), np.broadcast_to(allowed, (Hq, Lq, Lk)).copy())
    assert np.max(np.abs(r["O"] - ref)) < 1e-12


def test_chunked_varlen_equals_per_sequence_and_rejects_misaligned_chunks():
    rng = np.random.default_rng(22)
    B, Hq, Hkv, d = 8, 2, 1, 4
    lk, lq = [40, 75], [8, 19]
    q, _, _ = rand_qkv(rng, sum(lq), Hq, Hkv, d)
    _, k, v = rand_qkv(rng, sum(lk), Hq, Hkv, d)
    cq, ck = np.concatenate([[0], np.cumsum(lq)]), np.concatenate([[0], np.cumsum(lk)])
    p = _params(block_size=B, alpha=0.4)
    both = O.prefill(q, k, v, cq, Hkv, p, cu_seqlens_k=ck)
    for r in range(2):
        one = O.prefill(q[cq[r]:cq[r + 1]], k[ck[r]:ck[r + 1]], v[ck[r]:ck[r + 1]], [0, lq[r]], Hkv, p,
                        cu_seqlens_k=[0, lk[r]])
        assert np.max(np.abs(one["O"] - both["O"][cq[r]:cq[r + 1]])) == 0.0
    rp, ci = both["row_ptr"], both["col_idx"]
    back = O.kept_from_csr(rp, ci, lq, B, Hkv, seqlens_k=lk)
    assert all(np.array_equal(a, b) for a, b in zip(back, both["kept"]))
    with pytest.raises(ValueError):
        O.prefill(q[:5], k[:40], v[:40], [0, 5], Hkv, p, cu_seqlens_k=[0, 40])   # prefix 35 not a block multiple
