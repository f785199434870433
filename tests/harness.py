"""Shared test machinery: run the CUDA library stage by stage and compare with the oracle.

Tolerances (FlashPrefill V2 build contract): bf16 (and f32 inputs, which run on
tf32 tensor cores) max-abs <= 2e-2 and relative L2 <= 5e-3; fp8 e4m3 max-abs
<= 6e-2 and relative L2 <= 2e-2, all against the fp64 oracle on dequantised
inputs.  Block masks must match bit for bit except for blocks within 1e-3 of
the threshold (counted, then attention is compared on the oracle's mask).
Pooled means are fp32 sums of at most 128 values: they must agree with the
oracle's fp64 means to 2e-5 relative to the block's magnitude.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

from oracle import fp2_oracle as O
from synth import workloads as W

TOL = {"bf16": (2e-2, 5e-3), "f32": (2e-2, 5e-3), "e4m3": (6e-2, 2e-2)}
# LSE (natural log) bounds.  bf16: inputs are exact bf16; rounding kbar to bf16 moves a pruned
# block's logit q.kbar*scale by <= 2^-9 of it (<= 2e-2 for pooled logits up to ~10).  e4m3: kbar
# rounded to e4m3 moves it by <= 2^-4 of q.kbar*scale (pooled logits <= ~2 -> 1.5e-1).  f32: the
# tf32 tensor cores keep 10 mantissa bits of fp32 Q and K, so a logit q.k*scale moves by up to
# ~2^-10 of sum|q_i k_i|*scale; needle pairs reach 9*sqrt(d) = 72 at d = 64 -> 1e-1.
LSE_TOL = {"bf16": 2e-2, "f32": 1e-1, "e4m3": 1.5e-1}


def oracle_params(w: W.Workload) -> O.SparseParams:
    return O.SparseParams(block_size=w.block_size, alpha=w.alpha, sink_blocks=w.sink_blocks,
                          window_blocks=w.window_blocks, last_n_blocks=w.last_n_blocks,
                          min_sparse_len=w.min_sparse_len, mean_correction=w.mean_correction)


@dataclass
class GpuRun:
    problem: object
    params: object
    ws: object
    pooled_struct: object
    pooled: dict
    index_struct: object
    index: dict
    scratch: object
    out: object = None
    lse: object = None
    dev: dict = field(default_factory=dict)


def to_device(inp: W.Inputs, device="cuda"):
    import torch
    d = {"q": inp.q.to(device), "k": inp.k.to(device), "v": inp.v.to(device)}
    if inp.page_table is not None:
        d["k_cache"] = inp.k_cache.to(device)
        d["v_cache"] = inp.v_cache.to(device)
        d["page_table"] = torch.from_numpy(inp.page_table).to(device)
    return d


def make_gpu_problem(inp: W.Inputs, dev: dict):
    from block_sparse_long_pooled_b200 import fp2
    w = inp.workload
    if inp.page_table is not None:
        return fp2.make_problem(dev["q"], dev["k_cache"], dev["v_cache"], inp.cu_seqlens, w.num_kv_heads,
                                inp.q_descale, inp.k_descale, inp.v_descale, page_table=dev["page_table"])
    return fp2.make_problem(dev["q"], dev["k"], dev["v"], inp.cu_seqlens, w.num_kv_heads,
                            inp.q_descale, inp.k_descale, inp.v_descale)


def gpu_params(w: W.Workload, **over):
    from block_sparse_long_pooled_b200 import fp2
    kw = dict(block_size=w.block_size, alpha=w.alpha, sink_blocks=w.sink_blocks, window_blocks=w.window_blocks,
              last_n_blocks=w.last_n_blocks, min_sparse_len=w.min_sparse_len, mean_correction=w.mean_correction)
    kw.update(over)
    return fp2.make_params(**kw)


def run_gpu(inp: W.Inputs, external_index: Optional[tuple] = None, lse: bool = True, kv_splits: int = 0) -> GpuRun:
    """pool -> discover -> attend through the C ABI (attend on external_index when given)."""
    import torch
    from block_sparse_long_pooled_b200 import fp2
    dev = to_device(inp)
    prob = make_gpu_problem(inp, dev)
    params = gpu_params(inp.workload, kv_splits=kv_splits)
    ws = fp2.fp2_workspace_query(prob, params)
    pst, pooled = fp2.alloc_pooled(ws, prob, "cuda")
    ist, index = fp2.alloc_index(ws, "cuda")
    scratch = fp2.alloc_scratch(ws.scratch_bytes, "cuda")
    run = GpuRun(prob, params, ws, pst, pooled, ist, index, scratch, dev=dev)
    fp2.fp2_pool(prob, params, pst, scratch)
    fp2.fp2_discover(prob, params, pst, ist, scratch)
    torch.cuda.synchronize()
    st, bits = fp2.fp2_get_device_status(scratch)
    assert st == fp2.FP2_OK and bits == 0, (st, bits)
    T, Hq, D = inp.q.shape
    run.out = torch.empty((T, Hq, D), dtype=fp2.out_dtype(prob), device="cuda")
    run.lse = torch.empty((Hq, T), dtype=torch.float32, device="cuda") if lse else None
    att_index = ist
    if external_index is not None:
        rp = torch.from_numpy(np.asarray(external_index[0], dtype=np.int32)).cuda()
        ci = torch.from_numpy(np.asarray(external_index[1], dtype=np.int32)).cuda()
        if ci.numel() == 0:
            ci = torch.zeros(1, dtype=torch.int32, device="cuda")
        run.dev["ext_row_ptr"], run.dev["ext_col_idx"] = rp, ci
        att_index = fp2.index_struct(rp, ci)
    fp2.fp2_attend(prob, params, pst, att_index, run.out, run.lse, scratch)
    torch.cuda.synchronize()
    st, bits = fp2.fp2_get_device_status(scratch)
    assert st == fp2.FP2_OK and bits == 0, (st, bits)
    return run


# ------------------------------------------------------------------ oracle side (full or sliced)

@dataclass
class OracleSeq:
    qbar: np.ndarray
    kbar: np.ndarray
    vbar: np.ndarray
    counts: np.ndarray
    kept: np.ndarray
    border: np.ndarray


def oracle_discovery(inp: W.Inputs, head_chunk: int = 8) -> list:
    """Pool + score + select per sequence, reading the inputs in head slices (bounded memory)."""
    w = inp.workload
    p = oracle_params(w)
    scale = 1.0 / math.sqrt(w.head_dim)
    out = []
    cu = inp.cu_seqlens
    kname, vname = ("k", "v")
    for r in range(len(cu) - 1):
        a, b = int(cu[r]), int(cu[r + 1])
        def pooled(name, H):
            parts, counts = [], None
            for h0 in range(0, H, head_chunk):
                x = inp.dequant(name, heads=range(h0, min(H, h0 + head_chunk)), tokens=slice(a, b))
                m, counts = O.pool_blocks(x, w.block_size)
                parts.append(m)
            return np.concatenate(parts, axis=1), counts
        qbar, counts = pooled("q", w.num_q_heads)
        kbar, _ = pooled(kname, w.num_kv_heads)
        vbar, _ = pooled(vname, w.num_kv_heads)
        s = O.block_scores(qbar, kbar, scale)
        kept, border = O.select_blocks(s, w.num_kv_heads, b - a, p)
        out.append(OracleSeq(qbar, kbar, vbar, counts, kept, border))
    return out


def oracle_paged_kv(inp: W.Inputs, r: int):
    """K/V of sequence r gathered by the oracle through the page table (fp64)."""
    w = inp.workload
    L = w.seqlens[r]
    ds_k, ds_v = inp.k_descale, inp.v_descale
    kc = inp.k_cache.to(__import__("torch").float64).numpy() * ds_k
    vc = inp.v_cache.to(__import__("torch").float64).numpy() * ds_v
    pt = inp.page_table[r:r + 1]
    return O.gather_paged(kc, pt, [L]), O.gather_paged(vc, pt, [L])


def seq_kv(inp: W.Inputs, r: int):
    a, b = int(inp.cu_seqlens[r]), int(inp.cu_seqlens[r + 1])
    if inp.page_table is not None:
        return oracle_paged_kv(inp, r)
    return inp.dequant("k", tokens=slice(a, b)), inp.dequant("v", tokens=slice(a, b))


# ------------------------------------------------------------------ comparisons

def compare_pooled(run: GpuRun, inp: W.Inputs, ora: list):
    import torch
    w = inp.workload
    g = {k: run.pooled[k].float().cpu().numpy().astype(np.float64) for k in ("qbar", "kbar", "vbar")}
    qb = np.concatenate([o.qbar for o in ora])
    kb = np.concatenate([o.kbar for o in ora])
    vb = np.concatenate([o.vbar for o in ora])
    for name, gv, ov in (("qbar", g["qbar"], qb), ("kbar", g["kbar"], kb), ("vbar", g["vbar"], vb)):
        scale = max(1.0, float(np.abs(ov).max()))
        err = float(np.abs(gv - ov).max())
        assert err <= 2e-5 * scale, (name, err, scale)
    # narrow MMA copies: one rounding of the fp32 mean to the operand type (the V side is f16 for
    # e4m3 inputs)
    for name, ov, ds in (("kbar_mma", kb, inp.k_descale), ("vbar_mma", vb, inp.v_descale)):
        t = run.pooled[name]
        if w.dtype == "e4m3" and name == "vbar_mma":
            gv = t.float().cpu().numpy().astype(np.float64) * ds
            tol = np.abs(ov) * 2.0 ** -10 + 2.0 ** -24 * ds + 1e-9
        elif w.dtype == "e4m3":
            gv = t.view(torch.float8_e4m3fn).float().cpu().numpy().astype(np.float64) * ds
            tol = np.abs(ov) * 2.0 ** -3 + 2.0 ** -9 * ds + 1e-6
        elif w.dtype == "bf16":
            gv = t.float().cpu().numpy().astype(np.float64)
            tol = np.abs(ov) * 2.0 ** -8 + 1e-6
        else:
            gv = t.cpu().numpy().astype(np.float64)
            tol = np.abs(ov) * 1e-5 + 1e-6
        assert np.all(np.abs(gv - ov) <= tol), name
    if w.dtype == "e4m3":
        # the f16 copy of V equals the stored e4m3 values exactly, rows in key-token order
        assert torch.equal(run.pooled["v16"].cpu(), inp.v.to(torch.float16)), "v16"


def gpu_kept(run: GpuRun, inp: W.Inputs) -> list:
    w = inp.workload
    rp = run.index["row_ptr"].cpu().numpy()
    ci = run.index["col_idx"].cpu().numpy()
    out, row = [], 0
    for L in w.seqlens:
        N = -(-L // w.block_size)
        kept = np.zeros((w.num_kv_heads, N, N), dtype=bool)
        for i in range(N):
            for gg in range(w.num_kv_heads):
                cols = ci[rp[row]:rp[row + 1]]
                assert np.all(np.diff(cols) > 0), "columns must ascend"
                kept[gg, i, cols] = True
                row += 1
        out.append(kept)
    assert rp[row] == sum(int(k.sum()) for k in out)
    return out


def compare_index(run: GpuRun, inp: W.Inputs, ora: list) -> dict:
    """Bit-exact masks except borderline blocks; returns mismatch statistics."""
    gk = gpu_kept(run, inp)
    n_border_mismatch = n_border = n_total = n_kept = 0
    for gkr, o in zip(gk, ora):
        diff = gkr != o.kept
        assert not np.any(diff & ~o.border), f"{int((diff & ~o.border).sum())} non-borderline mask mismatches"
        n_border_mismatch += int(diff.sum())
        n_border += int(o.border.sum())
        n_total += int(np.tri(o.kept.shape[1]).sum()) * o.kept.shape[0]
        n_kept += int(o.kept.sum())
    return {"borderline_mismatches": n_border_mismatch, "borderline_blocks": n_border,
            "density": n_kept / max(1, n_total)}


def oracle_csr(ora: list):
    return O.csr_from_kept([o.kept for o in ora])


def compare_attention_full(run: GpuRun, inp: W.Inputs, ora: list, kept_override: Optional[list] = None):
    """Every output row against the oracle (small problems)."""
    w = inp.workload
    scale = 1.0 / math.sqrt(w.head_dim)
    O_ref, L_ref = [], []
    for r in range(len(w.seqlens)):
        a, b = int(inp.cu_seqlens[r]), int(inp.cu_seqlens[r + 1])
        if b == a:
            continue
        k, v = seq_kv(inp, r)
        o = ora[r]
        kept = kept_override[r] if kept_override is not None else o.kept
        Or, Lr = O.attend(inp.dequant("q", tokens=slice(a, b)), k, v, o.kbar, o.vbar, o.counts, kept,
                          w.block_size, scale, w.mean_correction)
        O_ref.append(Or)
        L_ref.append(Lr)
    O_ref = np.concatenate(O_ref)
    g = run.out.float().cpu().numpy().astype(np.float64)
    maxabs, rel = check_tol(g, O_ref, w.dtype)
    if run.lse is not None:
        lse = run.lse.cpu().numpy().astype(np.float64)
        lse_ref = np.concatenate(L_ref, axis=1)
        assert float(np.abs(lse - lse_ref).max()) < LSE_TOL[w.dtype], float(np.abs(lse - lse_ref).max())
    return maxabs, rel


def check_tol(g, ref, dtype):
    ma, rl = TOL[dtype]
    maxabs = float(np.abs(g - ref).max())
    rel = float(np.linalg.norm(g - ref) / max(1e-30, np.linalg.norm(ref)))
    assert maxabs <= ma and rel <= rl, (maxabs, rel, dtype)
    return maxabs, rel


def seq_group_kv(inp: W.Inputs, r: int, g: int):
    """fp64 K and V of KV head g of sequence r, shaped [L, 1, d] (through the page table when paged)."""
    import torch
    a, b = int(inp.cu_seqlens[r]), int(inp.cu_seqlens[r + 1])
    if inp.page_table is None:
        return inp.dequant("k", heads=[g], tokens=slice(a, b)), inp.dequant("v", heads=[g], tokens=slice(a, b))
    L = b - a
    ps = inp.k_cache.shape[1]
    pages = inp.page_table[r, :-(-L // ps)]
    # the sequence's own pages, renumbered 0..n-1, then the oracle's page-table gather
    idx = torch.from_numpy(pages.astype(np.int64))
    kc = inp.k_cache[idx][:, :, g:g + 1].to(torch.float64).numpy() * inp.k_descale
    vc = inp.v_cache[idx][:, :, g:g + 1].to(torch.float64).numpy() * inp.v_descale
    pt = np.arange(len(pages), dtype=np.int32)[None, :]
    return O.gather_paged(kc, pt, [L]), O.gather_paged(vc, pt, [L])


def select_pairs(inp: W.Inputs, ora: list, n_random: int = 8, seed: int = 0) -> list:
    """Whole (sequence r, KV group g, query block i) pairs to compare at full size.

    Every pair covers all G query heads of group g and every token of block i.  Chosen per
    sequence: the first block and the last four blocks (all groups for the last two); for each
    planted needle key block j, the query block j itself (the needle keys sit in its diagonal
    tile) and one later block that attends to j; the four rows with the most kept blocks in the
    oracle's index over the whole batch; every block of sequences below min_sparse_len (the
    dense-cutoff requests) when they have at most 32 blocks, else eight of them; and n_random
    random (group, block) pairs.  A tenth of all query rows are planted needle queries, so every
    pair also holds needle rows.
    """
    w = inp.workload
    rng = np.random.default_rng(4242 + seed)
    B, Hkv = w.block_size, w.num_kv_heads
    pairs = set()
    heavy = []
    for r, L in enumerate(w.seqlens):
        if L == 0:
            continue
        N = -(-L // B)
        for i in (0,) + tuple(range(max(0, N - 4), N)):
            gs = range(Hkv) if i >= N - 2 else [int(rng.integers(Hkv))]
            for g in gs:
                pairs.add((r, g, i))
        for j in (inp.needle_key_blocks[r] if inp.needle_key_blocks else []):
            if j < N:
                pairs.add((r, int(rng.integers(Hkv)), int(j)))
                if j + 1 < N:
                    pairs.add((r, int(rng.integers(Hkv)), int(rng.integers(j + 1, N))))
        if L < w.min_sparse_len:
            blocks = range(N) if N <= 32 else sorted(rng.choice(N, size=8, replace=False))
            for i in blocks:
                pairs.add((r, int(rng.integers(Hkv)), int(i)))
        for _ in range(n_random):
            pairs.add((r, int(rng.integers(Hkv)), int(rng.integers(N))))
        nk = ora[r].kept.sum(axis=2)            # [Hkv, N] kept blocks per row
        for g in range(Hkv):
            for i in range(N):
                heavy.append((int(nk[g, i]), r, g, i))
    heavy.sort(reverse=True)
    for _, r, g, i in heavy[:4]:
        pairs.add((r, g, i))
    return sorted(pairs)


def oracle_pairs(inp: W.Inputs, ora: list, pairs: list, kept_override: Optional[list] = None):
    """Oracle output [n_rows, d] and LSE [n_rows] for whole (r, g, i) pairs, rows ordered pair by
    pair, then token, then head of the group; also the matching (token, head) indices."""
    w = inp.workload
    B, G = w.block_size, w.group
    scale = 1.0 / math.sqrt(w.head_dim)
    outs, lses, toks, heads = [], [], [], []
    by_group = {}
    for r, g, i in pairs:
        by_group.setdefault((r, g), []).append(i)
    for (r, g), blocks in sorted(by_group.items()):
        a, b = int(inp.cu_seqlens[r]), int(inp.cu_seqlens[r + 1])
        L = b - a
        hs = list(range(g * G, (g + 1) * G))
        q = inp.dequant("q", heads=hs, tokens=slice(a, b))            # [L, G, d]
        k, v = seq_group_kv(inp, r, g)                                   # [L, 1, d]
        o = ora[r]
        kept = (kept_override[r] if kept_override is not None else o.kept)[g:g + 1]
        for i in sorted(blocks):
            t = np.arange(i * B, min(L, (i + 1) * B))
            rows = np.stack([np.repeat(t, G), np.tile(np.arange(G), len(t))], axis=1)
            Or, Lr = O.attend(q, k, v, o.kbar[:, g:g + 1], o.vbar[:, g:g + 1], o.counts, kept, B, scale,
                              w.mean_correction, rows=rows, head_ids=list(range(G)), group=G)
            outs.append(Or)
            lses.append(Lr)
            toks.append(rows[:, 0] + a)
            heads.append(rows[:, 1] + g * G)
    return np.concatenate(outs), np.concatenate(lses), np.concatenate(toks), np.concatenate(heads)


def compare_attention_pairs(run: GpuRun, inp: W.Inputs, ref: tuple, lse: bool = True):
    """Every element of the selected pairs' outputs (and their LSE) against the oracle's."""
    import torch
    O_ref, L_ref, toks, heads = ref
    it = torch.from_numpy(toks).to(run.out.device)
    ih = torch.from_numpy(heads).to(run.out.device)
    g = run.out[it, ih].float().cpu().numpy().astype(np.float64)
    maxabs, rel = check_tol(g, O_ref, inp.workload.dtype)
    lse_err = None
    if lse and run.lse is not None:
        gl = run.lse[ih, it].cpu().numpy().astype(np.float64)
        lse_err = float(np.abs(gl - L_ref).max())
        assert lse_err < LSE_TOL[inp.workload.dtype], lse_err
    return {"rows": int(len(toks)), "max_abs": maxabs, "rel_l2": rel, "lse_max_abs": lse_err}
