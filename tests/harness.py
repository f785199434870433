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
    # narrow MMA copies: one rounding of the fp32 mean to the operand type
    for name, ov, ds in (("kbar_mma", kb, inp.k_descale), ("vbar_mma", vb, inp.v_descale)):
        t = run.pooled[name]
        if w.dtype == "e4m3":
            gv = t.view(torch.float8_e4m3fn).float().cpu().numpy().astype(np.float64) * ds
            tol = np.abs(ov) * 2.0 ** -3 + 2.0 ** -9 * ds + 1e-6
        elif w.dtype == "bf16":
            gv = t.float().cpu().numpy().astype(np.float64)
            tol = np.abs(ov) * 2.0 ** -8 + 1e-6
        else:
            gv = t.cpu().numpy().astype(np.float64)
            tol = np.abs(ov) * 1e-5 + 1e-6
        assert np.all(np.abs(gv - ov) <= tol), name


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


def sample_rows(inp: W.Inputs, r: int, n: int, seed: int = 0) -> np.ndarray:
    """(t, h) pairs of sequence r: first/last tokens, block edges, needle rows and random ones."""
    w = inp.workload
    L = w.seqlens[r]
    B = w.block_size
    rng = np.random.default_rng(1000 + seed + r)
    toks = {0, L - 1, min(L - 1, B - 1), min(L - 1, B), L // 2}
    toks.update(int(x) for x in rng.integers(0, L, size=n))
    hs = rng.integers(0, w.num_q_heads, size=len(toks))
    return np.array([[t, int(h)] for t, h in zip(sorted(toks), hs)], dtype=np.int64)


def compare_attention_sampled(run: GpuRun, inp: W.Inputs, ora: list, n_per_seq: int = 48):
    w = inp.workload
    scale = 1.0 / math.sqrt(w.head_dim)
    G = w.group
    g_all, r_all = [], []
    out = run.out
    for r in range(len(w.seqlens)):
        a, b = int(inp.cu_seqlens[r]), int(inp.cu_seqlens[r + 1])
        if b == a:
            continue
        rows = sample_rows(inp, r, n_per_seq)
        heads = sorted(set(int(h) for h in rows[:, 1]))
        hpos = {h: x for x, h in enumerate(heads)}
        q = inp.dequant("q", heads=heads, tokens=slice(a, b))
        k, v = seq_kv(inp, r)
        local = np.stack([rows[:, 0], [hpos[int(h)] for h in rows[:, 1]]], axis=1)
        o = ora[r]
        Or, _ = O.attend(q, k, v, o.kbar, o.vbar, o.counts, o.kept, w.block_size, scale, w.mean_correction,
                         rows=local, head_ids=heads, group=G)
        idx_t = __import__("torch").from_numpy(rows[:, 0] + a).cuda()
        idx_h = __import__("torch").from_numpy(rows[:, 1]).cuda()
        g_all.append(out[idx_t, idx_h].float().cpu().numpy().astype(np.float64))
        r_all.append(Or)
    return check_tol(np.concatenate(g_all), np.concatenate(r_all), w.dtype)
