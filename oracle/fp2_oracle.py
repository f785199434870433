"""fp64 NumPy oracle of FlashPrefill V2's mean-corrected block-sparse causal prefill attention.

TEST INFRASTRUCTURE.  This module is the slow, plain CPU statement of what the
CUDA library computes; only the test-suite, the smoke check and the CPU
baseline leg of the benchmark may import it.  It shares no code with the CUDA
path (the only shared module is ``synth``, which draws random inputs).

Sources (page title, then the passage):

* "FlashPrefill V2: Block-Sparse Prefill Attention for Long-Context LLM
  Serving" (metallab.ai paper page) -- Figure 3 caption (Stage 1: PackGQA,
  block-mean pooling, CSR index of selected blocks; Stage 2: sparse attention
  whose exact and mean-correction streams merge inside the online softmax),
  Figure 4 caption (each pruned block J adds |B_J| e^{s_J} (vbar_J, 1) to the
  softmax numerator and denominator), Table 7 (CSR per KV head), Table 9 and
  the abstract (max-based dynamic thresholding with parameter alpha).
* "128K context now demands Hopper hardware" (nestfrontier.com), section
  "A serving setup you can actually test" -- the backend flags: attention sink
  2, window 4, abs threshold 0.1, last-n-blocks 8, k-block-n 128, min sparse
  q len, use mean correction.
* ResearchPod episode on FlashPrefill V2 -- blocks are scored from a simple
  average of each block.

Readings of the pages that this oracle fixes (the CUDA path takes the same):

* Pooling is the arithmetic mean over the tokens actually present in a block
  (the last block of a sequence may be partial); n_j is that token count.
* Block score s[h,i,j] = (qbar_{i,h} . kbar_{j,g(h)}) * scale for j <= i,
  scale = 1/sqrt(d) unless overridden.
* Max-based threshold: head h keeps block j of query block i iff
  s[h,i,j] >= max_{j'<=i} s[h,i,j'] + ln(alpha); the row max runs over every
  causal block, forced ones included.  alpha = 0 keeps every block.
* A KV-head row keeps the union over the G query heads of its group.
* Forced blocks: the whole causal row when the sequence is shorter than
  min_sparse_len; j < sink; j > i - max(window, 1) (the diagonal block is
  always exact); every j of the last ``last_n`` query blocks.
* Mean correction uses the token's own query: a pruned block j contributes the
  logit q_t . kbar_j * scale + ln n_j with value vbar_j.  Every pruned block lies
  strictly left of the diagonal, so it is fully visible.
* Chunked prefill (the paper page's Table 6; ResearchPod: discovery re-runs per
  chunk): a query chunk is the last L_q tokens of a sequence whose keys number
  L_k >= L_q, with bottom-right causal alignment (chunk token t sits at absolute
  position L_k - L_q + t).  The chunk must start on a block boundary, so chunk
  block i is absolute block I = (L_k - L_q)/B + i; causality, the diagonal and the
  window refer to I; last_n and min_sparse_len refer to the chunk's queries.

Parity pins: tests/test_oracle_pins.py checks these functions against dense
softmax attention from torch (alpha = 0), the closed form in which mean
correction is exact (keys constant inside each block), brute force on tiny
inputs, and the invariants of the selection rule.
"""

from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np

BORDERLINE_BAND = 1e-3

__all__ = [
    "SparseParams", "num_blocks", "pool_blocks", "pool_varlen", "gather_paged", "block_scores",
    "forced_blocks", "select_blocks", "csr_from_kept", "kept_from_csr", "attend", "prefill",
    "BORDERLINE_BAND",
]


@dataclass(frozen=True)
class SparseParams:
    """The backend flags of the nestfrontier.com write-up, as block-sparse parameters."""
    block_size: int
    alpha: float = 0.1
    sink_blocks: int = 2
    window_blocks: int = 4
    last_n_blocks: int = 0
    min_sparse_len: int = 0
    mean_correction: bool = True
    softmax_scale: float = 0.0   # 0 -> 1/sqrt(d)


def num_blocks(L: int, B: int) -> int:
    return -(-L // B)


def pool_blocks(x: np.ndarray, B: int):
    """Block means of one sequence (paper page, Figure 3: "pools block-mean statistics").

    x: [L, H, d] fp64.  Returns (mean [N, H, d], count [N]) where block i holds
    tokens [iB, min(L, (i+1)B)) and the mean divides by that token count.
    """
    L = x.shape[0]
    N = num_blocks(L, B)
    means = np.empty((N,) + x.shape[1:], dtype=np.float64)
    counts = np.empty(N, dtype=np.int64)
    for i in range(N):
        a, b = i * B, min(L, (i + 1) * B)
        means[i] = x[a:b].sum(axis=0) / (b - a)
        counts[i] = b - a
    return means, counts


def pool_varlen(x: np.ndarray, cu_seqlens: Sequence[int], B: int):
    """Pool every sequence of a packed [T, H, d] batch; blocks are concatenated in sequence order."""
    means, counts = [], []
    for r in range(len(cu_seqlens) - 1):
        m, c = pool_blocks(x[cu_seqlens[r]:cu_seqlens[r + 1]], B)
        means.append(m)
        counts.append(c)
    return np.concatenate(means), np.concatenate(counts)


def gather_paged(cache: np.ndarray, page_table: np.ndarray, seqlens: Sequence[int]) -> np.ndarray:
    """Read a paged KV cache [P, page_size, H, d] into a packed [T, H, d] array.

    Token t of sequence r lives in page page_table[r, t // page_size] at row
    t % page_size (the paper page's abstract: native paged KV cache support).
    """
    ps = cache.shape[1]
    parts = []
    for r, L in enumerate(seqlens):
        t = np.arange(L)
        pages = page_table[r, t // ps]
        if np.any(pages < 0) or np.any(pages >= cache.shape[0]):
            raise ValueError("page table entry out of range")
        parts.append(cache[pages, t % ps])
    return np.concatenate(parts)


def _causal(Nq: int, Nk: int, off: int) -> np.ndarray:
    """[Nq, Nk] boolean: key block j is visible from query block i (absolute block i + off)."""
    return np.arange(Nk)[None, :] <= (np.arange(Nq)[:, None] + off)


def block_scores(qbar: np.ndarray, kbar: np.ndarray, scale: float, q_block_offset: int = 0) -> np.ndarray:
    """Pooled block scores of one sequence: s[h, i, j] = qbar[i,h] . kbar[j,g(h)] * scale, j <= i + off.

    qbar: [Nq, Hq, d]; kbar: [Nk, Hkv, d]; q_block_offset = prefix blocks before the query chunk
    (0 for a whole-sequence prefill, where Nq = Nk).  Entries with j > i + off are -inf.
    """
    Nq, Hq, _ = qbar.shape
    Nk, Hkv = kbar.shape[0], kbar.shape[1]
    G = Hq // Hkv
    s = np.empty((Hq, Nq, Nk), dtype=np.float64)
    for h in range(Hq):
        s[h] = (qbar[:, h, :] @ kbar[:, h // G, :].T) * scale
    s[:, ~_causal(Nq, Nk, q_block_offset)] = -np.inf
    return s


def forced_blocks(N: int, L: int, p: SparseParams, Nk: Optional[int] = None, q_block_offset: int = 0) -> np.ndarray:
    """Blocks kept regardless of score, as a causal [N, Nk] boolean (i = query block, j = key block).

    N, L: query blocks and query tokens of the sequence (or chunk); the query block i sits at
    absolute block i + q_block_offset, which is what the window and the causal limit refer to;
    last_n and min_sparse_len refer to the queries.
    """
    Nk = N if Nk is None else Nk
    i = np.arange(N)[:, None]
    I = i + q_block_offset
    j = np.arange(Nk)[None, :]
    causal = j <= I
    if L < p.min_sparse_len or p.alpha <= 0.0:
        return causal.copy()
    f = (j < p.sink_blocks) | (j > I - max(p.window_blocks, 1)) | (i >= N - p.last_n_blocks)
    return f & causal


def select_blocks(s: np.ndarray, num_kv_heads: int, L: int, p: SparseParams, q_block_offset: int = 0):
    """Max-based dynamic thresholding (abstract; Table 9) with the GQA union per KV head (Table 7).

    s: [Hq, N, Nk] block scores of one sequence (or query chunk); L is its query token count.
    Returns (kept [Hkv, N, Nk], borderline [Hkv, N, Nk]); a block is borderline when it is not
    forced and some head of the group has |s - (rowmax + ln alpha)| < 1e-3.
    """
    Hq, N, Nk = s.shape
    G = Hq // num_kv_heads
    if N == 0:
        empty = np.zeros((num_kv_heads, 0, Nk), dtype=bool)
        return empty, empty.copy()
    forced = forced_blocks(N, L, p, Nk, q_block_offset)
    causal = _causal(N, Nk, q_block_offset)
    kept = np.zeros((num_kv_heads, N, Nk), dtype=bool)
    border = np.zeros((num_kv_heads, N, Nk), dtype=bool)
    dense = L < p.min_sparse_len or p.alpha <= 0.0
    for g in range(num_kv_heads):
        keep_g = forced.copy()
        bord_g = np.zeros((N, Nk), dtype=bool)
        if not dense:
            for h in range(g * G, (g + 1) * G):
                rowmax = s[h].max(axis=1)                       # over j <= i (others are -inf)
                thr = rowmax + math.log(p.alpha)
                keep_g |= (s[h] >= thr[:, None]) & causal
                bord_g |= (np.abs(s[h] - thr[:, None]) < BORDERLINE_BAND) & causal
        kept[g] = keep_g
        border[g] = bord_g & ~forced
    return kept, border


def csr_from_kept(kept_per_seq: Sequence[np.ndarray]):
    """Compressed sparse rows of kept key blocks, one row per (sequence, query block, KV head).

    Row id = (block_offset_r + i) * Hkv + g; columns are sequence-local key-block
    ids in ascending order (Table 7: "CSR of selected blocks, per KV head").
    """
    rows = []
    for kept in kept_per_seq:
        Hkv, N, _ = kept.shape
        for i in range(N):
            for g in range(Hkv):
                rows.append(np.nonzero(kept[g, i])[0].astype(np.int32))
    row_ptr = np.zeros(len(rows) + 1, dtype=np.int32)
    row_ptr[1:] = np.cumsum([len(r) for r in rows])
    col_idx = np.concatenate(rows).astype(np.int32) if rows else np.zeros(0, dtype=np.int32)
    return row_ptr, col_idx


def kept_from_csr(row_ptr, col_idx, seqlens, B, Hkv, seqlens_k=None):
    """Inverse of csr_from_kept: per-sequence kept [Hkv, Nq, Nk] booleans."""
    out, row = [], 0
    for r, L in enumerate(seqlens):
        N = num_blocks(L, B)
        Nk = num_blocks(seqlens_k[r], B) if seqlens_k is not None else N
        kept = np.zeros((Hkv, N, Nk), dtype=bool)
        for i in range(N):
            for g in range(Hkv):
                kept[g, i, col_idx[row_ptr[row]:row_ptr[row + 1]]] = True
                row += 1
        out.append(kept)
    return out


def attend(q, k, v, kbar, vbar, counts, kept, B: int, scale: float, mean_correction: bool,
           rows: Optional[np.ndarray] = None, head_ids: Optional[Sequence[int]] = None,
           group: Optional[int] = None, q_offset: int = 0):
    """Exact attention over kept blocks plus mean correction for pruned ones, one sequence.

    Figure 4 caption: selected blocks are computed exactly; each pruned block J
    contributes |B_J| e^{q.kbar_J*scale} (vbar_J, 1) to numerator and
    denominator.  For query token t (block i) and head h with g = h // G:

        logits  z_tu = q_t . k_u * scale     for u in kept blocks j <= i, u <= t
                c_tj = q_t . kbar_j * scale + ln n_j   for pruned j <= i (if enabled)
        m = max of all logits
        O_t = (sum e^{z-m} v_u + sum e^{c-m} vbar_j) / (sum e^{z-m} + sum e^{c-m})
        LSE_t = m + ln(denominator)

    q: [Lq, Hq, d] at absolute positions q_offset + t (q_offset = the chunk's prefix length, a
    multiple of B; 0 for a whole sequence); k, v: [Lk, Hkv, d]; kbar, vbar: [Nk, Hkv, d];
    counts: [Nk]; kept: [Hkv, Nq, Nk].  rows: optional int array [n, 2] of (t, h) pairs; when
    given only those outputs are computed and O is [n, d], LSE [n].
    Otherwise O is [L, Hq, d] and LSE [Hq, L].  head_ids / group: when q holds
    only some query heads, head_ids[x] is the global head of q[:, x] and group
    is G; rows then index q's own head axis.
    """
    L, Hq, d = q.shape
    Lk = k.shape[0]
    Hkv = k.shape[1]
    G = group if group is not None else Hq // Hkv
    gid = (lambda x: int(head_ids[x]) // G) if head_ids is not None else (lambda x: x // G)
    N = num_blocks(L, B)
    if q_offset % B != 0:
        raise ValueError("the query chunk must start on a block boundary")
    ob = q_offset // B
    logn = np.log(counts.astype(np.float64))
    if rows is None:
        O = np.zeros((L, Hq, d))
        LSE = np.zeros((Hq, L))
        work = [(h, i, np.arange(i * B, min(L, (i + 1) * B)), None) for h in range(Hq) for i in range(N)]
    else:
        rows = np.asarray(rows, dtype=np.int64).reshape(-1, 2)
        O = np.zeros((len(rows), d))
        LSE = np.zeros(len(rows))
        work = []
        for h in np.unique(rows[:, 1]):
            sel_h = np.nonzero(rows[:, 1] == h)[0]
            blocks = rows[sel_h, 0] // B
            for i in np.unique(blocks):
                sel = sel_h[blocks == i]
                work.append((int(h), int(i), rows[sel, 0], sel))
    for h, i, toks, dest in work:
        g = gid(h)
        I = i + ob                                                  # absolute query block
        if not kept[g, i, I]:
            raise ValueError("the diagonal block must be kept (it is only partly visible)")
        kj = np.nonzero(kept[g, i, : I + 1])[0]
        key_idx = np.concatenate([np.arange(j * B, min(Lk, (j + 1) * B)) for j in kj])
        qt = q[toks, h, :]                                          # [n, d]
        z = (qt @ k[key_idx, g, :].T) * scale                       # [n, nk]
        z[key_idx[None, :] > (toks[:, None] + q_offset)] = -np.inf  # causal, bottom-right aligned
        vals = v[key_idx, g, :]
        if mean_correction:
            pj = np.array([j for j in range(I + 1) if not kept[g, i, j]], dtype=np.int64)
        else:
            pj = np.zeros(0, dtype=np.int64)
        if len(pj):
            c = (qt @ kbar[pj, g, :].T) * scale + logn[pj][None, :]
            z = np.concatenate([z, c], axis=1)
            vals = np.concatenate([vals, vbar[pj, g, :]], axis=0)
        m = z.max(axis=1, keepdims=True)
        w = np.exp(z - m)
        den = w.sum(axis=1)
        o = (w @ vals) / den[:, None]
        lse = m[:, 0] + np.log(den)
        if dest is None:
            O[toks, h, :] = o
            LSE[h, toks] = lse
        else:
            O[dest] = o
            LSE[dest] = lse
    return O, LSE


def prefill(q, k, v, cu_seqlens, num_kv_heads: int, p: SparseParams, k_cache=None, v_cache=None,
            page_table=None, kept_override=None, attention: bool = True, cu_seqlens_k=None):
    """The whole path for a packed batch: pool -> score -> select -> CSR -> attend.

    q: [T, Hq, d]; k, v: [Tk, Hkv, d] fp64 (ignored when a paged cache is given,
    which is gathered through the page table first).  cu_seqlens_k: key offsets when
    queries are a chunk at the end of each sequence (chunked prefill: the query chunk of
    sequence r is its last L_q tokens, and L_k - L_q must be a multiple of the block size);
    None means q_len == kv_len.  kept_override: optional list of per-sequence kept arrays
    to attend on instead of the selected ones.  Returns a dict of every intermediate result.
    """
    cu = [int(x) for x in cu_seqlens]
    cuk = cu if cu_seqlens_k is None else [int(x) for x in cu_seqlens_k]
    seqlens = [cu[r + 1] - cu[r] for r in range(len(cu) - 1)]
    seqlens_k = [cuk[r + 1] - cuk[r] for r in range(len(cuk) - 1)]
    if page_table is not None:
        k = gather_paged(k_cache, page_table, seqlens_k)
        v = gather_paged(v_cache, page_table, seqlens_k)
    d = q.shape[2]
    scale = p.softmax_scale if p.softmax_scale > 0 else 1.0 / math.sqrt(d)
    B = p.block_size
    out = {"qbar": [], "kbar": [], "vbar": [], "counts": [], "scores": [], "kept": [], "borderline": [],
           "q_offset": []}
    for r, L in enumerate(seqlens):
        off = seqlens_k[r] - L
        if off < 0 or off % B != 0:
            raise ValueError("each query chunk must end its sequence and start on a block boundary")
        qs, ks, vs = q[cu[r]:cu[r + 1]], k[cuk[r]:cuk[r + 1]], v[cuk[r]:cuk[r + 1]]
        qbar, _ = pool_blocks(qs, B)
        kbar, counts = pool_blocks(ks, B)
        vbar, _ = pool_blocks(vs, B)
        s = block_scores(qbar, kbar, scale, off // B)
        kept, border = select_blocks(s, num_kv_heads, L, p, off // B)
        for key, val in (("qbar", qbar), ("kbar", kbar), ("vbar", vbar), ("counts", counts),
                         ("scores", s), ("kept", kept), ("borderline", border), ("q_offset", off)):
            out[key].append(val)
    out["row_ptr"], out["col_idx"] = csr_from_kept(out["kept"])
    if attention:
        Os, LSEs = [], []
        for r, L in enumerate(seqlens):
            kept = kept_override[r] if kept_override is not None else out["kept"][r]
            O, LSE = attend(q[cu[r]:cu[r + 1]], k[cuk[r]:cuk[r + 1]], v[cuk[r]:cuk[r + 1]], out["kbar"][r],
                            out["vbar"][r], out["counts"][r], kept, B, scale, p.mean_correction,
                            q_offset=out["q_offset"][r])
            Os.append(O)
            LSEs.append(LSE)
        out["O"] = np.concatenate(Os)
        out["LSE"] = np.concatenate(LSEs, axis=1)
    return out
