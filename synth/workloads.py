"""Seeded synthetic workloads standing in for the pages' needle-in-a-haystack inputs.

The FlashPrefill V2 paper page (metallab.ai, Table 1 and Table 3) measures the
operator on needle-in-a-haystack (NIAH) prompts fed through Llama-3.1-8B,
Qwen3-4B and Qwen3-30B-A3B.  Neither the prompts nor the model weights are
available here, so these generators draw tensors with the same shapes, value
scale and structure instead:

* every head's Q/K/V rows are ``(eps_t + rho * w_block(t)) @ A_h`` with
  ``eps_t, w ~ N(0, I_16)`` and ``A_h`` a 16 x d matrix with N(0, 1/16) entries
  (rank-16 structure, unit variance per coordinate).  The block-persistent
  latent ``w`` survives block-mean pooling, so ``rho`` controls how spread the
  pooled block scores are; V uses rho = 0;
* "needle" key blocks (1 % of the key blocks of each sequence; 4 blocks for the
  tiny case) have every key set to ``3 sqrt(d) u_g`` for a random unit vector
  ``u_g`` per KV head, and a seeded 10 % of query rows are set to the same
  vector in every query head of group g;
* FP8 workloads quantise the bf16 values per tensor with scale absmax / 448
  (round-to-nearest-even, saturating) into float8 e4m3.

Nothing in this module computes a step of the attention method; it only draws
inputs.  All randomness is NumPy PCG64 keyed by (seed, stream, ...), so any
slice (one sequence, one head) can be regenerated on its own.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import numpy as np
import torch

E4M3_MAX = 448.0

# rho for the rank-16 Q/K generator of the Llama/Qwen-shaped workloads, fixed once
# so that the 128K bf16 workload lands at 4-6 % block density with alpha = 0.1,
# sink = 2, window = 4 (the paper page's Table 3 reports 4.6-4.9 % at 128K).
RHO_CALIBRATED = 0.7

_STREAM_IDS = {"q": 1, "k": 2, "v": 3, "A": 4, "u": 5, "needle_k": 6, "needle_q": 7,
               "pages": 8, "eps": 9, "w": 10, "iid": 11}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    seqlens: tuple
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    dtype: str                   # "f32" | "bf16" | "e4m3" (storage / MMA input type)
    paged: bool = False
    page_size: int = 64
    alpha: float = 0.1
    sink_blocks: int = 2
    window_blocks: int = 4
    last_n_blocks: int = 0
    min_sparse_len: int = 0
    mean_correction: bool = True
    seed: int = 1
    rho: float = RHO_CALIBRATED
    iid: bool = False            # plain iid N(0,1) Q/K/V (tiny case)
    needle_blocks: Optional[int] = None   # fixed count per sequence, else 1 % of blocks
    needle_query_frac: float = 0.10
    description: str = ""

    @property
    def total_tokens(self) -> int:
        return int(sum(self.seqlens))

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    def num_blocks(self, L: int) -> int:
        return -(-L // self.block_size)

    def dense_equiv_flops(self) -> float:
        """4 d Hq sum_r L_r (L_r + 1) / 2: QK^T and PV over the causal triangle."""
        return float(sum(4.0 * self.head_dim * self.num_q_heads * L * (L + 1) / 2 for L in self.seqlens))

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def _w(name, **kw):
    return Workload(name=name, **kw)


WORKLOADS = {
    # tiny causal prefill, iid inputs, 4 planted needle key blocks
    "tiny_1k_f32": _w("tiny_1k_f32", seqlens=(1024,), num_q_heads=1, num_kv_heads=1, head_dim=64,
                      block_size=64, dtype="f32", sink_blocks=1, window_blocks=1, seed=1, rho=0.0,
                      iid=True, needle_blocks=4,
                      description="batch 1, 1/1 heads, seq 1024, d 64, block 64, fp32, iid N(0,1) + 4 needle blocks"),
    "llama8b_32k_bf16": _w("llama8b_32k_bf16", seqlens=(32768,), num_q_heads=32, num_kv_heads=8,
                           head_dim=128, block_size=128, dtype="bf16", seed=2,
                           description="Llama-3.1-8B-shaped layer, seq 32768, GQA 4, d 128, block 128, bf16"),
    "llama8b_128k_bf16": _w("llama8b_128k_bf16", seqlens=(131072,), num_q_heads=32, num_kv_heads=8,
                            head_dim=128, block_size=128, dtype="bf16", seed=3,
                            description="Llama-3.1-8B-shaped layer, seq 131072, GQA 4, d 128, block 128, bf16"),
    "llama8b_128k_e4m3": _w("llama8b_128k_e4m3", seqlens=(131072,), num_q_heads=32, num_kv_heads=8,
                            head_dim=128, block_size=128, dtype="e4m3", seed=3,
                            description="same layer at 128K in FP8 e4m3 with per-tensor absmax scales"),
    "qwen30b_64k_paged_bf16": _w("qwen30b_64k_paged_bf16", seqlens=(65536,), num_q_heads=32, num_kv_heads=4,
                                 head_dim=128, block_size=128, dtype="bf16", paged=True, page_size=64, seed=4,
                                 description="Qwen3-30B-A3B-shaped layer, seq 65536, GQA 8, paged KV (64-token pages)"),
    # Qwen3-4B-shaped layer at 64K in FP8: the setting of the paper page's Table 9 (alpha sweep) and
    # Figures 5-6 (latency vs sparsity, correction overhead); used by the sweeps, not a parity config.
    "qwen4b_64k_e4m3": _w("qwen4b_64k_e4m3", seqlens=(65536,), num_q_heads=32, num_kv_heads=8, head_dim=128,
                          block_size=128, dtype="e4m3", seed=6,
                          description="Qwen3-4B-shaped layer, seq 65536, GQA 4, d 128, block 128, FP8 e4m3"),
    "varlen6_paged_e4m3": _w("varlen6_paged_e4m3", seqlens=(2048, 4096, 16384, 32768, 65536, 131072),
                             num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=128, dtype="e4m3",
                             paged=True, page_size=64, min_sparse_len=8192, seed=5,
                             description="6 packed requests (cu_seqlens), GQA 4, paged FP8, min-sparse-length 8192"),
}

# The served configuration of the nestfrontier.com write-up ("A serving setup you can actually
# test") adds last-n-blocks 8: the same layers with the last 8 query blocks of each sequence dense.
WORKLOADS["llama8b_128k_bf16_lastn8"] = WORKLOADS["llama8b_128k_bf16"].replace(
    name="llama8b_128k_bf16_lastn8", last_n_blocks=8,
    description="the 128K bf16 layer with last-n-blocks 8 (the served configuration)")
WORKLOADS["qwen4b_64k_e4m3_lastn8"] = WORKLOADS["qwen4b_64k_e4m3"].replace(
    name="qwen4b_64k_e4m3_lastn8", last_n_blocks=8,
    description="the Qwen3-4B-shaped 64K FP8 layer with last-n-blocks 8 (the served configuration)")


def get_workload(name: str) -> Workload:
    return WORKLOADS[name]


def _rng(seed: int, stream: str, *keys: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([seed, _STREAM_IDS[stream], *[int(k) for k in keys]]))


@dataclasses.dataclass
class Inputs:
    """Generated tensors, all on the CPU.

    q: [T, Hq, d]; k, v: [T, Hkv, d] contiguous (always present);
    k_cache, v_cache: [num_pages, page_size, Hkv, d] and page_table
    [num_seqs, max_pages] int32 (-1 = unused) when the workload is paged.
    Storage dtypes: torch.float32 / torch.bfloat16 / torch.float8_e4m3fn.
    """
    workload: Workload
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    q_descale: float
    k_descale: float
    v_descale: float
    cu_seqlens: np.ndarray
    k_cache: Optional[torch.Tensor] = None
    v_cache: Optional[torch.Tensor] = None
    page_table: Optional[np.ndarray] = None
    needle_key_blocks: Optional[list] = None

    def dequant(self, name: str, heads: Optional[Sequence[int]] = None,
                tokens: Optional[slice] = None) -> np.ndarray:
        """fp64 values the kernels see: storage value times the per-tensor descale."""
        t = {"q": self.q, "k": self.k, "v": self.v, "k_cache": self.k_cache, "v_cache": self.v_cache}[name]
        if tokens is not None:
            t = t[tokens]
        if heads is not None:
            t = t[..., list(heads), :]
        scale = {"q": self.q_descale, "k": self.k_descale, "k_cache": self.k_descale,
                 "v": self.v_descale, "v_cache": self.v_descale}[name]
        out = t.to(torch.float64).numpy()
        if scale != 1.0:
            out = out * scale
        return out


def _lowrank_rows(seed, which, r, h, L, B, d, rho):
    A = _rng(seed, "A", _STREAM_IDS[which], h).normal(0.0, 0.25, size=(16, d)).astype(np.float32)
    g = _rng(seed, "eps", _STREAM_IDS[which], r, h)
    eps = g.standard_normal((L, 16), dtype=np.float32)
    if rho != 0.0:
        nb = -(-L // B)
        w = _rng(seed, "w", _STREAM_IDS[which], r, h).standard_normal((nb, 16), dtype=np.float32)
        eps += np.float32(rho) * np.repeat(w, B, axis=0)[:L]
    return eps @ A


def _quantize_e4m3(x_bf16: torch.Tensor) -> tuple:
    amax = float(x_bf16.abs().max().to(torch.float32))
    descale = float(np.float32(amax / E4M3_MAX)) if amax > 0 else 1.0
    out = torch.empty(x_bf16.shape, dtype=torch.float8_e4m3fn)
    # slice along the first axis to bound temporary memory
    step = max(1, (1 << 24) // max(1, x_bf16[0].numel()))
    inv = torch.tensor(descale, dtype=torch.float32)
    for s in range(0, x_bf16.shape[0], step):
        xs = x_bf16[s:s + step].to(torch.float32) / inv
        out[s:s + step] = xs.clamp_(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn)
    return out, descale


def generate(w: Workload) -> Inputs:
    T, Hq, Hkv, d, B = w.total_tokens, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size
    G = w.group
    base_dtype = torch.float32 if w.dtype == "f32" else torch.bfloat16
    q = torch.empty((T, Hq, d), dtype=base_dtype)
    k = torch.empty((T, Hkv, d), dtype=base_dtype)
    v = torch.empty((T, Hkv, d), dtype=base_dtype)
    cu = np.zeros(len(w.seqlens) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(w.seqlens)

    nscale = 3.0 * math.sqrt(d)
    u = np.stack([_rng(w.seed, "u", g).standard_normal(d) for g in range(Hkv)])
    u = (u / np.linalg.norm(u, axis=1, keepdims=True)).astype(np.float32)
    needle_blocks_all = []
    for r, L in enumerate(w.seqlens):
        s0 = int(cu[r])
        N = w.num_blocks(L)
        for name, tensor, H, rho in (("q", q, Hq, w.rho), ("k", k, Hkv, w.rho), ("v", v, Hkv, 0.0)):
            for h in range(H):
                if w.iid:
                    rows = _rng(w.seed, "iid", _STREAM_IDS[name], r, h).standard_normal((L, d), dtype=np.float32)
                else:
                    rows = _lowrank_rows(w.seed, name, r, h, L, B, d, rho)
                tensor[s0:s0 + L, h] = torch.from_numpy(rows).to(base_dtype)
        # needle key blocks (never block 0, which is a sink block)
        n_needle = w.needle_blocks if w.needle_blocks is not None else max(1, round(0.01 * N))
        n_needle = min(n_needle, max(0, N - 1))
        nb = np.sort(_rng(w.seed, "needle_k", r).choice(np.arange(1, N), size=n_needle, replace=False)) \
            if n_needle > 0 else np.zeros(0, dtype=np.int64)
        needle_blocks_all.append([int(x) for x in nb])
        for j in nb:
            t0, t1 = s0 + int(j) * B, s0 + min(L, (int(j) + 1) * B)
            for g in range(Hkv):
                k[t0:t1, g] = torch.from_numpy(nscale * u[g]).to(base_dtype)
        nq = int(round(w.needle_query_frac * L))
        rows_q = _rng(w.seed, "needle_q", r).choice(L, size=nq, replace=False)
        for h in range(Hq):
            q[s0 + rows_q, h] = torch.from_numpy(np.broadcast_to(nscale * u[h // G], (nq, d)).copy()).to(base_dtype)

    qd = kd = vd = 1.0
    if w.dtype == "e4m3":
        q, qd = _quantize_e4m3(q)
        k, kd = _quantize_e4m3(k)
        v, vd = _quantize_e4m3(v)

    inp = Inputs(workload=w, q=q, k=k, v=v, q_descale=qd, k_descale=kd, v_descale=vd,
                 cu_seqlens=cu, needle_key_blocks=needle_blocks_all)
    if w.paged:
        ps = w.page_size
        npages = [-(-L // ps) for L in w.seqlens]
        total = int(sum(npages))
        perm = _rng(w.seed, "pages").permutation(total).astype(np.int32)
        maxp = max(npages)
        pt = np.full((len(w.seqlens), maxp), -1, dtype=np.int32)
        kc = torch.zeros((total, ps, Hkv, d), dtype=k.dtype)
        vc = torch.zeros((total, ps, Hkv, d), dtype=v.dtype)
        off = 0
        for r, L in enumerate(w.seqlens):
            s0 = int(cu[r])
            for p in range(npages[r]):
                pid = int(perm[off + p])
                pt[r, p] = pid
                a, b = p * ps, min(L, (p + 1) * ps)
                kc[pid, : b - a] = k[s0 + a: s0 + b]
                vc[pid, : b - a] = v[s0 + a: s0 + b]
            off += npages[r]
        inp.k_cache, inp.v_cache, inp.page_table = kc, vc, pt
    return inp
