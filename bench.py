"""Benchmark of mean-corrected block-sparse prefill attention (pool -> discover -> attend).

One step = the whole path over one synthetic batch resident in HBM:
fp2_pool, fp2_discover (score/threshold, scan, scatter) and fp2_attend.
Headline metric: dense-equivalent TFLOP/s (4 d Hq sum L(L+1)/2 per step / step time);
ms per step, achieved TFLOP/s, per-stage times, sparsity, the all-blocks-kept run of
the same library, and an FP8 line ride along.

  python bench.py [--gpus N --steps K --warmup W] [--workload NAME] [--impl reference]

Under torchrun every rank runs its own replica of the workload (the path has no
exchange step); the time is the max over ranks and the value counts all ranks' work.
--impl reference times the fp64 CPU oracle on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse prefill attn ms + dense-equiv & achieved TFLOPS @128K BF16/FP8, 1xB200"
UNIT = "TFLOP/s (dense-equivalent)"
DEFAULT_WORKLOAD = "llama8b_128k_bf16"
FP8_WORKLOAD = "llama8b_128k_e4m3"
# Every configuration of the benchmark contract, measured in the default run and reported inside
# the headline line (per_config): the tiny fp32 case, the 32K and 128K Llama-shaped layers (128K in
# BF16 and FP8), the paged Qwen3-30B-A3B-shaped layer and the varlen paged FP8 batch; then the
# served configuration's last-n-blocks 8 variants of the 128K BF16 and the 64K FP8 layers.
CONFIGS = [("C1", "tiny_1k_f32"), ("C2", "llama8b_32k_bf16"), ("C3", "llama8b_128k_bf16"),
           ("C3-fp8", "llama8b_128k_e4m3"), ("C4", "qwen30b_64k_paged_bf16"), ("C5", "varlen6_paged_e4m3"),
           ("served-lastn8", "llama8b_128k_bf16_lastn8"), ("served-lastn8", "qwen4b_64k_e4m3_lastn8")]
L2_BYTES = 126 * 1024 * 1024

# DRAM traffic of one attention launch, from an ncu capture (dram__bytes_read.sum +
# dram__bytes_write.sum, one pass) of the same workload; valid only for the kernel source it was
# taken on (sha256 prefix of csrc/attention.cu), otherwise reported as null.
ATTN_TRAFFIC = {"llama8b_128k_bf16": {"bytes": 7598519552 + 1040229120, "source_sha": "e1d1461b29023c2c"},
                "llama8b_128k_e4m3": {"bytes": 5427795200 + 1029442560, "source_sha": "e1d1461b29023c2c"}}


def max_over_ranks(pg, x, device=None):
    """The largest of x over all ranks of the process group (x itself when there is none)."""
    if pg is None:
        return x
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def attention_traffic(wname):
    """DRAM bytes of one attention launch from the committed ncu capture, or None when the kernel
    source changed since it was taken (or no capture exists for the workload)."""
    tr = ATTN_TRAFFIC.get(wname)
    sha = source_sha(os.path.join(ROOT, "block_sparse_long_pooled_b200", "csrc", "attention.cu"))
    return tr["bytes"] if tr is not None and tr["source_sha"] == sha else None


def whole_job_value(flops_per_rank_step, world, ms_per_step):
    """Whole-job throughput in TFLOP/s: every rank runs the same workload (weak scaling) and the
    step time is the slowest rank's."""
    return flops_per_rank_step * world / (ms_per_step * 1e-3) / 1e12


def source_sha(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def attention_peak(dtype, peaks):
    """Dense tensor peak for the attention kernel's operand type: the measured burst bf16 GEMM rate
    (the timed region is a fraction of a second and the kernel holds the maximum SM clock most of
    it, while the sustained GEMM figure was taken over seconds at a power-capped ~1.34 GHz), times
    the nominal ratio for e4m3 (2x, QK runs on e4m3 operands) and tf32 (1/2x, f32 inputs)."""
    ratio = {"bf16": 1.0, "e4m3": 2.0, "f32": 0.5}[dtype]
    note = {"bf16": "", "e4m3": " x2 (FP8 nominal ratio)", "f32": " x0.5 (tf32 nominal ratio)"}[dtype]
    return peaks["bf16_tflops"] * ratio, f"{peaks['source']} bf16 burst{note}"


def input_bytes(w):
    elt = {"f32": 4, "bf16": 2, "e4m3": 1}[w.dtype]
    return w.total_tokens * (w.num_q_heads + 2 * w.num_kv_heads) * w.head_dim * elt


# ------------------------------------------------------------------ clocks sampler

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, smax, reasons = [], None, set()
        for line in self.lines:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                smax = float(parts[1])
            except ValueError:
                continue
            for name, flag in zip(self.NAMES, parts[3:7]):
                if flag.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ GPU arm

_INPUTS = {}


def generate_inputs(w):
    """Inputs of a workload, generated once and kept until another workload's are asked for (the
    threshold parameters do not change the inputs, so the all-kept run and the oracle sample reuse
    them)."""
    from synth import workloads as W
    key = (w.name, w.seqlens, w.seed, w.dtype, w.paged)
    if key not in _INPUTS:
        _INPUTS.clear()
        _INPUTS[key] = W.generate(w)
    return _INPUTS[key]


class Path:
    """Device-resident inputs plus every buffer of the path for one workload."""

    def __init__(self, wname, device, alpha=None):
        import numpy as np
        import torch
        from block_sparse_long_pooled_b200 import fp2
        from synth import workloads as W
        self.fp2 = fp2
        self.w = W.WORKLOADS[wname]
        if alpha is not None:
            self.w = self.w.replace(alpha=alpha)
        w = self.w
        inp = generate_inputs(w)
        self.inp = inp
        self.dev = device
        self.q = inp.q.to(device)
        if w.paged:
            self.k, self.v = inp.k_cache.to(device), inp.v_cache.to(device)
            self.pt = torch.from_numpy(inp.page_table).to(device)
        else:
            self.k, self.v, self.pt = inp.k.to(device), inp.v.to(device), None
        self.prob = fp2.make_problem(self.q, self.k, self.v, inp.cu_seqlens, w.num_kv_heads, inp.q_descale,
                                     inp.k_descale, inp.v_descale, page_table=self.pt)
        self.params = fp2.make_params(w.block_size, w.alpha, w.sink_blocks, w.window_blocks, w.last_n_blocks,
                                      w.min_sparse_len, w.mean_correction)
        self.ws = fp2.fp2_workspace_query(self.prob, self.params)
        self.pooled_st, self.pooled = fp2.alloc_pooled(self.ws, self.prob, device)
        self.index_st, self.index = fp2.alloc_index(self.ws, device)
        self.scratch = fp2.alloc_scratch(self.ws.prefill_scratch_bytes, device)
        self.out = torch.empty(self.q.shape, dtype=fp2.out_dtype(self.prob), device=device)
        self.np = np

    def step(self, events=None):
        f = self.fp2
        if events:
            events[0].record()
        f.fp2_pool(self.prob, self.params, self.pooled_st, self.scratch)
        if events:
            events[1].record()
        f.fp2_discover(self.prob, self.params, self.pooled_st, self.index_st, self.scratch)
        if events:
            events[2].record()
        f.fp2_attend(self.prob, self.params, self.pooled_st, self.index_st, self.out, None, self.scratch)
        if events:
            events[3].record()

    def work_counts(self):
        """Kept and pruned (q head, query block, key block) tiles of the current index."""
        np = self.np
        w = self.w
        rp = self.index["row_ptr"].cpu().numpy().astype(np.int64)
        nnz_rows = np.diff(rp)
        i_of_row = []
        for L in w.seqlens:
            N = -(-L // w.block_size)
            i_of_row.append(np.repeat(np.arange(N), w.num_kv_heads))
        i_of_row = np.concatenate(i_of_row) if i_of_row else np.zeros(0, dtype=np.int64)
        G = w.group
        kept = int(nnz_rows.sum()) * G
        pruned = int(((i_of_row + 1) - nnz_rows).sum()) * G if w.mean_correction else 0
        causal = int(sum((-(-L // w.block_size)) * (-(-L // w.block_size) + 1) // 2 for L in w.seqlens)) * \
            w.num_q_heads
        return kept, pruned, causal

    def achieved_flops(self):
        w = self.w
        kept, pruned, causal = self.work_counts()
        d, B = w.head_dim, w.block_size
        return 4.0 * d * B * B * kept + 4.0 * d * B * pruned, kept, pruned, causal

    def launches_per_step(self):
        """Kernels one step launches: pool, discover (3), attention, and with kv_splits = 0 one more
        when the attention launch is short: the split combine (fewer than 296 row CTAs) or the
        split plan (fewer than 16 waves of 148 SMs), following the library's automatic rule."""
        w = self.w
        G = w.num_q_heads // w.num_kv_heads
        mtiles = -(-G * w.block_size // 128)
        nt = 2 if mtiles >= 2 else 1
        parts = -(-mtiles // nt)
        row_ctas = self.ws.index_rows * parts
        return 5 + (1 if row_ctas < 16 * 148 else 0)

    def discover_flops(self):
        """Algorithmic flops of the pooled block scores: 2 d per (q head, query block, causal key block)."""
        w = self.w
        nb = [-(-L // w.block_size) for L in w.seqlens]
        return 2.0 * w.head_dim * w.num_q_heads * sum(n * (n + 1) // 2 for n in nb)

    def pool_bytes(self):
        w = self.w
        elt = {"f32": 4, "bf16": 2, "e4m3": 1}[w.dtype]
        T = w.total_tokens
        nb = self.ws.total_q_blocks  # q_len == kv_len in the benchmark workloads
        read = T * (w.num_q_heads + 2 * w.num_kv_heads) * w.head_dim * elt
        write = nb * (w.num_q_heads + 2 * w.num_kv_heads) * w.head_dim * 4 + 2 * nb * w.num_kv_heads * w.head_dim * elt
        if w.dtype == "e4m3":
            # f16 vbar operand (2 bytes instead of 1) and the f16 copy of V
            write += nb * w.num_kv_heads * w.head_dim + T * w.num_kv_heads * w.head_dim * 2
        return read + write


def discover_peak_tflops(peaks):
    """Peak of the discovery kernel's arithmetic: each fp32-accurate pooled product is three bf16
    tensor-core products (hi.hi + hi.lo + lo.hi), so a third of the measured bf16 burst rate (the
    kernel is timed inside a short stage)."""
    return peaks["bf16_tflops"] / 3.0


def rooflines_stage1(path, stages, peaks):
    """discover_roofline: algorithmic pooled-score flops over the discovery stage time against the
    split-bf16 tensor peak; stage1_roofline: Stage 1 (pool + discover, one pass in the pages'
    design) as HBM traffic, the pooling bytes over the two stages' time."""
    disc = path.discover_flops() / (stages["discover"] * 1e-3) / 1e12
    dpk = discover_peak_tflops(peaks)
    st1 = path.pool_bytes() / ((stages["pool"] + stages["discover"]) * 1e-3) / 1e9
    return ({"bound": "tensor", "achieved": disc, "peak": dpk, "unit": "TFLOP/s", "frac": disc / dpk,
             "peak_source": f"{peaks['source']} bf16 burst / 3 (three bf16 products per fp32-accurate product)",
             "includes": "discover_kernel + scan_kernel + scatter_kernel"},
            {"bound": "hbm", "achieved": st1, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": st1 / peaks["hbm_gbs"],
             "includes": "pool + discover stages (one read of Q, K, V)"})


def time_path(path, steps, warmup, flush=False):
    """Device time of `steps` steps after `warmup` untimed ones (CUDA events on the launching
    stream).  Returns (total ms, mean ms per stage).  flush: inputs fit in L2, so a 256 MB buffer is
    written between steps and the total is the sum of the per-step (pool..attend) spans."""
    import torch
    buf = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=path.q.device) if flush else None
    for _ in range(warmup):
        path.step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for k in range(steps):
        if buf is not None:
            buf.fill_(float(k))
        path.step(evs[k])
    end.record()
    torch.cuda.synchronize()
    total = start.elapsed_time(end)
    st = {"pool": [], "discover": [], "attend": []}
    for e in evs:
        st["pool"].append(e[0].elapsed_time(e[1]))
        st["discover"].append(e[1].elapsed_time(e[2]))
        st["attend"].append(e[2].elapsed_time(e[3]))
    if buf is not None:
        total = sum(e[0].elapsed_time(e[3]) for e in evs)
    return total, {k: sum(v) / len(v) for k, v in st.items()}


def time_e2e(path, steps):
    """The same path through the public call fp2_prefill with HOST buffers: every step copies its
    Q/K/V from pinned host memory to the device and its output O back.  Returns (pipelined ms per
    step, serial ms per step, h2d bytes, d2h bytes).  Pipelined: copies in, compute and copies out
    run on three streams with two device buffer sets, so step k+1's upload and step k-1's download
    overlap step k's compute (PCIe is full duplex); serial: one stream, nothing overlapped."""
    import torch
    fp2 = path.fp2
    hq = path.q.cpu().pin_memory()
    hk = path.k.cpu().pin_memory()
    hv = path.v.cpu().pin_memory()
    houts = [torch.empty(path.out.shape, dtype=path.out.dtype).pin_memory() for _ in range(2)]
    h2d = hq.numel() * hq.element_size() + hk.numel() * hk.element_size() + hv.numel() * hv.element_size()
    d2h = houts[0].numel() * houts[0].element_size()
    w = path.w

    # serial reference
    def one():
        path.q.copy_(hq, non_blocking=True)
        path.k.copy_(hk, non_blocking=True)
        path.v.copy_(hv, non_blocking=True)
        fp2.fp2_prefill(path.prob, path.params, path.out, None, path.scratch)
        houts[0].copy_(path.out, non_blocking=True)

    one()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(steps):
        one()
    e.record()
    torch.cuda.synchronize()
    serial_ms = s.elapsed_time(e) / steps

    # pipelined: buffer set 0 is the Path's, set 1 a second copy
    bufs = [(path.q, path.k, path.v, path.out, path.prob),
            None]
    q1, k1, v1, o1 = torch.empty_like(path.q), torch.empty_like(path.k), torch.empty_like(path.v), \
        torch.empty_like(path.out)
    prob1 = fp2.make_problem(q1, k1, v1, path.inp.cu_seqlens, w.num_kv_heads, path.inp.q_descale,
                             path.inp.k_descale, path.inp.v_descale, page_table=path.pt)
    bufs[1] = (q1, k1, v1, o1, prob1)
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    cmp_done = [None, None]
    out_done = [None, None]

    def step(k):
        b = k % 2
        q, kk, vv, o, prob = bufs[b]
        with torch.cuda.stream(s_in):
            if cmp_done[b] is not None:
                s_in.wait_event(cmp_done[b])        # compute of step k-2 no longer reads buffer b
            q.copy_(hq, non_blocking=True)
            kk.copy_(hk, non_blocking=True)
            vv.copy_(hv, non_blocking=True)
            ev_in = torch.cuda.Event()
            ev_in.record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(ev_in)
            if out_done[b] is not None:
                s_cmp.wait_event(out_done[b])       # download of step k-2 no longer reads o
            fp2.fp2_prefill(prob, path.params, o, None, path.scratch, stream=s_cmp)
            cmp_done[b] = torch.cuda.Event()
            cmp_done[b].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(cmp_done[b])
            houts[b].copy_(o, non_blocking=True)
            out_done[b] = torch.cuda.Event()
            out_done[b].record(s_out)

    for k in range(2):
        step(k)
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    start.record(s_in)
    for k in range(steps):
        step(k)
    s_in.wait_stream(s_out)
    s_in.wait_stream(s_cmp)
    stop.record(s_in)
    torch.cuda.synchronize()
    pipe_ms = start.elapsed_time(stop) / steps
    st, bits = fp2.fp2_get_device_status(path.scratch)
    if st != fp2.FP2_OK:
        raise SystemExit(f"device status {bits:#x} in the end-to-end leg")
    del bufs, q1, k1, v1, o1
    return pipe_ms, serial_ms, h2d, d2h


# ------------------------------------------------------------------ CPU oracle (baseline / reference arm)

class OracleSampler:
    """The fp64 oracle on a bounded sample of a workload (generated once).

    A sample pools every block and runs discovery for every KV-head group of the
    longest sequence, then times exact + mean-corrected attention for n uniformly
    drawn (group, query block) pairs (all G heads, all tokens of the block).  The
    full-workload time is estimated as discovery time + mean pair time x pairs,
    scaled for varlen batches by the batch's dense-equivalent work over the
    sampled sequence's (both stages grow with the square of the length)."""

    def __init__(self, wname):
        import numpy as np
        from oracle import fp2_oracle as O
        from synth import workloads as W
        self.O, self.np = O, np
        self.w = w = W.WORKLOADS[wname]
        self.inp = generate_inputs(w)
        self.r = int(np.argmax(w.seqlens))
        self.p = O.SparseParams(block_size=w.block_size, alpha=w.alpha, sink_blocks=w.sink_blocks,
                                window_blocks=w.window_blocks, last_n_blocks=w.last_n_blocks,
                                min_sparse_len=w.min_sparse_len, mean_correction=w.mean_correction)

    def _group_inputs(self, g):
        O, inp, w = self.O, self.inp, self.w
        a, b = int(inp.cu_seqlens[self.r]), int(inp.cu_seqlens[self.r + 1])
        L = b - a
        heads = list(range(g * w.group, (g + 1) * w.group))
        q = inp.dequant("q", heads=heads, tokens=slice(a, b))
        if w.paged:
            import torch
            kc = inp.k_cache[:, :, g:g + 1].to(torch.float64).numpy() * inp.k_descale
            vc = inp.v_cache[:, :, g:g + 1].to(torch.float64).numpy() * inp.v_descale
            k = O.gather_paged(kc, inp.page_table[self.r:self.r + 1], [L])
            v = O.gather_paged(vc, inp.page_table[self.r:self.r + 1], [L])
        else:
            k = inp.dequant("k", heads=[g], tokens=slice(a, b))
            v = inp.dequant("v", heads=[g], tokens=slice(a, b))
        return q, k, v, L

    def run(self, n_pairs, seed=0):
        O, np, w = self.O, self.np, self.w
        B, G = w.block_size, w.group
        scale = 1.0 / math.sqrt(w.head_dim)
        rng = np.random.default_rng(seed)
        L = w.seqlens[self.r]
        N = -(-L // B)
        pairs = rng.integers(0, w.num_kv_heads * N, size=n_pairs)
        t_disc = t_attn = 0.0
        for g in range(w.num_kv_heads):
            q, k, v, L = self._group_inputs(g)
            t0 = time.perf_counter()
            qbar, counts = O.pool_blocks(q, B)
            kbar, _ = O.pool_blocks(k, B)
            vbar, _ = O.pool_blocks(v, B)
            kept, _ = O.select_blocks(O.block_scores(qbar, kbar, scale), 1, L, self.p)
            t1 = time.perf_counter()
            t_disc += t1 - t0
            for pr in pairs[pairs // N == g]:
                i = int(pr % N)
                rows = np.array([[t, h] for t in range(i * B, min(L, (i + 1) * B)) for h in range(G)])
                t2 = time.perf_counter()
                O.attend(q, k, v, kbar, vbar, counts, kept, B, scale, w.mean_correction, rows=rows)
                t_attn += time.perf_counter() - t2
        scale_up = w.dense_equiv_flops() / w.replace(seqlens=(L,)).dense_equiv_flops()
        est = (t_disc + t_attn / max(1, n_pairs) * w.num_kv_heads * N) * scale_up
        desc = (f"fp64 oracle: pooling + discovery of all {w.num_kv_heads} KV-head groups of the {L}-token "
                f"sequence, attention for {n_pairs} uniformly drawn (group, query block) pairs of "
                f"{w.num_kv_heads * N}; full time = discovery + mean pair time x pairs"
                + (f", x{scale_up:.3f} for the batch's other sequences (dense-equivalent work ratio)"
                   if len(w.seqlens) > 1 else ""))
        return t_disc + t_attn, est, desc


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def config_dict(w, world):
    """The `config` object of a bench line (the same for the GPU arm and the reference arm)."""
    ib = input_bytes(w)
    return {"workload": w.name, "seq_len": max(w.seqlens), "batch": len(w.seqlens),
            "heads": f"{w.num_q_heads}/{w.num_kv_heads}", "head_dim": w.head_dim, "block": w.block_size,
            "alpha": w.alpha, "sink": w.sink_blocks, "window": w.window_blocks, "last_n": w.last_n_blocks,
            "min_sparse_len": w.min_sparse_len, "kv": "paged (64-token pages)" if w.paged else "contiguous",
            "parallelism": f"replicas{world}",
            "l2": (f"inputs larger than L2 ({ib / 1e9:.2f} GB)" if ib > L2_BYTES
                   else f"inputs fit in L2 ({ib / 1e6:.2f} MB): 256 MB written between steps")}


def run_reference(args, rank, world):
    """The fp64 oracle on the host cores.  It cannot run a whole 128K step in a bounded time, so each
    step runs a bounded sample (pooling and discovery of every KV group of the longest sequence, and
    exact + corrected attention for `pairs` whole (group, query block) pairs).  ms_per_step is that
    sample's measured wall time; the whole-workload time is extrapolated from it
    (extrapolated_ms_per_full_step), and value = dense-equivalent work / extrapolated time, i.e. the
    sample's share of the work (sample_fraction = measured / extrapolated) over its measured time."""
    from synth import workloads as W
    if rank != 0:
        return
    w = W.WORKLOADS[args.workload]
    dense = w.dense_equiv_flops()
    pairs = 32
    sampler = OracleSampler(args.workload)
    for k in range(args.warmup):
        sampler.run(2, seed=1000 + k)
    times, ests, desc = [], [], ""
    for k in range(args.steps):
        t, est, desc = sampler.run(pairs, seed=k)
        times.append(t)
        ests.append(est)
    est = statistics.mean(ests)
    t_mean = statistics.mean(times)
    value = dense / est / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_mean * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(w, args.gpus),
            "extrapolated_from_pairs": pairs,
            "extrapolated_ms_per_full_step": est * 1e3,
            "sample_fraction": t_mean / est,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
                             "sample": desc + f"; each step is this sample ({t_mean:.2f} s measured, "
                                              f"{100 * t_mean / est:.3f} % of the extrapolated full step)"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ sweeps (ablations)

def run_sweep(kind, args):
    """Sweeps on the 64K FP8 workload (one JSON line per point).

    alpha:       block density and step / attention time for alpha in {0.2, 0.1, 0.05, 0.025, 0.0125}
                 (the paper page's Table 9 grid).
    correction:  attention time with mean correction on and off, and the relative L2 error of
                 each against the all-blocks-kept output of the same library (Figure 6, Table 8).
    sparsity:    attention time against density over a wide alpha range, next to the time the
                 computed tiles would take at the measured tensor peak (Figure 5).
    chunked:     the 128K bf16 layer as 8K / 16K chunks versus one pass (Table 6).
    """
    import torch
    from block_sparse_long_pooled_b200 import build, fp2
    build.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    wname = args.workload if args.workload != DEFAULT_WORKLOAD else "qwen4b_64k_e4m3"
    peak = attention_peak("e4m3" if "e4m3" in wname else "bf16", peaks)[0]
    if kind == "chunked":
        for line in chunked_sweep(args, dev, peaks):
            print(json.dumps(line), flush=True)
        return
    base = Path(wname, dev)
    steps, warm = max(5, args.steps // 2), max(3, args.warmup)

    def measure(path):
        ms, st = time_path(path, steps, warm)
        ach, kept, pruned, causal = path.achieved_flops()
        return {"ms_per_step": ms / steps, "attend_ms": st["attend"], "density": kept / causal,
                "attend_tflops": ach / (st["attend"] * 1e-3) / 1e12,
                "ideal_attend_ms": ach / (peak * 1e12) * 1e3}

    def retarget(alpha=None, correction=None):
        w = base.w
        base.params = fp2.make_params(w.block_size, w.alpha if alpha is None else alpha, w.sink_blocks,
                                      w.window_blocks, w.last_n_blocks, w.min_sparse_len,
                                      w.mean_correction if correction is None else correction)
        base.w = w.replace(alpha=base.w.alpha if alpha is None else alpha,
                           mean_correction=w.mean_correction if correction is None else correction)

    out = []
    if kind in ("alpha", "sparsity"):
        grid = [0.2, 0.1, 0.05, 0.025, 0.0125] if kind == "alpha" else \
            [0.9, 0.5, 0.2, 0.1, 0.05, 0.02, 0.01, 0.005, 0.002, 0.001, 1e-4, 0.0]
        for al in grid:
            retarget(alpha=al)
            out.append({"sweep": kind, "workload": wname, "alpha": al, **measure(base)})
    elif kind == "correction":
        retarget(alpha=0.0)
        base.step()
        dense = base.out.float().clone()
        for corr in (True, False):
            retarget(alpha=0.1, correction=corr)
            m = measure(base)
            o = base.out.float()
            m["rel_l2_vs_all_kept"] = float(torch.linalg.vector_norm(o - dense) / torch.linalg.vector_norm(dense))
            m["max_abs_vs_all_kept"] = float((o - dense).abs().max())
            out.append({"sweep": kind, "workload": wname, "alpha": 0.1, "mean_correction": corr, **m})
    for line in out:
        print(json.dumps(line), flush=True)


def chunked_sweep(args, dev, peaks):
    """Chunked prefill of the 128K bf16 layer: the sequence is processed in chunks of 8K / 16K
    tokens (each chunk's queries against all keys so far, bottom-right causal; pooled prefix K/V
    reused from earlier chunks) and as one 128K pass.  Reports per chunk size the summed
    pool / discover / attend time over all chunks and the share spent outside attention."""
    import torch
    from block_sparse_long_pooled_b200 import fp2
    from synth import workloads as W
    w = W.WORKLOADS["llama8b_128k_bf16"]
    inp = W.generate(w)
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    L, B = w.seqlens[0], w.block_size
    params = fp2.make_params(B, w.alpha, w.sink_blocks, w.window_blocks, w.last_n_blocks, w.min_sparse_len,
                             w.mean_correction)
    full = fp2.make_problem(q, k, v, [0, L], w.num_kv_heads)
    ws_full = fp2.fp2_workspace_query(full, params)
    _, pooled = fp2.alloc_pooled(ws_full, full, dev)
    pst = fp2.pooled_struct(pooled)
    scratch = fp2.alloc_scratch(ws_full.prefill_scratch_bytes, dev)
    out = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
    lines = []
    for C in (8192, 16384, L):
        chunks = []
        for s0 in range(0, L, C):
            prob = fp2.make_problem(q[s0:s0 + C], k, v, [0, C], w.num_kv_heads, cu_seqlens_k=[0, s0 + C],
                                    kv_prefix_pooled=s0 > 0)
            ws = fp2.fp2_workspace_query(prob, params)
            ist, ix = fp2.alloc_index(ws, dev)
            chunks.append((prob, ist, ix, s0))
            # one scratch serves every call: size it for the largest (short chunk launches carry
            # the adaptive-split buffers, the one-pass launch does not)
            if ws.scratch_bytes > scratch.numel():
                scratch = fp2.alloc_scratch(ws.scratch_bytes, dev)

        def run(evs=None):
            for n, (prob, ist, _, s0) in enumerate(chunks):
                if evs:
                    evs[n][0].record()
                fp2.fp2_pool(prob, params, pst, scratch)
                if evs:
                    evs[n][1].record()
                fp2.fp2_discover(prob, params, pst, ist, scratch)
                if evs:
                    evs[n][2].record()
                fp2.fp2_attend(prob, params, pst, ist, out[s0:s0 + C], None, scratch)
                if evs:
                    evs[n][3].record()

        run()
        torch.cuda.synchronize()
        t_h = time.perf_counter()
        run()
        host_ms = (time.perf_counter() - t_h) * 1e3   # enqueue time of all chunks' calls
        torch.cuda.synchronize()
        reps = 3
        tot = {"pool": 0.0, "discover": 0.0, "attend": 0.0}
        per_chunk = [0.0] * len(chunks)
        for _ in range(reps):
            evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in chunks]
            run(evs)
            torch.cuda.synchronize()
            for n, e in enumerate(evs):
                tot["pool"] += e[0].elapsed_time(e[1]) / reps
                tot["discover"] += e[1].elapsed_time(e[2]) / reps
                tot["attend"] += e[2].elapsed_time(e[3]) / reps
                per_chunk[n] += e[2].elapsed_time(e[3]) / reps
        total = sum(tot.values())
        lines.append({"sweep": "chunked", "workload": w.name, "chunk": C, "chunks": len(chunks),
                      "total_ms": total, "stages_ms": tot, "outside_attention_share": (total - tot["attend"]) / total,
                      "host_enqueue_ms": host_ms, "attend_ms_per_chunk": [round(x, 4) for x in per_chunk]})
    return lines


# ------------------------------------------------------------------ per-config measurement

def measure_config(wname, dev, peaks, steps, warmup, all_kept=True, cpu_pairs=0, label=None):
    """One workload: device-timed steps (pool, discover, attend), the rooflines of the three stages,
    the same library with every block kept, and optionally the oracle on a bounded sample."""
    import torch
    from synth import workloads as W
    w = W.WORKLOADS[wname]
    flush = input_bytes(w) <= L2_BYTES
    path = Path(wname, dev)
    sampler = ClockSampler(dev.index or 0)
    sampler.start()
    total, st = time_path(path, steps, warmup, flush=flush)
    clocks = sampler.stop()
    fst, bits = path.fp2.fp2_get_device_status(path.scratch)
    if fst != path.fp2.FP2_OK:
        raise SystemExit(f"device status {bits:#x} on {wname}")
    ms = total / steps
    dense = w.dense_equiv_flops()
    ach, kept, pruned, causal = path.achieved_flops()
    peak, peak_src = attention_peak(w.dtype, peaks)
    attn = ach / (st["attend"] * 1e-3) / 1e12
    pool_gbs = path.pool_bytes() / (st["pool"] * 1e-3) / 1e9
    disc_rl, st1_rl = rooflines_stage1(path, st, peaks)
    e = {"label": label, "workload": wname, "dtype": w.dtype, "config": config_dict(w, 1), "steps": steps,
         "ms_per_step": ms, "stages_ms": st, "dense_equiv_tflops": dense / (ms * 1e-3) / 1e12,
         "achieved_tflops": ach / (ms * 1e-3) / 1e12, "sparsity": kept / causal,
         "roofline": {"kernel": "attention_kernel", "bound": "tensor", "achieved": attn, "peak": peak,
                      "unit": "TFLOP/s", "frac": attn / peak, "peak_source": peak_src,
                      "traffic": attention_traffic(wname)},
         "pool_roofline": {"bound": "hbm", "achieved": pool_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                           "frac": pool_gbs / peaks["hbm_gbs"]},
         "discover_roofline": disc_rl, "stage1_roofline": st1_rl,
         "clocks": clocks, "launches_per_step": path.launches_per_step()}
    del path
    torch.cuda.empty_cache()
    if all_kept:
        dp = Path(wname, dev, alpha=0.0)
        k = max(3, steps // 4)
        dms, dst = time_path(dp, k, 2, flush=flush)
        dach, _, _, _ = dp.achieved_flops()
        e["all_kept"] = {"ms_per_step": dms / k, "attend_ms": dst["attend"],
                         "attend_tflops": dach / (dst["attend"] * 1e-3) / 1e12,
                         "attend_frac": dach / (dst["attend"] * 1e-3) / 1e12 / peak,
                         "speedup_of_sparse": (dms / k) / ms}
        del dp
        torch.cuda.empty_cache()
    if cpu_pairs > 0:
        secs, est, desc = OracleSampler(wname).run(cpu_pairs)
        e["cpu_baseline"] = {"value": dense / est / 1e12, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
                             "ms_per_step_extrapolated": est * 1e3,
                             "sample": desc + f" ({secs:.1f} s of CPU work)"}
    return e


# ------------------------------------------------------------------ main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-extras", action="store_true",
                    help="only the headline workload: skip the all-kept, e2e, CPU and per-config legs")
    ap.add_argument("--sweep", choices=["alpha", "correction", "sparsity", "chunked"], default=None,
                    help="ablation sweeps on the 64K FP8 workload instead of the benchmark line")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")
    if args.sweep:
        run_sweep(args.sweep, args)
        return
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import torch
    from block_sparse_long_pooled_b200 import build, fp2
    build.build()
    fp2.load_library()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
        pg = dist
    peaks = load_peaks()

    path = Path(args.workload, dev)
    w = path.w
    flush = input_bytes(w) <= L2_BYTES
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    sampler.start()
    total_ms, stages = time_path(path, args.steps, args.warmup, flush=flush)
    clocks = sampler.stop()
    total_ms = max_over_ranks(pg, total_ms, dev)
    if pg:
        pg.barrier()
    st, bits = fp2.fp2_get_device_status(path.scratch)
    if st != fp2.FP2_OK:
        raise SystemExit(f"device status {bits:#x}")
    ms = total_ms / args.steps
    dense = w.dense_equiv_flops()
    ach, kept, pruned, causal = path.achieved_flops()
    value = whole_job_value(dense, world, ms)
    attn_tflops = ach / (stages["attend"] * 1e-3) / 1e12
    peak, peak_src = attention_peak(w.dtype, peaks)
    traffic = attention_traffic(w.name)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic (seeded needle-in-a-haystack-style generator: low-rank block-persistent Q/K, planted needle key blocks and queries)",
        "config": config_dict(w, world),
        "achieved_tflops": ach / (ms * 1e-3) / 1e12,
        "sparsity": kept / causal,
        "stages_ms": stages,
        "roofline": {"kernel": "attention_kernel", "bound": "tensor", "achieved": attn_tflops, "peak": peak,
                     "unit": "TFLOP/s", "frac": attn_tflops / peak, "traffic": traffic, "peak_source": peak_src},
        "pool_roofline": {"bound": "hbm", "achieved": path.pool_bytes() / (stages["pool"] * 1e-3) / 1e9,
                          "peak": peaks["hbm_gbs"], "unit": "GB/s",
                          "frac": path.pool_bytes() / (stages["pool"] * 1e-3) / 1e9 / peaks["hbm_gbs"]},
        "discover_roofline": rooflines_stage1(path, stages, peaks)[0],
        "stage1_roofline": rooflines_stage1(path, stages, peaks)[1],
        "clocks": clocks,
        "gpu_launches": path.launches_per_step() * args.steps,
    }
    if not args.no_extras:
        # the same library with every block kept (alpha = 0) on the same inputs
        dense_path = Path(args.workload, dev, alpha=0.0)
        dms, dst = time_path(dense_path, max(3, args.steps // 8), 3, flush=flush)
        dach, _, _, _ = dense_path.achieved_flops()
        line["all_kept"] = {"ms_per_step": dms / max(3, args.steps // 8),
                            "attend_tflops": dach / (dst["attend"] * 1e-3) / 1e12,
                            "attend_frac": dach / (dst["attend"] * 1e-3) / 1e12 / peak}
        del dense_path
        # at least 32 pipelined steps, so the fill (first upload) and drain (last compute and
        # download) weigh little against the upload-bound steady state
        e2e_ms, serial_ms, h2d, d2h = time_e2e(path, max(32, args.steps))
        e2e_ms = max_over_ranks(pg, e2e_ms, dev)
        line["e2e"] = {"value": whole_job_value(dense, world, e2e_ms), "unit": UNIT, "ms_per_step": e2e_ms,
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                       "mode": "pipelined: upload, fp2_prefill and download on three streams",
                       "serial_ms_per_step": serial_ms}
        del path
        torch.cuda.empty_cache()
        if args.workload == DEFAULT_WORKLOAD and world == 1:
            per = []
            for label, wname in CONFIGS:
                if wname == args.workload:
                    per.append({"label": label, "workload": wname, "same_as": "headline line"})
                    continue
                per.append(measure_config(wname, dev, peaks, max(5, args.steps // 2), args.warmup,
                                          cpu_pairs=128 if rank == 0 else 0, label=label))
            line["per_config"] = per
            fp8 = next(e for e in per if e["workload"] == FP8_WORKLOAD)
            line["fp8"] = {"workload": FP8_WORKLOAD, "ms_per_step": fp8["ms_per_step"],
                           "value": fp8["dense_equiv_tflops"], "achieved_tflops": fp8["achieved_tflops"],
                           "sparsity": fp8["sparsity"], "stages_ms": fp8["stages_ms"],
                           "attend_tflops": fp8["roofline"]["achieved"],
                           "attend_frac_of_fp8_peak": fp8["roofline"]["frac"],
                           "attend_frac_of_bf16_peak": fp8["roofline"]["achieved"] / peaks["bf16_tflops"]}
        if rank == 0 and world == 1:
            secs, est, desc = OracleSampler(args.workload).run(400)
            line["cpu_baseline"] = {"value": dense / est / 1e12, "unit": UNIT, "cores": cpu_cores(),
                                    "kind": "oracle", "sample": desc + f" ({secs:.1f} s of CPU work)"}
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
