"""Host-side helpers of bench.py that feed its JSON line (no GPU): the peaks of the discovery and
Stage-1 rooflines and the kernel-launch count per step."""

import numpy as np
import torch

import bench
from block_sparse_long_pooled_b200 import fp2
from synth import workloads as W


def test_stage1_rooflines_from_peaks_and_stage_times():
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0, "bf16_tflops_sustained": 1400.0, "source": "test"}
    assert bench.discover_peak_tflops(peaks) == 500.0      # three bf16 products per fp32-accurate one

    class P:
        def discover_flops(self):
            return 5e12 * 1e-4                              # 5 TFLOP/s over 0.1 ms

        def pool_bytes(self):
            return 6000e9 * 0.3e-3 * 0.5                    # half of HBM over 0.3 ms
    d, st1 = bench.rooflines_stage1(P(), {"pool": 0.2, "discover": 0.1, "attend": 1.0}, peaks)
    assert abs(d["achieved"] - 5.0) < 1e-9 and abs(d["frac"] - 0.01) < 1e-12 and d["bound"] == "tensor"
    assert abs(st1["frac"] - 0.5) < 1e-12 and st1["bound"] == "hbm"


class _FakePath:
    def __init__(self, name):
        w = W.WORKLOADS[name]
        dt = {"bf16": torch.bfloat16, "e4m3": torch.float8_e4m3fn, "f32": torch.float32}[w.dtype]
        q = torch.empty((w.total_tokens, w.num_q_heads, w.head_dim), dtype=dt)
        k = torch.empty((w.total_tokens, w.num_kv_heads, w.head_dim), dtype=dt)
        cu = np.concatenate([[0], np.cumsum(w.seqlens)]).astype(np.int32)
        prob = fp2.make_problem(q, k, k, cu, w.num_kv_heads)
        params = fp2.make_params(w.block_size, w.alpha, w.sink_blocks, w.window_blocks, w.last_n_blocks,
                                 w.min_sparse_len, w.mean_correction)
        self.w = w
        self.ws = fp2.fp2_workspace_query(prob, params)


def test_launches_per_step_follow_the_split_rule():
    # 128K layer: 8192 index rows x 2 packed parts = 16384 row CTAs -> no split plan or combine
    assert bench.Path.launches_per_step(_FakePath("llama8b_128k_bf16")) == 5
    # tiny workload: 16 row CTAs -> uniform KV splits and their combine kernel
    assert bench.Path.launches_per_step(_FakePath("tiny_1k_f32")) == 6
