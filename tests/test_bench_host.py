"""Host-side helpers of bench.py that feed its JSON line (no GPU): the fp32 FMA peak used for the
discovery roofline and the kernel-launch count per step."""

import numpy as np
import torch

import bench
from block_sparse_long_pooled_b200 import fp2
from synth import workloads as W


def test_fp32_fma_peak_from_unit_counts():
    # 148 SMs x 128 FMA lanes x 2 flops x clock
    assert abs(bench.fp32_fma_peak_tflops({"sm_max_mhz": 1965.0}) - 148 * 128 * 2 * 1.965e9 / 1e12) < 1e-9
    assert bench.fp32_fma_peak_tflops(None) == bench.fp32_fma_peak_tflops({"sm_max_mhz": 1965.0})


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
