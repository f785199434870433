"""Accuracy ablation of the mean correction against dense attention (the paper page's Table 8
measures task accuracy with and without the correction; here the numerical analogue).

On the Qwen3-4B-shaped 64K FP8 layer at alpha = 0.1, the GPU outputs with the correction on and off
are compared with the fp64 oracle's DENSE causal attention (every block kept) on whole (KV group,
query block) pairs.  The correction must bring the output closer to dense attention, and the
kernel's own error (GPU against the oracle's sparse output) must be small next to the method's
(the oracle's sparse output against its dense one).
"""

import dataclasses

import numpy as np
import pytest

from synth import workloads as W
from tests import harness as Hn

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from block_sparse_long_pooled_b200 import build
    build.build()


def _rel(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def test_mean_correction_error_against_dense_oracle():
    import torch
    w = W.WORKLOADS["qwen4b_64k_e4m3"]
    inp = W.generate(w)
    ora = Hn.oracle_discovery(inp)
    pairs = Hn.select_pairs(inp, ora, n_random=16)
    dense_kept = [np.broadcast_to(np.tril(np.ones(o.kept.shape[1:], dtype=bool)), o.kept.shape).copy() for o in ora]
    O_dense, _, toks, heads = Hn.oracle_pairs(inp, ora, pairs, kept_override=dense_kept)
    res = {}
    for corr in (True, False):
        inp_c = dataclasses.replace(inp, workload=w.replace(mean_correction=corr))
        O_sp, _, t2, h2 = Hn.oracle_pairs(inp_c, ora, pairs)
        assert np.array_equal(t2, toks) and np.array_equal(h2, heads)
        run = Hn.run_gpu(inp_c, external_index=Hn.oracle_csr(ora), lse=False)
        g = run.out[torch.from_numpy(toks).cuda(), torch.from_numpy(heads).cuda()].float().cpu().numpy()
        res[corr] = {"gpu_vs_dense": _rel(g.astype(np.float64), O_dense),
                     "oracle_vs_dense": _rel(O_sp, O_dense),
                     "gpu_vs_oracle": _rel(g.astype(np.float64), O_sp)}
        del run
        torch.cuda.empty_cache()
    print(f"correction on : {res[True]}\ncorrection off: {res[False]}  ({len(pairs)} pairs, {len(toks)} rows)")
    assert res[True]["gpu_vs_dense"] < res[False]["gpu_vs_dense"]
    assert res[True]["oracle_vs_dense"] < res[False]["oracle_vs_dense"]
    for corr in (True, False):
        assert res[corr]["gpu_vs_oracle"] < 0.2 * res[corr]["oracle_vs_dense"]
