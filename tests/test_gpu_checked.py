"""The checked build, libfp2_checked.so (the same sources with FP2_CHECKED=1; include/fp2.h says
what it checks), on the small parity cases, the KV-split and one-call cases and the chunked-prefill
cases, in a child process that loads it through FP2_LIBRARY.  Every output must still match the
oracle and no check may fire: those tests assert a zero device status word, and a failed
hand-off count or bound sets FP2_DEV_CHECK in it.  And the checks do fire: with the testing hook
FP2_DEBUG_MISCOUNT_LOAD the producer counts one K/V load twice (the data path is untouched), and
the consumer's exact-count check must report it; the normal build ignores the hook."""

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_parity_cases_pass_under_the_checked_build():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from block_sparse_long_pooled_b200 import build
    lib = build.build(checked=True)
    env = dict(os.environ, FP2_LIBRARY=lib)
    probe = subprocess.run(
        [sys.executable, "-c",
         "from block_sparse_long_pooled_b200 import fp2; import sys; sys.exit(0 if fp2.fp2_build_flags() == "
         "fp2.FP2_BUILD_CHECKED else 3)"],
        cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert probe.returncode == 0, probe.stdout + probe.stderr
    r = subprocess.run(
        [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", "-m", "gpu",
         "tests/test_gpu_parity.py", "tests/test_gpu_chunked.py",
         "-k", "small_full_parity or kv_splits or tiny or chunk or prefix"],
        cwd=ROOT, env=env, capture_output=True, text=True, timeout=1800)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout and "failed" not in r.stdout


# One small prefill with the miscount hook on, then one without; prints the two status pairs.
_MISCOUNT = r"""
import sys, torch
from block_sparse_long_pooled_b200 import fp2
from synth import workloads as W
w = W.WORKLOADS["tiny_1k_f32"].replace(seqlens=(1000, 333), num_q_heads=8, num_kv_heads=2, head_dim=128,
                                       block_size=128, dtype="bf16", iid=False)
inp = W.generate(w)
dev = torch.device("cuda:0")
q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
prob = fp2.make_problem(q, k, v, inp.cu_seqlens, w.num_kv_heads)
params = fp2.make_params(w.block_size, 0.0)   # every block kept: each CTA streams several key tiles
ws = fp2.fp2_workspace_query(prob, params)
out = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
res = []
for load in (2, -1):
    fp2.fp2_debug_set(fp2.FP2_DEBUG_MISCOUNT_LOAD, load)
    scratch = fp2.alloc_scratch(ws.prefill_scratch_bytes, dev)
    fp2.fp2_prefill(prob, params, out, None, scratch)
    torch.cuda.synchronize(dev)
    res.append(fp2.fp2_get_device_status(scratch))
print("RESULT", fp2.fp2_build_flags(), res[0][0], res[0][1], res[1][0], res[1][1])
"""


def _run_miscount(env):
    r = subprocess.run([sys.executable, "-c", _MISCOUNT], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    line = [l for l in r.stdout.splitlines() if l.startswith("RESULT")][-1]
    return [int(x) for x in line.split()[1:]]


def test_a_miscounted_hand_off_is_reported_by_the_checked_build_only():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from block_sparse_long_pooled_b200 import build, fp2
    checked_lib = build.build(checked=True)
    flags, st0, bits0, st1, bits1 = _run_miscount(dict(os.environ, FP2_LIBRARY=checked_lib))
    assert flags == fp2.FP2_BUILD_CHECKED
    assert st0 == fp2.FP2_ERR_CHECK_FAILED and bits0 == fp2.FP2_DEV_CHECK, (st0, bits0)
    assert (st1, bits1) == (fp2.FP2_OK, 0)                      # the next clean call is unaffected
    env = {k: v for k, v in os.environ.items() if k != "FP2_LIBRARY"}
    flags, st0, bits0, st1, bits1 = _run_miscount(dict(env, FP2_LIBRARY=build.build()))
    assert flags == 0 and (st0, bits0) == (fp2.FP2_OK, 0) and (st1, bits1) == (fp2.FP2_OK, 0)

