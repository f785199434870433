"""The checked build, libfp2_checked.so (the same sources with FP2_CHECKED=1; include/fp2.h says
what it checks), on the small parity cases, the KV-split and one-call cases and the chunked-prefill
cases, in a child process that loads it through FP2_LIBRARY.  Every output must still match the
oracle and no check may fire: those tests assert a zero device status word, and a failed
hand-off count or bound sets FP2_DEV_CHECK in it."""

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
