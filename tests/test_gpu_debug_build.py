"""The bounds-checked build (libs2attn_debug.so, compiled with S2ATTN_DEBUG) on the GPU:
every computed global store or reduction index is checked against its tensor's extent,
and an out-of-range one is skipped and recorded in the error word (site bit 0x80).  The
core parity suites run against it in a child process (the library is selected with
S2ATTN_LIBRARY before the binding loads it): on valid shapes no check may fire, and the
results must still match the oracle."""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_parity_suites_pass_on_the_bounds_checked_build():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from shifted_sparse_attention_s2attn_b200 import _build
    env = dict(os.environ, S2ATTN_LIBRARY=_build.build(debug=True))
    cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
           os.path.join(ROOT, "tests", "test_gpu_parity.py"), os.path.join(ROOT, "tests", "test_gpu_decode.py"),
           "-k", "small or rope or deterministic or matches_oracle or back_to_back"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
