"""Both decode-attention kernels on every decode parity case.

The library picks the TMA-fed tensor-core kernel or the CUDA-core kernel by
(head_dim, GQA group); LLAMA_DECODE_ATTN=mma | simt forces one of them.  The
choice is read once per process, so each kernel runs the decode parity tests
of ``test_gpu_layer.py`` (head_dim 64 / 96 / 128, groups 1 / 4 / 8, against
the fp64 oracle) in a child process, together with the full-size 13B-shaped
decode check.
"""

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("kernel", ["mma", "simt"])
def test_decode_parity_with_each_attention_kernel(kernel):
    env = dict(os.environ, LLAMA_DECODE_ATTN=kernel)
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider", "-m", "gpu",
                        "tests/test_gpu_layer.py", "-k", "decode"], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=1200)
    print(r.stdout[-3000:])
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
    assert " passed" in r.stdout
