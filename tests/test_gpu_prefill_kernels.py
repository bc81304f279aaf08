"""Both prefill-attention kernels on every prefill parity case.

The library runs the 64-key-step kernel (two S buffers per query tile) for
head_dim below 128 and the 128-key-step kernel at 128; LLAMA_ATTN_FORM=k64 or
pair takes one of them for every shape.  The choice is read once per process,
so each kernel runs the prefill parity tests of ``test_gpu_layer.py`` (head_dim
64 / 96 / 128, MHA and GQA head pairs, chunked prefill over a cache, the
rescale path of large scores) and the ragged batches of ``test_gpu_ragged.py``
against the fp64 oracle in a child process.
"""

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("form", ["pair", "k64"])
def test_prefill_parity_with_each_attention_kernel(form):
    env = dict(os.environ, LLAMA_ATTN_FORM=form)
    targets = ["tests/test_gpu_layer.py", "tests/test_gpu_ragged.py", "-k", "prefill or ragged"]
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider", "-m", "gpu"] + targets,
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1200)
    print(r.stdout[-3000:])
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
    assert " passed" in r.stdout
