"""Both decode-attention kernels on every decode parity case.

The library picks the TMA-fed tensor-core kernel or the CUDA-core kernel by
(head_dim, GQA group); LLAMA_DECODE_ATTN=mma | simt forces one of them.  The
choice is read once per process, so each kernel runs the decode parity tests
of ``test_gpu_layer.py`` (head_dim 64 / 96 / 128, groups 1 / 4 / 8, against
the fp64 oracle) in a child process, together with the full-size 13B-shaped
decode check.  The same child runs cover the other decode forms: RoPE + KV
append kept apart from the CUDA-core attention (LLAMA_FUSE_ROPE=0), the
persistent decode-block kernel at batch <= 16 instead of a kernel per step
(LLAMA_DECODE_LAYER=1), the RMSNorms taken into the ends of the residual
GEMMs (LLAMA_FUSE_NORM=1), the decode GEMMs split over thread-block
clusters whatever the SM share (LLAMA_DECODE_CLUSTER=2, where by default only
the full-size shapes take clusters), and every decode GEMM kept stream-K
(LLAMA_DECODE_CLUSTER=0).
"""

import os
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("kernel,extra", [("mma", {}), ("simt", {}), ("simt", {"LLAMA_FUSE_ROPE": "0"}),
                                          ("simt", {"LLAMA_DECODE_LAYER": "1"}),
                                          ("mma", {"LLAMA_FUSE_NORM": "1"}), ("simt", {"LLAMA_FUSE_NORM": "1"}),
                                          ("mma", {"LLAMA_DECODE_CLUSTER": "2"}),
                                          ("mma", {"LLAMA_DECODE_CLUSTER": "2", "LLAMA_FUSE_NORM": "1"}),
                                          ("simt", {"LLAMA_DECODE_CLUSTER": "0"})],
                         ids=["mma", "simt", "simt-rope-apart", "simt-decode-block", "mma-norm-fused",
                              "simt-norm-fused", "mma-cluster-split", "mma-cluster-split-norm-fused",
                              "simt-stream-k-only"])
def test_decode_parity_with_each_attention_kernel(kernel, extra):
    env = dict(os.environ, LLAMA_DECODE_ATTN=kernel, **extra)
    targets = ["tests/test_gpu_layer.py", "-k", "decode"]
    if extra.get("LLAMA_FUSE_NORM") == "1" or extra.get("LLAMA_DECODE_CLUSTER"):
        # a whole model chains each down GEMM into the next block's first RMSNorm
        targets = ["tests/test_gpu_layer.py", "tests/test_gpu_fullsize.py", "-k", "decode or phi3_two_layer"]
    if extra.get("LLAMA_DECODE_CLUSTER"):
        # the ragged batches' decode rows take the same GEMM forms
        targets = targets[:-2] + ["tests/test_gpu_ragged.py", "-k", "decode or phi3_two_layer or ragged"]
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider", "-m", "gpu"] + targets,
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1200)
    print(r.stdout[-3000:])
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
    assert " passed" in r.stdout


# Two decode steps of a block, written out by a child process: the rotated q,
# the appended k / v rows and the block output (argv: path, rope style, batch).
_CHILD = r"""
import sys, numpy as np, synth
from tests.harness import LayerRun
name, dim, nh, nkv, hd, ffn, T0, rope = "c", 384, 4, 4, 96, 1024, 700, sys.argv[2]
B = int(sys.argv[3])
w = synth.Workload(name, dim, nh, nkv, hd, ffn, 1e-5, 1e4, rope, "bf16", 0.02, 91,
                   cache_len=T0, decode_batch=B, decode_steps=2)
inp = synth.decode_inputs(w)
run = LayerRun(w, inp.weights, B, T0 + 8, 1, k0=inp.k_cache, v0=inp.v_cache)
out = {}
for t, xs in enumerate(inp.steps):
    out[f"y{t}"] = run.step(xs)
    it = run.intermediates()
    for n in ("q", "k", "v"):
        out[f"{n}{t}"] = it[n]
np.savez(sys.argv[1], **out)
"""


def _child_runs(tmp_path, rope, batch, envs):
    res = {}
    for tag, extra in envs.items():
        env = dict(os.environ, PYTHONPATH=ROOT, **extra)
        path = str(tmp_path / f"{tag}.npz")
        r = subprocess.run([sys.executable, "-c", _CHILD, path, rope, str(batch)], cwd=ROOT, env=env,
                           capture_output=True, text=True, timeout=600)
        assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
        res[tag] = np.load(path)
    return res


@pytest.mark.parametrize("kernel", ["simt", "mma"])
@pytest.mark.parametrize("rope", ["half", "interleaved"])
def test_rope_inside_attention_is_bit_identical_to_the_rope_kernel(tmp_path, rope, kernel):
    """RoPE + KV append inside either decode attention kernel (batch 40: one key
    split per (sequence, KV head)) rounds exactly like the stand-alone kernel:
    the same rotated q and appended k / v bits; the block output differs only
    by the order in which the new key joins the softmax."""
    res = _child_runs(tmp_path, rope, 40, {
        "fused": {"LLAMA_DECODE_ATTN": kernel, "LLAMA_FUSE_ROPE": "1"},
        "apart": {"LLAMA_DECODE_ATTN": kernel, "LLAMA_FUSE_ROPE": "0"}})
    a, b = res["fused"], res["apart"]
    for t in range(2):
        for n in ("q", "k", "v"):
            assert np.array_equal(a[f"{n}{t}"], b[f"{n}{t}"]), f"step {t}: {n} differs"
        ya, yb = a[f"y{t}"], b[f"y{t}"]
        rms = np.sqrt(np.mean(yb ** 2))
        assert np.max(np.abs(ya - yb)) <= 1e-3 * rms, f"step {t}: {np.max(np.abs(ya - yb)) / rms:.3g}"


@pytest.mark.parametrize("rope", ["half", "interleaved"])
def test_decode_block_kernel_matches_kernel_per_step(tmp_path, rope):
    """Batch 8: the persistent decode-block kernel against the kernel-per-step
    path on the same inputs.  The projections split and sum their k-blocks the
    same way; RMSNorm-1 sums its squares in another order and the attention
    runs one key split instead of several, so values agree to within bf16
    rounding of the tensors the block stores."""
    res = _child_runs(tmp_path, rope, 8, {"block": {"LLAMA_DECODE_LAYER": "1"}, "steps": {}})
    a, b = res["block"], res["steps"]
    for t in range(2):
        for n in ("q", "k", "v", "y"):
            x, ref = a[f"{n}{t}"], b[f"{n}{t}"]
            rms = np.sqrt(np.mean(ref ** 2))
            d = np.abs(x - ref)
            assert np.sqrt(np.mean(d ** 2)) <= 2e-3 * rms and d.max() <= 3e-2 * rms, \
                f"step {t}: {n} rms {np.sqrt(np.mean(d ** 2)) / rms:.3g} max {d.max() / rms:.3g}"
