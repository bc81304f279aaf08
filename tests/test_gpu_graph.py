"""GPU test: a decode step captured in a CUDA graph replays exactly.

A serving loop captures its decode step once and replays it.  The library
enqueues only kernels (no host synchronisation, no allocation) and every
launch leaves the workspace's flag words as it found them, so a captured
layer decode at cache length P, replayed after the cache is reset to P, must
give the eager step's output bit for bit -- on every replay.
"""

import numpy as np
import pytest

import llama_decoder_only_b200 as L
import synth
from synth import device as sd

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def test_decode_step_replays_from_a_cuda_graph():
    w = synth.Workload("graph_gqa", 512, 8, 2, 64, 1376, 1e-5, 1e4, "half", "bf16", 0.02, 31,
                       batch=2, prefill_len=100)
    dims = L.make_dims(w.dim, w.n_heads, w.n_kv_heads, w.head_dim, w.ffn_dim, w.eps, w.rope_theta,
                       w.rope_style, w.dtype)
    inp = synth.prefill_inputs(w, with_steps=False)
    dev = sd.upload_layer(inp.weights, w.dtype)   # keeps the device weights alive
    lw = L.layer_weights(dev)
    B, P = w.batch, w.prefill_len
    cache = L.KVCache(dims, B, 256)
    ws = torch.zeros(L.workspace_size(dims, B, P), dtype=torch.uint8, device="cuda")
    x = torch.from_numpy(np.ascontiguousarray(inp.x)).cuda().reshape(B * P, w.dim)
    y = torch.empty_like(x)
    L.layer_prefill(dims, lw, cache, B, P, x, y, ws)
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    xd = torch.randn(B, w.dim, generator=g, device="cuda")

    eager = torch.empty_like(xd)
    cache.set_length(P)
    L.layer_decode(dims, lw, cache, B, xd, eager, ws)
    torch.cuda.synchronize()

    out = torch.full_like(xd, float("nan"))
    graph = torch.cuda.CUDAGraph()
    cache.set_length(P)
    with torch.cuda.graph(graph):
        L.layer_decode(dims, lw, cache, B, xd, out, ws)   # enqueued on the capture stream
    for _ in range(2):
        out.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        assert L.device_status(ws) == 0
        assert torch.equal(out, eager)
