"""GPU test of llama_attention_decode_noalloc, the allocation-free decode attention.

Some callers cannot allocate device memory (a plug-in inside a serving
framework that reserved all GPU memory for its own pool and passes no
workspace, or a latency-critical loop that must not call cudaMalloc).  For
them the library offers the split-KV decode attention with its partial
results in a fixed array inside the library.  This test calls it through the
C ABI and checks its output against the attention output that the existing
entry point, llama_layer_decode, leaves in its workspace -- on two calls in a
row, each after a fresh decode step (so the second call reuses the array the
first one filled, at a different length).  The file is named so that pytest
collects it last; it does not depend on any other test.
"""

import numpy as np
import pytest

import llama_decoder_only_b200 as L
import synth
from tests.harness import LayerRun, rel_errors

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

TOL = 1e-2   # max-abs / RMS, the bf16 bar of the parity tests


@pytest.mark.parametrize("case", [
    # name, dim, nh, nkv, hd, ffn, B, T0
    ("gqa4_hd128", 1024, 16, 4, 128, 2816, 6, 700),
    ("mha_hd96", 384, 4, 4, 96, 1024, 8, 333),
])
def test_noalloc_matches_layer_decode_attention(case):
    name, dim, nh, nkv, hd, ffn, B, T0 = case
    w = synth.Workload(name, dim, nh, nkv, hd, ffn, 1e-5, 1e4, "half", "bf16", 0.02, 123,
                       cache_len=T0, decode_batch=B, decode_steps=2)
    inp = synth.decode_inputs(w)
    run = LayerRun(w, inp.weights, B, T0 + 4, 1, k0=inp.k_cache, v0=inp.v_cache)
    qkvn = (nh + 2 * nkv) * hd
    off_qkv, _, off_attn, _ = L.workspace_offsets(run.dims, B, 1)
    out = torch.empty(B, nh * hd, dtype=torch.bfloat16, device="cuda")
    for call, xs in enumerate(inp.steps):
        run.step(xs)                                   # existing entry point: llama_layer_decode
        T = run.cache.length
        q = run.ws[off_qkv:off_qkv + B * qkvn * 2].view(torch.bfloat16)
        ref = run.ws[off_attn:off_attn + B * nh * hd * 2].view(torch.bfloat16).reshape(B, nh * hd)
        out.fill_(float("nan"))
        L.attention_decode_noalloc(run.dims, B, q, qkvn, run.cache.k, run.cache.v, run.cache.capacity, T, out)
        torch.cuda.synchronize()
        got = out.double().cpu().numpy()
        want = ref.double().cpu().numpy()
        assert np.all(np.isfinite(got)), f"call {call}: non-finite output"
        mx, rms = rel_errors(got, want)
        print(f"[noalloc] {name} call {call} (length {T}): max/RMS {mx:.3g} rms {rms:.3g}")
        assert mx <= TOL, f"call {call}: max-abs/RMS {mx:.3g}"


def test_noalloc_rejects_beyond_its_scratch():
    d = L.make_dims(8192, 64, 8, 128, 28672, 1e-5, 1e4, "half", "bf16")
    t = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    # 1024 sequences x 64 heads x 130 floats x 2 splits x 4 bytes = 68 MB > 8 MiB
    with pytest.raises(L.LlamaError) as e:
        L.attention_decode_noalloc(d, 1024, t, 64 * 128, t, t, 4096, 100, t)
    assert e.value.status == 8
