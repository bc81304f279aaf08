"""GPU tests of llama_attention_decode_noalloc, the allocation-free decode attention.

Some callers cannot allocate device memory (a plug-in inside a serving
framework that reserved all GPU memory for its own pool and passes no
workspace, or a latency-critical loop that must not call cudaMalloc).  For
them the library offers the split-KV decode attention with its partial
results in a fixed array inside the library.

* The entry point is called through the C ABI on seeded synthetic q and K/V
  caches and compared with the fp64 oracle's causal GQA attention on the same
  values (the query is the newest position, so every cached key is visible),
  at the bar the other attention checks use: error against the exact oracle
  within 1.5x (RMS) / 2x (max-abs) of the bf16 floor (the oracle with bf16
  probabilities and a bf16 output) and RMS error <= 1e-2 x RMS.  Two calls in
  a row per case: the second reuses the array the first one filled.
* Cases cover the CUDA-core kernel (head_dim 96 and 64) and the tensor-core
  kernel (GQA groups 4 and 8, head_dim 128), a single key split (length <= 32,
  and <= 64 on the tensor-core kernel), and a batch whose two splits fill the
  8 MiB array to its last 0.05 %.  The split-count clamp of the fixed array
  never binds below the heuristic's own count for supported shapes (the
  heuristic needs at most group x (hd + 2) x 4 x 1184 bytes per KV head pair,
  under 5 MB), so the clamp is exercised only at its lower end of two splits.
* As an extra, the output is compared with the attention output that the
  existing entry point, llama_layer_decode, leaves in its workspace.

The file is named so that pytest collects it last; it depends on no other test.
"""

import math

import numpy as np
import pytest

import llama_decoder_only_b200 as L
import synth
from oracle import block as ob
from tests.harness import LayerRun, floor_ratios, rel_errors

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

TOL = 1e-2          # max-abs / RMS against the layer call's own attention (same kernels)
EXACT_RMS = 1e-2    # RMS error / RMS against the exact oracle
FLOOR_RMS = 1.5
FLOOR_MAX = 2.0
SCRATCH_BYTES = 8 << 20

CASES = [
    # name, nh, nkv, hd, batch, (length of call 1, length of call 2), capacity
    ("gqa4_hd128_mma", 16, 4, 128, 6, (700, 1701), 1800),
    ("gqa8_hd128_mma_short", 64, 8, 128, 4, (1500, 61), 1600),
    ("mha_hd96_cuda_core", 4, 4, 96, 8, (333, 334), 400),
    ("mha_hd64_single_split", 8, 8, 64, 3, (20, 64), 80),
    ("gqa8_hd128_full_scratch", 64, 8, 128, 126, (300, 301), 320),
]


def _inputs(case, seed):
    name, nh, nkv, hd, B, lengths, cap = case
    rng = np.random.default_rng(seed)
    q = synth.bf16_round(rng.standard_normal((B, nh * hd), dtype=np.float32))
    k = synth.bf16_round(rng.standard_normal((B, nkv, cap, hd), dtype=np.float32))
    v = synth.bf16_round(rng.standard_normal((B, nkv, cap, hd), dtype=np.float32))
    return q, k, v


def _oracle(q, k, v, T, nh, nkv, hd, bf16):
    """[B, nh*hd]: causal GQA attention of a query at position T-1 over keys 0..T-1."""
    rnd = ob.to_bf16 if bf16 else (lambda a: a)
    B = q.shape[0]
    out = np.empty((B, nh * hd))
    for b in range(B):
        kb = np.transpose(k[b, :, :T], (1, 0, 2)).astype(np.float64)
        vb = np.transpose(v[b, :, :T], (1, 0, 2)).astype(np.float64)
        o = ob.causal_gqa_attention(q[b].reshape(1, nh, hd), kb, vb, np.array([T - 1]), nh // nkv,
                                    round_p=rnd)
        out[b] = rnd(o).reshape(nh * hd)
    return out


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_noalloc_matches_oracle(case):
    name, nh, nkv, hd, B, lengths, cap = case
    if name.endswith("full_scratch"):
        used = B * nh * (hd + 2) * 4 * 2
        assert SCRATCH_BYTES - 8192 < used <= SCRATCH_BYTES, used
    q, k, v = _inputs(case, seed=500 + nh + B)
    dims = L.make_dims(nh * hd, nh, nkv, hd, 4 * nh * hd, 1e-5, 1e4, "half", "bf16")
    qd = torch.from_numpy(q).to(torch.bfloat16).cuda()
    kd = torch.from_numpy(k).to(torch.bfloat16).cuda()
    vd = torch.from_numpy(v).to(torch.bfloat16).cuda()
    out = torch.empty(B, nh * hd, dtype=torch.bfloat16, device="cuda")
    for call, T in enumerate(lengths):
        out.fill_(float("nan"))
        L.attention_decode_noalloc(dims, B, qd, nh * hd, kd, vd, cap, T, out)
        torch.cuda.synchronize()
        got = out.double().cpu().numpy()
        assert np.all(np.isfinite(got)), f"{name} call {call}: non-finite output"
        ye = _oracle(q, k, v, T, nh, nkv, hd, bf16=False)
        yb = _oracle(q, k, v, T, nh, nkv, hd, bf16=True)
        mx, rms = rel_errors(got, ye)
        r_rms, r_max = floor_ratios(got, yb, ye)
        print(f"[noalloc] {name} call {call} (length {T}): vs exact max/RMS {mx:.3g} rms {rms:.3g}; "
              f"ratio to bf16 floor rms {r_rms:.2f} max {r_max:.2f}")
        assert rms <= EXACT_RMS, f"{name} call {call}: rms/RMS {rms:.3g}"
        assert r_rms <= FLOOR_RMS and r_max <= FLOOR_MAX, f"{name} call {call}: floor ratios {r_rms:.3g} {r_max:.3g}"


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
        print(f"[noalloc] {name} call {call} (length {T}) vs llama_layer_decode: max/RMS {mx:.3g} rms {rms:.3g}")
        assert mx <= TOL, f"call {call}: max-abs/RMS {mx:.3g}"


def test_noalloc_rejects_beyond_its_scratch():
    d = L.make_dims(8192, 64, 8, 128, 28672, 1e-5, 1e4, "half", "bf16")
    t = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    # 1024 sequences x 64 heads x 130 floats x 2 splits x 4 bytes = 68 MB > 8 MiB
    with pytest.raises(L.LlamaError) as e:
        L.attention_decode_noalloc(d, 1024, t, 64 * 128, t, t, 4096, 100, t)
    assert e.value.status == 8
    # one sequence past the largest batch whose two splits fit: 127 x 64 x 130 x 4 x 2 > 8 MiB
    assert 127 * 64 * 130 * 4 * 2 > SCRATCH_BYTES >= 126 * 64 * 130 * 4 * 2
    with pytest.raises(L.LlamaError) as e:
        L.attention_decode_noalloc(d, 127, t, 64 * 128, t, t, 4096, 100, t)
    assert e.value.status == 8
