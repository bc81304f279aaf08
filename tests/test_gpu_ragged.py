"""GPU parity of ragged batches (llama_layer_forward_ragged) against the fp64
oracle's ``layer_forward_ragged``: every sequence keeps its own cache length
and brings its own number of new tokens; decode rows and prefill chunks mix in
one call ([MLX-13B] KV 缓存实现片段 keeps one offset for the batch; [HandsOn]
第三章: prefill and token-by-token decode are the same block).

Each call's output (packed rows) is compared per sequence with the oracle
run on that sequence alone, at the bars of the uniform bf16 parity tests:
max-abs / RMS <= 1e-2 against the oracle with bf16 rounding of the stored
tensors, RMS error <= 1e-2 and max-abs <= 5e-2 against the exact oracle.
"""

import numpy as np
import pytest

import llama_decoder_only_b200 as L
import synth
from oracle import block as ob
from synth import device as sd
from tests.harness import oracle_dims, rel_errors

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

CASES = [
    # name, dim, nh, nkv, hd, ffn, rope, initial lengths, then calls of new tokens per sequence
    ("mixed_gqa4_hd64", 512, 8, 2, 64, 1376, "half", [0, 37, 300, 5],
     [[130, 1, 1, 257], [1, 1, 40, 1], [1, 1, 1, 1]]),
    ("decode_only_mha_hd128", 768, 6, 6, 128, 2048, "interleaved", [513, 2, 129, 64, 1000],
     [[1, 1, 1, 1, 1], [1, 1, 1, 1, 1]]),
    ("decode_only_gqa8_hd128", 1024, 16, 2, 128, 2816, "half", [700, 3, 1500],
     [[1, 1, 1], [1, 1, 1]]),
    ("mixed_hd96_many_rows", 384, 4, 4, 96, 1024, "half", [0, 0, 17],
     [[300, 1, 129], [1, 200, 1]]),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_ragged_matches_oracle_per_sequence(case):
    name, dim, nh, nkv, hd, ffn, rope, lens0, calls = case
    B = len(lens0)
    w = synth.Workload(name, dim, nh, nkv, hd, ffn, 1e-5, 1e4, rope, "bf16", 0.02, 411)
    rng = np.random.default_rng(412)
    W = synth.layer_weights(w, rng)
    cap = max(l0 + sum(c[b] for c in calls) for b, l0 in enumerate(lens0)) + 8
    # synthetic cache contents for the initial lengths, N(0, 1), bf16 values
    k0 = synth.bf16_round(rng.standard_normal((B, nkv, cap, hd), dtype=np.float32))
    v0 = synth.bf16_round(rng.standard_normal((B, nkv, cap, hd), dtype=np.float32))
    dims = L.make_dims(dim, nh, nkv, hd, ffn, w.eps, w.rope_theta, rope, "bf16")
    dev = sd.upload_layer(W, "bf16")
    lw = L.layer_weights(dev)
    cache = L.KVCache(dims, B, cap, k=torch.from_numpy(k0).to(torch.bfloat16).cuda(),
                      v=torch.from_numpy(v0).to(torch.bfloat16).cuda())
    cache.set_lengths(lens0)
    assert cache.lengths == lens0
    d = oracle_dims(w)
    ce = [ob.KVCache(1, nkv, hd, cap, k0[b:b + 1, :, :l0].astype(np.float64),
                     v0[b:b + 1, :, :l0].astype(np.float64)) for b, l0 in enumerate(lens0)]
    cb = [ob.KVCache(1, nkv, hd, cap, k0[b:b + 1, :, :l0].astype(np.float64),
                     v0[b:b + 1, :, :l0].astype(np.float64)) for b, l0 in enumerate(lens0)]
    lens = list(lens0)
    for call, n_new in enumerate(calls):
        xs = [rng.standard_normal((n, dim), dtype=np.float32) for n in n_new]
        M = sum(n_new)
        xi = torch.from_numpy(np.concatenate(xs)).cuda()
        xo = torch.empty_like(xi)
        ws = torch.zeros(L.workspace_size_ragged(dims, B, M), dtype=torch.uint8, device="cuda")
        L.layer_forward_ragged(dims, lw, cache, n_new, xi, xo, ws)
        torch.cuda.synchronize()
        assert L.device_status(ws) == 0
        lens = [l + n for l, n in zip(lens, n_new)]
        assert cache.lengths == lens
        y = xo.double().cpu().numpy()
        ye = ob.layer_forward_ragged(d, W, xs, ce)
        yb = ob.layer_forward_ragged(d, W, xs, cb, rounding="bf16")
        r0 = 0
        for b, n in enumerate(n_new):
            yb_, ye_ = yb[b], ye[b]
            mx, _ = rel_errors(y[r0:r0 + n], yb_)
            mxe, rmse = rel_errors(y[r0:r0 + n], ye_)
            print(f"[ragged] {name} call {call} seq {b} ({n} new at {lens[b] - n}): vs bf16-oracle max {mx:.3g}; "
                  f"vs exact max {mxe:.3g} rms {rmse:.3g}")
            assert mx <= 1e-2 and rmse <= 1e-2 and mxe <= 5e-2, f"{name} call {call} seq {b}"
            r0 += n


def test_uniform_calls_refuse_a_ragged_cache_and_equal_lengths_are_uniform():
    dims = L.make_dims(512, 8, 2, 64, 1376, 1e-5, 1e4, "half", "bf16")
    cache = L.KVCache(dims, 2, 16)
    cache.set_lengths([3, 5])
    assert cache.length == -2 and cache.lengths == [3, 5]
    w = synth.Workload("r", 512, 8, 2, 64, 1376, 1e-5, 1e4, "half", "bf16", 0.02, 1)
    lw = L.layer_weights(sd.upload_layer(synth.layer_weights(w), "bf16"))
    x = torch.zeros(2, 512, device="cuda")
    y = torch.empty_like(x)
    ws = torch.zeros(L.workspace_size(dims, 2, 1), dtype=torch.uint8, device="cuda")
    with pytest.raises(L.LlamaError) as e:
        L.layer_decode(dims, lw, cache, 2, x, y, ws)
    assert e.value.status == 1
    cache.set_lengths([4, 4])
    assert cache.length == 4
    with pytest.raises(L.LlamaError) as e:
        cache.set_lengths([4, 17])
    assert e.value.status == 3
