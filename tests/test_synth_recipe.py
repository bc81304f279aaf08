"""CPU tests of the seeded input recipe in ``synth`` (shared by the oracle
side and the CUDA side).

They pin what the recipe states, on shrunken shapes: the draws are
deterministic per seed and in the stated order, bf16 workloads hold values
rounded to nearest-even bf16 (checked against torch's own conversion), norm
weights are ones except for the tiny fp32 workload, every weight has the
shape the block expects, and a fused qkv / gate_up weight is one draw whose
row blocks are the q, k, v (gate, up) weights.
"""

import numpy as np
import pytest

import synth

torch = pytest.importorskip("torch")


def small(name, **kw):
    w = synth.WORKLOADS[name]
    base = dict(dim=256, n_heads=4, n_kv_heads=2 if w.n_kv_heads < w.n_heads else 4, head_dim=64,
                ffn_dim=512, prefill_len=32, cache_len=48 if w.cache_len else 0, decode_steps=3)
    base.update(kw)
    return synth.shrink(w, **base)


def test_bf16_round_is_torch_round_to_nearest_even():
    rng = np.random.default_rng(0)
    a = np.concatenate([rng.standard_normal(4096).astype(np.float32) * 3,
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 0.0, -0.0],
                                 np.float32)])
    ref = torch.from_numpy(a).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(synth.bf16_round(a), ref)
    # the two ties above go to the even neighbour
    assert synth.bf16_round(np.float32(1.0 + 2 ** -8)) == np.float32(1.0)
    assert synth.bf16_round(np.float32(1.0 + 3 * 2 ** -8)) == np.float32(1.0 + 2 ** -6)


@pytest.mark.parametrize("name", ["llama7b_prefill", "llama13b_decode", "gqa70b", "phi3mini_model", "tiny_fp32"])
def test_layer_weights_shapes_dtype_and_norms(name):
    w = small(name)
    W = synth.layer_weights(w)
    nh, nkv, hd, d, f = w.n_heads, w.n_kv_heads, w.head_dim, w.dim, w.ffn_dim
    assert W["wq"].shape == (nh * hd, d) and W["wk"].shape == (nkv * hd, d) and W["wv"].shape == (nkv * hd, d)
    assert W["wo"].shape == (d, nh * hd) and W["w1"].shape == (f, d) and W["w3"].shape == (f, d)
    assert W["w2"].shape == (d, f)
    for k in ("wq", "wk", "wv", "wo", "w1", "w3", "w2"):
        assert W[k].dtype == np.float32
        if w.dtype == "bf16":
            assert np.array_equal(synth.bf16_round(W[k]), W[k]), k   # already on the bf16 grid
    if name == "tiny_fp32":
        for k in ("attn_norm", "ffn_norm"):
            assert 0.0 < np.std(W[k] - 1.0) < 0.05 and not np.all(W[k] == 1.0)
    else:
        assert np.all(W["attn_norm"] == 1.0) and np.all(W["ffn_norm"] == 1.0)
    # weight scale is the workload's std (loose: a few thousand draws)
    assert abs(np.std(W["wo"]) / w.w_std - 1.0) < 0.1


def test_draws_are_deterministic_and_seed_dependent():
    w = small("llama7b_prefill")
    a, b = synth.prefill_inputs(w), synth.prefill_inputs(w)
    assert np.array_equal(a.x, b.x) and all(np.array_equal(a.weights[k], b.weights[k]) for k in a.weights)
    c = synth.prefill_inputs(synth.shrink(w, seed=w.seed + 1))
    assert not np.array_equal(a.x, c.x)


def test_draw_order_weights_then_input_then_steps():
    # the input x is the next draw after the layer's weights from the same stream
    w = small("tiny_fp32")
    rng = np.random.default_rng(w.seed)
    synth.layer_weights(w, rng)
    x = rng.standard_normal((w.batch, w.prefill_len, w.dim), dtype=np.float32)
    s0 = rng.standard_normal((w.batch, 1, w.dim), dtype=np.float32)
    inp = synth.prefill_inputs(w)
    assert np.array_equal(inp.x, x) and np.array_equal(inp.steps[0], s0)


def test_decode_inputs_cache_layout_and_order():
    w = small("llama13b_decode")
    inp = synth.decode_inputs(w)
    shape = (w.decode_batch, w.n_kv_heads, w.cache_len, w.head_dim)
    assert inp.k_cache.shape == shape and inp.v_cache.shape == shape
    assert np.array_equal(synth.bf16_round(inp.k_cache), inp.k_cache)
    rng = np.random.default_rng(w.seed)
    synth.layer_weights(w, rng)
    k = synth.bf16_round(rng.standard_normal(shape, dtype=np.float32))
    assert np.array_equal(inp.k_cache, k)          # the K cache is the first draw after the weights
    assert len(inp.steps) == w.decode_steps and inp.steps[0].shape == (w.decode_batch, 1, w.dim)


def test_fused_weights_are_one_draw_split_by_rows():
    w = small("phi3mini_model")
    W = synth.layer_weights(w)
    nq, nk = w.n_heads * w.head_dim, w.n_kv_heads * w.head_dim
    assert np.array_equal(W["qkv"][:nq], W["wq"]) and np.array_equal(W["qkv"][nq:nq + nk], W["wk"])
    assert np.array_equal(W["qkv"][nq + nk:], W["wv"])
    assert np.array_equal(W["gate_up"][:w.ffn_dim], W["w1"]) and np.array_equal(W["gate_up"][w.ffn_dim:], W["w3"])
