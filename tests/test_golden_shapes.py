"""The synthetic workloads and the oracle's constants against values the
pages print (CPU only).

Each fixture under ``tests/golden/`` holds numbers copied by hand from one
page, with the page title and section in its ``source`` field: the MLX
LLaMA-2-13B module listing and config ([MLX-13B] "LLaMA 2 的结构分析",
"模型配置"), the printed Phi-3-mini module tree ([HandsOn] 第三章) and the
LLaMAConfig defaults ([DeepDive] 二、LLaMA架构组件).  A workload shape that
drifts from the page it stands for (a wrong ffn width, a fused qkv width
that does not add up, the wrong eps or RoPE pairing) fails here.
"""

import inspect
import json
import os

import pytest

import synth
from oracle import quant as oq
from oracle import sampling as osm

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load(name):
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        g = json.load(f)
    assert g["source"].startswith("[")   # every fixture names its page
    return g


def test_llama13b_decode_workload_is_the_mlx_13b_block():
    g = load("mlx13b_block.json")
    w = synth.WORKLOADS["llama13b_decode"]
    assert w.dim == g["dim"] and w.n_heads == g["n_heads"]
    assert w.head_dim == g["rope_dims"]
    # wq / wk / wv all map dim -> dim: no grouped K/V heads in this model
    assert w.n_heads * w.head_dim == g["wq"][1]
    assert w.n_kv_heads * w.head_dim == g["wk"][1] == g["wv"][1]
    assert (w.n_heads * w.head_dim, w.dim) == tuple(g["wo"])
    assert (w.dim, w.ffn_dim) == tuple(g["w1"]) == tuple(g["w3"])
    assert (w.ffn_dim, w.dim) == tuple(g["w2"])
    assert w.eps == g["norm_eps"]
    # MLX's RoPE(traditional=True) rotates adjacent pairs
    assert g["rope_traditional"] and w.rope_style == "interleaved"


def test_quantiser_defaults_are_the_mlx_quantization_config():
    g = load("mlx13b_block.json")["quantization"]
    params = inspect.signature(oq.quantize).parameters
    assert params["group_size"].default == g["group_size"]
    assert params["bits"].default == g["bits"]


def test_phi3mini_model_workload_is_the_printed_module_tree():
    g = load("phi3mini_modules.json")
    w = synth.WORKLOADS["phi3mini_model"]
    assert (w.vocab, w.dim) == tuple(g["embed_tokens"]) and (w.dim, w.vocab) == tuple(g["lm_head"])
    assert w.n_layers == g["n_layers"]
    # one fused qkv_proj: q (n_heads) + k, v (n_kv_heads) heads of head_dim
    assert (w.n_heads + 2 * w.n_kv_heads) * w.head_dim == g["qkv_proj"][1] and w.dim == g["qkv_proj"][0]
    assert (w.n_heads * w.head_dim, w.dim) == tuple(g["o_proj"])
    # one fused gate_up_proj: gate rows then up rows, each ffn_dim wide
    assert (w.dim, 2 * w.ffn_dim) == tuple(g["gate_up_proj"])
    assert (w.ffn_dim, w.dim) == tuple(g["down_proj"])
    assert w.eps == g["rms_norm_eps"]
    assert w.fused
    assert 0 <= g["padding_idx"] < w.vocab


def test_llama7b_prefill_workload_is_the_deepdive_config():
    g = load("deepdive_config.json")
    w = synth.WORKLOADS["llama7b_prefill"]
    assert w.dim == g["hidden_size"] and w.ffn_dim == g["intermediate_size"]
    assert w.n_heads == g["num_attention_heads"] and w.n_kv_heads == g["num_kv_heads"]
    assert w.head_dim == g["hidden_size"] // g["num_attention_heads"]
    assert w.eps == g["rms_norm_eps"] and w.rope_theta == g["rope_theta"]
    # the prefill length stays inside the config's position range
    assert w.prefill_len <= g["max_position_embeddings"]


def test_sampling_oracle_runs_at_the_generate_defaults():
    g = load("deepdive_config.json")
    np = pytest.importorskip("numpy")
    rng = np.random.default_rng(5)
    logits = rng.standard_normal((4, 64)) * 2.0
    u = rng.uniform(size=4)
    ids = osm.sample_top_p(logits, g["generate_temperature"], g["generate_top_p"], u)
    kept = [set(osm.nucleus(logits[b], g["generate_temperature"], g["generate_top_p"])[0].tolist())
            for b in range(4)]
    assert all(int(ids[b]) in kept[b] for b in range(4))
