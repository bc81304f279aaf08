"""Seeded synthetic inputs shared by the oracle side and the CUDA side.

This module holds NO arithmetic of the decoder block: only workload shapes,
seeded random draws and the storage-format conversion of those draws
(float32 -> bfloat16 bit patterns, round-to-nearest-even).  Both the oracle
tests and the GPU harness read the same arrays from here.

Recipe (every workload): NumPy ``default_rng(seed)``, ``standard_normal``
in float32 times the stated std, then rounded to bfloat16 for the bf16
workloads.  Draw order per layer: attn_norm, wq, wk, wv, wo, ffn_norm, w1,
w3, w2 (a fused qkv / gate_up weight is one draw); then the prefill input
(or tokens), then the K cache and V cache, then the decode inputs step by
step.  Norm weights are ones, except the tiny fp32 workload, whose norm
weights are 1 + N(0, 0.01).  The residual stream (x) is always float32.
"""

from __future__ import annotations

from dataclasses import dataclass, field, replace

import numpy as np

__all__ = ["Workload", "WORKLOADS", "bf16_bits", "bf16_round", "bits_to_f32",
           "layer_weights", "LayerInputs", "prefill_inputs", "decode_inputs",
           "model_weights", "model_tokens", "shrink"]


@dataclass(frozen=True)
class Workload:
    name: str
    dim: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    ffn_dim: int
    eps: float
    rope_theta: float
    rope_style: str          # "half" | "interleaved"
    dtype: str               # "f32" | "bf16"
    w_std: float
    seed: int
    batch: int = 1
    prefill_len: int = 0     # tokens per sequence in the prefill call
    cache_len: int = 0       # synthetic pre-filled cache length (decode workloads)
    decode_batch: int = 0
    decode_steps: int = 0
    fused: bool = False      # qkv and gate_up drawn as one matrix each
    vocab: int = 0
    n_layers: int = 1
    norm_std: float = 0.0    # norm weight = 1 + N(0, norm_std); 0 -> ones
    extra: dict = field(default_factory=dict)

    @property
    def qkv_n(self):
        return (self.n_heads + 2 * self.n_kv_heads) * self.head_dim


WORKLOADS = {
    # tiny single layer, fp32, GQA 8/2, prefill 64 then 16 decode steps
    "tiny_fp32": Workload("tiny_fp32", 256, 8, 2, 32, 688, 1e-5, 1e4, "half", "f32",
                          0.02, 1001, batch=1, prefill_len=64, decode_batch=1,
                          decode_steps=16, norm_std=0.01),
    # LLaMA-2-7B-shaped layer, bf16, causal prefill 1 x 2048
    "llama7b_prefill": Workload("llama7b_prefill", 4096, 32, 32, 128, 11008, 1e-6, 1e4,
                                "half", "bf16", 0.02, 1002, batch=1, prefill_len=2048),
    # LLaMA-2-13B-shaped layer, bf16, interleaved RoPE, decode batch 16 on a 4096 cache
    "llama13b_decode": Workload("llama13b_decode", 5120, 40, 40, 128, 13824, 1e-5, 1e4,
                                "interleaved", "bf16", 0.02, 1003, cache_len=4096,
                                decode_batch=16, decode_steps=128),
    # 70B-shaped GQA (64/8) layer: prefill 2 x 4096, then decode batch 64 on a 4096 cache
    "gqa70b": Workload("gqa70b", 8192, 64, 8, 128, 28672, 1e-5, 1e4, "half", "bf16",
                       0.015, 1004, batch=2, prefill_len=4096, cache_len=4096,
                       decode_batch=64, decode_steps=128),
    # Phi-3-mini-shaped model: 32 layers, fused qkv / gate_up, vocab 32064
    "phi3mini_model": Workload("phi3mini_model", 3072, 32, 32, 96, 8192, 1e-5, 1e4, "half",
                               "bf16", 0.02, 1005, batch=8, prefill_len=512,
                               decode_batch=8, decode_steps=128, fused=True,
                               vocab=32064, n_layers=32),
}


def shrink(w: Workload, **kw) -> Workload:
    """A copy of ``w`` with some fields replaced (smaller parity cases)."""
    return replace(w, **kw)


# ---------------------------------------------------------------- storage format

def bf16_bits(a):
    """float32 -> bfloat16 bit patterns (uint16), round to nearest, ties to even."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    bias = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + bias) >> 16).astype(np.uint16)


def bits_to_f32(b):
    """bfloat16 bit patterns -> the float32 values they hold (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def bf16_round(a):
    """float32 values rounded to the nearest bfloat16 value, kept as float32."""
    return bits_to_f32(bf16_bits(a))


def _normal(rng, shape, std):
    return rng.standard_normal(shape, dtype=np.float32) * np.float32(std)


def _store(w: Workload, a):
    return bf16_round(a) if w.dtype == "bf16" else a


# ---------------------------------------------------------------- layer weights

def _one_layer(w: Workload, rng):
    d, nh, nkv, hd, f = w.dim, w.n_heads, w.n_kv_heads, w.head_dim, w.ffn_dim

    def norm():
        if w.norm_std:
            return (1.0 + _normal(rng, (d,), w.norm_std)).astype(np.float32)
        return np.ones((d,), dtype=np.float32)

    out = {"attn_norm": norm()}
    if w.fused:
        qkv = _store(w, _normal(rng, (w.qkv_n, d), w.w_std))
        out["wq"] = qkv[: nh * hd]
        out["wk"] = qkv[nh * hd: (nh + nkv) * hd]
        out["wv"] = qkv[(nh + nkv) * hd:]
        out["qkv"] = qkv
    else:
        out["wq"] = _store(w, _normal(rng, (nh * hd, d), w.w_std))
        out["wk"] = _store(w, _normal(rng, (nkv * hd, d), w.w_std))
        out["wv"] = _store(w, _normal(rng, (nkv * hd, d), w.w_std))
    out["wo"] = _store(w, _normal(rng, (d, nh * hd), w.w_std))
    out["ffn_norm"] = norm()
    if w.fused:
        gu = _store(w, _normal(rng, (2 * f, d), w.w_std))
        out["w1"], out["w3"], out["gate_up"] = gu[:f], gu[f:], gu
    else:
        out["w1"] = _store(w, _normal(rng, (f, d), w.w_std))
        out["w3"] = _store(w, _normal(rng, (f, d), w.w_std))
    out["w2"] = _store(w, _normal(rng, (d, f), w.w_std))
    return out


def layer_weights(w: Workload, rng=None):
    """One layer's weights (float32 arrays holding bf16 values for bf16 workloads)."""
    rng = rng if rng is not None else np.random.default_rng(w.seed)
    return _one_layer(w, rng)


@dataclass
class LayerInputs:
    weights: dict
    x: np.ndarray | None = None          # [B, L, dim] float32
    k_cache: np.ndarray | None = None    # [B, nkv, cache_len, hd]
    v_cache: np.ndarray | None = None
    steps: list = field(default_factory=list)   # decode inputs, each [B, 1, dim]


def prefill_inputs(w: Workload, with_steps=True) -> LayerInputs:
    """Weights and the prefill input ``x ~ N(0, 1)`` of shape ``[batch, prefill_len, dim]``.

    For a workload that decodes after its own prefill (no synthetic cache),
    the ``decode_steps`` follow-up rows ``[batch, 1, dim]`` come next in the
    same stream.
    """
    rng = np.random.default_rng(w.seed)
    W = _one_layer(w, rng)
    x = rng.standard_normal((w.batch, w.prefill_len, w.dim), dtype=np.float32)
    steps = []
    if with_steps and w.cache_len == 0:
        steps = [rng.standard_normal((w.batch, 1, w.dim), dtype=np.float32)
                 for _ in range(w.decode_steps)]
    return LayerInputs(W, x=x, steps=steps)


def decode_inputs(w: Workload, steps=None, batch=None, cache_len=None) -> LayerInputs:
    """Weights, a synthetic N(0, 1) cache and N(0, 1) decode rows.

    The cache holds ``cache_len`` positions per sequence (already in the
    stored dtype).  ``steps`` decode inputs of shape ``[batch, 1, dim]``.
    """
    rng = np.random.default_rng(w.seed)
    W = _one_layer(w, rng)
    B = batch if batch is not None else w.decode_batch
    T = cache_len if cache_len is not None else w.cache_len
    shape = (B, w.n_kv_heads, T, w.head_dim)
    k = _store(w, rng.standard_normal(shape, dtype=np.float32))
    v = _store(w, rng.standard_normal(shape, dtype=np.float32))
    n = w.decode_steps if steps is None else steps
    xs = [rng.standard_normal((B, 1, w.dim), dtype=np.float32) for _ in range(n)]
    return LayerInputs(W, k_cache=k, v_cache=v, steps=xs)


# ---------------------------------------------------------------- whole model

def model_weights(w: Workload, n_layers=None):
    """Embedding, layers, final norm and lm_head (bf16 values, float32 arrays)."""
    rng = np.random.default_rng(w.seed)
    E = _store(w, _normal(rng, (w.vocab, w.dim), w.w_std))
    layers = [_one_layer(w, rng) for _ in range(n_layers or w.n_layers)]
    final = np.ones((w.dim,), dtype=np.float32)
    lm = _store(w, _normal(rng, (w.vocab, w.dim), w.w_std))
    return {"embed": E, "layers": layers, "final_norm": final, "lm_head": lm}


def model_tokens(w: Workload, batch=None, prefill_len=None, steps=None):
    """Uniform token ids: the prompt ``[B, L]`` and the teacher-forced ids per step ``[B]``."""
    rng = np.random.default_rng(w.seed + 100000)
    B = batch or w.batch
    L = prefill_len or w.prefill_len
    n = w.decode_steps if steps is None else steps
    prompt = rng.integers(0, w.vocab, size=(B, L), dtype=np.int32)
    forced = [rng.integers(0, w.vocab, size=(B,), dtype=np.int32) for _ in range(n)]
    return prompt, forced
