"""fp64 NumPy oracle of the LLaMA-style pre-norm decoder block (test infrastructure).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU-baseline legs, never by the product path.  It shares no
code with the CUDA library.

Every function states the passage it follows.  Pages are cited by title:

* [MLX-13B]  "iOS设备上运行LLaMA2-13B：基于苹果MLX框架的完整技术指南" (geoz.com.cn)
* [DeepDive] "LLaMA架构深度解析：从开源大模型设计到高效推理的工程实现全流程"
             (Tencent Cloud), section 二 "LLaMA架构组件"
* [Decoder]  "老码农和你一起学AI系列：关于LLaMA解码器" (jsqmd.com)
* [HandsOn]  "《Hands-On Large Language Models》阅读笔记(二)" (yanbin.blog)

Arithmetic is IEEE float64 throughout.  The optional ``rounding="bf16"`` mode
rounds (round-to-nearest-even, 8 significant bits) exactly the tensors that a
"bf16 weights/activations, fp32 accumulate" block stores in bf16 -- the norm
outputs, the q/k/v projection outputs, q/k after RoPE (hence the cache
entries), the attention probabilities (DeepDive, class LLaMAAttention: the
fp32 softmax is cast back to the activation dtype), the attention output and
the SwiGLU product -- and nothing else; the residual stream stays unrounded.
It exists to measure the rounding floor a bf16 implementation cannot go
below; ``rounding=None`` (the default) is the exact definition.

Readings where the pages are silent or garbled (each also listed in the
design notes):

* interleaved ("traditional") RoPE, named in [MLX-13B] "LLaMA 2 的结构分析"
  (``RoPE(128, traditional=True)``) but never defined: adjacent pairs
  ``(x[2i], x[2i+1])`` rotate by ``p * theta**(-2i/hd)`` -- the same frequency
  ladder as the rotate-half form, applied to adjacent pairs.
* positions of appended tokens start at the cache length ([MLX-13B] KV 缓存
  实现片段: ``offset=key_cache.shape[2]``); cached keys are stored after RoPE.
* GQA maps query head ``h`` to KV head ``h // n_rep`` ([DeepDive]
  LLaMAAttention: ``unsqueeze(2).expand(...).reshape``).
* the causal mask excludes key ``j`` from query position ``p`` iff ``j > p``
  ([MLX-13B] 5. 因果掩码: the code ``indices[:, None] < indices[None]`` masks
  the strict upper triangle; its comment's "lower triangular" is wrong).
* argmax ties resolve to the lowest index.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

__all__ = [
    "Dims", "to_bf16", "rms_norm", "rope_inv_freq", "rope_rotate_half",
    "rope_interleaved", "apply_rope", "silu", "causal_gqa_attention",
    "KVCache", "layer_forward", "final_logits", "greedy_argmax",
    "model_forward", "embed",
]


@dataclass(frozen=True)
class Dims:
    """Layer hyper-parameters ([MLX-13B] 模型配置 config.json; [DeepDive] LLaMAConfig)."""

    dim: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    ffn_dim: int
    eps: float
    rope_theta: float = 10000.0
    rope_style: str = "half"  # "half" (DeepDive LLaMARoPE) or "interleaved"

    @property
    def n_rep(self) -> int:
        assert self.n_heads % self.n_kv_heads == 0
        return self.n_heads // self.n_kv_heads


def to_bf16(a):
    """Round float64 values to the nearest bfloat16 value (ties to even).

    bfloat16 keeps 8 significant bits: ``x = m * 2**e`` with ``m`` in
    [0.5, 1) is rounded to ``rint(m * 2**8) * 2**(e-8)`` (``rint`` rounds half
    to even).  Exact in float64 for every finite input in the normal range.
    """
    a = np.asarray(a, dtype=np.float64)
    m, e = np.frexp(a)
    return np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)


def _identity(a):
    return a


def rms_norm(x, g, eps):
    """RMSNorm over the last axis: ``g * x / sqrt(mean(x**2) + eps)``.

    [MLX-13B] 4. RMSNorm (``x * rsqrt(mean(x**2) + eps)``); [DeepDive]
    class LLaMARMSNorm (the weight multiplies the normalised x).
    """
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return np.asarray(g, dtype=np.float64) * (x / np.sqrt(ms + eps))


def rope_inv_freq(head_dim, theta):
    """``theta ** (-2i / head_dim)`` for i = 0 .. head_dim/2 - 1 ([DeepDive] LLaMARoPE)."""
    i2 = np.arange(0, head_dim, 2, dtype=np.float64)
    return 1.0 / (float(theta) ** (i2 / head_dim))


def _angles(pos, head_dim, theta):
    return np.outer(np.asarray(pos, dtype=np.float64), rope_inv_freq(head_dim, theta))


def rope_rotate_half(x, pos, theta):
    """Rotate-half RoPE: ``x * cos(emb) + rot(x) * sin(emb)``.

    [DeepDive] class LLaMARoPE: ``freqs = outer(positions, inv_freq)``,
    ``emb = cat(freqs, freqs)``, ``rot(x) = cat(-x2, x1)`` with x1, x2 the
    two halves of the head vector.  ``x``: ``[..., L, H, hd]``; ``pos``: ``[L]``.
    """
    x = np.asarray(x, dtype=np.float64)
    hd = x.shape[-1]
    f = _angles(pos, hd, theta)                       # [L, hd/2]
    emb = np.concatenate([f, f], axis=-1)[:, None, :]  # [L, 1, hd]
    x1, x2 = x[..., : hd // 2], x[..., hd // 2:]
    rot = np.concatenate([-x2, x1], axis=-1)
    return x * np.cos(emb) + rot * np.sin(emb)


def rope_interleaved(x, pos, theta):
    """Interleaved ("traditional") RoPE -- reading of [MLX-13B] "LLaMA 2 的结构分析".

    Pair ``(x[2i], x[2i+1])`` is rotated by angle ``p * inv_freq[i]``:
    ``y0 = x0 cos - x1 sin``, ``y1 = x0 sin + x1 cos``.
    """
    x = np.asarray(x, dtype=np.float64)
    hd = x.shape[-1]
    f = _angles(pos, hd, theta)[:, None, :]           # [L, 1, hd/2]
    c, s = np.cos(f), np.sin(f)
    x0, x1 = x[..., 0::2], x[..., 1::2]
    y = np.empty_like(x)
    y[..., 0::2] = x0 * c - x1 * s
    y[..., 1::2] = x0 * s + x1 * c
    return y


def apply_rope(x, pos, theta, style):
    if style == "half":
        return rope_rotate_half(x, pos, theta)
    if style == "interleaved":
        return rope_interleaved(x, pos, theta)
    raise ValueError(f"unknown rope style {style!r}")


def silu(z):
    """``z / (1 + exp(-z))`` ([MLX-13B] 3. 前馈网络; [DeepDive] LLaMAMLP uses F.silu)."""
    z = np.asarray(z, dtype=np.float64)
    return z / (1.0 + np.exp(-z))


def causal_gqa_attention(q, k, v, q_pos, n_rep, round_p=_identity):
    """Causal grouped-query scaled-dot-product attention for ONE sequence.

    ``q``: ``[L, nh, hd]`` queries at absolute positions ``q_pos`` (``[L]``);
    ``k``, ``v``: ``[T, nkv, hd]``, key ``j`` at absolute position ``j``.
    For query head ``h`` (KV head ``h // n_rep``):
    ``out = softmax(q k^T / sqrt(hd) masked to j <= p) v``.

    [MLX-13B] 2. 注意力机制 (``softmax((Q @ K^T) / sqrt(d_head)) @ V``) and
    5. 因果掩码; [DeepDive] LLaMAAttention (masked_fill with -inf, fp32
    softmax).  Subtracting the row maximum before ``exp`` is the usual exact
    rewrite of softmax.
    """
    q = np.asarray(q, dtype=np.float64)
    L, nh, hd = q.shape
    T = k.shape[0]
    q_pos = np.asarray(q_pos)
    masked = np.arange(T)[None, :] > q_pos[:, None]          # [L, T]
    out = np.empty((L, nh, hd), dtype=np.float64)
    scale = 1.0 / math.sqrt(hd)
    for h in range(nh):
        kv = h // n_rep
        s = (q[:, h, :] @ k[:, kv, :].T) * scale
        s = np.where(masked, -np.inf, s)
        e = np.exp(s - s.max(axis=1, keepdims=True))
        a = round_p(e / e.sum(axis=1, keepdims=True))
        out[:, h, :] = a @ v[:, kv, :]
    return out


class KVCache:
    """Per-layer KV cache ``k, v: [B, n_kv, T, hd]``, grown along the sequence axis.

    [MLX-13B] KV 缓存实现片段: new (already rotated) keys/values are
    concatenated after the cached ones on axis 2; the next tokens' RoPE offset
    is ``key_cache.shape[2]``.  Storage is preallocated to ``capacity`` and
    filled in order, which gives the same contents as repeated concatenation.
    """

    def __init__(self, batch, n_kv_heads, head_dim, capacity, k0=None, v0=None):
        self.k = np.zeros((batch, n_kv_heads, capacity, head_dim), dtype=np.float64)
        self.v = np.zeros_like(self.k)
        self.length = 0
        if k0 is not None:
            t = k0.shape[2]
            self.k[:, :, :t] = k0
            self.v[:, :, :t] = v0
            self.length = t

    def append(self, k_new, v_new):
        """``k_new``, ``v_new``: ``[B, L, n_kv, hd]`` at positions length .. length+L-1."""
        L = k_new.shape[1]
        if self.length + L > self.k.shape[2]:
            raise ValueError("cache full")
        t0 = self.length
        self.k[:, :, t0:t0 + L] = np.transpose(k_new, (0, 2, 1, 3))
        self.v[:, :, t0:t0 + L] = np.transpose(v_new, (0, 2, 1, 3))
        self.length += L

    def view(self, b):
        """Sequence ``b``'s visible keys/values as ``[T, n_kv, hd]``."""
        t = self.length
        return (np.transpose(self.k[b, :, :t], (1, 0, 2)),
                np.transpose(self.v[b, :, :t], (1, 0, 2)))


def layer_forward(d: Dims, W, x, cache: KVCache, rounding=None, rows=None):
    """One pre-norm decoder block over ``x: [B, L, dim]`` (prefill, or decode when L == 1).

    [DeepDive] LLaMABlock: ``x = x + attn(norm1(x)); x = x + mlp(norm2(x))``;
    [Decoder] 数据流动 (the six steps in the same order).  ``W`` holds
    ``attn_norm, wq, wk, wv, wo, ffn_norm, w1, w3, w2`` with every Linear
    weight ``[out, in]`` and ``y = x W^T`` (no bias).  Positions start at the
    cache length; the rotated k and v are appended to ``cache`` before
    attention.

    ``rows``: optional token indices (within L); when given, only those query
    rows are pushed through attention, o_proj and the FFN (all rows still
    feed the cache), and the returned arrays hold just those rows.

    Returns ``(x_out, parts)``: ``parts`` holds the intermediates ``h``
    (norm-1 output), ``q`` (after RoPE, selected rows), ``k`` (after RoPE),
    ``v``, ``attn`` (attention output, heads concatenated), ``x_mid`` (residual
    stream after the attention branch), ``h2`` (norm-2 output) and ``m``
    (SwiGLU product).
    """
    rnd = to_bf16 if rounding == "bf16" else _identity
    x = np.asarray(x, dtype=np.float64)
    B, L, _ = x.shape
    nh, nkv, hd = d.n_heads, d.n_kv_heads, d.head_dim
    p0 = cache.length
    pos = p0 + np.arange(L)

    h = rnd(rms_norm(x, W["attn_norm"], d.eps))
    k_raw = rnd(h @ np.asarray(W["wk"], np.float64).T).reshape(B, L, nkv, hd)
    v = rnd(h @ np.asarray(W["wv"], np.float64).T).reshape(B, L, nkv, hd)
    k = rnd(apply_rope(k_raw, pos, d.rope_theta, d.rope_style))
    cache.append(k, v)

    sel = np.arange(L) if rows is None else np.asarray(rows)
    hs = h[:, sel]
    q = rnd(hs @ np.asarray(W["wq"], np.float64).T).reshape(B, len(sel), nh, hd)
    q = rnd(apply_rope(q, pos[sel], d.rope_theta, d.rope_style))

    o = np.empty((B, len(sel), nh, hd), dtype=np.float64)
    for b in range(B):
        kb, vb = cache.view(b)
        o[b] = causal_gqa_attention(q[b], kb, vb, pos[sel], d.n_rep, round_p=rnd)
    o = rnd(o).reshape(B, len(sel), nh * hd)

    xs = x[:, sel]
    x_mid = xs + o @ np.asarray(W["wo"], np.float64).T
    h2 = rnd(rms_norm(x_mid, W["ffn_norm"], d.eps))
    gate = h2 @ np.asarray(W["w1"], np.float64).T
    up = h2 @ np.asarray(W["w3"], np.float64).T
    m = rnd(silu(gate) * up)
    x_out = x_mid + m @ np.asarray(W["w2"], np.float64).T
    return x_out, {"h": h, "q": q, "k_raw": k_raw, "k": k, "v": v, "attn": o, "x_mid": x_mid,
                   "h2": h2, "m": m}


def embed(E, tokens):
    """Token embedding lookup ``x[t] = E[tok[t]]`` ([DeepDive] class LLaMA, nn.Embedding)."""
    return np.asarray(E, dtype=np.float64)[np.asarray(tokens)]


def final_logits(x_last, g_final, W_lm, eps, rounding=None):
    """``logits = norm(x) W_lm^T`` without bias ([DeepDive] class LLaMA: norm, lm_head)."""
    rnd = to_bf16 if rounding == "bf16" else _identity
    h = rnd(rms_norm(x_last, g_final, eps))
    return h @ np.asarray(W_lm, np.float64).T


def layer_forward_ragged(d: Dims, W, xs, caches, rounding=None):
    """A ragged batch: sequence ``b`` brings ``xs[b]`` of shape ``[L_b, dim]`` at
    positions ``caches[b].length .. + L_b - 1`` of its own single-sequence cache
    (decode rows, L_b = 1, and prefill chunks may be mixed).

    The block never mixes sequences: attention runs within one sequence
    ([DeepDive] LLaMAAttention, per batch row; [MLX-13B] KV 缓存实现片段, one
    cache per sequence) and the norms, projections and FFN act per token.  So a
    ragged batch is ``layer_forward`` applied to each sequence with its own
    offset.  Returns the list of ``[L_b, dim]`` outputs.
    """
    return [layer_forward(d, W, np.asarray(x)[None], c, rounding)[0][0] for x, c in zip(xs, caches)]


def greedy_argmax(logits):
    """Greedy decoding: index of the largest logit, lowest index on ties.

    [HandsOn] 第三章 (``lm_head_output[0, -1].argmax(-1)``); [MLX-13B] 生成过程
    (temp = 0 uses argmax).  ``numpy.argmax`` returns the first maximal index.
    """
    return np.argmax(np.asarray(logits), axis=-1)


def model_forward(d: Dims, model, tokens, caches, rounding=None):
    """Embedding -> all blocks -> final norm -> lm_head on the last row -> argmax.

    [DeepDive] class LLaMA forward; [Decoder] 数据流动 overview (token
    embedding, N decoder blocks, final RMSNorm, LM head); only the last row's
    logits pick the next token ([HandsOn] 第三章).  ``model`` holds
    ``embed [vocab, dim]``, ``layers`` (list of weight dicts), ``final_norm``
    and ``lm_head [vocab, dim]``.  Returns ``(logits [B, vocab], ids [B])``.
    """
    x = embed(model["embed"], tokens)
    for W, cache in zip(model["layers"], caches):
        x, _ = layer_forward(d, W, x, cache, rounding=rounding)
    logits = final_logits(x[:, -1, :], model["final_norm"], model["lm_head"], d.eps,
                          rounding=rounding)
    return logits, greedy_argmax(logits)
