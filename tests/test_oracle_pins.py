"""Pins of the fp64 oracle against facts fixed outside itself (CPU only).

Each test names what it pins and why a plausible mistake fails it: closed
forms, invariants the pages' definitions imply, special cases that reduce to
a library routine, and a pure-Python brute force on tiny shapes.  The
planted-mistake tests at the end show that these pins catch a dropped term,
a wrong sign, a wrong index and a transposed operand in the oracle.
"""

import math

import numpy as np
import pytest

from oracle import block as ob
from oracle import brute

RNG = np.random.default_rng(7)


def tiny_dims(style="half", nh=4, nkv=2, hd=8, dim=16, ffn=24):
    return ob.Dims(dim=dim, n_heads=nh, n_kv_heads=nkv, head_dim=hd, ffn_dim=ffn,
                   eps=1e-5, rope_theta=10000.0, rope_style=style)


def rand_weights(d, rng, std=0.3, norm_std=0.1):
    nh, nkv, hd, D, F = d.n_heads, d.n_kv_heads, d.head_dim, d.dim, d.ffn_dim
    g = lambda *s: rng.standard_normal(s) * std  # noqa: E731
    return {
        "attn_norm": 1 + rng.standard_normal(D) * norm_std,
        "wq": g(nh * hd, D), "wk": g(nkv * hd, D), "wv": g(nkv * hd, D),
        "wo": g(D, nh * hd),
        "ffn_norm": 1 + rng.standard_normal(D) * norm_std,
        "w1": g(F, D), "w3": g(F, D), "w2": g(D, F),
    }


# ------------------------------------------------------------------ RMSNorm (I-1)

def test_rmsnorm_closed_form():
    # x = [3, 4], eps = 0: mean(x^2) = 12.5, out = x / sqrt(12.5) (times weight)
    out = ob.rms_norm(np.array([3.0, 4.0]), np.array([1.0, 2.0]), 0.0)
    assert np.allclose(out, [3 / math.sqrt(12.5), 8 / math.sqrt(12.5)], rtol=0, atol=1e-15)


def test_rmsnorm_unit_weight_unit_rms():
    x = RNG.standard_normal((5, 64)) * 3.0
    eps = 1e-5
    out = ob.rms_norm(x, np.ones(64), eps)
    ms = np.mean(x * x, axis=-1)
    rms = np.sqrt(np.mean(out * out, axis=-1))
    assert np.allclose(rms, np.sqrt(ms / (ms + eps)), rtol=1e-13)
    # eps = 0: exactly unit RMS and invariant to positive scaling of x
    assert np.allclose(np.sqrt(np.mean(ob.rms_norm(x, np.ones(64), 0.0) ** 2, -1)), 1.0, rtol=1e-14)
    assert np.allclose(ob.rms_norm(7.5 * x, np.ones(64), 0.0), ob.rms_norm(x, np.ones(64), 0.0),
                       rtol=1e-13)


def test_rmsnorm_weight_is_per_feature():
    x = RNG.standard_normal((3, 8))
    g = RNG.standard_normal(8)
    assert np.allclose(ob.rms_norm(x, g, 1e-5), g * ob.rms_norm(x, np.ones(8), 1e-5), rtol=1e-14)


# ------------------------------------------------------------------ RoPE (I-2..I-4)

@pytest.mark.parametrize("style", ["half", "interleaved"])
def test_rope_position_zero_is_identity(style):
    x = RNG.standard_normal((1, 3, 16))
    assert np.array_equal(ob.apply_rope(x, [0], 1e4, style), x)


def test_rope_two_dim_closed_form():
    # head_dim 2: inv_freq = theta**0 = 1, so position p rotates by p radians
    for p in [1, 2, 5, 37]:
        for style in ["half", "interleaved"]:
            y = ob.apply_rope(np.array([[[1.0, 0.0]]]), [p], 1e4, style)[0, 0]
            assert np.allclose(y, [math.cos(p), math.sin(p)], atol=1e-15)


def test_rope_inv_freq_ladder():
    f = ob.rope_inv_freq(8, 10000.0)
    assert np.allclose(f, [1.0, 10000 ** -0.25, 10000 ** -0.5, 10000 ** -0.75], rtol=1e-15)


@pytest.mark.parametrize("style", ["half", "interleaved"])
def test_rope_preserves_pair_norms(style):
    hd = 16
    x = RNG.standard_normal((6, 2, hd))
    pos = np.arange(100, 106)
    y = ob.apply_rope(x, pos, 1e4, style)
    if style == "half":
        pn = lambda a: a[..., : hd // 2] ** 2 + a[..., hd // 2:] ** 2  # noqa: E731
    else:
        pn = lambda a: a[..., 0::2] ** 2 + a[..., 1::2] ** 2  # noqa: E731
    assert np.allclose(pn(y), pn(x), rtol=1e-12)
    assert np.allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)


@pytest.mark.parametrize("style", ["half", "interleaved"])
def test_rope_dot_depends_on_relative_position(style):
    hd = 32
    q = RNG.standard_normal((1, 1, hd))
    k = RNG.standard_normal((1, 1, hd))
    base = None
    for shift in [0, 3, 250, 4000]:
        pq, pk = 17 + shift, 5 + shift
        d = float(np.sum(ob.apply_rope(q, [pq], 1e4, style) * ob.apply_rope(k, [pk], 1e4, style)))
        base = d if base is None else base
        assert abs(d - base) < 1e-10
    # and it does depend on the offset
    d2 = float(np.sum(ob.apply_rope(q, [18], 1e4, style) * ob.apply_rope(k, [5], 1e4, style)))
    assert abs(d2 - base) > 1e-6


def test_rope_interleaved_is_permuted_rotate_half():
    # I-4: interleaved == P^-1 rotate_half(P x), P de-interleaves [x0, x2, .., x1, x3, ..]
    hd = 16
    x = RNG.standard_normal((4, 3, hd))
    pos = np.array([0, 9, 130, 4095])
    perm = np.concatenate([np.arange(0, hd, 2), np.arange(1, hd, 2)])
    inv = np.argsort(perm)
    y_half = ob.rope_rotate_half(x[..., perm], pos, 1e4)[..., inv]
    assert np.allclose(ob.rope_interleaved(x, pos, 1e4), y_half, rtol=0, atol=1e-13)


# ------------------------------------------------------------------ attention (I-5..I-10)

def _attn_inputs(L=6, T=None, nh=4, nkv=2, hd=8):
    T = T or L
    return (RNG.standard_normal((L, nh, hd)), RNG.standard_normal((T, nkv, hd)),
            RNG.standard_normal((T, nkv, hd)))


def test_attention_row0_returns_v0():
    q, k, v = _attn_inputs()
    o = ob.causal_gqa_attention(q, k, v, np.arange(6), n_rep=2)
    for h in range(4):
        assert np.allclose(o[0, h], v[0, h // 2], rtol=0, atol=1e-15)


def test_attention_convex_hull_and_zero_query_mean():
    q, k, v = _attn_inputs(L=8)
    o = ob.causal_gqa_attention(q, k, v, np.arange(8), n_rep=2)
    for i in range(8):
        for h in range(4):
            vis = v[: i + 1, h // 2]
            assert np.all(o[i, h] <= vis.max(0) + 1e-12) and np.all(o[i, h] >= vis.min(0) - 1e-12)
    o0 = ob.causal_gqa_attention(np.zeros_like(q), k, v, np.arange(8), n_rep=2)
    for i in range(8):
        assert np.allclose(o0[i, 0], v[: i + 1, 0].mean(0), atol=1e-14)


def test_attention_is_causal():
    q, k, v = _attn_inputs(L=7)
    o = ob.causal_gqa_attention(q, k, v, np.arange(7), n_rep=2)
    k2, v2 = k.copy(), v.copy()
    k2[5:] += 10.0
    v2[5:] -= 3.0
    o2 = ob.causal_gqa_attention(q, k2, v2, np.arange(7), n_rep=2)
    assert np.array_equal(o[:5], o2[:5])
    assert not np.allclose(o[5:], o2[5:])


def test_attention_matches_explicit_softmax_formula():
    # Closed form on a 2-key case: weights e^{s0}, e^{s1} normalised.
    hd = 4
    q = np.array([[[1.0, 0.0, 0.0, 0.0]]])
    k = np.array([[[2.0, 0, 0, 0]], [[-2.0, 0, 0, 0]]])
    v = np.array([[[1.0, 0, 0, 0]], [[0.0, 1, 0, 0]]])
    o = ob.causal_gqa_attention(q, k, v, np.array([1]), n_rep=1)
    s0, s1 = 2 / math.sqrt(hd), -2 / math.sqrt(hd)
    a0 = math.exp(s0) / (math.exp(s0) + math.exp(s1))
    assert np.allclose(o[0, 0], [a0, 1 - a0, 0, 0], atol=1e-15)


def test_gqa_equals_mha_with_repeated_kv_heads():
    q, k, v = _attn_inputs(L=5, nh=6, nkv=2)
    o = ob.causal_gqa_attention(q, k, v, np.arange(5), n_rep=3)
    rep = np.array([h // 3 for h in range(6)])
    o_mha = ob.causal_gqa_attention(q, k[:, rep], v[:, rep], np.arange(5), n_rep=1)
    assert np.allclose(o, o_mha, rtol=0, atol=1e-15)


def test_gqa_mapping_is_contiguous_groups_not_modulo():
    q, k, v = _attn_inputs(L=4, nh=4, nkv=2)
    o = ob.causal_gqa_attention(q, k, v, np.arange(4), n_rep=2)
    # head 1 must use kv head 0 (1 // 2), not kv head 1 (1 % 2)
    o_h1 = ob.causal_gqa_attention(q[:, 1:2], k[:, 0:1], v[:, 0:1], np.arange(4), n_rep=1)
    assert np.allclose(o[:, 1], o_h1[:, 0], atol=1e-15)


# ------------------------------------------------------------------ block and cache (I-11..I-14)

def _run_block(d, W, x, cache):
    return ob.layer_forward(d, W, x, cache)[0]


@pytest.mark.parametrize("style", ["half", "interleaved"])
def test_block_matches_pure_python_brute_force(style):
    d = tiny_dims(style)
    W = rand_weights(d, RNG)
    p_cache, L = 3, 4
    x_hist = RNG.standard_normal((1, p_cache, d.dim))
    x = RNG.standard_normal((1, L, d.dim))
    cache = ob.KVCache(1, d.n_kv_heads, d.head_dim, 16)
    _run_block(d, W, x_hist, cache)
    y = _run_block(d, W, x, cache)
    Wl = {k: np.asarray(v).tolist() for k, v in W.items()}
    kc, vc = [], []
    brute.block_forward(d, Wl, x_hist[0].tolist(), kc, vc)
    yb = np.array(brute.block_forward(d, Wl, x[0].tolist(), kc, vc))
    assert np.allclose(y[0], yb, rtol=0, atol=1e-12)


def test_decode_with_cache_reproduces_full_prefill_rows():
    d = tiny_dims()
    W = rand_weights(d, RNG)
    x = RNG.standard_normal((2, 9, d.dim))
    full = _run_block(d, W, x, ob.KVCache(2, d.n_kv_heads, d.head_dim, 16))
    cache = ob.KVCache(2, d.n_kv_heads, d.head_dim, 16)
    _run_block(d, W, x[:, :5], cache)
    for t in range(5, 9):
        y = _run_block(d, W, x[:, t:t + 1], cache)
        assert np.allclose(y[:, 0], full[:, t], rtol=0, atol=1e-12)


def test_chunked_prefill_equals_single_prefill():
    d = tiny_dims("interleaved")
    W = rand_weights(d, RNG)
    x = RNG.standard_normal((1, 10, d.dim))
    full = _run_block(d, W, x, ob.KVCache(1, d.n_kv_heads, d.head_dim, 16))
    cache = ob.KVCache(1, d.n_kv_heads, d.head_dim, 16)
    a = _run_block(d, W, x[:, :4], cache)
    b = _run_block(d, W, x[:, 4:], cache)
    assert np.allclose(np.concatenate([a, b], 1), full, rtol=0, atol=1e-12)


def test_row_subset_equals_full_rows():
    d = tiny_dims()
    W = rand_weights(d, RNG)
    x = RNG.standard_normal((2, 9, d.dim))
    full = _run_block(d, W, x, ob.KVCache(2, d.n_kv_heads, d.head_dim, 16))
    rows = [0, 4, 8]
    part, _ = ob.layer_forward(d, W, x, ob.KVCache(2, d.n_kv_heads, d.head_dim, 16), rows=rows)
    assert np.allclose(part, full[:, rows], rtol=0, atol=1e-13)


def test_zero_output_projections_make_block_identity():
    d = tiny_dims()
    W = rand_weights(d, RNG)
    W["wo"] = np.zeros_like(W["wo"])
    W["w2"] = np.zeros_like(W["w2"])
    x = RNG.standard_normal((1, 5, d.dim))
    assert np.array_equal(_run_block(d, W, x, ob.KVCache(1, 2, 8, 8)), x)
    W = rand_weights(d, RNG)
    W["w2"] = np.zeros_like(W["w2"])
    y, parts = ob.layer_forward(d, W, x, ob.KVCache(1, 2, 8, 8))
    assert np.array_equal(y, parts["x_mid"])


def test_silu_values():
    assert ob.silu(0.0) == 0.0
    assert math.isclose(float(ob.silu(1.0)), 1.0 / (1.0 + math.exp(-1.0)), rel_tol=1e-15)
    assert math.isclose(float(ob.silu(-2.0)), -2.0 / (1.0 + math.exp(2.0)), rel_tol=1e-15)


def test_batch_permutation_equivariance():
    d = tiny_dims()
    W = rand_weights(d, RNG)
    x = RNG.standard_normal((3, 6, d.dim))
    y = _run_block(d, W, x, ob.KVCache(3, 2, 8, 8))
    perm = [2, 0, 1]
    yp = _run_block(d, W, x[perm], ob.KVCache(3, 2, 8, 8))
    assert np.allclose(yp, y[perm], rtol=0, atol=1e-14)


def test_block_wiring_against_hand_composition():
    # one token at position 0: attention returns v, so the block is a plain
    # composition of norm, matvecs and SwiGLU that can be written out directly
    d = tiny_dims(nh=2, nkv=1)
    W = rand_weights(d, RNG)
    x = RNG.standard_normal((1, 1, d.dim))
    y = _run_block(d, W, x, ob.KVCache(1, 1, 8, 4))[0, 0]
    x0 = x[0, 0]
    ms = np.mean(x0 ** 2)
    h = W["attn_norm"] * x0 / np.sqrt(ms + d.eps)
    vv = W["wv"] @ h
    o = np.concatenate([vv, vv])          # both query heads read kv head 0
    xm = x0 + W["wo"] @ o
    h2 = W["ffn_norm"] * xm / np.sqrt(np.mean(xm ** 2) + d.eps)
    g, u = W["w1"] @ h2, W["w3"] @ h2
    expect = xm + W["w2"] @ (g / (1 + np.exp(-g)) * u)
    assert np.allclose(y, expect, rtol=0, atol=1e-13)


# ------------------------------------------------------------------ model (I-15)

def test_zero_layer_model_closed_form_and_argmax():
    d = tiny_dims()
    vocab = 50
    E = RNG.standard_normal((vocab, d.dim))
    lm = RNG.standard_normal((vocab, d.dim))
    g = 1 + 0.1 * RNG.standard_normal(d.dim)
    tok = RNG.integers(0, vocab, size=(3, 4))
    model = {"embed": E, "layers": [], "final_norm": g, "lm_head": lm}
    logits, ids = ob.model_forward(d, model, tok, [])
    xl = E[tok[:, -1]]
    hn = g * xl / np.sqrt(np.mean(xl ** 2, -1, keepdims=True) + d.eps)
    assert np.allclose(logits, hn @ lm.T, rtol=0, atol=1e-12)
    assert np.array_equal(ids, np.argmax(hn @ lm.T, axis=-1))


def test_argmax_tie_breaks_to_lowest_index():
    assert ob.greedy_argmax(np.array([[1.0, 3.0, 3.0, 2.0]]))[0] == 1


def test_model_one_layer_equals_block_then_head():
    d = tiny_dims()
    vocab = 40
    W = rand_weights(d, RNG)
    E = RNG.standard_normal((vocab, d.dim))
    lm = RNG.standard_normal((vocab, d.dim))
    tok = RNG.integers(0, vocab, size=(2, 5))
    model = {"embed": E, "layers": [W], "final_norm": np.ones(d.dim), "lm_head": lm}
    logits, _ = ob.model_forward(d, model, tok, [ob.KVCache(2, 2, 8, 8)])
    y = _run_block(d, W, E[tok], ob.KVCache(2, 2, 8, 8))
    expect = ob.rms_norm(y[:, -1], np.ones(d.dim), d.eps) @ lm.T
    assert np.allclose(logits, expect, rtol=0, atol=1e-12)


# ------------------------------------------------------------------ bf16 rounding (library special case)

def test_bf16_rounding_matches_torch_conversion():
    torch = pytest.importorskip("torch")
    x = np.concatenate([RNG.standard_normal(20000) * s for s in (1e-3, 1.0, 300.0)])
    # values exactly half-way between bf16 neighbours (ties -> even)
    ties = (np.arange(1, 200, dtype=np.float64) * 2 + 1) * 2.0 ** -9
    x = np.concatenate([x, ties, -ties]).astype(np.float32).astype(np.float64)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(ob.to_bf16(x), ref)


def test_bf16_mode_only_perturbs_at_rounding_level():
    d = tiny_dims()
    W = rand_weights(d, RNG)
    x = RNG.standard_normal((1, 6, d.dim))
    y = _run_block(d, W, x, ob.KVCache(1, 2, 8, 8))
    yb, _ = ob.layer_forward(d, W, x, ob.KVCache(1, 2, 8, 8), rounding="bf16")
    rel = np.max(np.abs(yb - y)) / np.sqrt(np.mean(y ** 2))
    assert 0 < rel < 3e-2


# ------------------------------------------------------------------ planted mistakes

def _planted(monkeypatch, name, fn):
    monkeypatch.setattr(ob, name, fn)


def test_pin_catches_rotate_half_sign_error(monkeypatch):
    orig = ob.rope_rotate_half

    def wrong(x, pos, theta):   # rot(x) = cat(x2, -x1) instead of cat(-x2, x1)
        x = np.asarray(x, dtype=np.float64)
        hd = x.shape[-1]
        f = ob._angles(pos, hd, theta)
        emb = np.concatenate([f, f], -1)[:, None, :]
        rot = np.concatenate([x[..., hd // 2:], -x[..., : hd // 2]], -1)
        return x * np.cos(emb) + rot * np.sin(emb)

    _planted(monkeypatch, "rope_rotate_half", wrong)
    with pytest.raises(AssertionError):
        test_rope_two_dim_closed_form()
    _planted(monkeypatch, "rope_rotate_half", orig)


def test_pin_catches_gqa_modulo_mapping(monkeypatch):
    orig = ob.causal_gqa_attention

    def wrong(q, k, v, q_pos, n_rep, round_p=lambda a: a):
        nkv = k.shape[1]
        kk = k[:, [h % nkv for h in range(q.shape[1])]]
        vv = v[:, [h % nkv for h in range(q.shape[1])]]
        return orig(q, kk, vv, q_pos, 1, round_p)

    _planted(monkeypatch, "causal_gqa_attention", wrong)
    with pytest.raises(AssertionError):
        test_gqa_mapping_is_contiguous_groups_not_modulo()


def test_pin_catches_dropped_norm_eps_and_transposed_weight(monkeypatch):
    _planted(monkeypatch, "rms_norm",
             lambda x, g, eps: np.asarray(g) * np.asarray(x) / np.sqrt(np.mean(np.asarray(x) ** 2, -1,
                                                                                  keepdims=True)))
    with pytest.raises(AssertionError):
        test_rmsnorm_unit_weight_unit_rms()
    monkeypatch.undo()
    # a transposed o_proj (square here) must change the result
    d = tiny_dims(nh=2, nkv=2)
    W = rand_weights(d, RNG)
    x = RNG.standard_normal((1, 3, d.dim))
    y = _run_block(d, W, x, ob.KVCache(1, 2, 8, 8))
    Wt = dict(W, wo=W["wo"].T.copy())
    yt = _run_block(d, Wt, x, ob.KVCache(1, 2, 8, 8))
    assert not np.allclose(y, yt, atol=1e-6)


def test_pin_catches_off_by_one_causal_mask(monkeypatch):
    orig = ob.causal_gqa_attention

    def wrong(q, k, v, q_pos, n_rep, round_p=lambda a: a):
        return orig(q, k, v, np.asarray(q_pos) - 1 + (np.asarray(q_pos) == 0), n_rep, round_p)

    _planted(monkeypatch, "causal_gqa_attention", wrong)
    with pytest.raises(AssertionError):
        test_block_matches_pure_python_brute_force("half")


def test_ragged_batch_matches_batched_and_full_prefill():
    """Ragged batches (per-sequence offsets and chunk lengths): with equal
    lengths they equal the batched block; with different ones each
    sequence's rows equal the matching rows of a one-shot prefill of its
    whole prefix (a different code path: one call, no chunking)."""
    d = tiny_dims()
    W = rand_weights(d, RNG)
    # equal lengths: per-sequence caches vs one batched cache
    x = RNG.standard_normal((3, 5, d.dim))
    batched, _ = ob.layer_forward(d, W, x, ob.KVCache(3, d.n_kv_heads, d.head_dim, 16))
    rag = ob.layer_forward_ragged(d, W, list(x), [ob.KVCache(1, d.n_kv_heads, d.head_dim, 16) for _ in range(3)])
    assert np.allclose(np.stack(rag), batched, rtol=0, atol=1e-12)
    # mixed: sequence 0 decodes its 8th token, sequence 1 prefills 4 tokens after 3 cached, sequence 2 starts fresh
    prefixes = [RNG.standard_normal((8, d.dim)), RNG.standard_normal((7, d.dim)), RNG.standard_normal((2, d.dim))]
    cached = [7, 3, 0]
    caches = []
    for pre, n in zip(prefixes, cached):
        c = ob.KVCache(1, d.n_kv_heads, d.head_dim, 16)
        if n:
            ob.layer_forward(d, W, pre[None, :n], c)
        caches.append(c)
    outs = ob.layer_forward_ragged(d, W, [pre[n:] for pre, n in zip(prefixes, cached)], caches)
    for pre, n, out in zip(prefixes, cached, outs):
        full, _ = ob.layer_forward(d, W, pre[None], ob.KVCache(1, d.n_kv_heads, d.head_dim, 16))
        assert out.shape == (len(pre) - n, d.dim)
        assert np.allclose(out, full[0, n:], rtol=0, atol=1e-12)
