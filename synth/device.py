"""Upload seeded synthetic arrays to the GPU (memory plumbing only, no arithmetic).

Weights go to device memory in the stored dtype.  q, k, v rows are packed
into one contiguous buffer (q, then k, then v) and gate/up rows into another
(gate first) -- the fused layout of the Phi-3 checkpoint -- so the library
can run each as one GEMM; ``wq``/``wk``/``wv`` and ``w1``/``w3`` are views.
"""

from __future__ import annotations

import numpy as np


def _torch():
    import torch
    return torch


def to_device(a, dtype, device="cuda"):
    """float32 numpy array -> device tensor of ``dtype`` ("bf16" or "f32")."""
    torch = _torch()
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    if dtype == "bf16":
        t = t.to(torch.bfloat16)
    return t.to(device)


def upload_layer(W, dtype, device="cuda"):
    """Device tensors for one layer's weight dict (see ``synth.layer_weights``)."""
    nq, nk = W["wq"].shape[0], W["wk"].shape[0]
    f = W["w1"].shape[0]
    qkv = to_device(np.concatenate([W["wq"], W["wk"], W["wv"]], axis=0), dtype, device)
    gu = to_device(np.concatenate([W["w1"], W["w3"]], axis=0), dtype, device)
    return {
        "attn_norm": to_device(W["attn_norm"], "f32", device),
        "ffn_norm": to_device(W["ffn_norm"], "f32", device),
        "qkv": qkv, "wq": qkv[:nq], "wk": qkv[nq:nq + nk], "wv": qkv[nq + nk:],
        "wo": to_device(W["wo"], dtype, device),
        "gate_up": gu, "w1": gu[:f], "w3": gu[f:],
        "w2": to_device(W["w2"], dtype, device),
    }


def upload_layer_separate(W, dtype, device="cuda"):
    """Like ``upload_layer`` but every projection in its own allocation."""
    out = {k: to_device(W[k], "f32" if k.endswith("norm") else dtype, device)
           for k in ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm", "w1", "w3", "w2")}
    return out


def random_layer_on_device(w, seed, device="cuda"):
    """A layer of workload ``w`` drawn directly on the device (torch generator).

    For timing runs where host-side generation of multi-GB weights would
    dominate; the distribution matches ``synth.layer_weights`` (N(0, w_std),
    bf16 storage, unit norm weights).
    """
    torch = _torch()
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    d, nh, nkv, hd, f = w.dim, w.n_heads, w.n_kv_heads, w.head_dim, w.ffn_dim

    def n(*shape):
        return (torch.randn(*shape, generator=g, device=device, dtype=torch.float32) * w.w_std).to(dt)

    qkv = n((nh + 2 * nkv) * hd, d)
    gu = n(2 * f, d)
    out = {
        "attn_norm": torch.ones(d, device=device, dtype=torch.float32),
        "ffn_norm": torch.ones(d, device=device, dtype=torch.float32),
        "qkv": qkv, "wq": qkv[: nh * hd], "wk": qkv[nh * hd:(nh + nkv) * hd], "wv": qkv[(nh + nkv) * hd:],
        "wo": n(d, nh * hd), "gate_up": gu, "w1": gu[:f], "w3": gu[f:], "w2": n(d, f),
    }
    return out


def random_q4_layer_on_device(w, seed, device="cuda"):
    """A 4-bit group-64 layer of workload ``w``'s shape drawn on the device, for timing
    runs: uniform codes (eight per int32 word), scales ~ U(0.3, 0.4) x w_std and
    offsets = -7.5 x scale (a group of N(0, w_std) weights spans about 15 steps),
    both bf16 and group-major ``[in / 64][out]``; unit norm weights.  Returns the
    dict ``layer_weights_q4`` takes: (codes, scales, offsets) per projection."""
    torch = _torch()
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    d, nh, nkv, hd, f = w.dim, w.n_heads, w.n_kv_heads, w.head_dim, w.ffn_dim

    def q(out_f, in_f):
        codes = torch.randint(-2 ** 31, 2 ** 31 - 1, (out_f, in_f // 8), generator=g, device=device,
                              dtype=torch.int64).to(torch.int32)
        s = (0.3 + 0.1 * torch.rand(in_f // 64, out_f, generator=g, device=device)) * w.w_std
        return codes, s.to(torch.bfloat16), (-7.5 * s).to(torch.bfloat16)

    return {
        "attn_norm": torch.ones(d, device=device, dtype=torch.float32),
        "ffn_norm": torch.ones(d, device=device, dtype=torch.float32),
        "wq": q(nh * hd, d), "wk": q(nkv * hd, d), "wv": q(nkv * hd, d), "wo": q(d, nh * hd),
        "w1": q(f, d), "w3": q(f, d), "w2": q(d, f),
    }
