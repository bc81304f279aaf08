"""Shared helpers of the GPU parity tests: run one block through the C ABI and
read back the output and the intermediates the call leaves in its workspace."""

from __future__ import annotations

import numpy as np

import llama_decoder_only_b200 as L
from oracle import block as ob
from synth import device as sd


def oracle_dims(w):
    return ob.Dims(dim=w.dim, n_heads=w.n_heads, n_kv_heads=w.n_kv_heads, head_dim=w.head_dim,
                   ffn_dim=w.ffn_dim, eps=w.eps, rope_theta=w.rope_theta, rope_style=w.rope_style)


def lib_dims(w):
    return L.make_dims(w.dim, w.n_heads, w.n_kv_heads, w.head_dim, w.ffn_dim, w.eps, w.rope_theta,
                       w.rope_style, w.dtype)


def rel_errors(gpu, ref):
    """(max-abs / RMS(ref), RMS(err) / RMS(ref))."""
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    rms = float(np.sqrt(np.mean(ref * ref)))
    d = gpu - ref
    return float(np.max(np.abs(d))) / rms, float(np.sqrt(np.mean(d * d))) / rms


def ulp_rms_err(gpu, ref, ulps=2, rms_frac=1e-2):
    """Largest |gpu - ref| / (ulps * 2**-8 |ref| + rms_frac RMS(ref)); <= 1 passes."""
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    rms = float(np.sqrt(np.mean(ref * ref)))
    return float(np.max(np.abs(gpu - ref) / (ulps * 2.0 ** -8 * np.abs(ref) + rms_frac * rms)))


def floor_ratios(gpu, rounded, exact):
    """Error of ``gpu`` against ``exact`` divided by the error of the bf16-rounded
    oracle against ``exact``: (RMS ratio, max-abs ratio)."""
    gpu, rounded, exact = (np.asarray(a, np.float64) for a in (gpu, rounded, exact))
    rms = float(np.sqrt(np.mean(exact * exact)))
    eg, eb = gpu - exact, rounded - exact
    tiny = 1e-4 * rms
    r_rms = float(np.sqrt(np.mean(eg * eg))) / (float(np.sqrt(np.mean(eb * eb))) + tiny)
    r_max = float(np.max(np.abs(eg))) / (float(np.max(np.abs(eb))) + tiny)
    return r_rms, r_max


class LayerRun:
    """One layer on the GPU: weights, a KV cache, a workspace and the dims."""

    def __init__(self, w, W, batch, capacity, max_tokens, separate=False, k0=None, v0=None):
        import torch
        self.torch = torch
        self.w = w
        self.dims = lib_dims(w)
        self.dev = (sd.upload_layer_separate if separate else sd.upload_layer)(W, w.dtype)
        self.lw = L.layer_weights(self.dev)
        dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
        shape = (batch, w.n_kv_heads, capacity, w.head_dim)
        k = torch.zeros(shape, dtype=dt, device="cuda")
        v = torch.zeros(shape, dtype=dt, device="cuda")
        if k0 is not None:
            t0 = k0.shape[2]
            k[:, :, :t0] = sd.to_device(k0, w.dtype)
            v[:, :, :t0] = sd.to_device(v0, w.dtype)
        self.cache = L.KVCache(self.dims, batch, capacity, k=k, v=v)
        if k0 is not None:
            self.cache.set_length(k0.shape[2])
        self.batch = batch
        self.ws_max_tokens = max_tokens
        nbytes = max(L.workspace_size(self.dims, batch, max_tokens), L.workspace_size(self.dims, batch, 1))
        self.ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")

    def step(self, x):
        """Run prefill (L > 1) or decode (L == 1) on ``x [B, L, dim]`` (numpy float32)."""
        torch = self.torch
        B, Lq, D = x.shape
        xi = torch.from_numpy(np.ascontiguousarray(x, np.float32)).cuda().reshape(B * Lq, D)
        xo = torch.empty_like(xi)
        self.p0 = self.cache.length
        if Lq == 1:
            L.layer_decode(self.dims, self.lw, self.cache, B, xi, xo, self.ws)
        else:
            L.layer_prefill(self.dims, self.lw, self.cache, B, Lq, xi, xo, self.ws)
        torch.cuda.synchronize()
        assert L.device_status(self.ws) == 0
        self.last_L = Lq
        return xo.reshape(B, Lq, D).double().cpu().numpy()

    def intermediates(self):
        """q (rotated), attn, h2, m of the last call plus the appended k and v (from the cache), as float64 numpy."""
        torch = self.torch
        w = self.w
        B, Lq = self.batch, self.last_L
        M = B * Lq
        off = L.workspace_offsets(self.dims, B, Lq)
        dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
        es = 2 if w.dtype == "bf16" else 4
        qkvn = (w.n_heads + 2 * w.n_kv_heads) * w.head_dim

        def view(o, n):
            return self.ws[o:o + M * n * es].view(dt).reshape(M, n).double().cpu().numpy()

        qkv = view(off[0], qkvn)
        nq = w.n_heads * w.head_dim
        p0 = self.p0
        kc = self.cache.k[:, :, p0:p0 + Lq].double().cpu().numpy()          # [B, nkv, L, hd]
        vc = self.cache.v[:, :, p0:p0 + Lq].double().cpu().numpy()
        return {
            "q": qkv[:, :nq].reshape(B, Lq, w.n_heads, w.head_dim),
            "v": np.transpose(vc, (0, 2, 1, 3)),
            "k": np.transpose(kc, (0, 2, 1, 3)),
            "attn": view(off[2], nq).reshape(B, Lq, nq),
            "h2": view(off[1], w.dim).reshape(B, Lq, w.dim),
            "m": view(off[3], w.ffn_dim).reshape(B, Lq, w.ffn_dim),
        }
