"""GPU parity of the decode step with 4-bit group-64 weights (llama_layer_decode_q4)
against the fp64 oracle ([MLX-13B] "LLaMA 2 的结构分析": QuantizedLinear;
"模型配置": group_size 64, bits 4).

Every projection of a seeded bf16 layer is quantised by the oracle's
quantiser (``oracle/quant.py``); the scales and offsets are rounded to bf16
(the stored form); both sides then see the same codes, scales and offsets.
The exact reference is the oracle's block with the exactly dequantised
weights s*q + b (fp64).  The bf16 floor is the same block with those weights
rounded to bf16 (what the kernel multiplies: one rounding of s*q + b) and
the oracle's bf16 rounding of stored activations.  Bars: the same as the bf16
decode parity tests -- max-abs / RMS <= 1e-2 against the floor oracle,
RMS <= 1e-2 and max-abs <= 5e-2 against the exact one, and every
intermediate within 1.5x (RMS) / 2x (max) of the floor's own error.
"""

import numpy as np
import pytest

import llama_decoder_only_b200 as L
import synth
from oracle import block as ob
from oracle import quant as oq
from tests.harness import floor_ratios, oracle_dims, rel_errors

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

PROJ = ("wq", "wk", "wv", "wo", "w1", "w3", "w2")


def quantise_layer(W):
    """(device q4 dict, exact dequantised weights, bf16-rounded dequantised weights)."""
    dev = {"attn_norm": torch.from_numpy(W["attn_norm"]).cuda(), "ffn_norm": torch.from_numpy(W["ffn_norm"]).cuda()}
    exact = {"attn_norm": W["attn_norm"], "ffn_norm": W["ffn_norm"]}
    rounded = dict(exact)
    for k in PROJ:
        codes, s, b = oq.quantize(W[k])
        s = synth.bf16_round(s.astype(np.float32)).astype(np.float64)
        b = synth.bf16_round(b.astype(np.float32)).astype(np.float64)
        words = oq.pack_int4(codes)
        wd = oq.dequantize(codes, s, b)
        exact[k] = wd
        rounded[k] = ob.to_bf16(wd)
        dev[k] = (torch.from_numpy(words.view(np.int32)).cuda(),
                  torch.from_numpy(np.ascontiguousarray(s.T).astype(np.float32)).to(torch.bfloat16).cuda(),
                  torch.from_numpy(np.ascontiguousarray(b.T).astype(np.float32)).to(torch.bfloat16).cuda())
    return dev, exact, rounded


CASES = [
    # name, dim, nh, nkv, hd, ffn, B, T0, rope
    ("mha_b16_inter", 1024, 8, 8, 128, 2816, 16, 300, "interleaved"),
    ("gqa4_b5", 768, 8, 2, 96, 2048, 5, 130, "half"),
    ("gqa8_b40", 1024, 16, 2, 64, 2752, 40, 77, "half"),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_q4_decode_parity(case):
    name, dim, nh, nkv, hd, ffn, B, T0, rope = case
    w = synth.Workload(name, dim, nh, nkv, hd, ffn, 1e-5, 1e4, rope, "bf16", 0.02, 321,
                       cache_len=T0, decode_batch=B, decode_steps=2)
    inp = synth.decode_inputs(w)
    dev, We, Wb = quantise_layer(inp.weights)
    lw = L.layer_weights_q4(dev)
    dims = L.make_dims(dim, nh, nkv, hd, ffn, w.eps, w.rope_theta, rope, "bf16")
    cap = T0 + 4
    k = torch.zeros(B, nkv, cap, hd, dtype=torch.bfloat16, device="cuda")
    v = torch.zeros_like(k)
    k[:, :, :T0] = torch.from_numpy(inp.k_cache).to(torch.bfloat16)
    v[:, :, :T0] = torch.from_numpy(inp.v_cache).to(torch.bfloat16)
    cache = L.KVCache(dims, B, cap, k=k, v=v)
    cache.set_length(T0)
    ws = torch.zeros(L.workspace_size(dims, B, 1), dtype=torch.uint8, device="cuda")
    off = L.workspace_offsets(dims, B, 1)
    d = oracle_dims(w)
    k0 = inp.k_cache.astype(np.float64)
    v0 = inp.v_cache.astype(np.float64)
    ce = ob.KVCache(B, nkv, hd, cap, k0, v0)
    cb = ob.KVCache(B, nkv, hd, cap, k0, v0)
    for t, xs in enumerate(inp.steps):
        xi = torch.from_numpy(np.ascontiguousarray(xs.reshape(B, dim))).cuda()
        xo = torch.empty_like(xi)
        p0 = cache.length
        L.layer_decode_q4(dims, lw, cache, B, xi, xo, ws)
        torch.cuda.synchronize()
        assert L.device_status(ws) == 0
        assert cache.length == p0 + 1
        y = xo.double().cpu().numpy().reshape(B, 1, dim)
        ye, pe = ob.layer_forward(d, We, xs, ce)
        yb, pb = ob.layer_forward(d, Wb, xs, cb, rounding="bf16")
        mx, _ = rel_errors(y, yb)
        mxe, rmse = rel_errors(y, ye)

        def view(o, n):
            return ws[o:o + B * n * 2].view(torch.bfloat16).reshape(B, n).double().cpu().numpy()
        qkvn = (nh + 2 * nkv) * hd
        got = {"q": view(off[0], qkvn)[:, :nh * hd].reshape(B, 1, nh, hd),
               "attn": view(off[2], nh * hd).reshape(B, 1, nh * hd),
               "h2": view(off[1], dim).reshape(B, 1, dim),
               "m": view(off[3], ffn).reshape(B, 1, ffn),
               "k": np.transpose(cache.k[:, :, p0:p0 + 1].double().cpu().numpy(), (0, 2, 1, 3)),
               "v": np.transpose(cache.v[:, :, p0:p0 + 1].double().cpu().numpy(), (0, 2, 1, 3))}
        ratios = {n: floor_ratios(got[n], pb[n], pe[n]) for n in got}
        print(f"[q4] {name} step {t}: out max/RMS vs floor oracle {mx:.3g}; vs exact max {mxe:.3g} rms {rmse:.3g}; "
              + " ".join(f"{n}=({r[0]:.2f},{r[1]:.2f})" for n, r in ratios.items()))
        for n, (r_rms, r_max) in ratios.items():
            assert r_rms <= 1.5 and r_max <= 2.0, f"{name} step {t}: {n} {r_rms:.3g} {r_max:.3g}"
        assert mx <= 1e-2 and rmse <= 1e-2 and mxe <= 5e-2


def test_q4_rejects_bad_shapes():
    dims = L.make_dims(1000, 8, 8, 125, 2816, 1e-5, 1e4, "half", "bf16")   # head_dim 125 unsupported
    t = torch.zeros(64, dtype=torch.int32, device="cuda")
    q = {k: (t, t, t) for k in PROJ}
    q.update(attn_norm=t, ffn_norm=t)
    lw = L.layer_weights_q4(q)
    with pytest.raises(L.LlamaError):
        L.layer_decode_q4(dims, lw, L.KVCache(L.make_dims(1024, 8, 8, 128, 2816, 1e-5), 1, 8), 1, t, t, t)
