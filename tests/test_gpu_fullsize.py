"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark times, checked on outputs the fp64 oracle can compute row by row.

* 7B-shaped prefill (1 x 2048): sampled query rows (the oracle computes K/V
  for every row and the rest of the block for the sampled rows only).
* 13B-shaped decode (batch 16, 4096-position cache, interleaved RoPE): three
  decode steps, sampled sequences (sequences are independent).
* 70B-shaped GQA layer: prefill 2 x 4096 on sampled rows; decode at batch 64
  on a 4096-position cache, sampled sequences.
* Phi-3-mini-shaped model: 2 full-width layers against the oracle (logits and
  argmax ids), and the full 32-layer model against properties that hold at
  any size: decode with the cache reproduces the prefill's last-row logits,
  and the ids are the argmax of the logits.

Tolerances.  At these widths the FFN branch dominates the block output, and
rounding the GEMM operands to bf16 -- which any bf16 tensor-core block must
do -- already moves the output by up to ~1.8e-2 x RMS (max-abs) against the
exact fp64 result; the bf16-rounded oracle is no closer to the exact result
than the GPU is, and the two round differently once any upstream element
lands one ulp apart.  So each full-size check asserts
  * RMS error <= 1e-2 x RMS against the exact oracle, and
  * error against the exact oracle within 1.5x (RMS) and 2x (max-abs) of the
    bf16 floor, i.e. of the bf16-rounded oracle's own error,
and prints the literal max-abs / RMS numbers.
"""

import numpy as np
import pytest

import llama_decoder_only_b200 as L
import synth
from oracle import block as ob
from synth import device as sd
from tests.harness import LayerRun, floor_ratios, oracle_dims, rel_errors

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
torch = pytest.importorskip("torch")

BF16_EXACT_RMS = 1e-2
FLOOR_RMS = 1.5
FLOOR_MAX = 2.0


def _check(label, y, yb, ye, absolute_rms=True):
    mx, _ = rel_errors(y, yb)
    mxe, rmse = rel_errors(y, ye)
    fmx, frms = rel_errors(yb, ye)
    r_rms, r_max = floor_ratios(y, yb, ye)
    print(f"[fullsize] {label}: vs exact max/RMS {mxe:.3g} rms/RMS {rmse:.3g}; bf16 floor max {fmx:.3g} "
          f"rms {frms:.3g}; ratio to floor rms {r_rms:.2f} max {r_max:.2f}; vs bf16-oracle max {mx:.3g}")
    if absolute_rms:
        assert rmse <= BF16_EXACT_RMS, label
    assert r_rms <= FLOOR_RMS and r_max <= FLOOR_MAX, label


def test_llama7b_prefill_full_size_sampled_rows():
    w = synth.WORKLOADS["llama7b_prefill"]
    inp = synth.prefill_inputs(w, with_steps=False)
    run = LayerRun(w, inp.weights, w.batch, w.prefill_len, w.prefill_len)
    y = run.step(inp.x)
    rows = [0, 1, 127, 128, 129, 1000, 2046, 2047]
    d = oracle_dims(w)
    yb, _ = ob.layer_forward(d, inp.weights, inp.x, ob.KVCache(1, w.n_kv_heads, w.head_dim, w.prefill_len),
                             rounding="bf16", rows=rows)
    ye, _ = ob.layer_forward(d, inp.weights, inp.x, ob.KVCache(1, w.n_kv_heads, w.head_dim, w.prefill_len),
                             rows=rows)
    _check("llama7b prefill", y[:, rows], yb, ye)


def _decode_full(name, seqs, steps=3):
    w = synth.WORKLOADS[name]
    inp = synth.decode_inputs(w, steps=steps)
    B, T0 = w.decode_batch, w.cache_len
    run = LayerRun(w, inp.weights, B, T0 + steps, 1, k0=inp.k_cache, v0=inp.v_cache)
    d = oracle_dims(w)
    kb = inp.k_cache[seqs].astype(np.float64)
    vb = inp.v_cache[seqs].astype(np.float64)
    cb = ob.KVCache(len(seqs), w.n_kv_heads, w.head_dim, T0 + steps, kb, vb)
    ce = ob.KVCache(len(seqs), w.n_kv_heads, w.head_dim, T0 + steps, kb.copy(), vb.copy())
    for t, xs in enumerate(inp.steps):
        y = run.step(xs)
        yb, _ = ob.layer_forward(d, inp.weights, xs[seqs], cb, rounding="bf16")
        ye, _ = ob.layer_forward(d, inp.weights, xs[seqs], ce)
        _check(f"{name} decode step {t}", y[seqs], yb, ye)


def test_llama13b_decode_full_size_sampled_sequences():
    _decode_full("llama13b_decode", [0, 7, 15])


def test_gqa70b_decode_full_size_sampled_sequences():
    _decode_full("gqa70b", [0, 33, 63], steps=2)


def test_gqa70b_prefill_full_size_sampled_rows():
    w = synth.WORKLOADS["gqa70b"]
    inp = synth.prefill_inputs(w, with_steps=False)
    run = LayerRun(w, inp.weights, w.batch, w.prefill_len, w.prefill_len)
    y = run.step(inp.x)
    rows = [0, 129, 4095]
    d = oracle_dims(w)
    yb, _ = ob.layer_forward(d, inp.weights, inp.x, ob.KVCache(2, w.n_kv_heads, w.head_dim, w.prefill_len),
                             rounding="bf16", rows=rows)
    ye, _ = ob.layer_forward(d, inp.weights, inp.x, ob.KVCache(2, w.n_kv_heads, w.head_dim, w.prefill_len),
                             rows=rows)
    _check("gqa70b prefill", y[:, rows], yb, ye)


# ------------------------------------------------------------------ whole model

class ModelRun:
    def __init__(self, w, M, batch, capacity, max_tokens, device_weights=None):
        self.w = w
        self.dims = L.make_dims(w.dim, w.n_heads, w.n_kv_heads, w.head_dim, w.ffn_dim, w.eps, w.rope_theta,
                                w.rope_style, w.dtype)
        if device_weights is not None:
            self.layers, self.emb, self.fn, self.lm = device_weights
        else:
            self.layers = [sd.upload_layer(W, w.dtype) for W in M["layers"]]
            self.emb = sd.to_device(M["embed"], w.dtype)
            self.lm = sd.to_device(M["lm_head"], w.dtype)
            self.fn = sd.to_device(M["final_norm"], "f32")
        self.model, self.keep = L.model_struct(self.dims, self.emb, self.fn, self.lm, self.layers)
        self.caches = [L.KVCache(self.dims, batch, capacity) for _ in self.layers]
        nbytes = max(L.model_workspace_size(self.model, batch, max_tokens),
                     L.model_workspace_size(self.model, batch, 1))
        self.ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
        self.batch = batch

    def forward(self, tokens):
        B, S = tokens.shape
        tok = torch.from_numpy(np.ascontiguousarray(tokens, np.int32)).cuda()
        logits = torch.empty(B, self.w.vocab, dtype=torch.float32, device="cuda")
        ids = torch.empty(B, dtype=torch.int32, device="cuda")
        L.model_forward(self.model, self.caches, tok, B, S, logits, ids, self.ws)
        torch.cuda.synchronize()
        assert L.device_status(self.ws) == 0
        return logits.double().cpu().numpy(), ids.cpu().numpy()


def _ids_agree(ids, logits_ref, tol):
    """Ids must match the oracle's argmax wherever its top-2 gap exceeds tol."""
    top2 = np.sort(logits_ref, axis=-1)[:, -2:]
    decisive = (top2[:, 1] - top2[:, 0]) > tol
    ref = ob.greedy_argmax(logits_ref)
    return bool(np.all(ids[decisive] == ref[decisive])), int(decisive.sum())


def test_phi3_two_layer_model_vs_oracle():
    w = synth.shrink(synth.WORKLOADS["phi3mini_model"], n_layers=2)
    M = synth.model_weights(w, n_layers=2)
    prompt, forced = synth.model_tokens(w, batch=2, prefill_len=96, steps=2)
    run = ModelRun(w, M, 2, 128, 96)
    d = oracle_dims(w)
    cb = [ob.KVCache(2, w.n_kv_heads, w.head_dim, 128) for _ in range(2)]
    ce = [ob.KVCache(2, w.n_kv_heads, w.head_dim, 128) for _ in range(2)]
    for t, tok in enumerate([prompt] + [f[:, None] for f in forced]):
        logits, ids = run.forward(tok)
        lb, _ = ob.model_forward(d, M, tok, cb, rounding="bf16")
        le, _ = ob.model_forward(d, M, tok, ce)
        # logits: held to the bf16 floor (whose own RMS error is ~1.1e-2 here)
        _check(f"phi3 2-layer logits call {t}", logits, lb, le, absolute_rms=False)
        # ids must agree wherever the exact oracle's top-2 gap exceeds 1e-2 x RMS(logits)
        # plus the largest logit error the bf16 floor allows (2x the rounded oracle's)
        floor = float(np.max(np.abs(lb - le)))
        tol = 1e-2 * float(np.sqrt(np.mean(le * le))) + 2 * floor
        ok, n = _ids_agree(ids, le, tol)
        print(f"[fullsize] phi3 2-layer call {t}: ids agree on {n} decisive rows of {len(ids)}")
        assert ok, f"argmax disagreement on decisive rows (call {t})"
        assert np.array_equal(ids, np.argmax(logits, axis=-1))


def test_phi3_full_model_properties():
    # full size: 32 layers, vocab 32064, B 8 (fewer prompt tokens keep it quick)
    w = synth.WORKLOADS["phi3mini_model"]
    # weights drawn on the device (same distribution): nothing here needs the oracle
    g = torch.Generator(device="cuda")
    g.manual_seed(w.seed)
    layers = [sd.random_layer_on_device(w, w.seed + 1 + i) for i in range(w.n_layers)]
    emb = (torch.randn(w.vocab, w.dim, generator=g, device="cuda") * w.w_std).to(torch.bfloat16)
    lm = (torch.randn(w.vocab, w.dim, generator=g, device="cuda") * w.w_std).to(torch.bfloat16)
    fn = torch.ones(w.dim, device="cuda", dtype=torch.float32)
    dw = (layers, emb, fn, lm)
    prompt, _ = synth.model_tokens(w, prefill_len=129, steps=0)
    a = ModelRun(w, None, 8, 160, 129, device_weights=dw)
    full_logits, full_ids = a.forward(prompt)
    assert np.all(np.isfinite(full_logits))
    assert np.array_equal(full_ids, np.argmax(full_logits, axis=-1))
    # prefill of 128 tokens then one decode step of token 129 == prefill of 129
    b = ModelRun(w, None, 8, 160, 128, device_weights=dw)
    b.forward(prompt[:, :128])
    dec_logits, dec_ids = b.forward(prompt[:, 128:129])
    mx, rms = rel_errors(dec_logits, full_logits)
    print(f"[fullsize] phi3 32-layer decode vs prefill logits: max/RMS {mx:.3g} rms {rms:.3g}")
    # Two bf16 evaluations that round differently drift apart by about the
    # per-layer floor (~4e-3 RMS) times sqrt(layers): sqrt(32) * 4e-3 ~ 2.3e-2.
    assert rms <= 3.5e-2
    # where the logit gap exceeds twice the largest difference, the ids are fixed
    delta = float(np.max(np.abs(dec_logits - full_logits)))
    ok, n = _ids_agree(dec_ids, full_logits, 2 * delta)
    assert ok
