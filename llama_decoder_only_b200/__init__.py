"""Python binding of the B200 decoder-block library (argument marshalling only).

Every call goes through the C ABI declared in ``include/llama_b200.h`` and
implemented by ``libllama_b200.so`` (built in-tree by ``build.py``).  There is
no fallback: if the library is missing or cannot be loaded, every entry point
raises ``LlamaError``.  PyTorch is used only to own device memory and to name
the CUDA stream.

The ``llama_*`` functions mirror the C names one to one and take raw
pointers / integers; the lower-case helpers (``layer_prefill`` ...) accept
torch tensors and pass their ``data_ptr()``.
"""

from __future__ import annotations

import ctypes
import os

from .build import LIB

__all__ = [
    "LlamaError", "Dims", "LayerWeights", "Model", "lib", "EXPORTS",
    "F32", "BF16", "ROPE_HALF", "ROPE_INTERLEAVED",
    "make_dims", "layer_weights", "model_struct", "KVCache",
    "workspace_size", "model_workspace_size", "layer_prefill", "layer_decode",
    "model_forward", "device_status", "workspace_offsets", "set_wait_limit_ns", "selftest_wait_timeout",
    "launch_count", "profile_enable", "profile_read", "profile_inflight", "attention_decode_noalloc",
    "sample_top_p", "model_forward_sample", "Q4Weight", "LayerWeightsQ4", "layer_weights_q4", "layer_decode_q4",
    "workspace_size_ragged", "layer_forward_ragged",
]

F32, BF16 = 0, 1
ROPE_HALF, ROPE_INTERLEAVED = 0, 1

STATUS = {
    0: "LLAMA_OK", 1: "LLAMA_ERR_INVALID_ARG", 2: "LLAMA_ERR_UNSUPPORTED", 3: "LLAMA_ERR_CACHE_FULL",
    4: "LLAMA_ERR_ALIGNMENT", 5: "LLAMA_ERR_WORKSPACE_TOO_SMALL", 6: "LLAMA_ERR_CUDA",
    7: "LLAMA_ERR_DEVICE_TIMEOUT", 8: "LLAMA_ERR_SCRATCH_LIMIT",
}


class LlamaError(RuntimeError):
    def __init__(self, status, what=""):
        self.status = int(status)
        super().__init__(f"{what}: {STATUS.get(self.status, self.status)}")


class Dims(ctypes.Structure):
    _fields_ = [("dim", ctypes.c_int32), ("n_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("ffn_dim", ctypes.c_int32), ("eps", ctypes.c_float),
                ("rope_theta", ctypes.c_float), ("rope_style", ctypes.c_int32), ("dtype", ctypes.c_int32)]


class LayerWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm", "w1", "w3", "w2")]


class Model(ctypes.Structure):
    _fields_ = [("dims", Dims), ("n_layers", ctypes.c_int32), ("vocab", ctypes.c_int32),
                ("embed", ctypes.c_void_p), ("final_norm", ctypes.c_void_p), ("lm_head", ctypes.c_void_p),
                ("layers", ctypes.POINTER(LayerWeights))]


class Q4Weight(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("offsets", ctypes.c_void_p)]


class LayerWeightsQ4(ctypes.Structure):
    _fields_ = [("attn_norm", ctypes.c_void_p), ("wq", Q4Weight), ("wk", Q4Weight), ("wv", Q4Weight),
                ("wo", Q4Weight), ("ffn_norm", ctypes.c_void_p), ("w1", Q4Weight), ("w3", Q4Weight),
                ("w2", Q4Weight)]


_P = ctypes.c_void_p
_I = ctypes.c_int32
_S = ctypes.c_size_t
_U64 = ctypes.c_uint64
_DP = ctypes.POINTER(Dims)
_WP = ctypes.POINTER(LayerWeights)
_MP = ctypes.POINTER(Model)

# name -> (restype, argtypes); the full export list of include/llama_b200.h
EXPORTS = {
    "llama_abi_version": (_I, []),
    "llama_status_string": (ctypes.c_char_p, [_I]),
    "llama_set_wait_limit_ns": (_U64, [_U64]),
    "llama_kv_cache_create": (_I, [_DP, _I, _I, _P, _P, ctypes.POINTER(_P)]),
    "llama_kv_cache_set_length": (_I, [_P, _I]),
    "llama_kv_cache_length": (_I, [_P]),
    "llama_kv_cache_capacity": (_I, [_P]),
    "llama_kv_cache_set_lengths": (_I, [_P, ctypes.POINTER(_I)]),
    "llama_kv_cache_lengths": (_I, [_P, ctypes.POINTER(_I)]),
    "llama_workspace_size_ragged": (_S, [_DP, _I, _I]),
    "llama_layer_forward_ragged": (_I, [_DP, _WP, _P, _I, ctypes.POINTER(_I), _P, _P, _P, _S, _P]),
    "llama_kv_cache_destroy": (None, [_P]),
    "llama_workspace_size": (_S, [_DP, _I, _I]),
    "llama_device_status": (_I, [_P, _I]),
    "llama_workspace_offsets": (_I, [_DP, _I, _I, ctypes.POINTER(_S), _I]),
    "llama_layer_prefill": (_I, [_DP, _WP, _P, _I, _I, _P, _P, _P, _S, _P]),
    "llama_layer_decode": (_I, [_DP, _WP, _P, _I, _P, _P, _P, _S, _P]),
    "llama_layer_decode_q4": (_I, [_DP, ctypes.POINTER(LayerWeightsQ4), _P, _I, _P, _P, _P, _S, _P]),
    "llama_model_workspace_size": (_S, [_MP, _I, _I]),
    "llama_model_forward": (_I, [_MP, ctypes.POINTER(_P), _P, _I, _I, _P, _P, _P, _S, _P]),
    "llama_selftest_wait_timeout": (_I, [_P, _U64, _P]),
    "llama_sample_top_p": (_I, [_P, _I, _I, ctypes.c_float, ctypes.c_float, _P, _P, _P]),
    "llama_model_forward_sample": (_I, [_MP, ctypes.POINTER(_P), _P, _I, _I, ctypes.c_float, ctypes.c_float, _P,
                                        _P, _P, _P, _S, _P]),
    "llama_attention_decode_noalloc": (_I, [_DP, _I, _P, _I, _P, _P, _I, _I, _P, _P]),
    "llama_launch_count": (_U64, []),
    "llama_profile_enable": (_I, [_I]),
    "llama_profile_inflight": (_I, [ctypes.POINTER(ctypes.c_char_p), _I]),
    "llama_profile_read": (_I, [ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(ctypes.c_double),
                                ctypes.POINTER(ctypes.c_longlong), _I, _I]),
}

_lib = None


def lib():
    """The loaded library (raises ``LlamaError`` if it is not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB):
            raise LlamaError(6, f"CUDA library not built ({LIB}); run python -m llama_decoder_only_b200.build")
        handle = ctypes.CDLL(LIB)
        for name, (res, args) in EXPORTS.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def _check(status, what):
    if status != 0:
        raise LlamaError(status, what)


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _ptr(t):
    return None if t is None else t.data_ptr()


# ------------------------------------------------------------------ structures

def make_dims(dim, n_heads, n_kv_heads, head_dim, ffn_dim, eps, rope_theta=10000.0,
              rope_style=ROPE_HALF, dtype=BF16):
    if isinstance(rope_style, str):
        rope_style = ROPE_HALF if rope_style == "half" else ROPE_INTERLEAVED
    if isinstance(dtype, str):
        dtype = BF16 if dtype == "bf16" else F32
    return Dims(dim, n_heads, n_kv_heads, head_dim, ffn_dim, eps, rope_theta, rope_style, dtype)


def layer_weights(t):
    """``LayerWeights`` from a dict of device tensors (keys attn_norm, wq, ... w2)."""
    return LayerWeights(*[_ptr(t[k]) for k in
                          ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm", "w1", "w3", "w2")])


def layer_weights_q4(t):
    """``LayerWeightsQ4`` from a dict: attn_norm, ffn_norm (device float32) and, for each of
    wq wk wv wo w1 w3 w2, a (codes, scales, offsets) triple of device tensors."""
    def q(k):
        c, sc, of = t[k]
        return Q4Weight(_ptr(c), _ptr(sc), _ptr(of))
    return LayerWeightsQ4(_ptr(t["attn_norm"]), q("wq"), q("wk"), q("wv"), q("wo"), _ptr(t["ffn_norm"]),
                          q("w1"), q("w3"), q("w2"))


def model_struct(dims, embed, final_norm, lm_head, layers):
    """``Model`` struct plus the ctypes array that must stay alive with it."""
    arr = (LayerWeights * len(layers))(*[layer_weights(w) for w in layers])
    m = Model(dims, len(layers), embed.shape[0], _ptr(embed), _ptr(final_norm), _ptr(lm_head),
              ctypes.cast(arr, ctypes.POINTER(LayerWeights)))
    return m, arr


class KVCache:
    """One layer's cache: device buffers (torch-owned) plus the library handle."""

    def __init__(self, dims, batch, capacity, device="cuda", k=None, v=None):
        import torch
        dt = torch.bfloat16 if dims.dtype == BF16 else torch.float32
        shape = (batch, dims.n_kv_heads, capacity, dims.head_dim)
        self.k = k if k is not None else torch.zeros(shape, dtype=dt, device=device)
        self.v = v if v is not None else torch.zeros(shape, dtype=dt, device=device)
        h = ctypes.c_void_p()
        _check(lib().llama_kv_cache_create(ctypes.byref(dims), batch, capacity, _ptr(self.k), _ptr(self.v),
                                           ctypes.byref(h)), "llama_kv_cache_create")
        self.handle = h
        self.batch, self.capacity = batch, capacity

    @property
    def length(self):
        return lib().llama_kv_cache_length(self.handle)

    def set_length(self, n):
        _check(lib().llama_kv_cache_set_length(self.handle, n), "llama_kv_cache_set_length")

    def set_lengths(self, lens):
        arr = (ctypes.c_int32 * self.batch)(*[int(x) for x in lens])
        _check(lib().llama_kv_cache_set_lengths(self.handle, arr), "llama_kv_cache_set_lengths")

    @property
    def lengths(self):
        arr = (ctypes.c_int32 * self.batch)()
        _check(lib().llama_kv_cache_lengths(self.handle, arr), "llama_kv_cache_lengths")
        return list(arr)

    def __del__(self):
        h = getattr(self, "handle", None)
        if h is not None and _lib is not None:
            _lib.llama_kv_cache_destroy(h)
            self.handle = None


# ------------------------------------------------------------------ calls

def workspace_size(dims, batch, seq_len):
    return lib().llama_workspace_size(ctypes.byref(dims), batch, seq_len)


def model_workspace_size(model, batch, seq_len):
    return lib().llama_model_workspace_size(ctypes.byref(model), batch, seq_len)


def layer_prefill(dims, w, cache, batch, seq_len, x_in, x_out, ws, stream=None):
    _check(lib().llama_layer_prefill(ctypes.byref(dims), ctypes.byref(w), cache.handle, batch, seq_len,
                                     _ptr(x_in), _ptr(x_out), _ptr(ws), ws.numel() * ws.element_size(),
                                     _stream(stream)), "llama_layer_prefill")


def layer_decode(dims, w, cache, batch, x_in, x_out, ws, stream=None):
    _check(lib().llama_layer_decode(ctypes.byref(dims), ctypes.byref(w), cache.handle, batch, _ptr(x_in),
                                    _ptr(x_out), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "llama_layer_decode")


def workspace_size_ragged(dims, batch, total_tokens):
    return lib().llama_workspace_size_ragged(ctypes.byref(dims), batch, total_tokens)


def layer_forward_ragged(dims, w, cache, n_new, x_in, x_out, ws, stream=None):
    """One block over a ragged batch: ``n_new[b]`` new tokens of sequence b, packed rows."""
    arr = (ctypes.c_int32 * len(n_new))(*[int(x) for x in n_new])
    _check(lib().llama_layer_forward_ragged(ctypes.byref(dims), ctypes.byref(w), cache.handle, len(n_new), arr,
                                            _ptr(x_in), _ptr(x_out), _ptr(ws), ws.numel() * ws.element_size(),
                                            _stream(stream)), "llama_layer_forward_ragged")


def layer_decode_q4(dims, w, cache, batch, x_in, x_out, ws, stream=None):
    _check(lib().llama_layer_decode_q4(ctypes.byref(dims), ctypes.byref(w), cache.handle, batch, _ptr(x_in),
                                       _ptr(x_out), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "llama_layer_decode_q4")


def model_forward(model, caches, tokens, batch, seq_len, logits, next_ids, ws, stream=None):
    arr = (ctypes.c_void_p * len(caches))(*[c.handle.value for c in caches])
    _check(lib().llama_model_forward(ctypes.byref(model), arr, _ptr(tokens), batch, seq_len, _ptr(logits),
                                     _ptr(next_ids), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "llama_model_forward")


def model_forward_sample(model, caches, tokens, batch, seq_len, temperature, top_p, u, logits, next_ids, ws,
                         stream=None):
    arr = (ctypes.c_void_p * len(caches))(*[c.handle.value for c in caches])
    _check(lib().llama_model_forward_sample(ctypes.byref(model), arr, _ptr(tokens), batch, seq_len,
                                            float(temperature), float(top_p), _ptr(u), _ptr(logits),
                                            _ptr(next_ids), _ptr(ws), ws.numel() * ws.element_size(),
                                            _stream(stream)), "llama_model_forward_sample")


def sample_top_p(logits, temperature, top_p, u, ids, stream=None):
    """ids [B] from logits [B, V] (device float32) and uniforms u [B] (device float32)."""
    B, V = logits.shape
    _check(lib().llama_sample_top_p(_ptr(logits), B, V, float(temperature), float(top_p), _ptr(u), _ptr(ids),
                                    _stream(stream)), "llama_sample_top_p")


def workspace_offsets(dims, batch, seq_len):
    """Offsets (bytes) of qkv, h, attn and m inside a layer call's workspace."""
    out = (_S * 4)()
    _check(lib().llama_workspace_offsets(ctypes.byref(dims), batch, seq_len, out, 4), "llama_workspace_offsets")
    return list(out)


def device_status(ws, clear=False):
    return lib().llama_device_status(_ptr(ws), 1 if clear else 0)


def launch_count():
    return int(lib().llama_launch_count())


def profile_enable(on=True):
    _check(lib().llama_profile_enable(1 if on else 0), "llama_profile_enable")


def profile_read(reset=True):
    """{kernel kind: (total ms, launches)} of the traced launches."""
    n = 32
    names = (ctypes.c_char_p * n)()
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_longlong * n)()
    k = lib().llama_profile_read(names, ms, cnt, n, 1 if reset else 0)
    return {names[i].decode(): (ms[i], cnt[i]) for i in range(min(k, n)) if cnt[i] > 0}


def profile_inflight(n=64):
    """Kinds of traced launches still running (non-blocking), oldest first."""
    names = (ctypes.c_char_p * n)()
    k = lib().llama_profile_inflight(names, n)
    return k, [names[i].decode() for i in range(min(k, n))]


def attention_decode_noalloc(dims, batch, q, ld_q, k_cache, v_cache, capacity, length, out, stream=None):
    """Decode attention with its scratch in the library's fixed array (see the C header)."""
    _check(lib().llama_attention_decode_noalloc(ctypes.byref(dims), batch, _ptr(q), ld_q, _ptr(k_cache),
                                                _ptr(v_cache), capacity, length, _ptr(out), _stream(stream)),
           "llama_attention_decode_noalloc")


def set_wait_limit_ns(ns):
    return lib().llama_set_wait_limit_ns(int(ns))


def selftest_wait_timeout(ws, limit_ns, stream=None):
    _check(lib().llama_selftest_wait_timeout(_ptr(ws), int(limit_ns), _stream(stream)),
           "llama_selftest_wait_timeout")
