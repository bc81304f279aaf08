"""Host-side checks of the C ABI (CPU only: nothing here launches a kernel).

* the library loads and exports every function ``include/llama_b200.h`` declares;
* argument validation rejects bad input before anything is enqueued
  (null pointers, unsupported shapes, misalignment, aliasing, cache overflow,
  a too-small workspace) and leaves the cache length unchanged;
* workspace sizing is monotone in the token count.

Fake device addresses are fine here: every rejected call returns before its
first CUDA call.
"""

import ctypes
import os
import re

import pytest

import llama_decoder_only_b200 as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "llama_b200.h")


def header_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(llama_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_function():
    lib = L.lib()
    declared = header_functions()
    assert len(declared) >= 15
    for name in declared:
        assert hasattr(lib, name), name
    assert set(declared) == set(L.EXPORTS)


def test_abi_version_and_status_strings():
    lib = L.lib()
    assert lib.llama_abi_version() == 1
    for s in range(8):
        assert lib.llama_status_string(s)
    assert lib.llama_status_string(99) == b"unknown status"


BF = dict(dim=512, n_heads=8, n_kv_heads=2, head_dim=64, ffn_dim=1376, eps=1e-5)
FAKE = 0x10000000  # aligned fake device address, never dereferenced


def dims(**kw):
    a = dict(BF, rope_theta=1e4, rope_style=L.ROPE_HALF, dtype=L.BF16)
    a.update(kw)
    return L.make_dims(**a)


def fake_weights(base=FAKE):
    return L.LayerWeights(*[base + i * 0x100000 for i in range(9)])


def cache(d, batch=2, cap=64):
    h = ctypes.c_void_p()
    st = L.lib().llama_kv_cache_create(ctypes.byref(d), batch, cap, FAKE, FAKE + 0x1000000, ctypes.byref(h))
    assert st == 0
    return h


@pytest.mark.parametrize("kw,expect", [
    (dict(n_heads=6, n_kv_heads=4), 1),       # not a multiple
    (dict(head_dim=48), 2),                   # unsupported head dim
    (dict(head_dim=32), 2),                   # 32 only on the fp32 path
    (dict(dim=100), 2),                       # dim % 8
    (dict(eps=0.0), 1),
    (dict(rope_theta=1.0), 1),
    (dict(rope_style=3), 1),
    (dict(dtype=7), 1),
    (dict(n_heads=24, n_kv_heads=2), 2),      # GQA group 12 not instantiated
])
def test_bad_dims_rejected(kw, expect):
    d = dims(**kw)
    assert L.lib().llama_workspace_size(ctypes.byref(d), 1, 16) == 0
    h = ctypes.c_void_p()
    assert L.lib().llama_kv_cache_create(ctypes.byref(d), 1, 16, FAKE, FAKE, ctypes.byref(h)) == expect


def test_fp32_head_dim_32_supported():
    d = dims(dtype=L.F32, head_dim=32)
    assert L.lib().llama_workspace_size(ctypes.byref(d), 1, 64) > 0


def test_cache_handle_lifecycle():
    d = dims()
    h = cache(d)
    lib = L.lib()
    assert lib.llama_kv_cache_length(h) == 0
    assert lib.llama_kv_cache_capacity(h) == 64
    assert lib.llama_kv_cache_set_length(h, 64) == 0
    assert lib.llama_kv_cache_set_length(h, 65) == 3        # LLAMA_ERR_CACHE_FULL
    assert lib.llama_kv_cache_set_length(h, -1) == 1
    assert lib.llama_kv_cache_length(None) == -1
    lib.llama_kv_cache_destroy(h)


def test_cache_create_rejects_null_and_misaligned():
    d = dims()
    h = ctypes.c_void_p()
    lib = L.lib()
    assert lib.llama_kv_cache_create(ctypes.byref(d), 1, 16, None, FAKE, ctypes.byref(h)) == 1
    assert lib.llama_kv_cache_create(ctypes.byref(d), 1, 16, FAKE + 8, FAKE, ctypes.byref(h)) == 4
    assert lib.llama_kv_cache_create(ctypes.byref(d), 0, 16, FAKE, FAKE, ctypes.byref(h)) == 1
    assert lib.llama_kv_cache_create(ctypes.byref(d), 1, 16, FAKE, FAKE, None) == 1


def _prefill(d, w, h, B, Lq, x_in, x_out, ws, ws_bytes):
    return L.lib().llama_layer_prefill(ctypes.byref(d), ctypes.byref(w), h, B, Lq, x_in, x_out, ws, ws_bytes, None)


def test_layer_call_validation_before_launch():
    d = dims()
    h = cache(d, batch=2, cap=64)
    w = fake_weights()
    lib = L.lib()
    need = lib.llama_workspace_size(ctypes.byref(d), 2, 16)
    X, Y, WS = 0x20000000, 0x30000000, 0x40000000
    assert _prefill(d, w, h, 2, 16, X, Y, WS, need - 1) == 5            # workspace too small
    assert _prefill(d, w, h, 2, 16, X, X + 256, WS, need) == 1          # x_out overlaps x_in
    assert _prefill(d, w, h, 2, 16, X + 4, Y, WS, need) == 4            # misaligned input
    assert _prefill(d, w, h, 3, 16, X, Y, WS, need) == 1                # batch != cache batch
    assert _prefill(d, w, h, 2, 0, X, Y, WS, need) == 1                 # empty call
    assert _prefill(d, w, h, 2, 65, X, Y, WS, 1 << 40) == 3             # exceeds capacity
    bad = fake_weights()
    bad.wk = None
    assert _prefill(d, bad, h, 2, 16, X, Y, WS, need) == 1              # null weight
    bad = fake_weights()
    bad.w2 = FAKE + 2
    assert _prefill(d, bad, h, 2, 16, X, Y, WS, need) == 4              # misaligned weight
    d2 = dims(ffn_dim=1408)
    assert _prefill(d2, w, h, 2, 16, X, Y, WS, need) == 1               # dims differ from the cache's
    assert lib.llama_kv_cache_length(h) == 0                            # nothing advanced
    lib.llama_kv_cache_destroy(h)


def test_decode_rejects_full_cache():
    d = dims()
    h = cache(d, batch=1, cap=8)
    lib = L.lib()
    lib.llama_kv_cache_set_length(h, 8)
    w = fake_weights()
    st = lib.llama_layer_decode(ctypes.byref(d), ctypes.byref(w), h, 1, 0x20000000, 0x30000000, 0x40000000,
                                1 << 40, None)
    assert st == 3
    assert lib.llama_kv_cache_length(h) == 8
    lib.llama_kv_cache_destroy(h)


def test_workspace_grows_with_tokens():
    d = dims()
    lib = L.lib()
    sizes = [lib.llama_workspace_size(ctypes.byref(d), 1, n) for n in (1, 64, 512, 4096)]
    assert all(a < b for a, b in zip(sizes, sizes[1:]))


def test_workspace_tensors_start_past_the_fixed_header():
    """The first 4096 bytes of every workspace (status word, decode-GEMM flags,
    chunk and tile counters) sit at the same place for every call shape and are
    never part of a tensor: a prefill call's data must not land on the words a
    later decode call expects to read zero, whatever the two calls' shapes."""
    header = 4096
    for dims in [L.make_dims(4096, 32, 32, 128, 11008, 1e-6, 1e4, "half", "bf16"),
                 L.make_dims(3072, 32, 32, 96, 8192, 1e-5, 1e4, "half", "bf16"),
                 L.make_dims(256, 8, 2, 32, 688, 1e-5, 1e4, "half", "f32")]:
        for batch, seq_len in [(1, 1), (16, 1), (64, 1), (1, 2048), (2, 4096), (8, 512)]:
            offs = L.workspace_offsets(dims, batch, seq_len)
            assert min(offs) >= header, (batch, seq_len, offs)
            assert all(o % 256 == 0 for o in offs)
            assert L.workspace_size(dims, batch, seq_len) > max(offs)


def test_model_call_validation():
    d = dims()
    lib = L.lib()
    layers = (L.LayerWeights * 2)(fake_weights(), fake_weights())
    m = L.Model(d, 2, 1000, FAKE, FAKE, FAKE, ctypes.cast(layers, ctypes.POINTER(L.LayerWeights)))
    need = lib.llama_model_workspace_size(ctypes.byref(m), 2, 8)
    assert need > lib.llama_workspace_size(ctypes.byref(d), 2, 8)
    h0, h1 = cache(d, 2, 16), cache(d, 2, 16)
    arr = (ctypes.c_void_p * 2)(h0.value, h1.value)
    call = lambda ws_bytes, tok=0x50000000: lib.llama_model_forward(  # noqa: E731
        ctypes.byref(m), arr, tok, 2, 8, None, 0x60000000, 0x40000000, ws_bytes, None)
    assert call(need - 1) == 5
    assert call(need, tok=0x50000004) == 4
    lib.llama_kv_cache_set_length(h1, 3)                                # lengths disagree
    assert call(need) == 1
    lib.llama_kv_cache_destroy(h0)
    lib.llama_kv_cache_destroy(h1)


def test_selftest_rejects_bad_args():
    lib = L.lib()
    assert lib.llama_selftest_wait_timeout(None, 1000, None) == 1
    assert lib.llama_selftest_wait_timeout(FAKE + 4, 1000, None) == 4
    assert lib.llama_selftest_wait_timeout(FAKE, 10 ** 10, None) == 1


def test_noalloc_attention_validates_before_any_launch():
    """Every rejection of the allocation-free decode attention happens on the
    host, before the library touches the device: too large for its fixed
    scratch (SCRATCH_LIMIT), fp32 dims (UNSUPPORTED), bad sizes (INVALID_ARG),
    misaligned pointers or ld_q (ALIGNMENT)."""
    lib = L.lib()
    d = L.make_dims(8192, 64, 8, 128, 28672, 1e-5, 1e4, "half", "bf16")
    q, k, v, o = FAKE, FAKE + (1 << 30), FAKE + (2 << 30), FAKE + (3 << 30)
    call = lambda dd, b, qq, ld, kk, vv, cap, n, oo: lib.llama_attention_decode_noalloc(  # noqa: E731
        ctypes.byref(dd), b, qq, ld, kk, vv, cap, n, oo, None)
    # 1024 sequences x 64 heads x 130 floats x 2 splits x 4 bytes = 68 MB > 8 MiB
    assert call(d, 1024, q, 64 * 128, k, v, 4096, 100, o) == 8
    f32 = L.make_dims(8192, 64, 8, 128, 28672, 1e-5, 1e4, "half", "f32")
    assert call(f32, 1, q, 64 * 128, k, v, 4096, 100, o) == 2
    assert call(d, 1, q, 64 * 128, k, v, 100, 101, o) == 1          # length > capacity
    assert call(d, 1, q, 64 * 128 - 8, k, v, 4096, 100, o) == 1     # ld_q < n_heads * head_dim
    assert call(d, 1, None, 64 * 128, k, v, 4096, 100, o) == 1
    assert call(d, 1, q + 8, 64 * 128, k, v, 4096, 100, o) == 4     # misaligned q
    assert call(d, 1, q, 64 * 128 + 4, k, v, 4096, 100, o) == 4     # ld_q not a multiple of 8


# ------------------------------------------------------------------ ragged batches, 4-bit weights, sampling

def test_ragged_lengths_and_validation():
    lib = L.lib()
    d = dims()
    h = cache(d, batch=3, cap=64)
    lens = (ctypes.c_int32 * 3)(5, 9, 5)
    assert lib.llama_kv_cache_set_lengths(h, lens) == 0
    assert lib.llama_kv_cache_length(h) == -2
    out = (ctypes.c_int32 * 3)()
    assert lib.llama_kv_cache_lengths(h, out) == 0 and list(out) == [5, 9, 5]
    # a uniform call refuses a cache whose lengths differ (before any launch)
    w = fake_weights()
    ws = lib.llama_workspace_size(ctypes.byref(d), 3, 1)
    assert lib.llama_layer_decode(ctypes.byref(d), ctypes.byref(w), h, 3, FAKE, FAKE + 0x4000000, FAKE + 0x8000000,
                                  ws, None) == 1
    n_new = (ctypes.c_int32 * 3)(1, 60, 1)          # 9 + 60 > 64
    wsr = lib.llama_workspace_size_ragged(ctypes.byref(d), 3, 62)
    assert wsr > 0
    assert lib.llama_layer_forward_ragged(ctypes.byref(d), ctypes.byref(w), h, 3, n_new, FAKE, FAKE + 0x4000000,
                                          FAKE + 0x8000000, wsr, None) == 3
    n_new = (ctypes.c_int32 * 3)(1, 0, 1)           # every sequence brings at least one token
    assert lib.llama_layer_forward_ragged(ctypes.byref(d), ctypes.byref(w), h, 3, n_new, FAKE, FAKE + 0x4000000,
                                          FAKE + 0x8000000, wsr, None) == 1
    n_new = (ctypes.c_int32 * 3)(1, 2, 1)
    small = lib.llama_workspace_size_ragged(ctypes.byref(d), 3, 3)
    assert lib.llama_layer_forward_ragged(ctypes.byref(d), ctypes.byref(w), h, 3, n_new, FAKE, FAKE + 0x4000000,
                                          FAKE + 0x8000000, small, None) == 5
    assert out[1] == 9 and lib.llama_kv_cache_lengths(h, out) == 0 and list(out) == [5, 9, 5]   # unchanged
    assert lib.llama_workspace_size_ragged(ctypes.byref(d), 129, 200) == 0                        # > 128 sequences
    assert lib.llama_workspace_size_ragged(ctypes.byref(d), 3, 62) >= lib.llama_workspace_size_ragged(
        ctypes.byref(d), 3, 3)
    equal = (ctypes.c_int32 * 3)(7, 7, 7)
    assert lib.llama_kv_cache_set_lengths(h, equal) == 0 and lib.llama_kv_cache_length(h) == 7
    big = (ctypes.c_int32 * 3)(7, 65, 7)
    assert lib.llama_kv_cache_set_lengths(h, big) == 3
    lib.llama_kv_cache_destroy(h)


def test_q4_layer_validation():
    lib = L.lib()
    d = dims(ffn_dim=1408)                                                      # every K a multiple of 64
    h = cache(d, batch=2, cap=64)
    q = L.Q4Weight(FAKE, FAKE + 0x100000, FAKE + 0x200000)
    w = L.LayerWeightsQ4(FAKE, q, q, q, q, FAKE, q, q, q)
    ws = lib.llama_workspace_size(ctypes.byref(d), 2, 1)
    bad = L.LayerWeightsQ4(FAKE, q, q, L.Q4Weight(FAKE + 4, FAKE, FAKE), q, FAKE, q, q, q)
    assert lib.llama_layer_decode_q4(ctypes.byref(d), ctypes.byref(bad), h, 2, FAKE, FAKE + 0x4000000,
                                     FAKE + 0x8000000, ws, None) == 4          # misaligned codes
    d1 = dims(ffn_dim=1352)                                                     # 1352 % 64 != 0
    h1 = cache(d1, batch=2, cap=64)
    assert lib.llama_layer_decode_q4(ctypes.byref(d1), ctypes.byref(w), h1, 2, FAKE, FAKE + 0x4000000,
                                     FAKE + 0x8000000, lib.llama_workspace_size(ctypes.byref(d1), 2, 1), None) == 2
    assert lib.llama_layer_decode_q4(ctypes.byref(d), ctypes.byref(w), h, 2, FAKE, FAKE + 0x4000000,
                                     FAKE + 0x8000000, ws - 1, None) == 5      # workspace too small
    assert lib.llama_kv_cache_length(h) == 0
    lib.llama_kv_cache_destroy(h)
    lib.llama_kv_cache_destroy(h1)


@pytest.mark.parametrize("t,p,u,expect", [
    (-1.0, 0.9, FAKE, 1), (float("nan"), 0.9, FAKE, 1), (1.0, 0.0, FAKE, 1), (1.0, 1.01, FAKE, 1),
    (1.0, 0.9, None, 1), (1.0, 0.9, FAKE + 4, 4),
])
def test_sampling_validation(t, p, u, expect):
    lib = L.lib()
    assert lib.llama_sample_top_p(FAKE, 2, 100, t, p, u, FAKE + 0x100000, None) == expect


# runs last: it reloads the binding
def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    import importlib
    monkeypatch.setattr(L, "_lib", None)
    monkeypatch.setattr(L, "LIB", str(tmp_path / "missing.so"))
    with pytest.raises(L.LlamaError):
        L.lib()
    importlib.reload(L)
