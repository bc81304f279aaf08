"""fp64 oracle of the 4-bit group-wise quantised Linear (test infrastructure).

TEST INFRASTRUCTURE ONLY: imported by ``tests/`` and never by the product
path.  It shares no code with the CUDA library.

What the pages fix: [MLX-13B] "LLaMA 2 的结构分析" lists every projection of the
13B block (wq, wk, wv, wo, w1, w2, w3 and the output layer) as
``QuantizedLinear(input_dims=..., output_dims=...)``, and its config.json
("模型配置") carries ``"quantization": {"group_size": 64, "bits": 4}``.  They
name the scheme but never define it.

Reading taken (the plainest one those two facts support, listed in the design
notes): group-wise affine quantisation along the input dimension.  Each weight
row is cut into groups of ``group_size`` consecutive inputs; a group keeps a
scale ``s`` and an offset ``b``, and each weight of the group an unsigned code
``q`` in ``[0, 2**bits - 1]``, so that the Linear uses ``w = s * q + b``.  From
a float weight, ``b`` is the group minimum, ``s = (max - min) / (2**bits - 1)``
and ``q = round((w - b) / s)`` (nearest, ties to even; ``s = 0`` for a
constant group, whose codes are 0).  Codes are packed eight to a 32-bit word,
code ``k`` of the word in bits ``4k .. 4k+3`` (low nibble first).  The Linear
is then ``y = x W^T`` with the dequantised ``W`` ([DeepDive] nn.Linear,
bias-free), in float64.
"""

from __future__ import annotations

import numpy as np


def quantize(w, group_size=64, bits=4):
    """Float weight [out, in] -> (codes uint8 [out, in], scales, offsets [out, in/group_size]).

    The reading above: per group, offset = min, scale = (max - min) / (2**bits - 1),
    code = round((w - offset) / scale).
    """
    w = np.asarray(w, np.float64)
    out_f, in_f = w.shape
    if in_f % group_size:
        raise ValueError("in_features must be a multiple of group_size")
    g = w.reshape(out_f, in_f // group_size, group_size)
    lo = g.min(axis=2)
    hi = g.max(axis=2)
    levels = (1 << bits) - 1
    scale = (hi - lo) / levels
    safe = np.where(scale > 0, scale, 1.0)
    q = np.rint((g - lo[..., None]) / safe[..., None])
    q = np.where(scale[..., None] > 0, q, 0.0)
    q = np.clip(q, 0, levels).astype(np.uint8)
    return q.reshape(out_f, in_f), scale, lo


def dequantize(codes, scales, offsets, group_size=64):
    """w[o, i] = scales[o, i // group_size] * codes[o, i] + offsets[o, i // group_size]."""
    codes = np.asarray(codes, np.float64)
    out_f, in_f = codes.shape
    s = np.repeat(np.asarray(scales, np.float64), group_size, axis=1)
    b = np.repeat(np.asarray(offsets, np.float64), group_size, axis=1)
    assert s.shape == (out_f, in_f)
    return s * codes + b


def pack_int4(codes):
    """uint8 codes [out, in] (values 0..15, in % 8 == 0) -> uint32 words [out, in/8],
    code 8j+k of a row in bits 4k..4k+3 of word j."""
    c = np.asarray(codes, np.uint32)
    out_f, in_f = c.shape
    if in_f % 8 or c.max(initial=0) > 15:
        raise ValueError("need in % 8 == 0 and codes in 0..15")
    c = c.reshape(out_f, in_f // 8, 8)
    words = np.zeros((out_f, in_f // 8), np.uint32)
    for k in range(8):
        words |= c[:, :, k] << np.uint32(4 * k)
    return words


def unpack_int4(words, in_features):
    """Inverse of ``pack_int4``."""
    wds = np.asarray(words, np.uint32)
    out_f = wds.shape[0]
    c = np.zeros((out_f, wds.shape[1], 8), np.uint8)
    for k in range(8):
        c[:, :, k] = (wds >> np.uint32(4 * k)) & np.uint32(15)
    return c.reshape(out_f, -1)[:, :in_features]


def quantized_linear(x, words, scales, offsets, in_features, group_size=64):
    """y = x W^T with W the dequantised packed weight ([MLX-13B] QuantizedLinear;
    [DeepDive] nn.Linear without bias), float64."""
    w = dequantize(unpack_int4(words, in_features), scales, offsets, group_size)
    return np.asarray(x, np.float64) @ w.T
