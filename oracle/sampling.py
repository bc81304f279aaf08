"""fp64 oracle of temperature / top-p (nucleus) sampling (test infrastructure).

TEST INFRASTRUCTURE ONLY: imported by ``tests/`` and never by the product
path.  It shares no code with the CUDA library.

What the pages fix ([DeepDive] class LLaMA, ``generate``; [MLX-13B]
"生成过程"): the last position's logits are divided by the temperature, sorted
in descending order, and turned into cumulative softmax probabilities; a
token is dropped when the cumulative probability of the tokens sorted before
it already exceeds ``top_p`` (the first token is always kept, so the token
that crosses the threshold stays); the kept logits are renormalised by a
softmax and one token is drawn from them.  Temperature 0 means greedy argmax
([MLX-13B]: "temp=0 时使用贪心搜索（argmax）").

Readings (listed in the design notes): the random draw is an input -- one
uniform ``u`` in [0, 1) per sequence -- and the token is picked by inverse CDF
over the kept tokens in the sorted order (the first kept token whose
cumulative renormalised probability exceeds ``u``); equal logits sort by
ascending vocabulary index.
"""

from __future__ import annotations

import numpy as np

from .block import greedy_argmax


def nucleus(logits_row, temperature, top_p):
    """(sorted vocabulary ids, renormalised probabilities of the kept prefix) of one row."""
    z = np.asarray(logits_row, np.float64) / float(temperature)
    V = z.shape[0]
    order = np.lexsort((np.arange(V), -z))          # descending logit, ties by index
    zs = z[order]
    p = np.exp(zs - zs[0])
    p /= p.sum()
    before = np.concatenate([[0.0], np.cumsum(p)[:-1]])   # probability of the tokens sorted before
    keep = before <= top_p
    keep[0] = True
    k = int(np.argmin(keep)) if not keep.all() else V      # kept tokens form a prefix
    q = p[:k] / p[:k].sum()
    return order[:k], q


def sample_top_p(logits, temperature, top_p, u):
    """Next ids [B] from logits [B, V] and uniforms u [B] in [0, 1)."""
    logits = np.asarray(logits, np.float64)
    if temperature == 0:
        return greedy_argmax(logits)
    out = np.empty(logits.shape[0], np.int64)
    for b in range(logits.shape[0]):
        ids, q = nucleus(logits[b], temperature, top_p)
        c = np.cumsum(q)
        j = int(np.searchsorted(c, float(u[b]), side="right"))
        out[b] = ids[min(j, len(ids) - 1)]
    return out
