"""Plain fp64 CPU oracle of the LLaMA-style pre-norm decoder block.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
link this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code with the CUDA path (no kernels, headers, helpers, tables or constant
generators); the only module both sides read is ``synth`` (seeded inputs).

Modules
-------
block  -- NumPy float64 definition of every step (norm, projections, RoPE in
          both styles, KV-cache append, causal GQA attention, SwiGLU, residual
          wiring, embedding, final norm, lm_head, greedy argmax).
brute  -- pure-Python (``math`` only) triple-loop restatement of the same
          block, used to cross-check ``block`` on tiny shapes.
quant  -- the 4-bit group-64 quantised Linear the pages name (group-wise
          affine codes, packing, dequantised product), the oracle of the next
          row of the build; pinned by ``tests/test_oracle_quant.py``.
sampling -- temperature / top-p (nucleus) sampling after the lm_head, with
          the uniform draw as an input; pinned by ``tests/test_oracle_sampling.py``.

Parity status: every function in ``block`` is pinned by the CPU tests in
``tests/test_oracle_*.py`` (closed forms, invariants, library special cases,
brute force).  One reading is pinned only through an identity:
the interleaved ("traditional") RoPE variant, which the pages name but never
define; it is pinned by its permutation identity with the rotate-half form
(the pages print no value computed with it).
"""

from . import block, brute  # noqa: F401
