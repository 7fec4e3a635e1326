"""Float64 CPU oracle for TurboQuant KV-cache quantization.

TEST INFRASTRUCTURE ONLY. Nothing in the product path may import, call or
execute this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it. It shares
no code, tables or constants with the CUDA library under
``kv_cache_vector_quantize_b200/``; the two meet only in the seeded input
generators of ``tq_synth``.

What it computes, and the pages it follows:

* ``codebook`` -- the law of one coordinate of a uniformly random unit vector
  (a Beta-shaped density on [-1, 1]) and a Lloyd-Max scalar quantizer fitted
  to it. Pages: zubnet.ai news, "Google's TurboQuant quantizes LLM KV cache
  to 3.5 bits per channel" (es/pt/fr editions), second paragraph: the random
  rotation concentrates coordinates in a Beta distribution, so an optimal
  per-coordinate scalar quantizer applies.
* ``turboquant`` -- the two-stage encoder (rotation, MSE quantizer, 1-bit
  Johnson-Lindenstrauss sketch of the residual, L2 norm), the record packer,
  the attention-logit estimator on the packed cache and softmax-weighted V.
  Pages: the same zubnet.ai paragraph (storage = quantization indices, sign
  bits and an L2-norm scalar); winningdata.io, "TurboQuant: Google comprime
  KV cache para 3 bits sem perder acuracia", section "Como o TurboQuant
  funciona" (1. PolarQuant: multiply by a random orthogonal matrix;
  2. QJL Residual: one extra bit per value removes the inner-product bias).

* ``mixed_rate`` -- fractional bits per channel (the 3.5 and 2.5 bits per
  channel of the zubnet.ai title and paragraph 2): the first m rotated
  coordinates at one more code bit than the rest, each group with its own
  Lloyd-Max codebook of the same law; encoder, packer, estimator, softmax.V.

The pages print no estimator formula, codebook, QJL constant or layout; the
readings taken where they are silent are listed in the module docstrings and
marked "reading:".

Parity status: every function here is pinned by tests under ``tests/`` that
use closed forms, textbook special cases, an independently tabulated codebook
and MSE table at finite d, brute force or Monte Carlo. ``turboquant.topk`` is an
ordering convention (largest first, equal scores by lower index), pinned by a
hand-worked case; ``turboquant.padding_is_zero`` is pinned by planting a stray
bit at every unused position of a record.
"""

from . import codebook, mixed_rate, turboquant  # noqa: F401
