"""CPU oracle for TurboQuant-style vector quantization -- TEST INFRASTRUCTURE ONLY.

This package is a plain, slow, fp64 NumPy restatement of what the quantization
hot path computes. It exists to check the CUDA library against, and for nothing
else:

* only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
  ``--impl reference`` legs of ``bench.py`` may import it;
* the library (``embedding_vector_quantization_b200``) never imports it, and the
  two share no code, tables or constants: the only shared module is the seeded
  synthetic-input generator, which holds none of the method's arithmetic.

Sources (web pages on the method; cited by page title and section):

* "Google TurboQuant: 6x KV-cache compression" (ebisuda.net) -- sections
  "Stage 1: PolarQuant (MSE-optimal compression)" and "Stage 2: QJL residual
  correction (1 bit)". The most concrete description of the algorithm.
* "TurboQuant / PolarQuant / QJL technical deep dive" (gemilab.net) -- sections
  "KV cache basics: the attention mechanism", "PolarQuant: Cartesian to polar",
  "QJL: error correction via the Johnson-Lindenstrauss lemma".
* "TurboQuant: redefining AI efficiency with extreme compression"
  (hakusoku.com) -- sections "PolarQuant", "QJL: zero-overhead 1-bit
  compression", "Impact on high-dimensional vector search".

Where the pages leave a step open, the reading taken is stated in the function
that implements it. Modules:

* :mod:`oracle.rng`      -- SplitMix64 + Box-Muller Gaussian stream (spec).
* :mod:`oracle.rotation` -- seeded Haar rotation Pi (QR of a Gaussian) and QJL matrix S.
* :mod:`oracle.codebook` -- Lloyd-Max codebook on the sphere-coordinate density.
* :mod:`oracle.quant`    -- encode (norm, rotate, bucketize, pack), QJL sketch, dequantize;
  the QJL-only 1-bit encode (sign sketch of the whole vector plus its norm).
* :mod:`oracle.ops`      -- inner-product scores, decode attention, top-k search.
* :mod:`oracle.polar`    -- PolarQuant's recursive polar transform and its angle codebooks
  ("PolarQuant explainer" (aibr.jp); the next row after the TurboQuant path: oracle only so far).
"""

from . import rng, rotation, codebook, quant, ops, polar  # noqa: F401
