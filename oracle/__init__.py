"""CPU oracle for TurboQuant KV-cache compression and decode attention.

TEST INFRASTRUCTURE ONLY. Nothing in the product path may import, call or
execute this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.

It is a plain, slow, NumPy restatement of the method as the web pages on
TurboQuant describe it, written step by step in the pages' order, and it
shares no code with the CUDA path (``kv_cache_vector_13_b200``): neither
imports the other.  Each function names the passage it follows.

Modules
  prng       SplitMix64 counter generator, Rademacher signs, Gaussian S
  codebook   Lloyd-Max centroids/thresholds for N(0,1/d) and the exact
             sphere-coordinate (Beta) density
  rotation   Sylvester-Hadamard rotation, canonical fp32 FWHT; the dense
             Haar rotation (Q of a seeded Gaussian's QR)
  quantizer  encode (TurboQuant_mse / TurboQuant_prod), bit packing, dequant
  attention  decode attention on the packed cache (float64 and fp32)
  search     top-k vector search by the estimated inner product
  split      outlier-channel split: two channel groups at two bit widths
  metrics    distortion (MSE) and inner-product bias

Parity unpinned: the GPU's fp32 summation order for the QJL projection
S.r and for the dense rotation's product Pi.x (the oracle takes both in
float64; decisions within rounding of a threshold or of zero may differ and
are counted by the tests), and the Beta-codebook distortion values (the
pages print none; only the numerical integral pins them).
"""

from . import prng, codebook, rotation, quantizer, attention, metrics, search, split  # noqa: F401
