"""fp64 CPU oracle of the TurboQuant hot path. TEST INFRASTRUCTURE ONLY.

Only `tests/`, `__graft_entry__.smoke()` and the `cpu_baseline` / reference leg of
`bench.py` may import this package. The library (`vector_quantization_tq_b200`) never
imports it, and it imports nothing from the library: the two share no code. The one
shared module is `synth`, which draws the seeded inputs and holds none of the method's
arithmetic.

What it computes (each function cites the passage it follows):
  codebook   Lemma-1 density f_X, Lloyd-Max centroids / boundaries, D_mse,
             Panter-Dite constant, index entropy
  rotation   dense Haar rotation from a Gaussian matrix (QR with sign fix),
             randomized Hadamard transform H diag(eps)/sqrt(d)
  quantizer  TurboQuant_mse and TurboQuant_prod encode / decode, bit packing,
             inner-product estimate <q, x~>
  attention  decode attention over reconstructed K and V, top-k by estimate
  mixed      outlier-channel split: two channel groups, each its own quantizer at its
             own bit width; merge, effective width, outlier-channel choice

Every function is pinned by a `-m "not gpu"` test against values the pages print,
closed forms, textbook special cases or brute force (tests/test_oracle_*.py).
No function is "parity unpinned".
"""
from . import attention, codebook, mixed, quantizer, rotation  # noqa: F401
