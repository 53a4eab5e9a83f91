"""Block-sparse prefill attention with block routing (PISA style) for B200.

The product is the C-ABI library ``libpsa.so`` (``include/psa.h``); the
module :mod:`block_sparse_attention_psa_b200.psa` is its thin Python binding
and :mod:`block_sparse_attention_psa_b200.inputs` holds the seeded synthetic
input generators.  Nothing here computes the method on the CPU.
"""

__version__ = "0.1.0"
