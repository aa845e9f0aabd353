"""Pooled block-sparse attention (hybrid Top-k / Top-p block mask) and its
sparse + linear mix, as CUDA kernels for sm_100a behind a C ABI.

The CUDA entry points live in :mod:`block_sparse_attention_pooled_b200.sparge`
(importing it loads ``libsparge.so`` and fails loudly when it is missing).
:mod:`block_sparse_attention_pooled_b200.synth` generates seeded inputs.
"""

__all__ = ["sparge", "synth"]
