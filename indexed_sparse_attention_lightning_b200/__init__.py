"""Indexed sparse attention for NVIDIA B200 (sm_100a).

The lightning indexer, the per-query top-K and the sparse MLA attention run as
hand-written CUDA kernels behind the C ABI in ``include/sa.h`` (``libsa.so``);
``api`` is the thin Python binding over it and ``workloads`` the seeded
synthetic inputs.  Build with ``python -m indexed_sparse_attention_lightning_b200.build``.
"""
__version__ = "0.1.0"
