"""Tile-sparse video attention with a dense-exempt conditioning prefix, for B200 (sm_100a).

The layer runs as five CUDA kernels behind the C ABI of ``libvsa.so``
(``include/vsa.h``): tile pack, tile score, top-k select, block-sparse
attention, tile unpack. This package is the thin Python binding.
"""
from .vsa import (  # noqa: F401
    EXPORTS,
    LIB_PATH,
    Plan,
    VsaError,
    k_from_sparsity,
    library,
    make_desc,
)
from .layer import TileSparseAttention  # noqa: F401
