"""QSA sparse decode for B200 (sm_100a): Python binding of libqsa.so.

The five calls of the decode step -- qsa_append, qsa_index_score,
qsa_topk_select, qsa_sparse_decode, qsa_merge -- are hand-written CUDA
kernels behind a C ABI (include/qsa.h); ``block_sparse_decode_b200.qsa``
marshals torch tensors into that ABI. Build the library with
``python -m block_sparse_decode_b200.build``. There is no fallback: a call
raises if libqsa.so is missing.
"""

__version__ = "0.1.0"
