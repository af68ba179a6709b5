"""DLRMv1 sparse/interaction stage on B200 (sm_100a).

The compute path is a C-ABI shared library of hand-written CUDA kernels
(``libdlrm_sparse.so``, declared in ``include/dlrm_sparse.h``);
``dlrm_embedding_bag_b200.ops`` is the thin Python binding over it. Importing
``ops`` loads the library and fails if it is missing: there is no CPU
fallback. ``synthetic`` draws the seeded benchmark inputs and ``build``
compiles the library.
"""
