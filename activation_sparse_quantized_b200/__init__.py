"""activation_sparse_quantized_b200 -- activation-sparse GEMV over group-wise
int4 weights, as hand-written CUDA for B200 (sm_100a) behind a C ABI.

``sgq``        the thin ctypes binding to ``libsgq.so`` (same names as the C ABI)
``workloads``  seeded synthetic inputs (shapes and distributions only)
``build``      compiles ``libsgq.so`` in-tree with nvcc for sm_100a

Importing the package loads nothing; the binding loads the CUDA library on
first use and raises if it is missing.
"""
__all__ = ["sgq", "workloads", "build"]
