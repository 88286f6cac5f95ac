"""QUOKA-style query-oriented KV selection + sparse chunk attention for one B200.

The compute lives in ``libquoka.so`` (hand-written CUDA for sm_100a behind a C ABI,
declared in ``include/quoka.h``); ``query_oriented_sparse_b200.binding`` marshals torch
tensors into those calls.  Importing this package does not load the library; the
first call through the binding does, and fails loudly if it is missing.
"""
__all__ = ["binding", "workloads"]
