"""Exact route-set Query Sparse Attention (QSA) for NVIDIA B200 (sm_100a)."""
