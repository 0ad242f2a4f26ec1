"""Ragged varlen attention for token-pruned ViTs on B200 (sm_100a).

The CUDA library (``librra.so``) is loaded by :mod:`ragged_varlen_attention_rra_b200.rra` on
first use; every call raises if it is missing.  :mod:`.workloads` holds the seeded input
generators and does not need the library.
"""
__all__ = ["rra", "workloads"]
