"""Segmented chunkwise gated linear attention on B200 (sm_100a).

The product is the C-ABI library ``libla_seg.so`` built from ``csrc/``; ``la_seg`` is its
thin ctypes binding (argument marshalling only) and ``inputs`` draws the seeded synthetic
workloads.
"""
__all__ = ["la_seg", "inputs"]
