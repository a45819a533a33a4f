"""Paged decode attention for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libpa.so`` built from ``csrc/``; this
package loads it lazily (on first use of :mod:`.binding`) and fails loudly if
it is missing.  ``block_manager`` and ``workload`` are host-side helpers that
produce the integer tables and seeded synthetic inputs the calls consume.
"""
__all__ = ["binding", "block_manager", "workload"]
