"""Muon / MuonGS optimizer step for stacks of 2-D weight matrices on B200 (sm_100a).

The compute path is libmuon.so (C ABI, include/muon.h); `binding` is its ctypes
wrapper and `workloads` the seeded synthetic shape sets.
"""
__all__ = ["binding", "workloads", "build"]
