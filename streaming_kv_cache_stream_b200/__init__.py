"""Streaming KV-cache attention on B200 (sm_100a).

The compute path lives in the C-ABI library ``lib/libfsstream.so`` (built from
``csrc/``); ``abi`` is a thin ctypes binding with the same function names.
Importing this package does not load the library; ``abi.load()`` does, and it
raises if the library is missing -- there is no CPU fallback.
"""
from .inputs import WORKLOADS, Workload  # noqa: F401

__all__ = ["WORKLOADS", "Workload"]
