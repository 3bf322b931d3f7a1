"""VAR-Q packed KV-cache hot path on B200 (sm_100a).

``varq`` is the Python binding of ``libvarq.so`` (C ABI in
``include/varq.h``; the library is loaded on first use and its absence is an
error); ``synth`` draws the seeded synthetic workloads.
"""
from . import synth, varq  # noqa: F401

__all__ = ["synth", "varq"]
