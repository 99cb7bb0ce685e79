"""DHSA prefill hot path for B200 (sm_100a).

``workloads`` makes seeded inputs.  ``api`` is the thin binding over the C-ABI
library ``libdhsa.so`` (loaded on first use; a missing library is an error).
"""

__all__ = ["workloads", "api"]
