"""B200 (sm_100a) routed MoE expert FFN over prefix-decodable bitplane weights.

`dpa` is the binding of the C ABI (include/dpa.h); `workloads` holds the seeded synthetic
layer shapes. Importing the package loads nothing; the CUDA library is loaded on first use
and every call raises if it is missing.
"""
from . import workloads  # noqa: F401

__version__ = "0.1.0"
