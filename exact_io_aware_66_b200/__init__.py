"""B200-native (sm_100a) exact, IO-aware attention: forward and backward through a C-ABI
library (libfa.so, declared in include/fa.h) with hand-written TMA/tcgen05 kernels.

Importing the package does not load the library; the first call into ``fa`` does, and raises
if it is missing.
"""

__all__ = ["fa", "workloads", "build"]
