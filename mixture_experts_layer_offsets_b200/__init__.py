"""B200-native (sm_100a) token-routed Mixture-of-Experts FFN layer.

The compute path is the CUDA library ``libmoe_b200.so`` (C ABI in
``include/moe.h``); ``capi`` binds it with ctypes and ``layer.MoELayer``
chains its calls into one forward + backward pass.  ``inputs`` draws the
seeded synthetic workloads.  Importing this package does not load the
library; the first call does, and fails loudly if it has not been built.
"""

__all__ = ["capi", "inputs", "layer"]
