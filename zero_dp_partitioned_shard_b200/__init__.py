"""B200-native ZeRO-DP partitioned mixed-precision Adam shard step.

The compute path is the CUDA library ``libzero_shard.so`` (C ABI declared in
``include/zero_shard.h``); :mod:`.binding` marshals arguments to it through
ctypes.  The library is loaded on first use and a missing or unloadable build
raises -- there is no CPU fallback.
"""
__all__ = ["binding", "synth"]
