"""B200-native Kimi Delta Attention (KDA) operator.

The operator runs in hand-written sm_100a CUDA kernels behind the C ABI of
``include/kda.h`` (``libkda.so``).  ``gated_delta_rule_98_b200.kda`` is the
thin ctypes binding (argument marshalling only); ``synth`` draws the seeded
synthetic inputs.  Importing the package does not load the CUDA library;
``kda.lib()`` does, and fails loudly when it is missing.
"""
__all__ = ["kda", "synth"]
