"""Float64 CPU oracle for the Kimi Delta Attention (KDA) operator.

TEST INFRASTRUCTURE ONLY.  Nothing in the library's product path imports,
links or runs anything in this package: only ``tests/``, the smoke check in
``__graft_entry__.py`` and the CPU-baseline leg of ``bench.py`` use it.  It
shares no code with the CUDA sources; the seeded input generators
(``gated_delta_rule_98_b200.synth``) are the only thing both sides consume.

Modules
-------
ref           ctypes wrapper around ``kda_ref.c``, the plain sequential float64
              recurrence (the oracle proper).
brute         numpy float64 brute force: materialised products of per-token
              transition matrices (position-interaction view), tiny sizes only.
prologue      numpy float64 input prologue (causal short convolution per
              channel, then Swish).
epilogue      numpy float64 output epilogue (head-wise RMSNorm, then the
              sigmoid output gate).
chunk_mirror  numpy float64 restatement of the chunkwise (WY/UT) algorithm the
              GPU kernels implement; a debugging aid pinned to ``ref``.
"""
