"""libkda: the Kimi Delta Attention forward pass (chunked prefill and recurrent decode) as a C-ABI
library of hand-written sm_100a CUDA kernels, with a thin Python binding.

The binding (``gated_delta_rule_127_b200.kda``) only marshals pointers and sizes; every step of the
computation runs in the CUDA library.  Importing this package does not load the library; the first
call through the binding does, and fails loudly if it is missing.
"""
