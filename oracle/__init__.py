"""fp64 CPU oracle for the KDA forward pass.

Test infrastructure: only the tests, ``__graft_entry__.smoke()`` and the bench's CPU-baseline
leg use it.  It never imports the CUDA package, and the CUDA package never imports it.
"""
from .oracle import (forward, decode_step, gdn_forward, gdn_decode_step, l2_normalise, sigmoid,  # noqa: F401
                     output_epilogue,
                     max_threads, RULE_DELTA, RULE_ADDITIVE)
