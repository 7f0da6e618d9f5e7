"""fp64 CPU oracle for the GDN recurrence -- test infrastructure only.

Imported by tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg;
never by the product package.
"""
from .oracle import (  # noqa: F401
    decode_e4m3, gdn_forward, gdn_forward_blockcausal, gdn_forward_fp8, gdn_forward_normalized, gdn_rollout,
    load,
)
