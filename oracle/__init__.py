"""fp64 CPU oracle for the GDN recurrence -- test infrastructure only.

Imported by tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg;
never by the product package.
"""
from .oracle import gdn_forward, gdn_forward_blockcausal, gdn_rollout, load  # noqa: F401
