"""gated_delta_rule_149_b200 -- the Gated-Delta-Net recurrence on B200 (sm_100a).

The compute runs in libgdn.so (hand-written CUDA behind a C ABI, include/gdn.h);
this package only marshals arguments.  Importing it does not load the library;
the first call does, and fails loudly if the library is missing.
"""
from .gdn import (  # noqa: F401
    GDN_BIDI, GDN_CAUSAL, GDN_FP32, GDN_RECURRENT, GDNError, gdn_device_status,
    gdn_forward, gdn_forward_blockcausal, gdn_forward_fp8, gdn_forward_host, gdn_forward_host_async,
    gdn_forward_normalized, gdn_forward_segmented, gdn_rollout, gdn_workspace_release,
    gdn_workspace_reserved, lib_path, load_library,
)
