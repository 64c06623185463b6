"""B200-native Video DeltaNet hybrid video-video attention forward.

The operation lives in libvdn.so (CUDA, sm_100a) behind the C ABI of
include/vdn.h; ``vdn`` is its ctypes binding and ``synth`` the seeded input
generator. Importing the package does not load the library; the first call
does, and fails loudly if it is missing.
"""

from .synth import Layout, WORKLOADS, make_inputs  # noqa: F401
from .vdn import (  # noqa: F401
    device_status,
    hybrid_attn_fwd,
    vda_scan_fwd,
    window_softmax_fwd,
    workspace_bytes,
)
