"""nmoe: the expert-choice MoE feed-forward layer of NucleusMoE-Image's DiT blocks,
as hand-written CUDA kernels for NVIDIA B200 (sm_100a) behind a C ABI (include/nmoe.h).

This package is the thin Python binding (argument marshalling only) plus the seeded
synthetic workload generators. The shared library ``libnmoe.so`` is built in place by
``python -m diffusion_transformer_moe_b200.build``; calls raise if it is missing.
"""

from . import inputs  # noqa: F401
from ._lib import (  # noqa: F401
    EXPORTS, LIB_PATH, NmoeError, Trace, build_info, forward, gather_rows, get_last_error,
    kernels_per_call, lib, router, select, workspace_size,
)
