"""B200-native paged MLA decode: a C-ABI CUDA library (libpagedmla.so) and its binding.

The decode path -- split-KV scheduler, page-gather loader, fused QK^T / online softmax /
PV kernel and log-sum-exp combine -- runs in hand-written sm_100a kernels; ``ops`` only
marshals arguments.  ``workloads`` draws seeded synthetic inputs.
"""

from .ops import (  # noqa: F401
    MlaError,
    device_sm_count,
    flash_mla_with_kvcache,
    get_mla_metadata,
    load_library,
    metadata_size,
    mla_combine,
    mla_decode_paged,
    new_workspace,
    num_parts_for,
    query_status,
    watchdog_selftest,
    workspace_size,
)
