"""Grouped NVFP4 weight-quantised MoE expert forward for B200 (sm_100a).

The compute lives in ``libnvfp4moe.so`` (hand-written CUDA, C ABI in
include/nvfp4_moe.h); this package is its thin Python binding plus device
containers.  Importing it without the built library raises ImportError.
"""

from ._binding import (  # noqa: F401
    ACTIVATIONS,
    LIB_PATH,
    PATH_AUTO,
    PATH_DECODE,
    PATH_PREFILL,
    SHARD_COLUMN,
    SHARD_ROW,
    Buffers,
    ExpertTables,
    LaunchOpts,
    NVFP4MoEError,
    active_cap,
    append_shared,
    blend,
    check_scales,
    device_error,
    wait_selftest,
    down,
    down_ws,
    exported_symbols,
    forward,
    forward_nongated,
    gate_up_silu,
    gate_up_silu_ws,
    route_sort,
    shard_nvfp4,
    shard_nvfp4_into,
    shared_slots,
    transpose_concat,
    transpose_concat_into,
    transpose_u8,
    up_act,
    up_act_ws,
    workspace_bytes,
)
from .layer import (  # noqa: F401
    MoEBuffers,
    NVFP4MoE,
    NVFP4Projection,
    all_reduce_out,
    expert_owner_range,
)
