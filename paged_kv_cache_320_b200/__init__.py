"""B200-native paged KV-cache decode path (sm_100a CUDA behind a C-ABI library).

``synth`` builds seeded synthetic workloads. The device entry points and the host
block manager are bound from ``libpagedkv.so`` (built in-tree by
``python -m paged_kv_cache_320_b200.build``); calling any of them without the
library raises — there is no CPU fallback.
"""
from ._binding import (  # noqa: F401
    BlockManager,
    PagedKVError,
    lib,
    pkv_copy_blocks,
    pkv_decode_partition_size,
    pkv_decode_shared_prefix_partition_size,
    pkv_decode_step_launches,
    pkv_decode_step_workspace_size,
    pkv_device_append,
    pkv_paged_decode_step,
    pkv_paged_decode_step_partitions,
    pkv_decode_workspace_size,
    pkv_get_device_status,
    pkv_paged_attention_decode,
    pkv_paged_attention_decode_noalloc,
    pkv_paged_attention_decode_partitions,
    pkv_paged_attention_merge,
    pkv_paged_attention_decode_shared_prefix,
    pkv_paged_attention_decode_shared_prefix_planned,
    pkv_shared_prefix_plan,
    pkv_decode_shared_prefix_workspace_size,
    pkv_reshape_and_cache,
    pkv_swap_blocks,
    pkv_swap_blocks_staged,
)
from ._binding import PKV_BF16, PKV_F16  # noqa: F401
