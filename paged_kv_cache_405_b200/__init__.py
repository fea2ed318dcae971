"""pagedkv -- paged KV cache decode on B200 (sm_100a).

A thin Python face over ``libpagedkv.so`` (C ABI in ``include/pagedkv.h``):
``kv_append``, ``paged_attention_decode``, ``block_copy``, the host
``BlockAllocator``, and ``DecodeSession`` which strings one decode step
together.  PyTorch supplies device memory and streams only.
"""
from .binding import (BlockAllocator, PagedKVError, attention_partition_size,  # noqa: F401
                      attention_chunk_workspace_bytes, attention_shared_workspace_bytes, attention_workspace_bytes, block_copy, device_error,
                      find_shared_prefix_groups, kv_append, kv_append_fp8, launch_count, paged_attention_chunk, paged_attention_decode,
                      paged_attention_decode_fp8, paged_attention_decode_shared, paged_attention_decode_static,
                      PkvCopy, PkvStep, raw_call, set_nvtx, step_from_host, workspace_for)
from .session import ChunkPlan, DecodeSession, DevicePlan, StepPlan  # noqa: F401,E402
