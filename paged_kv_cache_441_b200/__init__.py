"""Paged KV-cache decode attention for B200 (sm_100a).

The compute lives in ``libpa.so`` (CUDA kernels behind the C ABI in
``include/pa.h``); this package is its Python binding.  Public calls:

* ``kv_write(key, value, slot_mapping, k_cache, v_cache)`` -- scatter new tokens
  into their cache slots;
* ``copy_blocks(k_cache, v_cache, pairs)`` -- copy-on-write block copies;
* ``decode(out, q, k_cache, v_cache, block_tables, context_lens, scale, ...)`` --
  single-query attention through the block tables (single pass or split-K with a
  log-sum-exp merge; GQA served from one page read per kv head);
* ``decode_append(out, q, key, value, k_cache, v_cache, ...)`` -- the step's cache
  write fused into the decode;
* ``decode_cow(out, q, k_cache, v_cache, block_tables, context_lens, cow, scale, ...)``
  -- each sequence's copy-on-write of a shared block folded into the decode;
* ``decode_planned(..., host_context_lens, scale, key=None, value=None, ...)`` -- decode
  launched from a host-side plan of the partitions that exist, longest first;
* ``prefill(out, q, k_cache, v_cache, block_tables, context_lens, query_start_loc,
  scale)`` -- causal multi-query attention for prompts and prompt chunks (tcgen05);
* ``swap_blocks(...)`` -- block copies between the GPU cache and a pinned host pool;
* ``BlockManager`` -- the host owner of the page tables: on-demand allocation,
  fork (shared blocks), copy-on-write pairs, free, usage ratio, swap, sliding window.
Every attention call takes ``sliding_window`` (0 = whole context).
"""
from ._lib import (  # noqa: F401
    DEVERR,
    EXPORTS,
    LIB_PATH,
    PARTITION_BALANCED,
    PARTITION_DYNAMIC,
    PAError,
    STATIC_SCRATCH_BYTES,
    WORKSPACE_ZERO_BYTES,
    copy_blocks,
    decode,
    decode_append,
    decode_cow,
    decode_planned,
    decode_planned_units,
    decode_static_scratch,
    decode_partition_tokens,
    decode_workspace_bytes,
    device_error,
    kv_write,
    load,
    prefill,
    swap_blocks,
    version,
)
from .block_manager import BlockManager, blocks_needed  # noqa: F401
