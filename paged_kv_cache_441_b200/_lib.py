"""ctypes binding of libpa (include/pa.h).  Argument marshalling only.

Every function takes torch CUDA tensors, reads their pointers, shapes and the
current CUDA stream, and calls the C entry point of the same name.  There is no
fallback: if ``libpa.so`` is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpa.so")

PA_FP16, PA_BF16 = 0, 1
DEVERR = {"block_id": 0x1, "slot": 0x2, "pair": 0x4, "context": 0x8, "timeout": 0x10}
EXPORTS = ("pa_kv_write", "pa_copy_blocks", "pa_decode", "pa_decode_workspace_bytes",
           "pa_decode_partition_tokens", "pa_get_device_error", "pa_status_str", "pa_version",
           "pa_decode_static_scratch", "pa_decode_append", "pa_swap_blocks", "pa_prefill",
           # host block manager (include/pa_block_manager.h)
           "pa_bm_create", "pa_bm_destroy", "pa_bm_blocks_needed", "pa_bm_num_free_blocks",
           "pa_bm_usage_ratio", "pa_bm_can_allocate", "pa_bm_allocate", "pa_bm_fork",
           "pa_bm_free", "pa_bm_append_slots", "pa_bm_slot", "pa_bm_seq_len",
           "pa_bm_block_refcount", "pa_bm_block_tables", "pa_bm_set_cpu_pool",
           "pa_bm_num_free_cpu_blocks", "pa_bm_is_swapped", "pa_bm_swap_out", "pa_bm_swap_in",
           "pa_bm_set_sliding_window")
STATIC_SCRATCH_BYTES = 16 << 20  # PA_STATIC_SCRATCH_BYTES in include/pa.h

_lib = None


class PAError(RuntimeError):
    pass


def load(path: str = LIB_PATH):
    """Load libpa.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise PAError(f"libpa.so not found at {path}; build it with "
                      "`python -m paged_kv_cache_441_b200.build`")
    lib = ctypes.CDLL(path)
    P, i32, i64, sz, f32 = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t,
                            ctypes.c_float)
    lib.pa_kv_write.argtypes = [P, P, P, i32, i32, i32, i64, i64, P, P, i32, i32, i32, P]
    lib.pa_kv_write.restype = i32
    lib.pa_copy_blocks.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, P]
    lib.pa_copy_blocks.restype = i32
    lib.pa_swap_blocks.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, i32, i32, P]
    lib.pa_swap_blocks.restype = i32
    lib.pa_decode.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, i32, f32, i32, i32,
                              i32, P, sz, i32, P]
    lib.pa_decode.restype = i32
    lib.pa_decode_workspace_bytes.argtypes = [i32] * 9
    lib.pa_decode_workspace_bytes.restype = sz
    lib.pa_decode_partition_tokens.argtypes = [i32] * 9
    lib.pa_decode_partition_tokens.restype = i32
    lib.pa_decode_static_scratch.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, i32,
                                             f32, i32, i32, i32, i32, P]
    lib.pa_decode_static_scratch.restype = i32
    lib.pa_decode_append.argtypes = [P, P, P, P, i64, i64, P, P, P, P, i32, i32, i32, i32, i32,
                                     i32, i32, f32, i32, i32, i32, P, sz, i32, P]
    lib.pa_decode_append.restype = i32
    lib.pa_prefill.argtypes = [P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, i32, i32, f32,
                               i32, i32, P]
    lib.pa_prefill.restype = i32
    lib.pa_get_device_error.argtypes = [i32, ctypes.POINTER(ctypes.c_uint32), i32]
    lib.pa_get_device_error.restype = i32
    lib.pa_status_str.argtypes = [i32]
    lib.pa_status_str.restype = ctypes.c_char_p
    lib.pa_version.argtypes = []
    lib.pa_version.restype = i32
    _lib = lib
    return lib


def _check(status: int, what: str):
    if status != 0:
        msg = load().pa_status_str(status).decode()
        raise PAError(f"{what} failed: status {status} ({msg})")


def _dtype(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return PA_BF16
    if t.dtype == torch.float16:
        return PA_FP16
    raise PAError(f"unsupported dtype {t.dtype}")


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def kv_write(key, value, slot_mapping, k_cache, v_cache, stream=None) -> None:
    """key/value [T, Hkv, d] (token stride may exceed Hkv*d), slot_mapping int64 [T]."""
    T, hkv, d = key.shape
    assert key.stride(2) == 1 and key.stride(1) == d and value.stride(1) == d
    nb, _, bs, _ = k_cache.shape
    _check(load().pa_kv_write(_ptr(key), _ptr(value), _ptr(slot_mapping), T, hkv, d,
                              key.stride(0), value.stride(0), _ptr(k_cache), _ptr(v_cache), nb, bs,
                              _dtype(k_cache), _stream(stream)), "pa_kv_write")


def copy_blocks(k_cache, v_cache, pairs, stream=None) -> None:
    """pairs int64 [P, 2] (src, dst) on the device."""
    nb, hkv, bs, d = k_cache.shape
    _check(load().pa_copy_blocks(_ptr(k_cache), _ptr(v_cache), _ptr(pairs), pairs.shape[0], hkv,
                                 bs, d, nb, _dtype(k_cache), _stream(stream)), "pa_copy_blocks")


def swap_blocks(dst_k_cache, dst_v_cache, src_k_cache, src_v_cache, pairs, stream=None) -> None:
    """Copy blocks pairs[:, 0] of the source pool to blocks pairs[:, 1] of the destination
    pool; either pool may be a pinned host tensor.  pairs: int64 [P, 2] (device or pinned)."""
    snb, hkv, bs, d = src_k_cache.shape
    dnb = dst_k_cache.shape[0]
    _check(load().pa_swap_blocks(_ptr(dst_k_cache), _ptr(dst_v_cache), _ptr(src_k_cache),
                                 _ptr(src_v_cache), _ptr(pairs), pairs.shape[0], hkv, bs, d, snb,
                                 dnb, _dtype(src_k_cache), _stream(stream)), "pa_swap_blocks")


def decode_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                           max_blocks_per_seq, max_context_len=0, partition_size=0,
                           sliding_window=0) -> int:
    return int(load().pa_decode_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                                block_size, max_blocks_per_seq, max_context_len,
                                                sliding_window, partition_size))


def decode_partition_tokens(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                            max_blocks_per_seq, max_context_len=0, partition_size=0,
                            sliding_window=0) -> int:
    return int(load().pa_decode_partition_tokens(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                                 block_size, max_blocks_per_seq, max_context_len,
                                                 sliding_window, partition_size))


def decode(out, q, k_cache, v_cache, block_tables, context_lens, scale, block_size=None,
           max_context_len=0, partition_size=0, workspace=None, stream=None,
           sliding_window=0) -> None:
    """out, q [B, Hq, d]; caches [NB, Hkv, bs, d]; block_tables int32 [B, W];
    context_lens int32 [B].  ``workspace`` (a uint8 CUDA tensor) is allocated here
    with torch when the plan needs one and none is given.  ``sliding_window`` > 0:
    each query attends to the last that many tokens of its context."""
    import torch
    B, hq, d = q.shape
    nb, hkv, bs, _ = k_cache.shape
    if block_size is not None and block_size != bs:
        raise PAError(f"block_size {block_size} != cache block size {bs}")
    W = block_tables.shape[1]
    need = decode_workspace_bytes(B, hq, hkv, d, bs, W, max_context_len, partition_size,
                                  sliding_window)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    wptr = _ptr(workspace) if workspace is not None else None
    wbytes = workspace.numel() if workspace is not None else 0
    _check(load().pa_decode(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                            _ptr(context_lens), B, hq, hkv, d, bs, nb, W, float(scale),
                            int(max_context_len), int(sliding_window), int(partition_size), wptr,
                            wbytes, _dtype(q), _stream(stream)), "pa_decode")


def decode_append(out, q, key, value, k_cache, v_cache, block_tables, context_lens, scale,
                  max_context_len=0, partition_size=0, workspace=None, stream=None,
                  sliding_window=0) -> None:
    """Cache write of each sequence's new token (key/value [B, Hkv, d], stored at
    position context_lens[s]-1) fused with decode; same result as kv_write + decode."""
    import torch
    B, hq, d = q.shape
    nb, hkv, bs, _ = k_cache.shape
    assert key.shape[0] == B and key.stride(2) == 1 and key.stride(1) == d
    assert value.stride(2) == 1 and value.stride(1) == d
    W = block_tables.shape[1]
    need = decode_workspace_bytes(B, hq, hkv, d, bs, W, max_context_len, partition_size,
                                  sliding_window)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    wptr = _ptr(workspace) if workspace is not None else None
    wbytes = workspace.numel() if workspace is not None else 0
    _check(load().pa_decode_append(_ptr(out), _ptr(q), _ptr(key), _ptr(value), key.stride(0),
                                   value.stride(0), _ptr(k_cache), _ptr(v_cache),
                                   _ptr(block_tables), _ptr(context_lens), B, hq, hkv, d, bs, nb,
                                   W, float(scale), int(max_context_len), int(sliding_window),
                                   int(partition_size), wptr, wbytes, _dtype(q), _stream(stream)),
           "pa_decode_append")


def decode_static_scratch(out, q, k_cache, v_cache, block_tables, context_lens, scale,
                          block_size=None, max_context_len=0, partition_size=0,
                          stream=None, sliding_window=0) -> None:
    """``decode`` for callers that cannot allocate device memory: the split-K partial
    results go to the library's own fixed scratch array (STATIC_SCRATCH_BYTES per
    GPU) instead of a workspace.  Calls that overlap on the GPU race on that array."""
    B, hq, d = q.shape
    nb, hkv, bs, _ = k_cache.shape
    if block_size is not None and block_size != bs:
        raise PAError(f"block_size {block_size} != cache block size {bs}")
    W = block_tables.shape[1]
    need = decode_workspace_bytes(B, hq, hkv, d, bs, W, max_context_len, partition_size,
                                  sliding_window)
    if need > STATIC_SCRATCH_BYTES:
        raise PAError(f"pa_decode_static_scratch: these sizes need {need} bytes of scratch, "
                      f"more than the library's fixed {STATIC_SCRATCH_BYTES}; use decode() "
                      "with a workspace")
    _check(load().pa_decode_static_scratch(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
        _ptr(context_lens), B, hq, hkv, d, bs, nb, W, float(scale), int(max_context_len),
        int(sliding_window), int(partition_size), _dtype(q), _stream(stream)),
        "pa_decode_static_scratch")


def prefill(out, q, k_cache, v_cache, block_tables, context_lens, query_start_loc, scale,
            sliding_window=0, stream=None) -> None:
    """Causal multi-query attention: q, out [T, Hq, d] (the new tokens of every sequence,
    sequence s in rows query_start_loc[s] .. [s+1]); caches [NB, Hkv, bs, d];
    block_tables int32 [B, W]; context_lens int32 [B] (tokens in the cache, the chunk
    included); query_start_loc int32 [B + 1]."""
    T, hq, d = q.shape
    nb, hkv, bs, _ = k_cache.shape
    B = context_lens.shape[0]
    assert query_start_loc.shape[0] == B + 1
    _check(load().pa_prefill(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                             _ptr(block_tables), _ptr(context_lens), _ptr(query_start_loc), B, T,
                             hq, hkv, d, bs, nb, block_tables.shape[1], float(scale),
                             int(sliding_window), _dtype(q), _stream(stream)), "pa_prefill")


def device_error(device: int = 0, clear: bool = True) -> int:
    """Synchronises `device` and returns (and by default clears) its error bits."""
    bits = ctypes.c_uint32(0)
    _check(load().pa_get_device_error(device, ctypes.byref(bits), 1 if clear else 0),
           "pa_get_device_error")
    return int(bits.value)


def version() -> int:
    return int(load().pa_version())
