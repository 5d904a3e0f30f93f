"""ctypes binding of libpa (include/pa.h).  Argument marshalling only.

Every function takes torch CUDA tensors, checks that they are what the C entry
point reads (device, dtype, contiguity, shapes that agree), then passes their
pointers, shapes and the tensors' device's current CUDA stream to the C entry
point of the same name.  A failed check raises PAError before anything reaches
the library.  There is no fallback: if ``libpa.so`` is missing or a call fails,
an exception is raised.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpa.so")

PA_FP16, PA_BF16 = 0, 1
DEVERR = {"block_id": 0x1, "slot": 0x2, "pair": 0x4, "context": 0x8, "timeout": 0x10,
          "workspace": 0x20}
EXPORTS = ("pa_kv_write", "pa_copy_blocks", "pa_decode", "pa_decode_workspace_bytes",
           "pa_decode_partition_tokens", "pa_get_device_error", "pa_status_str", "pa_version",
           "pa_decode_static_scratch", "pa_decode_append", "pa_decode_cow", "pa_decode_planned",
           "pa_decode_planned_units",
           "pa_swap_blocks",
           "pa_prefill",
           # host block manager (include/pa_block_manager.h)
           "pa_bm_create", "pa_bm_destroy", "pa_bm_blocks_needed", "pa_bm_num_free_blocks",
           "pa_bm_usage_ratio", "pa_bm_can_allocate", "pa_bm_allocate", "pa_bm_fork",
           "pa_bm_free", "pa_bm_append_slots", "pa_bm_append_slots_cow", "pa_bm_slot",
           "pa_bm_seq_len",
           "pa_bm_block_refcount", "pa_bm_block_tables", "pa_bm_set_cpu_pool",
           "pa_bm_num_free_cpu_blocks", "pa_bm_is_swapped", "pa_bm_swap_out", "pa_bm_swap_in",
           "pa_bm_set_sliding_window")
STATIC_SCRATCH_BYTES = 16 << 20  # PA_STATIC_SCRATCH_BYTES in include/pa.h
PARTITION_BALANCED = -1  # PA_PARTITION_BALANCED
PARTITION_DYNAMIC = -2  # PA_PARTITION_DYNAMIC
WORKSPACE_ZERO_BYTES = 8192  # PA_WORKSPACE_ZERO_BYTES

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
    lib.pa_decode_cow.argtypes = [P, P, P, P, i64, i64, P, P, P, P, P, i32, i32, i32, i32, i32,
                                  i32, i32, f32, i32, i32, i32, P, sz, i32, P]
    lib.pa_decode_cow.restype = i32
    lib.pa_decode_planned.argtypes = [P, P, P, P, i64, i64, P, P, P, P, P, i32, i32, i32, i32,
                                      i32, i32, i32, f32, i32, i32, i32, P, sz, i32, P]
    lib.pa_decode_planned.restype = i32
    lib.pa_decode_planned_units.argtypes = [P] + [i32] * 9 + [P, i32]
    lib.pa_decode_planned_units.restype = i32
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


# Device type every tensor of a launch must live on.  The marshalling tests run the
# same checks on CPU tensors against a stand-in library by switching this to "cpu".
_DEVICE_TYPE = "cuda"


def _fail(what: str, msg: str):
    raise PAError(f"{what}: {msg}")


def _args(what: str, half: dict, ints: dict = None, rows: dict = None):
    """Check the tensors of one call before their pointers reach the library.

    half: 16-bit float tensors (q, out, caches), one dtype, contiguous.
    ints: name -> (tensor, torch dtype); contiguous (block tables, lengths, slots).
    rows: 16-bit tensors [T, H, d] whose heads are contiguous but whose token stride
          is free (a key or value slice of a wider projection).
    All of them on the first half tensor's device, which must be of type _DEVICE_TYPE.
    Returns that device."""
    ints, rows = ints or {}, rows or {}
    first = next(iter(half.values()))
    dev = first.device
    if dev.type != _DEVICE_TYPE:
        _fail(what, f"tensors must be on a {_DEVICE_TYPE} device, got {dev}")
    for name, t in {**half, **rows}.items():
        if t.dtype != first.dtype:
            _fail(what, f"{name} is {t.dtype}, expected {first.dtype}")
        if t.device != dev:
            _fail(what, f"{name} is on device {t.device}, expected {dev}")
    _dtype(first)
    for name, t in half.items():
        if not t.is_contiguous():
            _fail(what, f"{name} must be contiguous")
    for name, t in rows.items():
        if not (t.dim() == 3 and t.stride(2) == 1 and t.stride(1) == t.shape[2]):
            _fail(what, f"{name} must be [tokens, heads, head_dim] with contiguous heads")
    for name, (t, dt) in ints.items():
        if t.dtype != dt:
            _fail(what, f"{name} is {t.dtype}, expected {dt}")
        if t.device != dev:
            _fail(what, f"{name} is on device {t.device}, expected {dev}")
        if not t.is_contiguous():
            _fail(what, f"{name} must be contiguous")
    return dev


def _cache_shape(what: str, k_cache, v_cache, num_kv_heads=None, head_dim=None):
    if not (k_cache.dim() == 4 and tuple(v_cache.shape) == tuple(k_cache.shape)):
        _fail(what, f"k_cache {tuple(k_cache.shape)} and v_cache {tuple(v_cache.shape)} must "
              "both be [num_blocks, num_kv_heads, block_size, head_dim]")
    nb, hkv, bs, d = k_cache.shape
    if num_kv_heads is not None and hkv != num_kv_heads:
        _fail(what, f"cache has {hkv} kv heads, the tokens {num_kv_heads}")
    if head_dim is not None and d != head_dim:
        _fail(what, f"cache head_dim {d} != {head_dim}")
    return nb, hkv, bs, d


def _tables(what: str, block_tables, context_lens, num_seqs):
    if not (block_tables.dim() == 2 and block_tables.shape[0] == num_seqs):
        _fail(what, f"block_tables {tuple(block_tables.shape)} must be "
              f"[{num_seqs}, max_blocks]")
    if tuple(context_lens.shape) != (num_seqs,):
        _fail(what, f"context_lens {tuple(context_lens.shape)} must be [{num_seqs}]")


def _stream(stream, device=None):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _on(device):
    """Make ``device`` current for the launch (the library launches on the current
    device; a tensor on another GPU would be read through the wrong context)."""
    import contextlib
    import torch
    if device is None or device.type != "cuda" or device.index is None or \
            device.index == torch.cuda.current_device():
        return contextlib.nullcontext()
    return torch.cuda.device(device)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def kv_write(key, value, slot_mapping, k_cache, v_cache, stream=None) -> None:
    """key/value [T, Hkv, d] (token stride may exceed Hkv*d), slot_mapping int64 [T]."""
    import torch
    what = "pa_kv_write"
    if not (key.dim() == 3 and tuple(value.shape) == tuple(key.shape)):
        _fail(what, f"key {tuple(key.shape)} and value {tuple(value.shape)} must both be "
              "[T, Hkv, d]")
    T, hkv, d = key.shape
    nb, _, bs, _ = _cache_shape(what, k_cache, v_cache, hkv, d)
    if tuple(slot_mapping.shape) != (T,):
        _fail(what, f"slot_mapping must be [{T}]")
    dev = _args(what, {"k_cache": k_cache, "v_cache": v_cache}, rows={"key": key, "value": value},
                ints={"slot_mapping": (slot_mapping, torch.int64)})
    with _on(dev):
        _check(load().pa_kv_write(_ptr(key), _ptr(value), _ptr(slot_mapping), T, hkv, d,
                                  key.stride(0), value.stride(0), _ptr(k_cache), _ptr(v_cache),
                                  nb, bs, _dtype(k_cache), _stream(stream, dev)), what)


def copy_blocks(k_cache, v_cache, pairs, stream=None) -> None:
    """pairs int64 [P, 2] (src, dst) on the device."""
    import torch
    what = "pa_copy_blocks"
    nb, hkv, bs, d = _cache_shape(what, k_cache, v_cache)
    if not (pairs.dim() == 2 and pairs.shape[1] == 2):
        _fail(what, "pairs must be [P, 2]")
    dev = _args(what, {"k_cache": k_cache, "v_cache": v_cache},
                ints={"pairs": (pairs, torch.int64)})
    with _on(dev):
        _check(load().pa_copy_blocks(_ptr(k_cache), _ptr(v_cache), _ptr(pairs), pairs.shape[0],
                                     hkv, bs, d, nb, _dtype(k_cache), _stream(stream, dev)), what)


def swap_blocks(dst_k_cache, dst_v_cache, src_k_cache, src_v_cache, pairs, stream=None) -> None:
    """Copy blocks pairs[:, 0] of the source pool to blocks pairs[:, 1] of the destination
    pool; either pool may be a pinned host tensor.  pairs: int64 [P, 2] (device or pinned).
    Whether a host pool is pinned is checked by the library."""
    import torch
    what = "pa_swap_blocks"
    snb, hkv, bs, d = _cache_shape(what, src_k_cache, src_v_cache)
    dnb, dh, dbs, dd = _cache_shape(what, dst_k_cache, dst_v_cache)
    if (dh, dbs, dd) != (hkv, bs, d):
        _fail(what, "source and destination blocks differ in shape")
    if not (pairs.dim() == 2 and pairs.shape[1] == 2):
        _fail(what, "pairs must be [P, 2]")
    pools = {"dst_k_cache": dst_k_cache, "dst_v_cache": dst_v_cache,
             "src_k_cache": src_k_cache, "src_v_cache": src_v_cache}
    for name, t in pools.items():
        if t.dtype != src_k_cache.dtype:
            _fail(what, f"{name} is {t.dtype}, expected {src_k_cache.dtype}")
        if not t.is_contiguous():
            _fail(what, f"{name} must be contiguous")
    if not (pairs.dtype == torch.int64 and pairs.is_contiguous()):
        _fail(what, "pairs must be contiguous int64")
    gpus = {t.device for t in (*pools.values(), pairs) if t.device.type == _DEVICE_TYPE}
    if len(gpus) > 1:
        _fail(what, f"tensors on more than one device: {sorted(map(str, gpus))}")
    dev = next(iter(gpus)) if gpus else None
    with _on(dev):
        _check(load().pa_swap_blocks(_ptr(dst_k_cache), _ptr(dst_v_cache), _ptr(src_k_cache),
                                     _ptr(src_v_cache), _ptr(pairs), pairs.shape[0], hkv, bs, d,
                                     snb, dnb, _dtype(src_k_cache), _stream(stream, dev)), what)


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


def _decode_shapes(what, out, q, k_cache, v_cache, block_tables, context_lens, block_size):
    """Shapes shared by the decode entry points: (B, Hq, d, NB, Hkv, bs, W)."""
    if not (q.dim() == 3 and tuple(out.shape) == tuple(q.shape)):
        _fail(what, f"q {tuple(q.shape)} and out {tuple(out.shape)} must both be [B, Hq, d]")
    B, hq, d = q.shape
    nb, hkv, bs, _ = _cache_shape(what, k_cache, v_cache, head_dim=d)
    if block_size is not None and block_size != bs:
        _fail(what, f"block_size {block_size} != cache block size {bs}")
    _tables(what, block_tables, context_lens, B)
    return B, hq, d, nb, hkv, bs, block_tables.shape[1]


def _workspace(what, workspace, need, dev):
    """(pointer, bytes) of the split-K workspace; allocated with torch when the plan needs
    one and the caller gave none (zero-filled: the dynamic split keeps its claim counters
    in the first WORKSPACE_ZERO_BYTES, which must start at zero)."""
    import torch
    if workspace is None:
        if not need:
            return None, 0
        workspace = torch.zeros(need, dtype=torch.uint8, device=dev)
    if not (workspace.device == dev and workspace.is_contiguous()):
        _fail(what, f"workspace must be a contiguous tensor on {dev}")
    return _ptr(workspace), workspace.numel() * workspace.element_size()


def decode(out, q, k_cache, v_cache, block_tables, context_lens, scale, block_size=None,
           max_context_len=0, partition_size=0, workspace=None, stream=None,
           sliding_window=0) -> None:
    """out, q [B, Hq, d]; caches [NB, Hkv, bs, d]; block_tables int32 [B, W];
    context_lens int32 [B].  ``workspace`` (a contiguous CUDA tensor) is allocated here
    with torch when the plan needs one and none is given.  ``sliding_window`` > 0:
    each query attends to the last that many tokens of its context."""
    import torch
    what = "pa_decode"
    B, hq, d, nb, hkv, bs, W = _decode_shapes(what, out, q, k_cache, v_cache, block_tables,
                                              context_lens, block_size)
    dev = _args(what, {"q": q, "out": out, "k_cache": k_cache, "v_cache": v_cache},
                ints={"block_tables": (block_tables, torch.int32),
                      "context_lens": (context_lens, torch.int32)})
    with _on(dev):
        need = decode_workspace_bytes(B, hq, hkv, d, bs, W, max_context_len, partition_size,
                                      sliding_window)
        wptr, wbytes = _workspace(what, workspace, need, dev)
        _check(load().pa_decode(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                _ptr(block_tables), _ptr(context_lens), B, hq, hkv, d, bs, nb, W,
                                float(scale), int(max_context_len), int(sliding_window),
                                int(partition_size), wptr, wbytes, _dtype(q),
                                _stream(stream, dev)), what)


def decode_append(out, q, key, value, k_cache, v_cache, block_tables, context_lens, scale,
                  max_context_len=0, partition_size=0, workspace=None, stream=None,
                  sliding_window=0) -> None:
    """Cache write of each sequence's new token (key/value [B, Hkv, d], stored at
    position context_lens[s]-1) fused with decode; same result as kv_write + decode."""
    import torch
    what = "pa_decode_append"
    B, hq, d, nb, hkv, bs, W = _decode_shapes(what, out, q, k_cache, v_cache, block_tables,
                                              context_lens, None)
    if not (tuple(key.shape) == (B, hkv, d) and tuple(value.shape) == (B, hkv, d)):
        _fail(what, f"key {tuple(key.shape)} and value {tuple(value.shape)} must both be "
              f"[{B}, {hkv}, {d}]")
    dev = _args(what, {"q": q, "out": out, "k_cache": k_cache, "v_cache": v_cache},
                rows={"key": key, "value": value},
                ints={"block_tables": (block_tables, torch.int32),
                      "context_lens": (context_lens, torch.int32)})
    with _on(dev):
        need = decode_workspace_bytes(B, hq, hkv, d, bs, W, max_context_len, partition_size,
                                      sliding_window)
        wptr, wbytes = _workspace(what, workspace, need, dev)
        _check(load().pa_decode_append(_ptr(out), _ptr(q), _ptr(key), _ptr(value),
                                       key.stride(0), value.stride(0), _ptr(k_cache),
                                       _ptr(v_cache), _ptr(block_tables), _ptr(context_lens), B,
                                       hq, hkv, d, bs, nb, W, float(scale), int(max_context_len),
                                       int(sliding_window), int(partition_size), wptr, wbytes,
                                       _dtype(q), _stream(stream, dev)), what)


def decode_cow(out, q, k_cache, v_cache, block_tables, context_lens, cow, scale, key=None,
               value=None, max_context_len=0, partition_size=0, workspace=None, stream=None,
               sliding_window=0) -> None:
    """``decode`` with each sequence's copy-on-write done by the CTAs that read the rows:
    cow int32 [B, 3] = (source block, logical block index, rows), source < 0 for none.
    With key/value ([B, Hkv, d]) the new token's cache write of ``decode_append`` too."""
    import torch
    what = "pa_decode_cow"
    B, hq, d, nb, hkv, bs, W = _decode_shapes(what, out, q, k_cache, v_cache, block_tables,
                                              context_lens, None)
    if (key is None) != (value is None):
        _fail(what, "key and value must be given together")
    if tuple(cow.shape) != (B, 3):
        _fail(what, f"cow {tuple(cow.shape)} must be [{B}, 3]")
    rows = {}
    if key is not None:
        if not (tuple(key.shape) == (B, hkv, d) and tuple(value.shape) == (B, hkv, d)):
            _fail(what, f"key {tuple(key.shape)} and value {tuple(value.shape)} must both be "
                  f"[{B}, {hkv}, {d}]")
        rows = {"key": key, "value": value}
    dev = _args(what, {"q": q, "out": out, "k_cache": k_cache, "v_cache": v_cache}, rows=rows,
                ints={"block_tables": (block_tables, torch.int32),
                      "context_lens": (context_lens, torch.int32),
                      "cow": (cow, torch.int32)})
    with _on(dev):
        need = decode_workspace_bytes(B, hq, hkv, d, bs, W, max_context_len, partition_size,
                                      sliding_window)
        wptr, wbytes = _workspace(what, workspace, need, dev)
        _check(load().pa_decode_cow(
            _ptr(out), _ptr(q), _ptr(key), _ptr(value), key.stride(0) if key is not None else 0, value.stride(0) if value is not None else 0,
            _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(context_lens), _ptr(cow), B,
            hq, hkv, d, bs, nb, W, float(scale), int(max_context_len), int(sliding_window),
            int(partition_size), wptr, wbytes, _dtype(q), _stream(stream, dev)), what)


def decode_planned(out, q, k_cache, v_cache, block_tables, context_lens, host_context_lens,
                   scale, key=None, value=None, max_context_len=0, partition_size=0,
                   workspace=None, stream=None, sliding_window=0) -> None:
    """``decode`` (with key/value: ``decode_append``) launched from a host-side plan:
    host_context_lens, an int32 host array (numpy or CPU tensor) with the values of
    context_lens, gives the units that exist, taken longest first."""
    import torch
    what = "pa_decode_planned"
    B, hq, d, nb, hkv, bs, W = _decode_shapes(what, out, q, k_cache, v_cache, block_tables,
                                              context_lens, None)
    if (key is None) != (value is None):
        _fail(what, "key and value must be given together")
    hl = host_context_lens
    if isinstance(hl, torch.Tensor):
        if hl.device.type != "cpu":
            _fail(what, "host_context_lens must be in host memory")
        hl = hl.numpy()
    hl = np.ascontiguousarray(hl)
    if hl.dtype != np.int32 or hl.shape != (B,):
        _fail(what, f"host_context_lens must be int32 [{B}], got {hl.dtype} {hl.shape}")
    rows = {}
    if key is not None:
        if not (tuple(key.shape) == (B, hkv, d) and tuple(value.shape) == (B, hkv, d)):
            _fail(what, f"key {tuple(key.shape)} and value {tuple(value.shape)} must both be "
                  f"[{B}, {hkv}, {d}]")
        rows = {"key": key, "value": value}
    dev = _args(what, {"q": q, "out": out, "k_cache": k_cache, "v_cache": v_cache}, rows=rows,
                ints={"block_tables": (block_tables, torch.int32),
                      "context_lens": (context_lens, torch.int32)})
    with _on(dev):
        need = decode_workspace_bytes(B, hq, hkv, d, bs, W, max_context_len, partition_size,
                                      sliding_window)
        wptr, wbytes = _workspace(what, workspace, need, dev)
        _check(load().pa_decode_planned(
            _ptr(out), _ptr(q), _ptr(key), _ptr(value), key.stride(0) if key is not None else 0,
            value.stride(0) if value is not None else 0, _ptr(k_cache), _ptr(v_cache),
            _ptr(block_tables), _ptr(context_lens), hl.ctypes.data_as(ctypes.c_void_p), B, hq,
            hkv, d, bs, nb, W, float(scale), int(max_context_len), int(sliding_window),
            int(partition_size), wptr, wbytes, _dtype(q), _stream(stream, dev)), what)


def decode_planned_units(host_context_lens, num_q_heads, num_kv_heads, head_dim, block_size,
                         max_blocks_per_seq, max_context_len=0, sliding_window=0,
                         partition_size=0):
    """The units decode_planned launches for these arguments (host-side): uint32 array,
    each sequence << 16 | partition << 8 | partition count, in launch order; empty when
    it launches the full grid."""
    hl = np.ascontiguousarray(host_context_lens, np.int32)
    out = np.zeros(4096, np.uint32)
    n = load().pa_decode_planned_units(
        hl.ctypes.data_as(ctypes.c_void_p), int(hl.shape[0]), int(num_q_heads),
        int(num_kv_heads), int(head_dim), int(block_size), int(max_blocks_per_seq),
        int(max_context_len), int(sliding_window), int(partition_size),
        out.ctypes.data_as(ctypes.c_void_p), out.shape[0])
    if n < 0:
        _fail("pa_decode_planned_units", "invalid arguments")
    return out[:n].copy()


def decode_static_scratch(out, q, k_cache, v_cache, block_tables, context_lens, scale,
                          block_size=None, max_context_len=0, partition_size=0,
                          stream=None, sliding_window=0) -> None:
    """``decode`` for callers that cannot allocate device memory: the split-K partial
    results go to the library's own fixed scratch array (STATIC_SCRATCH_BYTES per
    GPU) instead of a workspace.  Calls that overlap on the GPU race on that array."""
    import torch
    what = "pa_decode_static_scratch"
    B, hq, d, nb, hkv, bs, W = _decode_shapes(what, out, q, k_cache, v_cache, block_tables,
                                              context_lens, block_size)
    dev = _args(what, {"q": q, "out": out, "k_cache": k_cache, "v_cache": v_cache},
                ints={"block_tables": (block_tables, torch.int32),
                      "context_lens": (context_lens, torch.int32)})
    with _on(dev):
        # sized on the tensors' device: the balanced split's need grows with its SM count
        need = decode_workspace_bytes(B, hq, hkv, d, bs, W, max_context_len, partition_size,
                                      sliding_window)
        if need > STATIC_SCRATCH_BYTES:
            _fail(what, f"these sizes need {need} bytes of scratch, more than the library's "
                  f"fixed {STATIC_SCRATCH_BYTES}; use decode() with a workspace")
        _check(load().pa_decode_static_scratch(
            _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
            _ptr(context_lens), B, hq, hkv, d, bs, nb, W, float(scale), int(max_context_len),
            int(sliding_window), int(partition_size), _dtype(q), _stream(stream, dev)), what)


def prefill(out, q, k_cache, v_cache, block_tables, context_lens, query_start_loc, scale,
            sliding_window=0, stream=None) -> None:
    """Causal multi-query attention: q, out [T, Hq, d] (the new tokens of every sequence,
    sequence s in rows query_start_loc[s] .. [s+1]); caches [NB, Hkv, bs, d];
    block_tables int32 [B, W]; context_lens int32 [B] (tokens in the cache, the chunk
    included); query_start_loc int32 [B + 1]."""
    import torch
    what = "pa_prefill"
    if not (q.dim() == 3 and tuple(out.shape) == tuple(q.shape)):
        _fail(what, f"q {tuple(q.shape)} and out {tuple(out.shape)} must both be [T, Hq, d]")
    T, hq, d = q.shape
    nb, hkv, bs, _ = _cache_shape(what, k_cache, v_cache, head_dim=d)
    if context_lens.dim() != 1:
        _fail(what, "context_lens must be [B]")
    B = context_lens.shape[0]
    _tables(what, block_tables, context_lens, B)
    if tuple(query_start_loc.shape) != (B + 1,):
        _fail(what, f"query_start_loc must be [{B + 1}]")
    dev = _args(what, {"q": q, "out": out, "k_cache": k_cache, "v_cache": v_cache},
                ints={"block_tables": (block_tables, torch.int32),
                      "context_lens": (context_lens, torch.int32),
                      "query_start_loc": (query_start_loc, torch.int32)})
    with _on(dev):
        _check(load().pa_prefill(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                 _ptr(block_tables), _ptr(context_lens), _ptr(query_start_loc),
                                 B, T, hq, hkv, d, bs, nb, block_tables.shape[1], float(scale),
                                 int(sliding_window), _dtype(q), _stream(stream, dev)), what)


def device_error(device: int = 0, clear: bool = True) -> int:
    """Synchronises `device` and returns (and by default clears) its error bits."""
    bits = ctypes.c_uint32(0)
    _check(load().pa_get_device_error(device, ctypes.byref(bits), 1 if clear else 0),
           "pa_get_device_error")
    return int(bits.value)


def version() -> int:
    return int(load().pa_version())
