"""ctypes binding of the host block manager (include/pa_block_manager.h).

Marshalling only; the logic is the C++ in libpa.so.
"""
from __future__ import annotations

import ctypes

import numpy as np

from ._lib import PAError, _check, load

_declared = False


def _lib():
    global _declared
    lib = load()
    if not _declared:
        P, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
        lib.pa_bm_create.argtypes = [i32, i32]
        lib.pa_bm_create.restype = P
        lib.pa_bm_destroy.argtypes = [P]
        lib.pa_bm_destroy.restype = None
        lib.pa_bm_blocks_needed.argtypes = [i32, i32]
        lib.pa_bm_blocks_needed.restype = i32
        lib.pa_bm_num_free_blocks.argtypes = [P]
        lib.pa_bm_num_free_blocks.restype = i32
        lib.pa_bm_usage_ratio.argtypes = [P]
        lib.pa_bm_usage_ratio.restype = ctypes.c_double
        lib.pa_bm_can_allocate.argtypes = [P, i32]
        lib.pa_bm_can_allocate.restype = i32
        lib.pa_bm_allocate.argtypes = [P, i64, i32]
        lib.pa_bm_allocate.restype = i32
        lib.pa_bm_fork.argtypes = [P, i64, i64]
        lib.pa_bm_fork.restype = i32
        lib.pa_bm_free.argtypes = [P, i64]
        lib.pa_bm_free.restype = i32
        lib.pa_bm_append_slots.argtypes = [P, P, i32, P, P, i32, ctypes.POINTER(i32)]
        lib.pa_bm_append_slots.restype = i32
        lib.pa_bm_append_slots_cow.argtypes = [P, P, i32, P, P, ctypes.POINTER(i32)]
        lib.pa_bm_append_slots_cow.restype = i32
        lib.pa_bm_slot.argtypes = [P, i64, i32]
        lib.pa_bm_slot.restype = i64
        lib.pa_bm_seq_len.argtypes = [P, i64]
        lib.pa_bm_seq_len.restype = i32
        lib.pa_bm_block_refcount.argtypes = [P, i32]
        lib.pa_bm_block_refcount.restype = i32
        lib.pa_bm_block_tables.argtypes = [P, P, i32, P, i32, P]
        lib.pa_bm_block_tables.restype = i32
        lib.pa_bm_set_cpu_pool.argtypes = [P, i32]
        lib.pa_bm_set_cpu_pool.restype = i32
        lib.pa_bm_num_free_cpu_blocks.argtypes = [P]
        lib.pa_bm_num_free_cpu_blocks.restype = i32
        lib.pa_bm_is_swapped.argtypes = [P, i64]
        lib.pa_bm_is_swapped.restype = i32
        for f in (lib.pa_bm_swap_out, lib.pa_bm_swap_in):
            f.argtypes = [P, P, i32, P, i32, ctypes.POINTER(i32)]
            f.restype = i32
        lib.pa_bm_set_sliding_window.argtypes = [P, i32]
        lib.pa_bm_set_sliding_window.restype = i32
        _declared = True
    return lib


def blocks_needed(num_tokens: int, block_size: int) -> int:
    return int(_lib().pa_bm_blocks_needed(num_tokens, block_size))


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


class BlockManager:
    """Reference-counted block pool with per-sequence page tables.  Not thread-safe: one
    manager per engine thread."""

    def __init__(self, num_blocks: int, block_size: int):
        self._h = None  # so that __del__ is safe if the library cannot be loaded
        self._lib = _lib()
        self._h = self._lib.pa_bm_create(num_blocks, block_size)
        if not self._h:
            raise PAError("pa_bm_create failed (bad sizes or out of host memory)")
        self.num_blocks = num_blocks
        self.block_size = block_size

    def close(self):
        if self._h:
            self._lib.pa_bm_destroy(self._h)
            self._h = None

    def __del__(self):
        self.close()

    def _live(self):
        if not self._h:
            raise PAError("the block manager has been closed")
        return self._h

    @property
    def num_free_blocks(self) -> int:
        return int(self._lib.pa_bm_num_free_blocks(self._live()))

    @property
    def usage_ratio(self) -> float:
        return float(self._lib.pa_bm_usage_ratio(self._live()))

    def can_allocate(self, num_tokens: int) -> bool:
        return bool(self._lib.pa_bm_can_allocate(self._live(), num_tokens))

    def allocate(self, seq_id: int, num_tokens: int) -> None:
        _check(self._lib.pa_bm_allocate(self._live(), seq_id, num_tokens), "pa_bm_allocate")

    def fork(self, parent_id: int, child_id: int) -> None:
        _check(self._lib.pa_bm_fork(self._live(), parent_id, child_id), "pa_bm_fork")

    def free(self, seq_id: int) -> None:
        _check(self._lib.pa_bm_free(self._live(), seq_id), "pa_bm_free")

    def append_slots(self, seq_ids):
        """One new token per sequence -> (slot_mapping int64 [n], copy pairs int64 [p, 2])."""
        ids = np.ascontiguousarray(seq_ids, np.int64)
        n = ids.shape[0]
        slots = np.empty(n, np.int64)
        pairs = np.empty((max(n, 1), 2), np.int64)
        npairs = ctypes.c_int(0)
        _check(self._lib.pa_bm_append_slots(self._live(), _p(ids), n, _p(slots), _p(pairs), n,
                                            ctypes.byref(npairs)), "pa_bm_append_slots")
        return slots, pairs[:npairs.value].copy()

    def append_slots_cow(self, seq_ids):
        """One new token per sequence -> (slot_mapping int64 [n], copy list int32 [n, 3]):
        the same reservations as append_slots, each private copy given per sequence as
        (source block, logical block index, rows filled before the token), (-1, 0, 0)
        where nothing is copied -- the copy list of decode_cow."""
        ids = np.ascontiguousarray(seq_ids, np.int64)
        n = ids.shape[0]
        slots = np.empty(n, np.int64)
        cow = np.empty((max(n, 1), 3), np.int32)
        ncopies = ctypes.c_int(0)
        _check(self._lib.pa_bm_append_slots_cow(self._live(), _p(ids), n, _p(slots), _p(cow),
                                                ctypes.byref(ncopies)), "pa_bm_append_slots_cow")
        return slots, cow[:n].copy()

    def slot(self, seq_id: int, pos: int) -> int:
        """Slot of token position ``pos``; -1 where the position has no block (past the
        sequence's end, or released by the sliding window), which a cache write skips."""
        return int(self._lib.pa_bm_slot(self._live(), seq_id, pos))

    def seq_len(self, seq_id: int) -> int:
        """Context length of a sequence; -1 for an unknown sequence."""
        return int(self._lib.pa_bm_seq_len(self._live(), seq_id))

    def refcount(self, block: int) -> int:
        """Reference count of a physical block (0 = free); -1 for an id outside the pool."""
        return int(self._lib.pa_bm_block_refcount(self._live(), block))

    def set_sliding_window(self, window: int) -> None:
        """Keep only each sequence's last ``window`` positions: blocks wholly before them
        go back to the pool (table entry -1).  Only while no sequence exists."""
        _check(self._lib.pa_bm_set_sliding_window(self._live(), window), "pa_bm_set_sliding_window")

    def set_cpu_pool(self, num_cpu_blocks: int) -> None:
        _check(self._lib.pa_bm_set_cpu_pool(self._live(), num_cpu_blocks), "pa_bm_set_cpu_pool")

    @property
    def num_free_cpu_blocks(self) -> int:
        return int(self._lib.pa_bm_num_free_cpu_blocks(self._live()))

    def is_swapped(self, seq_id: int) -> bool:
        return self._lib.pa_bm_is_swapped(self._live(), seq_id) == 1

    def _move(self, fn, seq_ids, what):
        ids = np.ascontiguousarray(seq_ids, np.int64)
        cap = max(1, int(self.num_blocks))
        pairs = np.empty((cap, 2), np.int64)
        npairs = ctypes.c_int(0)
        _check(fn(self._live(), _p(ids), ids.shape[0], _p(pairs), cap, ctypes.byref(npairs)), what)
        return pairs[:npairs.value].copy()

    def swap_out(self, seq_ids):
        """Move a group of sequences to the host pool -> pairs (gpu block, host block)."""
        return self._move(self._lib.pa_bm_swap_out, seq_ids, "pa_bm_swap_out")

    def swap_in(self, seq_ids):
        """Move a swapped-out group back to the GPU -> pairs (host block, gpu block)."""
        return self._move(self._lib.pa_bm_swap_in, seq_ids, "pa_bm_swap_in")

    def block_tables(self, seq_ids, width: int):
        """(block_tables int32 [n, width], context_lens int32 [n]) for the decode call."""
        ids = np.ascontiguousarray(seq_ids, np.int64)
        n = ids.shape[0]
        bt = np.empty((n, width), np.int32)
        cl = np.empty(n, np.int32)
        _check(self._lib.pa_bm_block_tables(self._live(), _p(ids), n, _p(bt), width, _p(cl)),
               "pa_bm_block_tables")
        return bt, cl
